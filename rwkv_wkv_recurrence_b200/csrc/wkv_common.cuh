// Device helpers shared by the WKV kernels: TMA / mbarrier PTX wrappers, the
// bounded wait, and the numerically stable WKV-4 state step.
//
// WKV-4 state representation used by every kernel and by the C-ABI:
//   (a, b, p) stands for numerator A = a * 2^p and denominator B = b * 2^p of
//   the recurrent form of "RWKV - Transformer 시대에 RNN을 재발명하다",
//   Method / (2) Time-mixing (WKV):  WKV_t = (A_{t-1} + e^{u+k_t} v_t) /
//   (B_{t-1} + e^{u+k_t}),  A_t = e^{-w} A_{t-1} + e^{k_t} v_t,  likewise B.
// p is kept integer-valued, so rescaling the state (a, b) by 2^-s is exact and
// the represented (A, B) never changes when p moves.  Between rescales the
// state decays by a precomputed e^{-w} (one rounding per step, like the plain
// recurrence), so no per-step rounding of p accumulates.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace rwkv {

// Bit set in the library's device error word when a bounded wait gives up.
// Read and cleared by rwkv_check_device_error().
constexpr unsigned int kErrTmaTimeout = 1u;

// Default limit of a bounded wait.  A TMA load or an MMA chain completes in
// microseconds; a wait that lasts this long means its arrival will not come.
constexpr unsigned long long kDefaultWaitLimitNs = 1000000000ull;  // 1 s

// The library's device control block (one per device), whose address every
// kernel with a wait receives:
//   err            error bits (kErrTmaTimeout), set by a wait that gives up;
//   withhold       test hook: when nonzero the TMA-issuing thread arms its
//                  barriers but issues no load, so the first wait runs out with
//                  nothing in flight (set by rwkv_debug_withhold_loads);
//   wait_limit_ns  how long a bounded wait polls before giving up.
struct DevCtl {
  unsigned int err;
  unsigned int withhold;
  unsigned long long wait_limit_ns;
};

// ---------------------------------------------------------------- PTX helpers
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void fence_proxy_async() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t phase) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred P;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 P, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, P;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(phase)
      : "memory");
  return ok != 0;
}

// Nanoseconds of the GPU's global timer.
__device__ __forceinline__ unsigned long long global_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// Wait for phase `phase` of an mbarrier, giving up once ctl->wait_limit_ns
// have passed (each poll may suspend the thread for a hardware-chosen
// interval).  Returns false, and records kErrTmaTimeout, if the phase never
// completed.  The first poll needs no clock read.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t phase, DevCtl* ctl) {
  if (mbar_try_wait(bar, phase)) return true;
  const unsigned long long t0 = global_ns();
  const unsigned long long limit = *reinterpret_cast<volatile unsigned long long*>(&ctl->wait_limit_ns);
  while (!mbar_try_wait(bar, phase)) {
    if (global_ns() - t0 > limit) {
      atomicOr(&ctl->err, kErrTmaTimeout);
      return false;
    }
  }
  return true;
}

// Flags one CTA publishes for others of the same launch (release / acquire at GPU scope).
__device__ __forceinline__ void flag_release(unsigned int* f, unsigned int v) {
  asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(f), "r"(v) : "memory");
}
__device__ __forceinline__ unsigned int flag_acquire(const unsigned int* f) {
  unsigned int v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(f) : "memory");
  return v;
}
// Polls a flag until it is non-zero or the control block's time limit passes; 0 then (and the
// timeout bit is set in the error word).
__device__ __forceinline__ unsigned int flag_wait_bounded(const unsigned int* f, DevCtl* ctl) {
  unsigned int v = flag_acquire(f);
  if (v != 0u) return v;
  const unsigned long long t0 = global_ns();
  const unsigned long long limit = *reinterpret_cast<volatile unsigned long long*>(&ctl->wait_limit_ns);
  while ((v = flag_acquire(f)) == 0u) {
    if (global_ns() - t0 > limit) {
      atomicOr(&ctl->err, kErrTmaTimeout);
      return 0u;
    }
    __nanosleep(64);
  }
  return v;
}

// True when the test hook asks the issuing thread to withhold its loads.
__device__ __forceinline__ bool loads_withheld(const DevCtl* ctl) {
  return *reinterpret_cast<const volatile unsigned int*>(&ctl->withhold) != 0u;
}

// Abort path of a `stages`-deep load pipeline whose wait for iteration i gave up: the loads
// issued for iterations i .. (refills run stages - 1 iterations ahead, never past ntile) may
// still be in flight, so the issuing thread waits for each, bounded again, before its CTA
// leaves.  Nothing was issued when the loads were withheld.  Not inlined: it runs only on the
// abort path and keeps its registers out of the kernel's main loop.
static __device__ __noinline__ void drain_loads(uint64_t* bars, int stages, int i, int ntile, DevCtl* ctl) {
  if (loads_withheld(ctl)) return;
  const int issued = min(ntile, max(stages, i - 1 + stages));
  for (int j = i; j < issued; ++j) mbar_wait_bounded(&bars[j % stages], (uint32_t)(j / stages) & 1u, ctl);
}

// 3-D tiled TMA load (no multicast) into shared memory, completing on `bar`.
__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* map, uint64_t* bar, int c0, int c1,
                                            int c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(smem_u32(bar))
      : "memory");
}

// Contiguous bulk copy global -> shared (no multicast), completing on `bar`; both addresses
// 16-byte aligned, `bytes` a multiple of 16.
__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                   smem_u32(dst)),
               "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(smem_u32(bar))
               : "memory");
}

// 3-D tiled TMA store (shared -> global) of one box, tracked by the issuing
// thread's bulk async-group; the box is clipped at the tensor's bounds.
__device__ __forceinline__ void tma_store_3d(const CUtensorMap* map, const void* src, int c0, int c1, int c2) {
  asm volatile("cp.async.bulk.tensor.3d.global.shared::cta.tile.bulk_group [%0, {%2, %3, %4}], [%1];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(smem_u32(src)), "r"(c0), "r"(c1), "r"(c2)
               : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// The thread's bulk stores have finished reading shared memory.
__device__ __forceinline__ void bulk_wait_read() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
// The thread's bulk stores are complete.
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

__device__ __forceinline__ void prefetch_tensormap(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// 2^x on the special-function unit (PTX ex2.approx.ftz.f32).
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// 1/x on the special-function unit (PTX rcp.approx.ftz.f32, ~1 ulp); callers
// only pass normal x (x >= FLT_MIN), the denominators of the WKV ratio.
__device__ __forceinline__ float rcp_approx(float x) {
  float y;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Logistic sigmoid 1 / (1 + e^{-x}) (the receptance gate); saturates to 0 and 1
// without NaN: e^{-x} = inf gives 0, e^{-x} = 0 gives 1.
__device__ __forceinline__ float sigmoid(float x) { return rcp_approx(1.f + __expf(-x)); }

// A WKV denominator too small to divide by: it is below FLT_MIN only when a
// token arrives with no history and its own weight e^{u+k} underflowed at the
// segment's scale, where the ratio is v itself.  The kernels test !(d < kMinDen)
// so that a NaN denominator (a NaN input upstream) still divides and propagates.
constexpr float kMinDen = 1.17549435e-38f;

// ---------------------------------------------------------------- I/O types
template <typename T>
struct IO;
template <>
struct IO<float> {
  __device__ __forceinline__ static float load(const float* p) { return *p; }
  __device__ __forceinline__ static float to_f(float x) { return x; }
  __device__ __forceinline__ static float from_f(float x) { return x; }
};
template <>
struct IO<__nv_bfloat16> {
  __device__ __forceinline__ static float load(const __nv_bfloat16* p) { return __bfloat162float(*p); }
  __device__ __forceinline__ static float to_f(__nv_bfloat16 x) { return __bfloat162float(x); }
  __device__ __forceinline__ static __nv_bfloat16 from_f(float x) { return __float2bfloat16_rn(x); }
};

// Plain-access path of the WKV-4 kernels (any element-aligned base, any C):
// warp-local copy of rows [ts, ts + cnt) of one [B,T,C] tensor into ROWS
// shared-memory rows of 32 channels (lane = channel; rows past cnt and lanes
// past C get zeros, as the TMA fill would), plus an L2 prefetch of the rows
// `ahead` steps later for the warp's next visit.
template <typename T, int ROWS>
__device__ __forceinline__ void warp_rows_in(T* rows, const T* __restrict__ g, int bb, int T_, int C, int ts,
                                             int cnt, int c, bool valid, int lane, int ahead) {
  const size_t base = ((size_t)bb * T_ + (size_t)max(ts, 0)) * C + (size_t)c;
#pragma unroll
  for (int j = 0; j < ROWS; ++j)
    rows[j * 32 + lane] = (valid && j < cnt) ? g[base + (size_t)j * C] : IO<T>::from_f(0.f);
  const int tn = ts + ahead + lane;
  if (lane < ROWS && tn >= 0 && tn < T_ && valid)
    asm volatile("prefetch.global.L2 [%0];" ::"l"(g + ((size_t)bb * T_ + tn) * C + c) : "memory");
}

// ---------------------------------------------------------------- WKV-4 state
// log2(e) split into an fp32 head and tail: x = k*kL2eHi + k*kL2eLo carries
// the product k log2(e) to ~2^-40 relative, so a key of 40 is not shifted by
// the 1e-6 that rounding log2(e) to fp32 alone would cost.
constexpr float kL2eHi = 1.44269502162933349609375f;
constexpr float kL2eLo = 1.9259629911266175e-08f;

// 2^e as a double, e clamped to the normal range [-1022, 1023].  Callers
// scale values whose true factor would leave that range only when the value is
// negligible (a state or carry below 2^-1000 of the other terms).
__device__ __forceinline__ double pow2d(int e) {
  e = min(max(e, -1022), 1023);
  return __longlong_as_double((long long)(e + 1023) << 52);
}

// floor(log2 x) of a positive normal double (exponent field); -1023 for 0.
__device__ __forceinline__ int ilogb_d(double x) {
  return (int)((__double_as_longlong(x) >> 52) & 0x7ff) - 1023;
}

// 2^e as a float for integer e <= 0 (0 below the normal range).
__device__ __forceinline__ float pow2f_neg(int e) {
  return e < -126 ? 0.f : __int_as_float((e + 127) << 23);
}

// Token weight e^{k} 2^{-p}: the exponent k log2(e) - p is formed with the
// split log2(e), then raised on the special-function unit.
__device__ __forceinline__ float tok_weight(float k, float p) {
  return ex2(fmaf(k, kL2eLo, fmaf(k, kL2eHi, -p)));
}

// State (A, B) = (a, b) * 2^p carried between 16-step segments, a and b in
// fp64: the fp64 carry keeps the decayed sums of thousands of steps to ~1e-16
// relative, which the gradients need (they cancel terms of similar size).
struct State {
  double a, b;
  int p;
};

constexpr int kScaleMax = 1 << 20;  // |p| bound (keys beyond ±7e5 are out of range)

__device__ __forceinline__ int clamp_scale(int q) { return min(max(q, -kScaleMax), kScaleMax); }

// Moves a state to scale q (exact: multiplies by a power of two).
__device__ __forceinline__ State rescale(State s, int q) {
  const double f = pow2d(s.p - q);
  s.a *= f;
  s.b *= f;
  s.p = q;
  return s;
}

// Associative step of the time-parallel form: the state S decays over a
// segment (factor lamL = e^{-w len}) and the segment's own contribution X
// (its scan from a zero state) is added:  S' = lamL * S (+) X.  The common
// scale follows the larger of the two magnitudes, so the result's b stays
// near 1 and never drifts towards the end of the fp64 range.
__device__ __forceinline__ State fold(State s, double lamL, State x) {
  s.a *= lamL;
  s.b *= lamL;
  const int q = max(x.p, s.p + ilogb_d(s.b) + 1);
  s = rescale(s, q);
  x = rescale(x, q);
  s.a += x.a;
  s.b += x.b;
  return s;
}

// Writes a state as fp32 (a, b, p) with b moved into [1, 2), so that rounding
// to fp32 neither underflows nor overflows.
__device__ __forceinline__ void store_state(const State& s0, float* a, float* b, float* p) {
  State s = s0;
  if (s.b > 0.0) s = rescale(s, s.p + ilogb_d(s.b));
  *a = (float)s.a;
  *b = (float)s.b;
  *p = (float)s.p;
}

// Loads an fp32 (a, b, p) state, moving a fractional part of p into (a, b).
__device__ __forceinline__ State load_state(float a, float b, float p) {
  State s;
  if (!(fabsf(p) < (float)kScaleMax)) p = 0.f;  // inf / NaN / huge p only make sense for a zero state
  const float pi = floorf(p);
  s.a = (double)a;
  s.b = (double)b;
  if (p != pi) {
    const double f = exp2((double)(p - pi));
    s.a *= f;
    s.b *= f;
  }
  s.p = (int)pi;
  return s;
}

// Scale that puts both the state and every token weight of a segment at or
// below 2^1: q = max(ceil(max k log2 e), p + floor(log2 b) + 1).
__device__ __forceinline__ int segment_scale(float kmax2, const State& s) {
  const float kq = fminf(fmaxf(ceilf(kmax2), -(float)kScaleMax), (float)kScaleMax);
  return clamp_scale(max((int)kq, s.p + ilogb_d(s.b) + 1));
}

// s e^{-w} + x in fp32 with e^{-w} = lh + ll: the low part keeps the decay
// unbiased (a rounded e^{-w} alone would bias every step the same way).
__device__ __forceinline__ float decay_add(float s, float x, float lh, float ll) {
  return fmaf(lh, s, fmaf(ll, s, x));
}

// e^{-w len} in fp64 for len <= 16 by repeated multiplication of e^{-w}.
__device__ __forceinline__ double lam_pow(double lam, int len) {
  double r = 1.0;
  for (int i = 0; i < len; ++i) r *= lam;
  return r;
}

// ------------------------------------------------ single recurrent step (decode)
// Limits of the stable single step: rescale when the new token's relative log2
// weight exceeds kSlowXHi or b leaves [kSlowBLo, kSlowBHi].
constexpr float kSlowXHi = 20.f;
constexpr float kSlowBLo = 0x1p-20f;
constexpr float kSlowBHi = 0x1p+80f;

struct Lane4 {
  float lam;     // e^{-w} rounded to fp32
  float lam_lo;  // e^{-w} - lam (the rounding remainder)
  float U;       // e^{u}
};

// The decode state outlives a call, so its decay uses e^{-w} as lam + lam_lo
// (bias-free to ~2^-48 per step) instead of the rounded fp32 value alone.
__device__ __forceinline__ Lane4 lane4_step_consts(float w, float u) {
  Lane4 L;
  const double lam_d = exp(-(double)w);
  L.lam = (float)lam_d;
  L.lam_lo = (float)(lam_d - (double)L.lam);
  L.U = expf(u);
  return L;
}

// Rescale (a, b, p) so that max(x, log2 b) lands in [0, 1); x is the new
// token's log2 weight relative to 2^p and is shifted the same way.
__device__ __forceinline__ void wkv4_rescale(float& a, float& b, float& p, float& x) {
  const float xc = fminf(fmaxf(x, -2000.f), 2000.f);
  int s = static_cast<int>(floorf(xc));
  if (b > 0.f) s = max(s, ilogbf(b));
  a = ldexpf(a, -s);
  b = ldexpf(b, -s);
  p += static_cast<float>(s);
  x -= static_cast<float>(s);
}

// Bring an externally supplied fp32 state to an integer p.
__device__ __forceinline__ void wkv4_snap(float& a, float& b, float& p) {
  if (!(fabsf(p) < 1e30f)) {
    p = 0.f;
    return;
  }
  const float pi = floorf(p);
  const float f = exp2f(p - pi);
  a *= f;
  b *= f;
  p = pi;
}

// One recurrent step in fp32 with a compensated decay: rescale if needed,
// emit WKV_t, advance the state.
__device__ __forceinline__ float wkv4_step_careful(float& a, float& b, float& p, float kt, float vt,
                                                   const Lane4& L) {
  float x = fmaf(kt, kL2eLo, fmaf(kt, kL2eHi, -p));
  if (!(x <= kSlowXHi && b >= kSlowBLo && b <= kSlowBHi)) wkv4_rescale(a, b, p, x);
  const float e = ex2(x);
  const float eu = e * L.U;
  const float d = b + eu;
  const float n = fmaf(eu, vt, a);
  const float y = !(d < kMinDen) ? n * rcp_approx(d) : vt;  // a NaN d propagates
  a = fmaf(L.lam, a, fmaf(L.lam_lo, a, e * vt));
  b = fmaf(L.lam, b, fmaf(L.lam_lo, b, e));
  return y;
}

}  // namespace rwkv
