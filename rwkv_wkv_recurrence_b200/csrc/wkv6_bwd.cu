// Finch / RWKV-6 WKV backward on the CUDA cores (sm_100a).
//
// Operator: "RWKV-5 Eagle과 RWKV-6 Finch", section Finch: per head, for each token t,
//   y_t = r_t (s + diag(u) k_tᵀ v_t),   then   s <- diag(w_t) s + k_tᵀ v_t,   w_t = exp(-exp(ω_t)),
// with s[d][j] (key d, value j).  The pages print no backward; this is the chain rule through
// that recurrence for L = Σ gy·y + Σ gs_out ∘ s_T.  With s^(t) the state before token t and
// G^(t) = ∂L/∂s^(t) (G^(T) = gs_out, G^(t) = r_tᵀ gy_t + diag(w_t) G^(t+1)):
//   gr_t = s^(t) gy_tᵀ + u ⊙ k_t (v_t·gy_t)
//   gk_t = G^(t+1) v_tᵀ + u ⊙ r_t (v_t·gy_t)
//   gv_t = G^(t+1)ᵀ k_t + (Σ_d r_t u k_t) gy_t
//   gω_t = -e^{ω_t} w_t ⊙ Σ_j G^(t+1)[.][j] s^(t)[.][j]     (one value per token and key channel)
//   gu   = Σ_{b,t} r_t ⊙ k_t (v_t·gy_t),   gs_in = G^(0).
//
// The decay changes with every token, so the chunked factorization the Eagle kernels use would
// need per-token cumulative factors and a fallback wherever they leave the fp32 range; this
// kernel runs the recurrence itself, token by token, which holds for any w in [0, 1].
//
// The recurrence is linear in s and in G, so a 64-token chunk depends on the rest of the sequence
// only through the state entering it and the gradient leaving it.  Three kernels:
//   1. per chunk, in parallel: the chunk's own state increment ΔS (its tokens from a zero state),
//      its own gradient increment ΔG = Σ_τ diag(Π_{a<=m<τ} w_m) r_τᵀ gy_τ (a = the chunk's first
//      token) and its decay product D = Π_m w_m;
//   2. per (batch row, head), sequentially over the chunks, one CTA per scan: the state entering
//      every chunk, S_{c+1} = D_c ⊙ S_c + ΔS_c, and the gradient leaving it,
//      G_{c-1} = ΔG_c + D_c ⊙ G_c (in place over the increments), and gs_in;
//   3. per chunk, in parallel: the chunk's tokens forward from its entering state (gr_t, and the
//      state every 8 tokens into shared memory), then backwards from its leaving gradient, 8
//      tokens at a time: the 8 states are recomputed into registers and walked with G, forming gk,
//      the gω row sums and gv.
// So all B·H·ceil(T/64) chunks are spread evenly over the SMs (one CTA per (batch row, head) would
// leave some SMs with two whole sequences).  In every kernel thread t of 256 owns the 4 x 4 block
// of keys 4 (t / 16) .. + 3 and values 4 (t % 16) .. + 3; sums over the values (gr, gk, gω) run
// over the 16 lanes of a half-warp as a shuffle butterfly, sums over the keys (gv) as one shuffle
// across the warp's two key groups and then through shared memory.  A chunk's inputs (r, k, v, gy,
// ω: 48 KB) arrive by cp.async.  gu is summed per (chunk, key) in fp32 and reduced over batch rows
// and chunks in fixed order, so the results are deterministic.
#include <cuda_bf16.h>

#include "launch.h"
#include "wkv_common.cuh"

namespace rwkv {
namespace {

constexpr int kN = 64;        // channels per head
constexpr int kL = 64;        // tokens per chunk
constexpr int kS = 8;         // tokens per sub-chunk (states held in registers)
constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kBlock = 16;    // floats of s (or G) per thread
static_assert(kThreads * kBlock == kN * kN, "256 threads x 16 elements cover one 64 x 64 state");

struct __align__(16) Stage {
  __nv_bfloat16 r[kL][kN], k[kL][kN], v[kL][kN], g[kL][kN];
  float om[kL][kN];  // ω; the chunk kernel overwrites it with dw/dω = -e^ω w
};

struct __align__(16) SumsSmem {  // kernel 1
  Stage st;
  float w[kL][kN];
};

struct __align__(16) ChunkSmem {  // kernel 3
  Stage st;
  float w[kL][kN];                       // w_t[d] of the chunk
  float4 sub[kL / kS][4][kThreads];      // the state every kS tokens, each thread's block as 4 float4
  float red[kS][kWarps][kN];             // gv parts of a sub-chunk: [token][warp][value]
  float vg[kL];                          // v_t · gy_t
  float ruk[kL];                         // Σ_d r_t[d] u_d k_t[d]
  float uu[kN];
};

__device__ __forceinline__ void cp_async16(void* dst, const void* src, bool full) {
  const uint32_t d = (uint32_t)__cvta_generic_to_shared(dst);
  // src-size 0 fills the 16 bytes with zeros (rows past the end of the sequence)
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(d), "l"(src), "r"(full ? 16 : 0) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }

__device__ __forceinline__ void bf16x4(const __nv_bfloat16* p, float (&f)[4]) {
  const uint2 x = *reinterpret_cast<const uint2*>(p);
  f[0] = __uint_as_float(x.x << 16);
  f[1] = __uint_as_float(x.x & 0xFFFF0000u);
  f[2] = __uint_as_float(x.y << 16);
  f[3] = __uint_as_float(x.y & 0xFFFF0000u);
}

__device__ __forceinline__ float bf(const __nv_bfloat16 x) { return __bfloat162float(x); }

// Element offset of token t, channel 0 of head h, batch row bb in a [B,T,H,64] tensor.
__device__ __forceinline__ size_t tok_off(const Wkv6BwdParams& p, int bb, int h, int t) {
  return ((size_t)bb * p.T + t) * (size_t)p.H * kN + (size_t)h * kN;
}

// The tokens [t0, t0 + cnt) of (bb, h) into a stage (rows past cnt are zero) and wait for them.
__device__ __forceinline__ void stage_chunk(Stage& S, const Wkv6BwdParams& p, int bb, int h, int t0, int cnt) {
  const int tid = threadIdx.x;
  const size_t rs = (size_t)p.H * kN;  // elements from one token to the next
  const size_t base = tok_off(p, bb, h, t0);
#pragma unroll
  for (int i = tid; i < kL * 8; i += kThreads) {  // bf16 rows: 8 pieces of 16 bytes
    const int row = i >> 3, pc = (i & 7) * 8;
    const bool ok = row < cnt;
    const size_t off = base + (size_t)(ok ? row : 0) * rs + pc;
    cp_async16(&S.r[row][pc], p.r + off, ok);
    cp_async16(&S.k[row][pc], p.k + off, ok);
    cp_async16(&S.v[row][pc], p.v + off, ok);
    cp_async16(&S.g[row][pc], p.gy + off, ok);
  }
#pragma unroll
  for (int i = tid; i < kL * 16; i += kThreads) {  // fp32 rows: 16 pieces
    const int row = i >> 4, pc = (i & 15) * 4;
    const bool ok = row < cnt;
    cp_async16(&S.om[row][pc], p.omega + base + (size_t)(ok ? row : 0) * rs + pc, ok);
  }
  cp_async_commit();
  cp_async_wait_all();
  __syncthreads();
}

// Sums x[i] (i = 0..3, rows d0 + i) over the 16 lanes of a half-warp (the value groups).  On return
// the lane holds the sum for row 2 b3 + b2 (b3, b2: bits 3 and 2 of the lane), the same in the four
// lanes that differ in bits 0 and 1.
__device__ __forceinline__ float butterfly4(const float (&x)[4], int lane) {
  const bool b3 = (lane >> 3) & 1, b2 = (lane >> 2) & 1;
  float k0 = b3 ? x[2] : x[0], k1 = b3 ? x[3] : x[1];
  const float s0 = b3 ? x[0] : x[2], s1 = b3 ? x[1] : x[3];
  k0 += __shfl_xor_sync(0xffffffffu, s0, 8);
  k1 += __shfl_xor_sync(0xffffffffu, s1, 8);
  float k = b2 ? k1 : k0;
  k += __shfl_xor_sync(0xffffffffu, b2 ? k0 : k1, 4);
  k += __shfl_xor_sync(0xffffffffu, k, 2);
  k += __shfl_xor_sync(0xffffffffu, k, 1);
  return k;
}

// The same for two quantities of four rows each, x[0..3] and y[0..3]: on return the lane holds,
// for row 2 b3 + b2, the x sum if bit 1 of the lane is clear and the y sum if it is set (the same
// in the two lanes that differ in bit 0).
__device__ __forceinline__ float butterfly8(const float (&x)[4], const float (&y)[4], int lane) {
  const bool b3 = (lane >> 3) & 1, b2 = (lane >> 2) & 1, b1 = (lane >> 1) & 1;
  // bit 3: keep rows 2 b3, 2 b3 + 1 of both quantities
  float kx0 = b3 ? x[2] : x[0], kx1 = b3 ? x[3] : x[1], ky0 = b3 ? y[2] : y[0], ky1 = b3 ? y[3] : y[1];
  kx0 += __shfl_xor_sync(0xffffffffu, b3 ? x[0] : x[2], 8);
  kx1 += __shfl_xor_sync(0xffffffffu, b3 ? x[1] : x[3], 8);
  ky0 += __shfl_xor_sync(0xffffffffu, b3 ? y[0] : y[2], 8);
  ky1 += __shfl_xor_sync(0xffffffffu, b3 ? y[1] : y[3], 8);
  // bit 2: keep row 2 b3 + b2
  float kx = b2 ? kx1 : kx0, ky = b2 ? ky1 : ky0;
  kx += __shfl_xor_sync(0xffffffffu, b2 ? kx0 : kx1, 4);
  ky += __shfl_xor_sync(0xffffffffu, b2 ? ky0 : ky1, 4);
  // bit 1: keep x or y
  float k = b1 ? ky : kx;
  k += __shfl_xor_sync(0xffffffffu, b1 ? kx : ky, 2);
  k += __shfl_xor_sync(0xffffffffu, k, 1);
  return k;
}

// This thread's 16 elements of a [64][64] fp32 state (rows d0 .. d0 + 3, columns j0 .. j0 + 3).
__device__ __forceinline__ void load_block(const float* m, int d0, int j0, float (&s)[kBlock]) {
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float4 x = *reinterpret_cast<const float4*>(m + (d0 + i) * kN + j0);
    s[4 * i + 0] = x.x;
    s[4 * i + 1] = x.y;
    s[4 * i + 2] = x.z;
    s[4 * i + 3] = x.w;
  }
}
__device__ __forceinline__ void store_block(float* m, int d0, int j0, const float (&s)[kBlock]) {
#pragma unroll
  for (int i = 0; i < 4; ++i)
    *reinterpret_cast<float4*>(m + (d0 + i) * kN + j0) = make_float4(s[4 * i], s[4 * i + 1], s[4 * i + 2], s[4 * i + 3]);
}
// The per-chunk [64][64] blocks of the workspace are kept in thread order: float4 i of thread t at
// [i][t], so that a warp's accesses are contiguous.
__device__ __forceinline__ void save_own(float* m, const float (&s)[kBlock]) {
  float4* q = reinterpret_cast<float4*>(m) + threadIdx.x;
#pragma unroll
  for (int i = 0; i < 4; ++i) q[i * kThreads] = make_float4(s[4 * i], s[4 * i + 1], s[4 * i + 2], s[4 * i + 3]);
}
__device__ __forceinline__ void load_own(const float* m, float (&s)[kBlock]) {
  const float4* q = reinterpret_cast<const float4*>(m) + threadIdx.x;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float4 x = q[i * kThreads];
    s[4 * i + 0] = x.x;
    s[4 * i + 1] = x.y;
    s[4 * i + 2] = x.z;
    s[4 * i + 3] = x.w;
  }
}

// One token of the state recurrence on the thread's block: s <- diag(w_t) s + k_tᵀ v_t.
__device__ __forceinline__ void state_step(float (&s)[kBlock], const Stage& S, const float (*w)[kN], int t, int d0,
                                           int j0) {
  float kf[4], vf[4];
  bf16x4(&S.k[t][d0], kf);
  bf16x4(&S.v[t][j0], vf);
  const float4 w4 = *reinterpret_cast<const float4*>(&w[t][d0]);
  const float wf[4] = {w4.x, w4.y, w4.z, w4.w};
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int c = 0; c < 4; ++c) s[4 * i + c] = fmaf(wf[i], s[4 * i + c], kf[i] * vf[c]);
}

// 1. Per chunk: ΔS (the chunk's tokens from a zero state), ΔG = Σ_τ diag(P_τ) r_τᵀ gy_τ with
//    P_τ = Π_{a<=m<τ} w_m, and D = P at the chunk's end.
__global__ void __launch_bounds__(kThreads) wkv6_bwd_sums_kernel(const Wkv6BwdParams p) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  SumsSmem& sm = *reinterpret_cast<SumsSmem*>(smem_raw);
  const int tid = threadIdx.x;
  const int d0 = 4 * (tid >> 4), j0 = 4 * (tid & 15);
  const int nch = (p.T + kL - 1) / kL;
  const int bh = blockIdx.x / nch, c = blockIdx.x % nch;
  const int bb = bh / p.H, h = bh % p.H;
  const int t0 = c * kL, cnt = min(kL, p.T - t0);
  stage_chunk(sm.st, p, bb, h, t0, cnt);
  for (int i = tid; i < kL * kN; i += kThreads) sm.w[i >> 6][i & 63] = expf(-expf(sm.st.om[i >> 6][i & 63]));
  __syncthreads();
  const Stage& S = sm.st;
  float ds[kBlock], dg[kBlock], P[4] = {1.f, 1.f, 1.f, 1.f};
#pragma unroll
  for (int e = 0; e < kBlock; ++e) ds[e] = dg[e] = 0.f;
#pragma unroll 4
  for (int t = 0; t < cnt; ++t) {
    float rf[4], gf[4];
    bf16x4(&S.r[t][d0], rf);
    bf16x4(&S.g[t][j0], gf);
    const float4 w4 = *reinterpret_cast<const float4*>(&sm.w[t][d0]);
    const float wf[4] = {w4.x, w4.y, w4.z, w4.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float rp = P[i] * rf[i];
#pragma unroll
      for (int cc = 0; cc < 4; ++cc) dg[4 * i + cc] = fmaf(rp, gf[cc], dg[4 * i + cc]);
      P[i] *= wf[i];
    }
    state_step(ds, S, sm.w, t, d0, j0);
  }
  const size_t slot = ((size_t)bh * nch + c) * kN * kN;
  save_own(p.xs + slot, ds);
  save_own(p.xg + slot, dg);
  if ((tid & 15) == 0)
    *reinterpret_cast<float4*>(p.dec + ((size_t)bh * nch + c) * kN + d0) = make_float4(P[0], P[1], P[2], P[3]);
}

// 2. Per (batch row, head), two CTAs: the state entering every chunk (even CTA) and the gradient
//    leaving it with gs_in (odd CTA), each in place over its increments.  The two scans are
//    independent.
__global__ void __launch_bounds__(kThreads) wkv6_bwd_carry_kernel(const Wkv6BwdParams p) {
  const int tid = threadIdx.x;
  const int d0 = 4 * (tid >> 4), j0 = 4 * (tid & 15);
  const int nch = (p.T + kL - 1) / kL;
  const int bh = blockIdx.x >> 1;
  const bool grad = blockIdx.x & 1;
  const size_t state_off = (size_t)bh * kN * kN;
  float* xs = (grad ? p.xg : p.xs) + (size_t)bh * nch * kN * kN;
  const float* dec = p.dec + (size_t)bh * nch * kN;
  const float* init = grad ? p.gs_out : p.s_in;
  float a[kBlock], x[kBlock], xn[kBlock];
  if (init != nullptr)
    load_block(init + state_off, d0, j0, a);
  else
#pragma unroll
    for (int e = 0; e < kBlock; ++e) a[e] = 0.f;
  // the state runs forward over the chunks, the gradient backward
  const int c0 = grad ? nch - 1 : 0, dc = grad ? -1 : 1;
  load_own(xs + (size_t)c0 * kN * kN, x);
  for (int i = 0, c = c0; i < nch; ++i, c += dc) {
    if (i + 1 < nch) load_own(xs + (size_t)(c + dc) * kN * kN, xn);  // the next increment, ahead of the chain
    const float4 D = *reinterpret_cast<const float4*>(dec + (size_t)c * kN + d0);
    const float df[4] = {D.x, D.y, D.z, D.w};
    save_own(xs + (size_t)c * kN * kN, a);
#pragma unroll
    for (int ii = 0; ii < 4; ++ii)
#pragma unroll
      for (int cc = 0; cc < 4; ++cc) a[4 * ii + cc] = fmaf(df[ii], a[4 * ii + cc], x[4 * ii + cc]);
#pragma unroll
    for (int e = 0; e < kBlock; ++e) x[e] = xn[e];
  }
  if (grad && p.gs_in != nullptr) store_block(p.gs_in + state_off, d0, j0, a);
}

// 3. Per chunk: gr forward in time from the entering state; gk, gv, gω backward from the leaving
//    gradient; the chunk's gu parts.
__global__ void __launch_bounds__(kThreads, 1) wkv6_bwd_chunk_kernel(const Wkv6BwdParams p) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  ChunkSmem& sm = *reinterpret_cast<ChunkSmem*>(smem_raw);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int d0 = 4 * (tid >> 4), j0 = 4 * (tid & 15);
  const int nch = (p.T + kL - 1) / kL;
  const int bh = blockIdx.x / nch, c = blockIdx.x % nch;
  const int bb = bh / p.H, h = bh % p.H;
  const int t0 = c * kL, cnt = min(kL, p.T - t0);
  const size_t slot = ((size_t)bh * nch + c) * kN * kN;
  // the lane that holds a butterfly result writes row dr (bits 3, 2 of the lane)
  const int dr = d0 + 2 * ((lane >> 3) & 1) + ((lane >> 2) & 1);

  if (tid < kN) sm.uu[tid] = p.u[h * kN + tid];
  stage_chunk(sm.st, p, bb, h, t0, cnt);
  Stage& S = sm.st;
  for (int i = tid; i < kL * kN; i += kThreads) {
    const int t = i >> 6, d = i & 63;
    const float om = S.om[t][d];
    sm.w[t][d] = expf(-expf(om));
    S.om[t][d] = -expf(om - expf(om));  // dw/dω = -e^ω w, finite (0) where w underflows
  }
  {  // v_t·gy_t and Σ_d r_t u k_t: token t = tid / 4, quarter q = tid % 4 of the channels
    const int t = tid >> 2, q = tid & 3;
    float a = 0.f, b = 0.f;
#pragma unroll
    for (int g = 0; g < 4; ++g) {
      const int c0 = 16 * q + 4 * g;
      float vf[4], gf[4], rf[4], kf[4];
      bf16x4(&S.v[t][c0], vf);
      bf16x4(&S.g[t][c0], gf);
      bf16x4(&S.r[t][c0], rf);
      bf16x4(&S.k[t][c0], kf);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        a = fmaf(vf[i], gf[i], a);
        b = fmaf(rf[i] * sm.uu[c0 + i], kf[i], b);
      }
    }
    a += __shfl_xor_sync(0xffffffffu, a, 1);
    a += __shfl_xor_sync(0xffffffffu, a, 2);
    b += __shfl_xor_sync(0xffffffffu, b, 1);
    b += __shfl_xor_sync(0xffffffffu, b, 2);
    if (q == 0) {
      sm.vg[t] = a;
      sm.ruk[t] = b;
    }
  }
  __syncthreads();
  if (tid < kN) {  // gu parts: Σ_t r_t[d] k_t[d] (v_t·gy_t), d = tid
    float a = 0.f;
    for (int t = 0; t < cnt; ++t) a = fmaf(bf(S.r[t][tid]) * bf(S.k[t][tid]), sm.vg[t], a);
    p.part[((size_t)bh * nch + c) * kN + tid] = a;
  }

  // forward in time: gr, and the state every kS tokens
  {
    float s[kBlock];
    load_own(p.xs + slot, s);
    const float ud = sm.uu[dr];
    for (int tb = 0; tb < cnt; tb += kS) {
#pragma unroll
      for (int i = 0; i < 4; ++i)
        sm.sub[tb / kS][i][tid] = make_float4(s[4 * i], s[4 * i + 1], s[4 * i + 2], s[4 * i + 3]);
#pragma unroll
      for (int m = 0; m < kS; ++m) {
        const int t = tb + m;
        if (t < cnt) {
          float gf[4], part[4];
          bf16x4(&S.g[t][j0], gf);
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            part[i] = s[4 * i] * gf[0];
#pragma unroll
            for (int cc = 1; cc < 4; ++cc) part[i] = fmaf(s[4 * i + cc], gf[cc], part[i]);
          }
          const float x = butterfly4(part, lane);
          if ((lane & 3) == 0)
            p.gr[tok_off(p, bb, h, t0 + t) + dr] = __float2bfloat16_rn(fmaf(ud * bf(S.k[t][dr]), sm.vg[t], x));
          state_step(s, S, sm.w, t, d0, j0);
        }
      }
    }
  }

  // backward in time, kS tokens at a time
  float G[kBlock];
  load_own(p.xg + slot, G);
  const int nsub = (cnt + kS - 1) / kS;
  for (int sc = nsub - 1; sc >= 0; --sc) {
    const int tb = sc * kS;
    float hs[kS][kBlock];  // hs[m] = s^(t0 + tb + m)
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float4 x = sm.sub[sc][i][tid];
      hs[0][4 * i + 0] = x.x;
      hs[0][4 * i + 1] = x.y;
      hs[0][4 * i + 2] = x.z;
      hs[0][4 * i + 3] = x.w;
    }
#pragma unroll
    for (int m = 1; m < kS; ++m) {
#pragma unroll
      for (int e = 0; e < kBlock; ++e) hs[m][e] = hs[m - 1][e];
      if (tb + m - 1 < cnt) state_step(hs[m], S, sm.w, tb + m - 1, d0, j0);
    }
#pragma unroll
    for (int m = kS - 1; m >= 0; --m) {
      const int t = tb + m;
      if (t < cnt) {
        float kf[4], vf[4], rf[4], gf[4];
        bf16x4(&S.k[t][d0], kf);
        bf16x4(&S.v[t][j0], vf);
        bf16x4(&S.r[t][d0], rf);
        bf16x4(&S.g[t][j0], gf);
        const float4 w4 = *reinterpret_cast<const float4*>(&sm.w[t][d0]);
        const float wf[4] = {w4.x, w4.y, w4.z, w4.w};
        float xk[4], xw[4], pv[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          xk[i] = G[4 * i] * vf[0];
          xw[i] = G[4 * i] * hs[m][4 * i];
#pragma unroll
          for (int cc = 1; cc < 4; ++cc) {
            xk[i] = fmaf(G[4 * i + cc], vf[cc], xk[i]);
            xw[i] = fmaf(G[4 * i + cc], hs[m][4 * i + cc], xw[i]);
          }
        }
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) {
          pv[cc] = G[cc] * kf[0];
#pragma unroll
          for (int i = 1; i < 4; ++i) pv[cc] = fmaf(G[4 * i + cc], kf[i], pv[cc]);
        }
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
          for (int cc = 0; cc < 4; ++cc) G[4 * i + cc] = fmaf(wf[i], G[4 * i + cc], rf[i] * gf[cc]);
        const float x = butterfly8(xk, xw, lane);
        if ((lane & 1) == 0) {
          const size_t o = tok_off(p, bb, h, t0 + t) + dr;
          if (lane & 2)
            p.gomega[o] = x * S.om[t][dr];
          else
            p.gk[o] = __float2bfloat16_rn(fmaf(sm.uu[dr] * bf(S.r[t][dr]), sm.vg[t], x));
        }
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) pv[cc] += __shfl_xor_sync(0xffffffffu, pv[cc], 16);
        if (lane < 16) *reinterpret_cast<float4*>(&sm.red[m][warp][j0]) = make_float4(pv[0], pv[1], pv[2], pv[3]);
      }
    }
    __syncthreads();
#pragma unroll
    for (int h2 = 0; h2 < 2; ++h2) {  // kS tokens x 64 values: two per thread
      const int m = 4 * h2 + (tid >> 6), j = tid & 63, t = tb + m;
      if (t < cnt) {
        float a = (sm.red[m][0][j] + sm.red[m][1][j]) + (sm.red[m][2][j] + sm.red[m][3][j]);
        a += (sm.red[m][4][j] + sm.red[m][5][j]) + (sm.red[m][6][j] + sm.red[m][7][j]);
        p.gv[tok_off(p, bb, h, t0 + t) + j] = __float2bfloat16_rn(fmaf(sm.ruk[t], bf(S.g[t][j]), a));
      }
    }
    __syncthreads();
  }
}

// gu[h][d] = Σ_b Σ_c part[b][h][c][d] in batch and chunk order (deterministic).
__global__ void wkv6_bwd_reduce_kernel(int B, int H, int nch, const float* __restrict__ part, float* __restrict__ gu) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= H * kN) return;
  const int h = i / kN, d = i % kN;
  double su = 0.0;
  for (int bb = 0; bb < B; ++bb)
    for (int c = 0; c < nch; ++c) su += (double)part[(((size_t)bb * H + h) * nch + c) * kN + d];
  gu[i] = (float)su;
}

}  // namespace

size_t wkv6_bwd_block_floats(int B, int T, int H) { return (size_t)B * H * ((T + kL - 1) / kL) * kN * kN; }
size_t wkv6_bwd_row_floats(int B, int T, int H) { return (size_t)B * H * ((T + kL - 1) / kL) * kN; }

cudaError_t launch_wkv6_bwd(const Wkv6BwdParams& p, cudaStream_t st) {
  const int nch = (p.T + kL - 1) / kL;
  const unsigned nblk = (unsigned)((size_t)p.B * p.H * nch);
  static unsigned mask_s = 0, mask_c = 0;
  cudaError_t e = ensure_smem_attr(reinterpret_cast<const void*>(wkv6_bwd_sums_kernel), (int)sizeof(SumsSmem), &mask_s);
  if (e != cudaSuccess) return e;
  e = ensure_smem_attr(reinterpret_cast<const void*>(wkv6_bwd_chunk_kernel), (int)sizeof(ChunkSmem), &mask_c);
  if (e != cudaSuccess) return e;
  wkv6_bwd_sums_kernel<<<nblk, kThreads, sizeof(SumsSmem), st>>>(p);
  wkv6_bwd_carry_kernel<<<(unsigned)(2LL * p.B * p.H), kThreads, 0, st>>>(p);
  wkv6_bwd_chunk_kernel<<<nblk, kThreads, sizeof(ChunkSmem), st>>>(p);
  wkv6_bwd_reduce_kernel<<<(p.H * kN + 127) / 128, 128, 0, st>>>(p.B, p.H, nch, p.part, p.gu);
  return cudaGetLastError();
}

}  // namespace rwkv
