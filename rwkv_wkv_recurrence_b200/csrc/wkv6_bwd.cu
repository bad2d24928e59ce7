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
// One CTA of 256 threads per (batch row, head); thread t owns the 4 x 4 block of keys
// 4 (t / 16) .. + 3 and values 4 (t % 16) .. + 3 of both the state s and its gradient G.
//   1. Forward in time over 64-token chunks: gr_t (the state read with gy_t in place of r_t, summed
//      over the 16 value groups of a half-warp by a shuffle butterfly), and the state at every
//      chunk start, written to the workspace.
//   2. Backward in time, chunk by chunk: the chunk's states are recomputed from its checkpoint and
//      written every 8 tokens to a per-CTA scratch (L2-resident); each 8-token sub-chunk then
//      recomputes its 8 states into registers and walks them backwards with G, forming gk and the
//      gω row sums (one butterfly over 8 values) and gv (a shuffle across the warp's two key groups,
//      then the 8 warps' parts meet in shared memory).
// Inputs of a chunk (r, k, v, gy, ω: 48 KB) arrive by cp.async into one of two shared-memory
// stages while the chunk before is processed; outputs are staged in shared memory and leave as
// 16-byte rows.  gu is summed per (batch row, head, key) in fp64 and reduced over the batch in
// fixed order by a second kernel, so the results are deterministic.
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
  float om[kL][kN];
};

struct __align__(16) Smem {
  Stage st[2];
  float w[kL][kN];                  // w_t[d] of the chunk
  float red[kS][kWarps][kN];        // gv parts of a sub-chunk: [token][warp][value]
  __nv_bfloat16 o0[kL][kN];         // staged gr (forward pass) or gk (backward pass)
  __nv_bfloat16 o1[kL][kN];         // staged gv
  float ogw[kL][kN];                // staged gω
  float vg[kL];                     // v_t · gy_t
  float ruk[kL];                    // Σ_d r_t[d] u_d k_t[d]
  float uu[kN];
};

__device__ __forceinline__ void cp_async16(void* dst, const void* src, bool full) {
  const uint32_t d = (uint32_t)__cvta_generic_to_shared(dst);
  // src-size 0 fills the 16 bytes with zeros (rows past the end of the sequence)
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(d), "l"(src), "r"(full ? 16 : 0) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

__device__ __forceinline__ void bf16x4(const __nv_bfloat16* p, float (&f)[4]) {
  const uint2 x = *reinterpret_cast<const uint2*>(p);
  f[0] = __uint_as_float(x.x << 16);
  f[1] = __uint_as_float(x.x & 0xFFFF0000u);
  f[2] = __uint_as_float(x.y << 16);
  f[3] = __uint_as_float(x.y & 0xFFFF0000u);
}

__device__ __forceinline__ float bf(const __nv_bfloat16 x) { return __bfloat162float(x); }

// The chunk of tokens [t0, t0 + cnt) of (bb, h) into a stage; rows past cnt are zero.
// With `with_r` false the r rows are not fetched (the forward pass does not read them).
__device__ __forceinline__ void stage_chunk(Stage& S, const Wkv6BwdParams& p, int bb, int h, int t0, int cnt,
                                            bool with_r) {
  const int tid = threadIdx.x;
  const size_t rs = (size_t)p.H * kN;  // elements from one token to the next
  const size_t base = ((size_t)bb * p.T + t0) * rs + (size_t)h * kN;
#pragma unroll
  for (int i = tid; i < kL * 8; i += kThreads) {  // bf16 rows: 8 pieces of 16 bytes
    const int row = i >> 3, pc = (i & 7) * 8;
    const bool ok = row < cnt;
    const size_t off = base + (size_t)(ok ? row : 0) * rs + pc;
    if (with_r) cp_async16(&S.r[row][pc], p.r + off, ok);
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
}

// Per-chunk tables: w_t[d] from ω, v_t·gy_t and (with_ruk) Σ_d r_t u k_t.
__device__ __forceinline__ void chunk_tables(Smem& sm, const Stage& S, bool with_ruk) {
  const int tid = threadIdx.x;
#pragma unroll 4
  for (int i = tid; i < kL * kN; i += kThreads) {
    const int t = i >> 6, d = i & 63;
    sm.w[t][d] = expf(-expf(S.om[t][d]));
  }
  // token t = tid / 4, quarter q = tid % 4 of the channels
  const int t = tid >> 2, q = tid & 3;
  float a = 0.f, b = 0.f;
#pragma unroll
  for (int g = 0; g < 4; ++g) {
    const int c0 = 16 * q + 4 * g;
    float vf[4], gf[4], rf[4], kf[4];
    bf16x4(&S.v[t][c0], vf);
    bf16x4(&S.g[t][c0], gf);
#pragma unroll
    for (int i = 0; i < 4; ++i) a = fmaf(vf[i], gf[i], a);
    if (with_ruk) {
      bf16x4(&S.r[t][c0], rf);
      bf16x4(&S.k[t][c0], kf);
#pragma unroll
      for (int i = 0; i < 4; ++i) b = fmaf(rf[i] * sm.uu[c0 + i], kf[i], b);
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

// Staged [cnt][64] rows to the [B,T,H,64] tensor at token t0 of (bb, h), 16 bytes per store.
__device__ __forceinline__ void store_rows_bf16(const __nv_bfloat16 (*src)[kN], __nv_bfloat16* dst,
                                                const Wkv6BwdParams& p, int bb, int h, int t0, int cnt) {
  const size_t rs = (size_t)p.H * kN;
  const size_t base = ((size_t)bb * p.T + t0) * rs + (size_t)h * kN;
  for (int i = threadIdx.x; i < cnt * 8; i += kThreads) {
    const int row = i >> 3, pc = (i & 7) * 8;
    *reinterpret_cast<uint4*>(dst + base + (size_t)row * rs + pc) = *reinterpret_cast<const uint4*>(&src[row][pc]);
  }
}

__device__ __forceinline__ void store_rows_f32(const float (*src)[kN], float* dst, const Wkv6BwdParams& p, int bb,
                                               int h, int t0, int cnt) {
  const size_t rs = (size_t)p.H * kN;
  const size_t base = ((size_t)bb * p.T + t0) * rs + (size_t)h * kN;
  for (int i = threadIdx.x; i < cnt * 16; i += kThreads) {
    const int row = i >> 4, pc = (i & 15) * 4;
    *reinterpret_cast<float4*>(dst + base + (size_t)row * rs + pc) = *reinterpret_cast<const float4*>(&src[row][pc]);
  }
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
// A thread-private copy of the block (scratch laid out [thread][16] so that a warp's accesses are
// contiguous).
__device__ __forceinline__ void save_own(float* m, const float (&s)[kBlock]) {
  float4* q = reinterpret_cast<float4*>(m) + threadIdx.x * 4;
#pragma unroll
  for (int i = 0; i < 4; ++i) q[i] = make_float4(s[4 * i], s[4 * i + 1], s[4 * i + 2], s[4 * i + 3]);
}
__device__ __forceinline__ void load_own(const float* m, float (&s)[kBlock]) {
  const float4* q = reinterpret_cast<const float4*>(m) + threadIdx.x * 4;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float4 x = q[i];
    s[4 * i + 0] = x.x;
    s[4 * i + 1] = x.y;
    s[4 * i + 2] = x.z;
    s[4 * i + 3] = x.w;
  }
}

// One token of the state recurrence on the thread's block: s <- diag(w_t) s + k_tᵀ v_t.
__device__ __forceinline__ void state_step(float (&s)[kBlock], const Stage& S, const Smem& sm, int t, int d0,
                                           int j0) {
  float kf[4], vf[4];
  bf16x4(&S.k[t][d0], kf);
  bf16x4(&S.v[t][j0], vf);
  const float4 w4 = *reinterpret_cast<const float4*>(&sm.w[t][d0]);
  const float wf[4] = {w4.x, w4.y, w4.z, w4.w};
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int c = 0; c < 4; ++c) s[4 * i + c] = fmaf(wf[i], s[4 * i + c], kf[i] * vf[c]);
}

__global__ void __launch_bounds__(kThreads, 1) wkv6_bwd_kernel(const Wkv6BwdParams p) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  Smem& sm = *reinterpret_cast<Smem*>(smem_raw);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int kg = tid >> 4, cg = tid & 15;
  const int d0 = 4 * kg, j0 = 4 * cg;
  const int bh = blockIdx.x;
  const int bb = bh / p.H, h = bh % p.H;
  const int nch = (p.T + kL - 1) / kL;
  const size_t state_off = (size_t)bh * kN * kN;
  float* ck = p.ckpt + (size_t)bh * nch * kN * kN;          // [nch][256 threads][16]
  float* sub = p.sub + (size_t)bh * (kL / kS) * kN * kN;    // [8 sub-chunks][256 threads][16]
  // the lane that holds a butterfly result writes row dr (bits 3, 2 of the lane)
  const int dr = d0 + 2 * ((lane >> 3) & 1) + ((lane >> 2) & 1);

  if (tid < kN) sm.uu[tid] = p.u[h * kN + tid];

  // 1. forward in time: gr and the chunk-start states
  float s[kBlock];
  if (p.s_in != nullptr)
    load_block(p.s_in + state_off, d0, j0, s);
  else
#pragma unroll
    for (int e = 0; e < kBlock; ++e) s[e] = 0.f;

  stage_chunk(sm.st[0], p, bb, h, 0, min(kL, p.T), false);
  for (int c = 0; c < nch; ++c) {
    const int t0 = c * kL, cnt = min(kL, p.T - t0);
    if (c + 1 < nch) {
      stage_chunk(sm.st[(c + 1) & 1], p, bb, h, t0 + kL, min(kL, p.T - t0 - kL), false);
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();
    const Stage& S = sm.st[c & 1];
    chunk_tables(sm, S, false);
    save_own(ck + (size_t)c * kN * kN, s);
    __syncthreads();
    for (int t = 0; t < cnt; ++t) {
      float gf[4], part[4];
      bf16x4(&S.g[t][j0], gf);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        part[i] = s[4 * i] * gf[0];
#pragma unroll
        for (int cc = 1; cc < 4; ++cc) part[i] = fmaf(s[4 * i + cc], gf[cc], part[i]);
      }
      const float x = butterfly4(part, lane);
      if ((lane & 3) == 0) sm.o0[t][dr] = __float2bfloat16_rn(fmaf(sm.uu[dr] * bf(S.k[t][dr]), sm.vg[t], x));
      state_step(s, S, sm, t, d0, j0);
    }
    __syncthreads();
    store_rows_bf16(sm.o0, p.gr, p, bb, h, t0, cnt);
    // (the next iteration's first barrier orders these reads of o0 before its next writes)
  }
  __syncthreads();

  // 2. backward in time
  float G[kBlock];
  if (p.gs_out != nullptr)
    load_block(p.gs_out + state_off, d0, j0, G);
  else
#pragma unroll
    for (int e = 0; e < kBlock; ++e) G[e] = 0.f;
  double gu_acc = 0.0;

  {
    const int c = nch - 1;
    stage_chunk(sm.st[0], p, bb, h, c * kL, p.T - c * kL, true);
  }
  for (int it = 0; it < nch; ++it) {
    const int c = nch - 1 - it;
    const int t0 = c * kL, cnt = min(kL, p.T - t0);
    if (c >= 1) {
      stage_chunk(sm.st[(it + 1) & 1], p, bb, h, t0 - kL, kL, true);
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();
    const Stage& S = sm.st[it & 1];
    chunk_tables(sm, S, true);
    __syncthreads();
    if (tid < kN) {  // gu: Σ_t r_t[d] k_t[d] (v_t·gy_t), d = tid
      float a = 0.f;
      for (int t = 0; t < cnt; ++t) a = fmaf(bf(S.r[t][tid]) * bf(S.k[t][tid]), sm.vg[t], a);
      gu_acc += (double)a;
    }
    // the chunk's states, every kS tokens, into this CTA's scratch
    {
      float x[kBlock];
      load_own(ck + (size_t)c * kN * kN, x);
      for (int t = 0; t < cnt; ++t) {
        if (t % kS == 0) save_own(sub + (size_t)(t / kS) * kN * kN, x);
        state_step(x, S, sm, t, d0, j0);
      }
    }
    const int nsub = (cnt + kS - 1) / kS;
    for (int sc = nsub - 1; sc >= 0; --sc) {
      const int tb = sc * kS;
      float hs[kS][kBlock];  // hs[m] = s^(tb + m)
      load_own(sub + (size_t)sc * kN * kN, hs[0]);
#pragma unroll
      for (int m = 1; m < kS; ++m) {
#pragma unroll
        for (int e = 0; e < kBlock; ++e) hs[m][e] = hs[m - 1][e];
        if (tb + m - 1 < cnt) state_step(hs[m], S, sm, tb + m - 1, d0, j0);
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
            if (lane & 2)
              sm.ogw[t][dr] = x * -expf(S.om[t][dr] - expf(S.om[t][dr]));  // dw/dω = -e^ω w, finite at w = 0
            else
              sm.o0[t][dr] = __float2bfloat16_rn(fmaf(sm.uu[dr] * bf(S.r[t][dr]), sm.vg[t], x));
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
          sm.o1[t][j] = __float2bfloat16_rn(fmaf(sm.ruk[t], bf(S.g[t][j]), a));
        }
      }
      __syncthreads();
    }
    store_rows_bf16(sm.o0, p.gk, p, bb, h, t0, cnt);
    store_rows_bf16(sm.o1, p.gv, p, bb, h, t0, cnt);
    store_rows_f32(sm.ogw, p.gomega, p, bb, h, t0, cnt);
    __syncthreads();
  }
  if (p.gs_in != nullptr) store_block(p.gs_in + state_off, d0, j0, G);
  if (tid < kN) p.part[(size_t)bh * kN + tid] = gu_acc;
}

// gu[h][d] = Σ_b part[b][h][d] in batch order (deterministic).
__global__ void wkv6_bwd_reduce_kernel(int B, int H, const double* __restrict__ part, float* __restrict__ gu) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= H * kN) return;
  double su = 0.0;
  for (int bb = 0; bb < B; ++bb) su += part[(size_t)bb * H * kN + i];
  gu[i] = (float)su;
}

}  // namespace

size_t wkv6_bwd_ckpt_floats(int B, int T, int H) { return (size_t)B * H * ((T + kL - 1) / kL) * kN * kN; }
size_t wkv6_bwd_sub_floats(int B, int H) { return (size_t)B * H * (kL / kS) * kN * kN; }

cudaError_t launch_wkv6_bwd(const Wkv6BwdParams& p, cudaStream_t st) {
  const size_t smem = sizeof(Smem);
  static unsigned device_mask = 0;
  cudaError_t e = ensure_smem_attr(reinterpret_cast<const void*>(wkv6_bwd_kernel), (int)smem, &device_mask);
  if (e != cudaSuccess) return e;
  wkv6_bwd_kernel<<<(unsigned)(p.B * p.H), kThreads, smem, st>>>(p);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  wkv6_bwd_reduce_kernel<<<(p.H * kN + 127) / 128, 128, 0, st>>>(p.B, p.H, p.part, p.gu);
  return cudaGetLastError();
}

}  // namespace rwkv
