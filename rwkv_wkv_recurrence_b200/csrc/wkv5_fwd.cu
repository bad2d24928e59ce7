// Eagle / RWKV-5 multi-head matrix-state WKV forward (sm_100a), recurrent
// form on CUDA cores.
//
// "RWKV-5 Eagle과 RWKV-6 Finch", section Eagle: per head,
//   s' = diag(w) s + kᵀ v,   wkv' = s + diag(u) kᵀ v,   w = exp(-exp(ω)),
// and the receptance reads the state like a query: y_t = r_t (s + diag(u) k_tᵀ v_t),
// with s[i][j] indexed (key i, value j) as in the RWKV-7 page's update
// kv[d,e] = k_d v_e, out_e = Σ_d r_d state[d,e].
//
// Shape: one CTA of N = 64 threads per (batch, head); thread j owns value
// column j of the fp32 state (64 registers).  Tokens are staged 32 at a time
// in shared memory (converted to fp32 once), so r and k are read as
// broadcasts.  Columns never interact, so the only per-token dependency is the
// thread's own column.
#include "launch.h"
#include "wkv_common.cuh"

namespace rwkv {
namespace {

constexpr int kN = 64;
constexpr int kTok = 32;

__global__ void __launch_bounds__(kN) wkv5_fwd_recurrent_kernel(int B, int T, int H,
                                                                const __nv_bfloat16* __restrict__ r,
                                                                const __nv_bfloat16* __restrict__ k,
                                                                const __nv_bfloat16* __restrict__ v,
                                                                const float* __restrict__ omega,
                                                                const float* __restrict__ u,
                                                                __nv_bfloat16* __restrict__ y,
                                                                const float* s_in, float* s_out) {
  __shared__ float rs[kTok][kN];
  __shared__ float ks[kTok][kN];
  __shared__ float vs[kTok][kN];
  __shared__ float bonus[kTok];
  __shared__ float wd[kN];
  __shared__ float ud[kN];

  const int j = threadIdx.x;
  const int bh = blockIdx.x;
  const int b = bh / H, h = bh % H;
  wd[j] = expf(-expf(omega[h * kN + j]));
  ud[j] = u[h * kN + j];

  float s[kN];
  const size_t sbase = (size_t)bh * kN * kN;
#pragma unroll
  for (int i = 0; i < kN; ++i) s[i] = s_in ? s_in[sbase + (size_t)i * kN + j] : 0.f;

  for (int t0 = 0; t0 < T; t0 += kTok) {
    const int cnt = min(kTok, T - t0);
    __syncthreads();
    for (int tt = 0; tt < cnt; ++tt) {
      const size_t off = (((size_t)b * T + t0 + tt) * H + h) * kN + j;
      rs[tt][j] = __bfloat162float(r[off]);
      ks[tt][j] = __bfloat162float(k[off]);
      vs[tt][j] = __bfloat162float(v[off]);
    }
    __syncthreads();
    if (j < cnt) {
      float acc = 0.f;
      for (int i = 0; i < kN; ++i) acc = fmaf(rs[j][i] * ud[i], ks[j][i], acc);
      bonus[j] = acc;
    }
    __syncthreads();
    for (int tt = 0; tt < cnt; ++tt) {
      const float vj = vs[tt][j];
      float acc = bonus[tt] * vj;
#pragma unroll
      for (int i = 0; i < kN; ++i) acc = fmaf(rs[tt][i], s[i], acc);
#pragma unroll
      for (int i = 0; i < kN; ++i) s[i] = fmaf(wd[i], s[i], ks[tt][i] * vj);
      y[(((size_t)b * T + t0 + tt) * H + h) * kN + j] = __float2bfloat16_rn(acc);
    }
  }
  if (s_out != nullptr) {
    __syncthreads();  // s_out may alias s_in: every thread has read its column above
#pragma unroll
    for (int i = 0; i < kN; ++i) s_out[sbase + (size_t)i * kN + j] = s[i];
  }
}

}  // namespace

cudaError_t launch_wkv5_fwd(int B, int T, int H, const void* r, const void* k, const void* v, const float* omega,
                            const float* u, void* y, const float* s_in, float* s_out, cudaStream_t st) {
  const unsigned grid = (unsigned)(B * H);
  wkv5_fwd_recurrent_kernel<<<grid, kN, 0, st>>>(B, T, H, static_cast<const __nv_bfloat16*>(r),
                                                  static_cast<const __nv_bfloat16*>(k),
                                                  static_cast<const __nv_bfloat16*>(v), omega, u,
                                                  static_cast<__nv_bfloat16*>(y), s_in, s_out);
  return cudaGetLastError();
}

}  // namespace rwkv
