// Eagle / RWKV-5 recurrent decode step (sm_100a): one token for each of B
// independent streams, all heads at once.
//
// "RWKV-5 Eagle과 RWKV-6 Finch", section Eagle: per head, with the state s
// indexed (key i, value j),
//   y_j   = Σ_i r_i (s_ij + u_i k_i v_j) = Σ_i r_i s_ij + (Σ_i r_i u_i k_i) v_j,
//   s'_ij = w_i s_ij + k_i v_j,   w_i = exp(-exp(ω_i)),
// the one-token case of the forward.  The same kernel is the Finch / RWKV-6
// decode step (section Finch: the decay becomes data dependent), where ω is
// one [H, N] vector per stream, the current token's.
//
// The step is a pass over the fp32 state (16 KB per head, read once and
// written once); everything else is 64-element vectors.  One CTA of 256
// threads per (b, h): thread t owns rows 4 (t/16) .. +3 and columns
// 4 (t%16) .. +3 of the head's state, loads and stores them as float4 (a warp
// covers two 256-byte row segments per instruction), forms its partial y over
// its four rows, and the CTA sums the 16 row groups of every column.  s_in and
// s_out may be the same array: each element is read before it is written, by
// the same thread.
#include "launch.h"
#include "wkv_common.cuh"

namespace rwkv {
namespace {

constexpr int kN = 64;
constexpr int kThreads = 256;

__global__ void __launch_bounds__(kThreads) wkv5_step_kernel(Wkv5StepParams p) {
  __shared__ float sr[kN], sk[kN], sv[kN], sw[kN];
  __shared__ float part[kThreads / 16][kN];  // partial y_j per group of four rows
  __shared__ float bonus;
  const int tid = threadIdx.x;
  const int bh = blockIdx.x;  // b * H + h
  const int h = bh % p.H;
  const size_t tok = (size_t)bh * kN;  // [B,H,N]: this stream's token for head h

  if (tid < kN) {
    sr[tid] = __bfloat162float(p.r[tok + tid]);
    sk[tid] = __bfloat162float(p.k[tok + tid]);
    sv[tid] = __bfloat162float(p.v[tok + tid]);
    sw[tid] = expf(-expf(p.omega[(p.omega_per_stream ? tok : (size_t)h * kN) + tid]));
  }
  __syncthreads();
  if (tid < 32) {  // Σ_i r_i u_i k_i
    const float* u = p.u + h * kN;
    float x = fmaf(sr[tid] * u[tid], sk[tid], sr[tid + 32] * u[tid + 32] * sk[tid + 32]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    if (tid == 0) bonus = x;
  }

  const int j0 = 4 * (tid & 15), i0 = 4 * (tid >> 4);
  const size_t sb = (size_t)bh * kN * kN + (size_t)i0 * kN + j0;
  float4 s[4];
#pragma unroll
  for (int a = 0; a < 4; ++a)
    s[a] = p.s_in ? *reinterpret_cast<const float4*>(p.s_in + sb + (size_t)a * kN) : make_float4(0.f, 0.f, 0.f, 0.f);
  float4 yp = make_float4(0.f, 0.f, 0.f, 0.f);
  const float4 vj = make_float4(sv[j0], sv[j0 + 1], sv[j0 + 2], sv[j0 + 3]);
#pragma unroll
  for (int a = 0; a < 4; ++a) {
    const float ri = sr[i0 + a], wi = sw[i0 + a], ki = sk[i0 + a];
    yp.x = fmaf(ri, s[a].x, yp.x);
    yp.y = fmaf(ri, s[a].y, yp.y);
    yp.z = fmaf(ri, s[a].z, yp.z);
    yp.w = fmaf(ri, s[a].w, yp.w);
    const float4 o = make_float4(fmaf(wi, s[a].x, ki * vj.x), fmaf(wi, s[a].y, ki * vj.y),
                                 fmaf(wi, s[a].z, ki * vj.z), fmaf(wi, s[a].w, ki * vj.w));
    *reinterpret_cast<float4*>(p.s_out + sb + (size_t)a * kN) = o;
  }
  *reinterpret_cast<float4*>(&part[tid >> 4][j0]) = yp;
  __syncthreads();
  if (tid < kN) {
    float y = 0.f;
#pragma unroll
    for (int g = 0; g < kThreads / 16; ++g) y += part[g][tid];
    p.y[tok + tid] = __float2bfloat16_rn(fmaf(bonus, sv[tid], y));
  }
}

}  // namespace

cudaError_t launch_wkv5_step(const Wkv5StepParams& p, cudaStream_t st) {
  wkv5_step_kernel<<<(unsigned)(p.B * p.H), kThreads, 0, st>>>(p);
  return cudaGetLastError();
}

}  // namespace rwkv
