// RWKV-4 WKV recurrent decode step (sm_100a): one token for every lane.
//
// "RWKV - Transformer 시대에 RNN을 재발명하다", Method / (2) Time-mixing (WKV),
// recurrent form: WKV_t = (a_{t-1} + e^{u+k_t} v_t) / (b_{t-1} + e^{u+k_t}),
// a_t = e^{-w} a_{t-1} + e^{k_t} v_t, b_t = e^{-w} b_{t-1} + e^{k_t}; O(d) state
// per stream, constant work per token.  Pure streaming: 12 B of state in, 12 B
// out, k, v in and y out per lane, four lanes per thread with 16-byte accesses.
#include "launch.h"
#include "wkv_common.cuh"

namespace rwkv {
namespace {

template <typename T, int V>
struct Vec;
template <>
struct Vec<float, 4> {
  using type = float4;
};
template <>
struct Vec<float, 1> {
  using type = float;
};

template <typename T, int V>
__global__ void __launch_bounds__(256) wkv4_step_kernel(int B, int C, const float* __restrict__ w,
                                                        const float* __restrict__ u, const T* __restrict__ k,
                                                        const T* __restrict__ v, T* __restrict__ y,
                                                        const float* state_in, float* state_out) {
  // state_in may alias state_out: each thread reads its lanes before writing them.
  const size_t plane = (size_t)B * C;
  const size_t i0 = ((size_t)blockIdx.x * blockDim.x + threadIdx.x) * V;
  if (i0 >= plane) return;
  float a[V], b[V], pe[V], kk[V], vv[V], yy[V];
  if constexpr (V == 4 && sizeof(T) == 4) {
    const float4 a4 = *reinterpret_cast<const float4*>(state_in + i0);
    const float4 b4 = *reinterpret_cast<const float4*>(state_in + plane + i0);
    const float4 p4 = *reinterpret_cast<const float4*>(state_in + 2 * plane + i0);
    const float4 k4 = *reinterpret_cast<const float4*>(k + i0);
    const float4 v4 = *reinterpret_cast<const float4*>(v + i0);
    a[0] = a4.x; a[1] = a4.y; a[2] = a4.z; a[3] = a4.w;
    b[0] = b4.x; b[1] = b4.y; b[2] = b4.z; b[3] = b4.w;
    pe[0] = p4.x; pe[1] = p4.y; pe[2] = p4.z; pe[3] = p4.w;
    kk[0] = k4.x; kk[1] = k4.y; kk[2] = k4.z; kk[3] = k4.w;
    vv[0] = v4.x; vv[1] = v4.y; vv[2] = v4.z; vv[3] = v4.w;
  } else {
#pragma unroll
    for (int j = 0; j < V; ++j) {
      if (i0 + j < plane) {
        a[j] = state_in ? state_in[i0 + j] : 0.f;
        b[j] = state_in ? state_in[plane + i0 + j] : 0.f;
        pe[j] = state_in ? state_in[2 * plane + i0 + j] : 0.f;
        kk[j] = IO<T>::load(k + i0 + j);
        vv[j] = IO<T>::load(v + i0 + j);
      }
    }
  }
#pragma unroll
  for (int j = 0; j < V; ++j) {
    if (i0 + j < plane) {
      const int c = (int)((i0 + j) % C);
      const Lane4 L = lane4_step_consts(w[c], u[c]);
      wkv4_snap(a[j], b[j], pe[j]);
      yy[j] = wkv4_step_careful(a[j], b[j], pe[j], kk[j], vv[j], L);
    }
  }
  if constexpr (V == 4 && sizeof(T) == 4) {
    *reinterpret_cast<float4*>(y + i0) = make_float4(yy[0], yy[1], yy[2], yy[3]);
    *reinterpret_cast<float4*>(state_out + i0) = make_float4(a[0], a[1], a[2], a[3]);
    *reinterpret_cast<float4*>(state_out + plane + i0) = make_float4(b[0], b[1], b[2], b[3]);
    *reinterpret_cast<float4*>(state_out + 2 * plane + i0) = make_float4(pe[0], pe[1], pe[2], pe[3]);
  } else {
#pragma unroll
    for (int j = 0; j < V; ++j) {
      if (i0 + j < plane) {
        y[i0 + j] = IO<T>::from_f(yy[j]);
        state_out[i0 + j] = a[j];
        state_out[plane + i0 + j] = b[j];
        state_out[2 * plane + i0 + j] = pe[j];
      }
    }
  }
}

__global__ void copy_state_kernel(size_t n, const float* __restrict__ in, float* __restrict__ out) {
  const size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) out[i] = in ? in[i] : 0.f;
}

template <typename T, int V>
cudaError_t step_launch(int B, int C, const float* w, const float* u, const void* k, const void* v, void* y,
                        const float* si, float* so, cudaStream_t st) {
  const size_t lanes = (size_t)B * C;
  const size_t threads = (lanes + V - 1) / V;
  const unsigned grid = (unsigned)((threads + 255) / 256);
  wkv4_step_kernel<T, V><<<grid, 256, 0, st>>>(B, C, w, u, static_cast<const T*>(k), static_cast<const T*>(v),
                                               static_cast<T*>(y), si, so);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_wkv4_step(bool bf16, int B, int C, const float* w, const float* u, const void* k, const void* v,
                             void* y, const float* state_in, float* state_out, bool vec4, cudaStream_t st) {
  if (bf16) return step_launch<__nv_bfloat16, 1>(B, C, w, u, k, v, y, state_in, state_out, st);
  if (vec4 && state_in != nullptr) return step_launch<float, 4>(B, C, w, u, k, v, y, state_in, state_out, st);
  return step_launch<float, 1>(B, C, w, u, k, v, y, state_in, state_out, st);
}

cudaError_t launch_copy_state(int B, int C, const float* state_in, float* state_out, cudaStream_t st) {
  const size_t n = (size_t)3 * B * C;
  copy_state_kernel<<<(unsigned)((n + 255) / 256), 256, 0, st>>>(n, state_in, state_out);
  return cudaGetLastError();
}

cudaError_t ensure_smem_attr(const void* func, int bytes, unsigned* device_mask) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (bytes > 227 * 1024) return cudaErrorInvalidValue;
  const unsigned bit = 1u << (dev & 31);
  if (__atomic_load_n(device_mask, __ATOMIC_ACQUIRE) & bit) return cudaSuccess;
  e = cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024);
  if (e != cudaSuccess) return e;
  __atomic_fetch_or(device_mask, bit, __ATOMIC_ACQ_REL);
  return cudaSuccess;
}

}  // namespace rwkv
