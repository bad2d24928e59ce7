// Per-chunk WKV recurrence on the CUDA cores (sm_100a), used by the Finch
// tensor-core kernel for chunks whose decay is too fast for its chunked
// factorization (some channel's decay leaves the fp32 range there).
//
// "RWKV-5 Eagle과 RWKV-6 Finch", sections Eagle and Finch: per token t of the
// chunk, with the state s[d][j] (key d, value j) entering the chunk,
//   y_t[j] = Σ_d r_t[d] (s[d][j] + u_d k_t[d] v_t[j]),
//   s[d][j] <- w_t[d] s[d][j] + k_t[d] v_t[j],
// w_t the decay of token t (constant per channel for Eagle).  This is the
// recurrence itself, token by token, in fp32: it needs no factorization, so it
// holds for any decay in [0, 1].
//
// Work split: thread t owns the 4 x 4 state block of keys 4 kg .. 4 kg + 3
// (kg = t / 16) and values 4 cg .. 4 cg + 3 (cg = t % 16).  Per token it reads
// 4 r, 4 k, 4 v (and 4 w) from shared memory, forms its part of y for its 4
// values (16 FMAs), updates its block (32 operations), and the two key groups
// of a warp add their parts with one shuffle.  The 8 warps' parts of 8 tokens
// meet in shared memory and one pass adds them, with the bonus term, into the
// output rows: two barriers per 8 tokens.  A batch of 8 tokens is one 8-row
// group of the swizzled boxes, so every address is a fixed per-thread offset.  The state enters and leaves in the
// tensor-core kernels' fragment layout (rows drow, drow + 8, columns
// jcol + 4 q) through a padded shared-memory copy.
#pragma once

#include <cuda_bf16.h>

#include <cstddef>
#include <cstdint>

#include "wkv_common.cuh"

namespace rwkv {
namespace recur {

constexpr int kN = 64;
constexpr int kTB = 8;            // tokens per reduction batch (one box row group: the swizzle phase is fixed)
constexpr int kPad = 68;          // row stride (floats) of the state copy: conflict-free both ways
constexpr int kScratchFloats = kN * kPad;
constexpr int kRedFloats = kTB * 8 * kN;  // one batch of [token][warp][value] parts

struct Frag16 {
  float v[16];
};

// Byte offset of (box row, channel d) in a [64 x 64] bf16 box with the 128-byte swizzle.
__device__ __forceinline__ uint32_t box_off(int row, int d) {
  return (uint32_t)row * 128u + ((uint32_t)((d >> 3) ^ (row & 7)) << 4) + (uint32_t)(d & 7) * 2u;
}

// Four consecutive bf16 (channels d .. d + 3, d % 4 == 0) at byte offset `off` of a box, as fp32.
__device__ __forceinline__ void ld_bf16x4(const unsigned char* box, uint32_t off, float (&f)[4]) {
  const uint2 x = *reinterpret_cast<const uint2*>(box + off);
  f[0] = __uint_as_float(x.x << 16);
  f[1] = __uint_as_float(x.x & 0xFFFF0000u);
  f[2] = __uint_as_float(x.y << 16);
  f[3] = __uint_as_float(x.y & 0xFFFF0000u);
}

__device__ __forceinline__ float ld_bf16(const unsigned char* box, uint32_t off) {
  return __uint_as_float((uint32_t)(*reinterpret_cast<const unsigned short*>(box + off)) << 16);
}

struct ChunkArgs {
  const unsigned char *rawR, *rawK, *rawV;  // the r, k, v boxes in shared memory (token rows, 128-byte swizzle)
  const float* wconst;        // shared [64]: per-key decay w (Eagle), or nullptr
  const float* wtok;          // shared [64 tokens][64 keys]: per-token decay (Finch), or nullptr
  const float* u;             // [64] bonus u of this head (global or shared)
  float* scratch;             // shared, kScratchFloats: the state copy
  float* red;                 // shared, kRedFloats: the per-warp output parts
  float* bonus;               // shared [64]: Σ_d r u k per token
  __nv_bfloat16* y;           // output rows: token t at y + t * ystride (value j at + j)
  size_t ystride;
  int cnt;                    // tokens in the chunk
  int drow, jcol;             // the caller's fragment coordinates
};

// Runs the chunk's `cnt` tokens.  Token τ of the pass reads box row REV ? 63 - τ : τ and writes
// output row `yrow(τ)` = REV ? -τ : τ relative to `y` (the caller points y at the pass's first
// token).  All 256 threads call it; it returns the updated fragment.  Inlined, so that the
// arguments stay in registers and the compiler sees the shared-memory address space.
template <bool REV>
__device__ __forceinline__ Frag16 chunk_recur(Frag16 S, const ChunkArgs a) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int cg = tid & 15, kg = tid >> 4;
  const int d0 = 4 * kg, j0 = 4 * cg;

  // the bonus of every token: Σ_d r u k over the four key quarters of 16 keys
  {
    const int tau = tid >> 2, kq = tid & 3;
    const int row = REV ? kN - 1 - tau : tau;
    float part = 0.f;
    if (tau < a.cnt) {
#pragma unroll
      for (int g = 0; g < 4; ++g) {
        float rv[4], kv[4];
        ld_bf16x4(a.rawR, box_off(row, 16 * kq + 4 * g), rv);
        ld_bf16x4(a.rawK, box_off(row, 16 * kq + 4 * g), kv);
#pragma unroll
        for (int i = 0; i < 4; ++i) part = fmaf(rv[i] * a.u[16 * kq + 4 * g + i], kv[i], part);
      }
    }
    part += __shfl_xor_sync(0xffffffffu, part, 1);
    part += __shfl_xor_sync(0xffffffffu, part, 2);
    if (kq == 0) a.bonus[tau] = part;
  }
  // the state into the block layout
#pragma unroll
  for (int q = 0; q < 8; ++q)
#pragma unroll
    for (int r = 0; r < 2; ++r) a.scratch[(a.drow + 8 * r) * kPad + a.jcol + 4 * q] = S.v[2 * q + r];
  __syncthreads();
  float s[4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float4 x = *reinterpret_cast<const float4*>(&a.scratch[(d0 + i) * kPad + j0]);
    s[i][0] = x.x;
    s[i][1] = x.y;
    s[i][2] = x.z;
    s[i][3] = x.w;
  }
  float wk[4] = {1.f, 1.f, 1.f, 1.f};
  if (a.wconst != nullptr) {
#pragma unroll
    for (int i = 0; i < 4; ++i) wk[i] = a.wconst[d0 + i];
  }

  // per-thread byte offsets of this thread's keys and values in row e of an 8-row group (the
  // swizzle XORs the 16-byte chunk index with the row's low three bits)
  uint32_t offk[kTB], offv[kTB];
#pragma unroll
  for (int e = 0; e < kTB; ++e) {
    const int ph = REV ? 7 - e : e;
    offk[e] = ((uint32_t)((d0 >> 3) ^ ph) << 4) + (uint32_t)(d0 & 7) * 2u;
    offv[e] = ((uint32_t)((j0 >> 3) ^ ph) << 4) + (uint32_t)(j0 & 7) * 2u;
  }
  for (int t0 = 0; t0 < a.cnt; t0 += kTB) {
#pragma unroll
    for (int e = 0; e < kTB; ++e) {
      const int tau = t0 + e;
      if (tau < a.cnt) {
        const uint32_t rowb = (uint32_t)(REV ? kN - 1 - tau : tau) * 128u;
        float rv[4], kv[4], vv[4];
        ld_bf16x4(a.rawR, rowb + offk[e], rv);
        ld_bf16x4(a.rawK, rowb + offk[e], kv);
        ld_bf16x4(a.rawV, rowb + offv[e], vv);
        if (a.wtok != nullptr) {
          const float4 w4 = *reinterpret_cast<const float4*>(&a.wtok[tau * kN + d0]);
          wk[0] = w4.x;
          wk[1] = w4.y;
          wk[2] = w4.z;
          wk[3] = w4.w;
        }
        float part[4];
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          part[c] = rv[0] * s[0][c];
#pragma unroll
          for (int i = 1; i < 4; ++i) part[c] = fmaf(rv[i], s[i][c], part[c]);
        }
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
          for (int c = 0; c < 4; ++c) s[i][c] = fmaf(wk[i], s[i][c], kv[i] * vv[c]);
#pragma unroll
        for (int c = 0; c < 4; ++c) part[c] += __shfl_xor_sync(0xffffffffu, part[c], 16);
        if (lane < 16)
          *reinterpret_cast<float4*>(&a.red[(e * 8 + warp) * kN + j0]) =
              make_float4(part[0], part[1], part[2], part[3]);
      }
    }
    __syncthreads();
#pragma unroll
    for (int h2 = 0; h2 < 2; ++h2) {  // 8 tokens x 64 values: two per thread
      const int e = 4 * h2 + (tid >> 6), j = tid & 63, tau = t0 + e;
      if (tau < a.cnt) {
        const float* pr = a.red + e * 8 * kN + j;
        float yv = (pr[0] + pr[kN]) + (pr[2 * kN] + pr[3 * kN]);
        yv += (pr[4 * kN] + pr[5 * kN]) + (pr[6 * kN] + pr[7 * kN]);
        const int row = REV ? kN - 1 - tau : tau;
        yv = fmaf(a.bonus[tau], ld_bf16(a.rawV, box_off(row, j)), yv);
        const ptrdiff_t yrow = REV ? -(ptrdiff_t)tau : (ptrdiff_t)tau;
        a.y[yrow * (ptrdiff_t)a.ystride + j] = __float2bfloat16_rn(yv);
      }
    }
    __syncthreads();
  }

  // the state back into the fragment layout
#pragma unroll
  for (int i = 0; i < 4; ++i)
    *reinterpret_cast<float4*>(&a.scratch[(d0 + i) * kPad + j0]) = make_float4(s[i][0], s[i][1], s[i][2], s[i][3]);
  __syncthreads();
#pragma unroll
  for (int q = 0; q < 8; ++q)
#pragma unroll
    for (int r = 0; r < 2; ++r) S.v[2 * q + r] = a.scratch[(a.drow + 8 * r) * kPad + a.jcol + 4 * q];
  __syncthreads();
  return S;
}

}  // namespace recur
}  // namespace rwkv
