// Finch / RWKV-6 multi-head matrix-state WKV forward with a data-dependent
// (per-token) decay (sm_100a): chunked form on the tcgen05 tensor cores.
//
// "RWKV-5 Eagle과 RWKV-6 Finch", section Finch: the Eagle update with a decay
// that depends on the token,
//   y_t = r_t (s_t + diag(u) k_tᵀ v_t),   s_{t+1} = diag(w_t) s_t + k_tᵀ v_t,
//   w_t = exp(-exp(ω_t)),   ω [B,T,H,N]: one value per token and channel.
//
// Chunked form.  In a chunk of L = 64 tokens that starts at state S, with
// λ_τ = -exp(ω_τ) and the cumulative log-decay Λ_τ = Σ_{σ≤τ} λ_σ (Λ_{-1} = 0),
// token ι < τ reaches token τ multiplied by e^{Λ_{τ-1} - Λ_ι}, so
//   y[τ]   = Σ_d r[τ,d] e^{Λ_{τ-1,d}} S[d,:]
//          + Σ_{ι<τ} A[τ,ι] v[ι,:] + (Σ_d r[τ,d] u_d k[τ,d]) v[τ,:]
//   A[τ,ι] = Σ_d (r[τ,d] e^{Λ_{τ-1,d} - R_d}) (k[ι,d] e^{R_d - Λ_{ι,d}})
//   S'     = e^{Λ_last} ⊙ S + e^{Λ_last - R} ⊙ Σ_ι (k[ι,:] e^{R - Λ_ι})ᵀ v[ι,:]
// with a per-channel reference R and Λ_last the log-decay of the whole chunk.
// With r̃ = r e^{Λ_{τ-1} - R} and k̃ = k e^{R - Λ_ι} the chunk is the Eagle
// kernel's three tensor-core chains
//   [A | Y] = r̃ [k̃ ; e^{R} Sᵀ]ᵀ,   Y += A_masked v,   ΔS = k̃ᵀ v
// (the Eagle kernel is the case Λ_τ = λ (τ + 1), R = Λ_31).  Any R gives the
// same products; every factor stays within e^{±64} while -R and R - Λ_last
// are at most 64 in every channel (wider factors would push small operands
// into the subnormal range, where a tf32 operand keeps few bits).  The first chunk takes R = Λ_31, the middle
// of its own decay; every later chunk takes half the log-decay of the chunk
// before it (the middle again while the decay rate holds), which is known when
// the previous chunk folds its state, so that fold also writes e^{R} ⊙ Sᵀ for
// the next chunk's state read as in the Eagle kernel.  A chunk whose decay
// leaves that range in some channel (a fast decay, or one that jumps) is
// computed by the per-token recurrence on the CUDA cores instead (chunk_recur,
// all 256 threads), on the same state registers.
//
// Decay prologue per chunk: each thread forms λ for 8 tokens x 2 channels
// (ω arrives by TMA as two fp32 [64 tokens x 32 channels] boxes); the
// cumulative sums come from 8-lane shuffle scans, all 16 of a thread's scans
// advancing one shuffle step at a time so that their latencies overlap, plus a
// running carry; the factors are exponentials of differences of those sums, so
// the rounding of the cumulative decay never compounds from chunk to chunk
// beyond one fp32 product per chunk.
//
// CTA: one (batch, head), 8 warps, about 109 KB of shared memory and 256 TMEM
// columns, two CTAs per SM.  The fp32 master state lives in registers in the
// 16x128b fragment of the state-increment accumulator.
#include <cstddef>

#include "launch.h"
#include "tc_common.cuh"
#include "wkv_common.cuh"
#include "wkv_recur.cuh"

namespace rwkv {
namespace {

using namespace tc;

constexpr int kN = 64;                      // head size
constexpr int kL = 64;                      // tokens per chunk
constexpr int kThreads = 256;
constexpr uint32_t kRawBytes = kL * kN * 2;  // one bf16 [64 x 64] box
constexpr uint32_t kOmBytes = kL * 32 * 4;   // one fp32 [64 tokens x 32 channels] box
constexpr float kMaxHalfDecay = 64.f;       // largest log-decay of half a chunk the factorization takes
constexpr uint32_t kTmemCols = 256;         // [scores | output rows], state increment, k̃ᵀ

struct Wkv6Smem {
  alignas(1024) __nv_bfloat16 raw[3][kL * kN];  // r, k, v boxes [token][channel] (128-byte swizzle)
  alignas(1024) float om[2][kL * 32];           // ω, channels 0..31 and 32..63 [token][channel] (128-byte swizzle)
  alignas(128) float opRA[64 * 64];  // r̃ [τ][d] (A of the first product), then the masked scores [τ][ι]
  alignas(128) float opK[64 * 64];   // k̃ [ι][d]: B rows 0..63 of the first product
  alignas(128) float opS[64 * 64];   // e^{R} ⊙ Sᵀ [j][d]: B rows 64..127 of the first product
  alignas(128) float opVt[64 * 64];  // vᵀ [j][ι]: B of A v and of ΔS; reduction scratch of the recurrent path
  float diag_part[8][kL];            // per-warp parts of Σ_d r u k
  float diag[kL];
  float Rv[2][kN];                   // R per channel (the chunk's reference), by chunk parity
  float Lend[2][kN];                 // Λ_last per channel, by chunk parity
  alignas(8) uint64_t bar_tma;
  alignas(8) uint64_t bar_sc;
  alignas(8) uint64_t bar_av;
  alignas(8) uint64_t bar_ds;
  uint32_t tmem_base;
  int abort_flag;
};
static_assert(offsetof(Wkv6Smem, opK) == offsetof(Wkv6Smem, opRA) + 64 * 64 * sizeof(float) &&
                  recur::kScratchFloats <= 2 * 64 * 64 && recur::kRedFloats <= 64 * 64,
              "the recurrent path's state copy spans opRA and opK, its output parts fit opVt");
static_assert(offsetof(Wkv6Smem, opS) == offsetof(Wkv6Smem, opK) + 64 * 64 * sizeof(float),
              "the first product reads k̃ and e^{R} Sᵀ as one 128-row operand");

__device__ __forceinline__ float2 lds_f2(uint32_t addr) {
  float2 v;
  asm volatile("ld.shared.v2.f32 {%0, %1}, [%2];" : "=f"(v.x), "=f"(v.y) : "r"(addr) : "memory");
  return v;
}

__device__ __forceinline__ float lds_f32(uint32_t addr) {
  float v;
  asm volatile("ld.shared.f32 %0, [%1];" : "=f"(v) : "r"(addr) : "memory");
  return v;
}

// Byte offset of (token τ, channel d) in the two fp32 ω boxes with the 128-byte swizzle.
__device__ __forceinline__ uint32_t om_off(int tau, int d) {
  return (uint32_t)(d >> 5) * kOmBytes + (uint32_t)tau * 128u + ((uint32_t)(((d & 31) >> 2) ^ (tau & 7)) << 4) +
         (uint32_t)(d & 3) * 4u;
}

// Reference point of the next chunk's factorization: half of this chunk's log-decay
// (the middle of the chunk if the decay rate stays put), no lower than -79.
__device__ __forceinline__ float next_ref(float lend) { return fmaxf(0.5f * lend, -79.f); }

using recur::Frag16;

__global__ void __launch_bounds__(kThreads, 2) wkv6_fwd_tc_kernel(const __grid_constant__ CUtensorMap mr,
                                                                  const __grid_constant__ CUtensorMap mk,
                                                                  const __grid_constant__ CUtensorMap mv,
                                                                  const __grid_constant__ CUtensorMap mw,
                                                                  Wkv6Params p) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  const uint32_t base_s = smem_u32(smem_raw);
  Wkv6Smem& sm = *reinterpret_cast<Wkv6Smem*>(smem_raw + ((1024u - (base_s & 1023u)) & 1023u));
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int t4 = lane >> 2, tq = lane & 3;
  const int q4 = warp & 3, hc = warp >> 2;
  const int b = blockIdx.x / p.H, h = blockIdx.x % p.H;
  const int nchunk = (p.T + kL - 1) / kL;

  if (tid == 0) sm.abort_flag = 0;
  if (warp == 0) tmem_alloc(&sm.tmem_base, kTmemCols);
  // thread 0 issues every load; with the test hook set it arms the barrier and issues none
  const bool withheld = tid == 0 && loads_withheld(p.ctl);
  if (tid == 0) {
    prefetch_tensormap(&mr);
    prefetch_tensormap(&mk);
    prefetch_tensormap(&mv);
    prefetch_tensormap(&mw);
    mbar_init(&sm.bar_tma, 1);
    mbar_init(&sm.bar_sc, 1);
    mbar_init(&sm.bar_av, 1);
    mbar_init(&sm.bar_ds, 1);
    fence_mbar_init();
    mbar_arrive_expect_tx(&sm.bar_tma, 3 * kRawBytes + 2 * kOmBytes);
    if (!withheld) {
      tma_load_3d(sm.raw[0], &mr, &sm.bar_tma, h * kN, 0, b);
      tma_load_3d(sm.raw[1], &mk, &sm.bar_tma, h * kN, 0, b);
      tma_load_3d(sm.raw[2], &mv, &sm.bar_tma, h * kN, 0, b);
      tma_load_3d(sm.om[0], &mw, &sm.bar_tma, h * kN, 0, b);
      tma_load_3d(sm.om[1], &mw, &sm.bar_tma, h * kN + 32, 0, b);
    }
  }

  // ---- decay prologue and r̃, k̃: warp w owns channels 8w..8w+7; lane holds token rows 8 ib + rr
  // of channels dR, dR + 1.  The 8 lanes of equal rp hold all 64 tokens of their two channels.
  const int rr = lane & 7, rp = lane >> 3;
  const int dR = 8 * warp + 2 * rp;
  const float uA[2] = {p.u[h * kN + dR], p.u[h * kN + dR + 1]};
  const uint32_t offRK = (uint32_t)rr * 128u + (uint32_t)((warp ^ rr) << 4) + (uint32_t)rp * 4u;
  const uint32_t offW = (uint32_t)(warp >> 2) * kOmBytes + (uint32_t)rr * 128u +
                        ((uint32_t)((2 * (warp & 3) + (rp >> 1)) ^ rr) << 4) + (uint32_t)(rp & 1) * 8u;
  const int lrow = lane & 7, lmat = lane >> 3;
  // vᵀ: ldmatrix.trans of block column w; lanes whose bit 1 and bit 4 differ trade with lane ^ 18
  const int sw = ((lane >> 1) ^ (lane >> 4)) & 1;
  const int srow = t4 ^ (sw << 2), stq = tq ^ (sw << 1);
  const uint32_t offT = (uint32_t)(lmat * 8 + lrow) * 128u + (uint32_t)((warp ^ lrow) << 4);

  // ---- state S[d][j] (fp32 master copy), .16x128b fragment: d = 16 q4 + t4 + 8 r, j = 32 hc + 4 q + tq
  const int drow = 16 * q4 + t4;
  const int jcol = 32 * hc + tq;
  const uint32_t tquar = (uint32_t)(32 * q4) << 16;
  const size_t sbase = ((size_t)b * p.H + h) * kN * kN;
  Frag16 S;
#pragma unroll
  for (int q = 0; q < 8; ++q)
#pragma unroll
    for (int r = 0; r < 2; ++r)
      S.v[2 * q + r] = p.s_in ? p.s_in[sbase + (size_t)(drow + 8 * r) * kN + jcol + 4 * q] : 0.f;

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = sm.tmem_base;
  const uint32_t tSc = tbase, tY = tbase + 64, tDS = tbase + 128, tKt = tbase + 192;
  const uint32_t rawR = smem_u32(sm.raw[0]), rawK = smem_u32(sm.raw[1]), rawV = smem_u32(sm.raw[2]);
  const uint32_t omS = smem_u32(sm.om[0]);
  const uint32_t opKs = smem_u32(sm.opK);
  const bool issuer = tid == 0;
  uint32_t nfast = 0;  // chunks done on the tensor cores (phase of the MMA barriers)
  float Rnext[2] = {0.f, 0.f};  // reference of the next chunk: half the log-decay of this one

  int c = 0;
  bool aborted = false;
  for (; c < nchunk; ++c) {
    const int t0 = c * kL;
    const int cnt = min(kL, p.T - t0);
    const int par = c & 1;
    if (!mbar_wait_bounded(&sm.bar_tma, (uint32_t)c & 1u, p.ctl)) sm.abort_flag = 1;

    // T1a: λ, the cumulative log-decay, the reference R and the chunk decay; then r̃, k̃ and the
    // bonus parts.  Rows past the sequence end (zeros from the TMA fill) get λ = 0.
    int bad = 0;
    {
      float lam[8][2], lin[8][2], carry[2] = {0.f, 0.f}, R[2] = {Rnext[0], Rnext[1]};
      // stage-major: the 16 loads and exponentials, then each shuffle step for all 16 values at once
#pragma unroll
      for (int ib = 0; ib < 8; ++ib) {
        const bool live = 8 * ib + rr < cnt;
        const float2 om = lds_f2(omS + offW + ib * 1024u);
        lam[ib][0] = live ? -__expf(om.x) : 0.f;
        lam[ib][1] = live ? -__expf(om.y) : 0.f;
        lin[ib][0] = lam[ib][0];
        lin[ib][1] = lam[ib][1];
      }
#pragma unroll
      for (int o = 1; o < 8; o <<= 1) {
        float up[8][2];
#pragma unroll
        for (int ib = 0; ib < 8; ++ib)
#pragma unroll
          for (int e = 0; e < 2; ++e) up[ib][e] = __shfl_up_sync(0xffffffffu, lin[ib][e], o, 8);
#pragma unroll
        for (int ib = 0; ib < 8; ++ib)
#pragma unroll
          for (int e = 0; e < 2; ++e)
            if (rr >= o) lin[ib][e] += up[ib][e];
      }
      {
        float tot[8][2];
#pragma unroll
        for (int ib = 0; ib < 8; ++ib)
#pragma unroll
          for (int e = 0; e < 2; ++e) tot[ib][e] = __shfl_sync(0xffffffffu, lin[ib][e], 7, 8);
#pragma unroll
        for (int ib = 0; ib < 8; ++ib) {
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            lin[ib][e] += carry[e];
            carry[e] += tot[ib][e];
          }
          if (ib == 3 && c == 0) {
            R[0] = carry[0];
            R[1] = carry[1];
          }
        }
      }
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        bad |= !(-R[e] <= kMaxHalfDecay && R[e] - carry[e] <= kMaxHalfDecay);
        Rnext[e] = next_ref(carry[e]);
      }
      if (rr == 0) {
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          sm.Rv[par][dR + e] = R[e];
          sm.Lend[par][dR + e] = carry[e];
        }
      }
      float part[8];
#pragma unroll
      for (int ib = 0; ib < 8; ++ib) {
        const float2 rv = bf2_to_f2(lds_u32(rawR + offRK + ib * 1024u));
        const float2 kv = bf2_to_f2(lds_u32(rawK + offRK + ib * 1024u));
        const int row = 8 * ib + rr;
        const float fr0 = __expf(lin[ib][0] - lam[ib][0] - R[0]), fr1 = __expf(lin[ib][1] - lam[ib][1] - R[1]);
        const float fk0 = __expf(R[0] - lin[ib][0]), fk1 = __expf(R[1] - lin[ib][1]);
        // rounded to nearest tf32: truncation by the tensor core would bias both factors of every score
        *reinterpret_cast<float2*>(&sm.opRA[op_off(row, dR)]) = make_float2(to_tf32(rv.x * fr0), to_tf32(rv.y * fr1));
        *reinterpret_cast<float2*>(&sm.opK[op_off(row, dR)]) = make_float2(to_tf32(kv.x * fk0), to_tf32(kv.y * fk1));
        part[ib] = fmaf(rv.x * uA[0], kv.x, rv.y * uA[1] * kv.y);
      }
#pragma unroll
      for (int ib = 0; ib < 8; ++ib) part[ib] += __shfl_xor_sync(0xffffffffu, part[ib], 8);
#pragma unroll
      for (int ib = 0; ib < 8; ++ib) part[ib] += __shfl_xor_sync(0xffffffffu, part[ib], 16);
      if (rp == 0) {
#pragma unroll
        for (int ib = 0; ib < 8; ++ib) sm.diag_part[warp][8 * ib + rr] = part[ib];
      }
    }
    fence_proxy_async();
    tc_fence_before();
    const int slow = __syncthreads_or(bad);
    if (sm.abort_flag) {
      aborted = true;
      break;
    }

    if (slow) {  // some channel decays too fast for the factorization: per-token recurrence
      // the decay of every (token, key) into opS (rewritten below from the new state)
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const int tau = tid >> 2, d = 16 * (tid & 3) + i;
        sm.opS[tau * kN + d] = __expf(-__expf(lds_f32(omS + om_off(tau, d))));
      }
      recur::ChunkArgs ca;
      ca.rawR = reinterpret_cast<const unsigned char*>(sm.raw[0]);
      ca.rawK = reinterpret_cast<const unsigned char*>(sm.raw[1]);
      ca.rawV = reinterpret_cast<const unsigned char*>(sm.raw[2]);
      ca.wconst = nullptr;
      ca.wtok = sm.opS;
      ca.u = p.u + h * kN;
      ca.scratch = sm.opRA;
      ca.red = sm.opVt;
      ca.bonus = sm.diag;
      ca.ystride = (size_t)p.H * kN;
      ca.y = p.y + (((size_t)b * p.T + t0) * p.H + h) * kN;
      ca.cnt = cnt;
      ca.drow = drow;
      ca.jcol = jcol;
      S = recur::chunk_recur<false>(S, ca);
      if (c + 1 < nchunk) {
#pragma unroll
        for (int r = 0; r < 2; ++r) {
          const float eR = __expf(next_ref(sm.Lend[par][drow + 8 * r]));
#pragma unroll
          for (int q = 0; q < 8; ++q) sm.opS[op_off(jcol + 4 * q, drow + 8 * r)] = eR * S.v[2 * q + r];
        }
      }
      if (issuer && c + 1 < nchunk) {
        fence_proxy_async();
        mbar_arrive_expect_tx(&sm.bar_tma, 3 * kRawBytes + 2 * kOmBytes);
        tma_load_3d(sm.raw[0], &mr, &sm.bar_tma, h * kN, (c + 1) * kL, b);
        tma_load_3d(sm.raw[1], &mk, &sm.bar_tma, h * kN, (c + 1) * kL, b);
        tma_load_3d(sm.raw[2], &mv, &sm.bar_tma, h * kN, (c + 1) * kL, b);
        tma_load_3d(sm.om[0], &mw, &sm.bar_tma, h * kN, (c + 1) * kL, b);
        tma_load_3d(sm.om[1], &mw, &sm.bar_tma, h * kN + 32, (c + 1) * kL, b);
      }
      continue;
    }

    if (c == 0) {  // e^{R} ⊙ Sᵀ of the initial state (later chunks get it from the previous state fold)
#pragma unroll
      for (int r = 0; r < 2; ++r) {
        const float eR = __expf(sm.Rv[par][drow + 8 * r]);
#pragma unroll
        for (int q = 0; q < 8; ++q) sm.opS[op_off(jcol + 4 * q, drow + 8 * r)] = eR * S.v[2 * q + r];
      }
      fence_proxy_async();
      tc_fence_before();
      __syncthreads();
    }

    const uint32_t phm = nfast & 1u;
    auto issue_first = [&](int s0) {
      if (issuer) {
        if (s0 == 0) tc_fence_after();
#pragma unroll
        for (int s = s0; s < s0 + 2; ++s)
          umma_tf32(tSc, smem_desc(&sm.opRA[s * 64], kLbo, kSbo), smem_desc(&sm.opK[s * 64], kLbo, kSbo),
                    kIdesc128, s);
        if (s0 == 6) umma_commit(&sm.bar_sc);
      }
    };
    issue_first(0);

    // T1b: bonus sums; k̃ᵀ from opK into tensor memory (.16x256b fragment: rows d = 16 q4 + t4 + 8 r,
    // columns ι = 32 hc + 8 i + 2 tq + e -> register 4 i + 2 r + e); vᵀ into shared memory
    {
      if (tid < kL) {
        float sum = 0.f;
#pragma unroll
        for (int w = 0; w < 8; ++w) sum += sm.diag_part[w][tid];
        sm.diag[tid] = sum;
      }
      uint32_t kt[16];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
#pragma unroll
        for (int r = 0; r < 2; ++r)
#pragma unroll
          for (int e = 0; e < 2; ++e)
            kt[4 * i + 2 * r + e] = lds_u32(opKs + 4u * (uint32_t)op_off(32 * hc + 8 * i + 2 * tq + e, drow + 8 * r));
        if (i == 1) issue_first(2);
        if (i == 3) issue_first(4);
      }
      tmem_st16(tKt + tquar + (uint32_t)(32 * hc), kt);
#pragma unroll
      for (int pp = 0; pp < 2; ++pp) {
        uint32_t qv[4];
        ldsm_x4_t(rawV + offT + pp * 4096u, qv);
#pragma unroll
        for (int m = 0; m < 4; ++m) {
          const int ib = 4 * pp + m;
          const uint32_t xv = __shfl_xor_sync(0xffffffffu, qv[m], 18);
          *reinterpret_cast<float2*>(&sm.opVt[op_off(8 * warp + srow, 8 * ib + 2 * stq)]) =
              bf2_to_f2(sw ? xv : qv[m]);
        }
        if (pp == 0) issue_first(6);
      }
    }
    fence_proxy_async();
    tc_fence_before();
    __syncthreads();
    if (issuer) {
      tc_fence_after();
      if (c + 1 < nchunk) {  // every box of this chunk is consumed: load the next chunk
        fence_proxy_async();
        mbar_arrive_expect_tx(&sm.bar_tma, 3 * kRawBytes + 2 * kOmBytes);
        tma_load_3d(sm.raw[0], &mr, &sm.bar_tma, h * kN, (c + 1) * kL, b);
        tma_load_3d(sm.raw[1], &mk, &sm.bar_tma, h * kN, (c + 1) * kL, b);
        tma_load_3d(sm.raw[2], &mv, &sm.bar_tma, h * kN, (c + 1) * kL, b);
        tma_load_3d(sm.om[0], &mw, &sm.bar_tma, h * kN, (c + 1) * kL, b);
        tma_load_3d(sm.om[1], &mw, &sm.bar_tma, h * kN + 32, (c + 1) * kL, b);
      }
    }

    // T2a: causal mask of the scores (ι < τ kept, ι = τ the bonus, ι > τ zero) -> opRA
    if (!mbar_wait_bounded(&sm.bar_sc, phm, p.ctl)) sm.abort_flag = 1;
    tc_fence_after();
    {
      const int tau0 = 16 * q4 + t4;
      if (hc > (q4 >> 1)) {
#pragma unroll
        for (int q = 0; q < 8; ++q)
#pragma unroll
          for (int r = 0; r < 2; ++r) sm.opRA[op_off(tau0 + 8 * r, 32 * hc + 4 * q + tq)] = 0.f;
      } else {
        float a[16];
        tmem_ld16x128(tSc + tquar + (uint32_t)(32 * hc), a);
        float dg[2] = {0.f, 0.f};
        if ((q4 >> 1) == hc) {
          dg[0] = sm.diag[tau0];
          dg[1] = sm.diag[tau0 + 8];
        }
#pragma unroll
        for (int q = 0; q < 8; ++q)
#pragma unroll
          for (int r = 0; r < 2; ++r) {
            const int io = 32 * hc + 4 * q + tq, tau = tau0 + 8 * r;
            sm.opRA[op_off(tau, io)] = io < tau ? a[2 * q + r] : (io == tau ? dg[r] : 0.f);
          }
      }
    }
    fence_proxy_async();
    tc_fence_before();
    __syncthreads();
    if (issuer) {
      tc_fence_after();
#pragma unroll
      for (int s = 0; s < 8; ++s)
        umma_tf32(tY, smem_desc(&sm.opRA[s * 64], kLbo, kSbo), smem_desc(&sm.opVt[s * 64], kLbo, kSbo), kIdesc, 1);
      umma_commit(&sm.bar_av);
#pragma unroll
      for (int s = 0; s < 8; ++s) umma_tf32_ts(tDS, tKt + 8 * s, smem_desc(&sm.opVt[s * 64], kLbo, kSbo), kIdesc, s);
      umma_commit(&sm.bar_ds);
    }

    // T3: output rows -> bf16 -> global
    if (!mbar_wait_bounded(&sm.bar_av, phm, p.ctl)) sm.abort_flag = 1;
    tc_fence_after();
    {
      float yv[32];
      tmem_ld32(tY + tquar + (uint32_t)(32 * hc), yv);
      const int tau = 16 * q4 + lane;
      if (lane < 16 && tau < cnt) {
        __nv_bfloat16* yp = p.y + (((size_t)b * p.T + t0 + tau) * p.H + h) * kN + 32 * hc;
#pragma unroll
        for (int j = 0; j < 32; j += 8) {
          uint4 pk;
          __nv_bfloat162* q2 = reinterpret_cast<__nv_bfloat162*>(&pk);
#pragma unroll
          for (int e = 0; e < 4; ++e) q2[e] = __floats2bfloat162_rn(yv[j + 2 * e], yv[j + 2 * e + 1]);
          *reinterpret_cast<uint4*>(yp + j) = pk;
        }
      }
    }

    // T2b: S <- e^{Λ_last} S + e^{Λ_last - R} ΔS
    if (!mbar_wait_bounded(&sm.bar_ds, phm, p.ctl)) sm.abort_flag = 1;
    tc_fence_after();
    {
      float ds[16];
      tmem_ld16x128(tDS + tquar + (uint32_t)(32 * hc), ds);
#pragma unroll
      for (int r = 0; r < 2; ++r) {
        const float le = sm.Lend[par][drow + 8 * r], rv = sm.Rv[par][drow + 8 * r];
        const float gD = __expf(le), gS = __expf(le - rv), eR = __expf(next_ref(le));
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          S.v[2 * q + r] = fmaf(gD, S.v[2 * q + r], gS * ds[2 * q + r]);
          sm.opS[op_off(jcol + 4 * q, drow + 8 * r)] = eR * S.v[2 * q + r];
        }
      }
    }
    ++nfast;
  }

  if (aborted && tid == 0) {
    // a wait gave up at chunk c: the last committed MMA chains (bar_ds, one phase per chunk on
    // the tensor cores) and this chunk's loads must finish before the tensor memory and shared
    // memory are released, each wait bounded again
    if (nfast >= 1) mbar_wait_bounded(&sm.bar_ds, (nfast - 1) & 1u, p.ctl);
    if (!withheld) mbar_wait_bounded(&sm.bar_tma, (uint32_t)c & 1u, p.ctl);
  }
  if (p.s_out != nullptr) {
#pragma unroll
    for (int q = 0; q < 8; ++q)
#pragma unroll
      for (int r = 0; r < 2; ++r) p.s_out[sbase + (size_t)(drow + 8 * r) * kN + jcol + 4 * q] = S.v[2 * q + r];
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tbase, kTmemCols);
  }
}

}  // namespace

size_t wkv6_smem_bytes() { return sizeof(Wkv6Smem) + 1024; }  // + alignment slack

cudaError_t launch_wkv6_fwd(const CUtensorMap& mr, const CUtensorMap& mk, const CUtensorMap& mv,
                            const CUtensorMap& mw, const Wkv6Params& p, cudaStream_t st) {
  const size_t smem = wkv6_smem_bytes();
  static unsigned device_mask = 0;
  cudaError_t e = ensure_smem_attr(reinterpret_cast<const void*>(wkv6_fwd_tc_kernel), (int)smem, &device_mask);
  if (e != cudaSuccess) return e;
  wkv6_fwd_tc_kernel<<<(unsigned)(p.B * p.H), kThreads, smem, st>>>(mr, mk, mv, mw, p);
  return cudaGetLastError();
}

}  // namespace rwkv
