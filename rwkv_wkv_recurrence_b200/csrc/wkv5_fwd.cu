// Eagle / RWKV-5 multi-head matrix-state WKV forward (sm_100a): chunked form
// on the tcgen05 tensor cores.
//
// "RWKV-5 Eagle과 RWKV-6 Finch", section Eagle: per head,
//   s' = diag(w) s + kᵀ v,   wkv' = s + diag(u) kᵀ v,   w = exp(-exp(ω)),
// and the receptance reads the state like a query:
//   y_t = r_t (s_t + diag(u) k_tᵀ v_t),   s_{t+1} = diag(w) s_t + k_tᵀ v_t,
// with s[i][j] indexed (key i, value j) as in the RWKV-7 page's update
// kv[d,e] = k_d v_e, out_e = Σ_d r_d state[d,e].
//
// Chunked form (chunk of L = 64 tokens starting at state S, λ_d = -exp(ω_d),
// w_d = e^{λ_d}; τ, ι are positions inside the chunk):
//   y[τ]   = Σ_d r[τ,d] e^{λ_d τ} S[d,:]                          (inter-chunk)
//          + Σ_{ι<τ} A[τ,ι] v[ι,:] + (Σ_d r[τ,d] u_d k[τ,d]) v[τ,:]   (intra-chunk)
//   A[τ,ι] = Σ_d r[τ,d] e^{λ_d (τ-1-ι)} k[ι,d]
//          = Σ_d (r[τ,d] e^{λ_d (τ-32)}) (k[ι,d] e^{λ_d (31-ι)})       (a plain product)
//   S'     = e^{64 λ} ⊙ S + Σ_ι (k[ι,:] e^{λ (63-ι)})ᵀ v[ι,:]
// Per chunk the tensor cores (tcgen05, kind::tf32, fp32 accumulators in tensor
// memory) run three chains of eight K = 8 steps:
//   [A | Y] = r̃ [k̃ ; e^{32λ} Sᵀ]ᵀ          M = 64, N = 128: scores [τ][ι] and the
//                                           inter-chunk read [τ][j] share operand r̃
//   ΔS      = k̃ᵀ vᵀᵀ                       M = 64, N = 64, k̃ᵀ read from tensor memory
//   Y      += A_masked vᵀᵀ                 M = 64, N = 64 (intra-chunk term), the masked scores
//                                           read in place from tensor memory
// ΔS needs only the chunk's own operands, so it is issued as soon as they exist
// and runs while the scores are masked; the state fold then overlaps A v.
// with r̃ = r e^{λ(τ-32)}, k̃ = k e^{λ(31-ι)}, so that r̃·k̃ = r e^{λ(τ-1-ι)} k and
// e^{32λ} (r̃ S) = r e^{λτ} S; the state increment is scaled by e^{λ(cnt-32)} per
// key channel when it is folded into the fp32 master state, which lives in
// registers (S' = e^{cnt λ} S + e^{(cnt-32) λ} ΔS), so the state is never
// rounded below fp32.  Splitting e^{λ(τ-1-ι)} around the chunk middle keeps
// every factor within e^{±32|λ|}; a head with -λ > 2.5 in any channel
// (w < 0.082) would leave the fp32 range there: its chunks run token by token
// on the CUDA cores instead (chunk_recur), with the same TMA boxes and state.
//
// The tensor core takes tf32 operands K-major only, so the operand tiles are
// fp32 [rows][64] in the K-major core-matrix layout without swizzle (8 rows x
// 16 bytes per core matrix); k̃ᵀ and vᵀ are transposed on the way in with
// ldmatrix.trans.  Each tcgen05.mma of these sizes costs its issuing thread
// about 70 cycles whatever M and N are, so the kernel uses the widest shapes
// the data allows (N = 128 for the first chain) and the issuing thread hands
// the first chain out in pairs between the other work of its warp.
//
// CTA: one (batch, head), 8 warps, about 90 KB of shared memory and 256 TMEM
// columns, two CTAs per SM.  Thread 0 issues the TMA loads of the raw r, k, v
// tiles (one [64 tokens x 64] bf16 box each, 128-byte swizzle, no multicast)
// and the MMAs; all warps build operands, mask the scores, fold the state and
// write the output rows.
#include <cstddef>

#include "launch.h"
#include "tc_common.cuh"
#include "wkv_common.cuh"
#include "wkv_recur.cuh"

namespace rwkv {
namespace {

using namespace tc;

constexpr int kN = 64;                 // head size
constexpr int kL = 64;                 // tokens per chunk
constexpr int kThreads = 256;
constexpr uint32_t kRawBytes = kL * kN * 2;    // one bf16 [64 x 64] box
constexpr float kMaxRate = 2.5f;       // largest -λ the chunked factorization accepts
constexpr uint32_t kTmemCols = 256;  // [scores | output rows], state increment, k̃ᵀ (64 columns each)

struct Wkv5Smem {
  alignas(1024) __nv_bfloat16 raw[3][kL * kN];  // r, k, v boxes [token][channel] (128-byte swizzle)
  alignas(128) float opR[64 * 64];   // r̃ = r e^{λ(τ-32)}   [τ][d]: A of the scores and of the state read
  alignas(128) float opK[64 * 64];   // k̃ = k e^{λ(31-ι)}   [ι][d]: B rows 0..63 of the first product
  alignas(128) float opS[64 * 64];   // e^{32λ} ⊙ Sᵀ         [j][d]: B rows 64..127 of the first product
  alignas(128) float opVt[64 * 64];  // vᵀ                   [j][ι]: B of A v and of the state increment
  float diag_part[8][kL];            // per-warp parts of Σ_d r u k (the bonus term)
  float diag[kL];                    // Σ_d r u k per token
  float wdec[kN];                    // w per key channel (heads on the recurrent path)
  alignas(8) uint64_t bar_tma;
  alignas(8) uint64_t bar_sc;        // scores and state read done
  alignas(8) uint64_t bar_av;        // A v done
  alignas(8) uint64_t bar_ds;        // state increment done
  uint32_t tmem_base;
  int slow;
  int abort_flag;
};
static_assert(offsetof(Wkv5Smem, opK) == offsetof(Wkv5Smem, opR) + 64 * 64 * sizeof(float) &&
                  recur::kScratchFloats <= 2 * 64 * 64 && recur::kRedFloats <= 64 * 64,
              "the recurrent path's state copy spans opR and opK, its output parts fit opVt");
static_assert(offsetof(Wkv5Smem, opS) == offsetof(Wkv5Smem, opK) + 64 * 64 * sizeof(float),
              "the first product reads k̃ and e^{32λ} Sᵀ as one 128-row operand");

// REV: the operator over reversed time (position τ of chunk c is token T-1-(64c+τ)), reading and
// writing the tensors in their own order: chunk c's box starts at token T-64(c+1) (rows before
// token 0 read as zeros), its rows are taken bottom up, and y row τ goes to token T-1-(64c+τ).
template <bool REV>
__global__ void __launch_bounds__(kThreads, 2) wkv5_fwd_tc_kernel(const __grid_constant__ CUtensorMap mr,
                                                                  const __grid_constant__ CUtensorMap mk,
                                                                  const __grid_constant__ CUtensorMap mv,
                                                                  Wkv5Params p) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  // TMA destinations with the 128-byte swizzle need 1024-byte alignment: align by hand
  const uint32_t base_s = smem_u32(smem_raw);
  Wkv5Smem& sm = *reinterpret_cast<Wkv5Smem*>(smem_raw + ((1024u - (base_s & 1023u)) & 1023u));
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int t4 = lane >> 2, tq = lane & 3;
  const int q4 = warp & 3, hc = warp >> 2;  // TMEM lane quarter and column half of this warp
  const int b = blockIdx.x / p.H, h = blockIdx.x % p.H;
  const int nchunk = (p.T + kL - 1) / kL;
  const float* om = p.omega + h * kN;

  if (tid == 0) {
    sm.slow = 0;
    sm.abort_flag = 0;
  }
  __syncthreads();
  if (tid < kN && !(expf(om[tid]) <= kMaxRate)) atomicOr(&sm.slow, 1);
  if (tid < kN) sm.wdec[tid] = expf(-expf(om[tid]));
  __syncthreads();
  // a head with some channel outside the factorization's range runs every chunk by the recurrence
  const bool fast = sm.slow != 0;

  if (warp == 0) tmem_alloc(&sm.tmem_base, kTmemCols);
  // thread 0 issues every load; with the test hook set it arms the barrier and issues none
  const bool withheld = tid == 0 && loads_withheld(p.ctl);
  if (tid == 0) {
    prefetch_tensormap(&mr);
    prefetch_tensormap(&mk);
    prefetch_tensormap(&mv);
    mbar_init(&sm.bar_tma, 1);
    mbar_init(&sm.bar_sc, 1);
    mbar_init(&sm.bar_av, 1);
    mbar_init(&sm.bar_ds, 1);
    fence_mbar_init();
    mbar_arrive_expect_tx(&sm.bar_tma, 3 * kRawBytes);
    if (!withheld) {
      const int row0 = REV ? p.T - kL : 0;
      tma_load_3d(sm.raw[0], &mr, &sm.bar_tma, h * kN, row0, b);
      tma_load_3d(sm.raw[1], &mk, &sm.bar_tma, h * kN, row0, b);
      tma_load_3d(sm.raw[2], &mv, &sm.bar_tma, h * kN, row0, b);
    }
  }

  // ---- r̃, k̃: warp w owns channels 8w..8w+7; lane holds token row 8 ib + rr, channels dR, dR + 1.
  // A half-warp then writes one whole core matrix (eight 16-byte rows): no bank conflicts.
  const int rr = lane & 7, rp = lane >> 3;
  const int dR = 8 * warp + 2 * rp;
  float fr0[2], frs[2], fk0[2], fks[2], uA[2];
#pragma unroll
  for (int e = 0; e < 2; ++e) {
    const float rate = expf(om[dR + e]);  // -λ
    fr0[e] = expf(-rate * (float)(rr - 32));
    frs[e] = expf(-8.f * rate);
    fk0[e] = expf(-rate * (float)(31 - rr));
    fks[e] = expf(8.f * rate);
    uA[e] = p.u[h * kN + dR + e];
  }
  // box row of position 8 ib + rr: 8 ib + rr, or 63 - (8 ib + rr) = 8 (7 - ib) + (7 - rr) reversed
  const int rb = REV ? 7 - rr : rr;
  const uint32_t offRK = (uint32_t)rb * 128u + (uint32_t)((warp ^ rb) << 4) + (uint32_t)rp * 4u;
  const int lrow = lane & 7, lmat = lane >> 3;
  // ---- vᵀ (shared memory): ldmatrix.trans of block column w; lanes whose bit 1 and bit 4 differ
  // trade their pair with lane ^ 18 so that each half-warp again covers one core matrix.
  const int sw = ((lane >> 1) ^ (lane >> 4)) & 1;
  const int srow = t4 ^ (sw << 2), stq = tq ^ (sw << 1);
  // lane's row address for ldmatrix: position 8 lmat + lrow (+ 32 per pp), its box row bottom up when REV
  const uint32_t offT = REV ? (uint32_t)(63 - lmat * 8 - lrow) * 128u + (uint32_t)((warp ^ (7 - lrow)) << 4)
                            : (uint32_t)(lmat * 8 + lrow) * 128u + (uint32_t)((warp ^ lrow) << 4);
  // ---- k̃ᵀ (tensor memory, A of the state increment), .16x256b fragment of warp w:
  // rows d = 16 q4 + t4 + 8 r, columns ι = 32 hc + 8 i + 2 tq + e  ->  register 4 i + 2 r + e
  float fc0[2][2], fcs[2];
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    const float rate = expf(om[16 * q4 + 8 * r + t4]);
#pragma unroll
    for (int e = 0; e < 2; ++e) fc0[r][e] = expf(-rate * (float)(31 - 32 * hc - 2 * tq - e));
    fcs[r] = expf(8.f * rate);
  }
  // position 32 hc + 8 (lmat >> 1) + lrow (+ 16 per pp); its box row bottom up when REV
  const uint32_t offKt =
      REV ? (uint32_t)(63 - (4 * hc + (lmat >> 1)) * 8 - lrow) * 128u + (uint32_t)(((2 * q4 + (lmat & 1)) ^ (7 - lrow)) << 4)
          : (uint32_t)((4 * hc + (lmat >> 1)) * 8 + lrow) * 128u + (uint32_t)(((2 * q4 + (lmat & 1)) ^ lrow) << 4);

  // ---- state S[d][j] (fp32 master copy) in the .16x128b fragment of warp w:
  // d = 16 q4 + t4 + 8 r, j = 32 hc + 4 q + tq  ->  S[2 q + r]
  const int drow = 16 * q4 + t4;
  const int jcol = 32 * hc + tq;
  const uint32_t tquar = (uint32_t)(32 * q4) << 16;
  float e32[2];
#pragma unroll
  for (int r = 0; r < 2; ++r) e32[r] = expf(-32.f * expf(om[drow + 8 * r]));
  const size_t sbase = ((size_t)b * p.H + h) * kN * kN;
  float S[16];
#pragma unroll
  for (int q = 0; q < 8; ++q)
#pragma unroll
    for (int r = 0; r < 2; ++r)
      S[2 * q + r] = p.s_in ? p.s_in[sbase + (size_t)(drow + 8 * r) * kN + jcol + 4 * q] : 0.f;
#pragma unroll
  for (int q = 0; q < 8; ++q)
#pragma unroll
    for (int r = 0; r < 2; ++r) sm.opS[op_off(jcol + 4 * q, drow + 8 * r)] = e32[r] * S[2 * q + r];

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = sm.tmem_base;
  const uint32_t tSc = tbase, tY = tbase + 64, tDS = tbase + 128, tKt = tbase + 192;
  const uint32_t rawR = smem_u32(sm.raw[0]), rawK = smem_u32(sm.raw[1]), rawV = smem_u32(sm.raw[2]);
  const bool issuer = tid == 0;

  int c = 0;
  bool aborted = false;
  for (; c < nchunk; ++c) {
    const int t0 = c * kL;
    const int cnt = min(kL, p.T - t0);
    const uint32_t ph = (uint32_t)c & 1u;
    if (!mbar_wait_bounded(&sm.bar_tma, ph, p.ctl)) sm.abort_flag = 1;

    if (fast) {  // the chunk's tokens one by one on the CUDA cores (opR, opK, opVt, diag as scratch)
      __syncthreads();
      if (sm.abort_flag) {
        aborted = true;
        break;
      }
      recur::ChunkArgs ca;
      ca.rawR = reinterpret_cast<const unsigned char*>(sm.raw[0]);
      ca.rawK = reinterpret_cast<const unsigned char*>(sm.raw[1]);
      ca.rawV = reinterpret_cast<const unsigned char*>(sm.raw[2]);
      ca.wconst = sm.wdec;
      ca.wtok = nullptr;
      ca.u = p.u + h * kN;
      ca.scratch = sm.opR;
      ca.red = sm.opVt;
      ca.bonus = sm.diag;
      ca.ystride = (size_t)p.H * kN;
      ca.y = p.y + (((size_t)b * p.T + (REV ? p.T - 1 - t0 : t0)) * p.H + h) * kN;
      ca.cnt = cnt;
      ca.drow = drow;
      ca.jcol = jcol;
      recur::Frag16 f;
#pragma unroll
      for (int x = 0; x < 16; ++x) f.v[x] = S[x];
      f = recur::chunk_recur<REV>(f, ca);
#pragma unroll
      for (int x = 0; x < 16; ++x) S[x] = f.v[x];
      if (issuer && c + 1 < nchunk) {  // the boxes are consumed (the routine ends on a barrier)
        fence_proxy_async();
        mbar_arrive_expect_tx(&sm.bar_tma, 3 * kRawBytes);
        const int rown = REV ? p.T - (c + 2) * kL : (c + 1) * kL;
        tma_load_3d(sm.raw[0], &mr, &sm.bar_tma, h * kN, rown, b);
        tma_load_3d(sm.raw[1], &mk, &sm.bar_tma, h * kN, rown, b);
        tma_load_3d(sm.raw[2], &mv, &sm.bar_tma, h * kN, rown, b);
      }
      continue;
    }

    // T1a: r̃, k̃ and the bonus parts (rows past the sequence end hold zeros from the TMA fill)
    {
      float fr[2] = {fr0[0], fr0[1]}, fk[2] = {fk0[0], fk0[1]};
#pragma unroll
      for (int ib = 0; ib < 8; ++ib) {
        const uint32_t ibo = (uint32_t)(REV ? 7 - ib : ib) * 1024u;
        const float2 rv = bf2_to_f2(lds_u32(rawR + offRK + ibo));
        const float2 kv = bf2_to_f2(lds_u32(rawK + offRK + ibo));
        const int row = 8 * ib + rr;
        *reinterpret_cast<float2*>(&sm.opR[op_off(row, dR)]) = make_float2(rv.x * fr[0], rv.y * fr[1]);
        *reinterpret_cast<float2*>(&sm.opK[op_off(row, dR)]) = make_float2(kv.x * fk[0], kv.y * fk[1]);
        float part = fmaf(rv.x * uA[0], kv.x, rv.y * uA[1] * kv.y);
        part += __shfl_xor_sync(0xffffffffu, part, 8);
        part += __shfl_xor_sync(0xffffffffu, part, 16);
        if (rp == 0) sm.diag_part[warp][row] = part;
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          fr[e] *= frs[e];
          fk[e] *= fks[e];
        }
      }
    }
    fence_proxy_async();
    tc_fence_before();
    __syncthreads();
    if (sm.abort_flag) {
      aborted = true;
      break;
    }
    // [scores | Y] = r̃ [k̃ ; e^{32λ} Sᵀ]ᵀ: causal scores [τ][ι] and the state read [τ][j].  The
    // issuing thread hands the eight K steps out in pairs between its warp's T1b steps, so that
    // the warp never waits on a full MMA queue.
    auto issue_first = [&](int s0) {
      if (issuer) {
        if (s0 == 0) tc_fence_after();
#pragma unroll
        for (int s = s0; s < s0 + 2; ++s)
          umma_tf32(tSc, smem_desc(&sm.opR[s * 64], kLbo, kSbo), smem_desc(&sm.opK[s * 64], kLbo, kSbo),
                    kIdesc128, s);
        if (s0 == 6) umma_commit(&sm.bar_sc);
      }
    };
    issue_first(0);

    // T1b: k̃ᵀ into tensor memory, vᵀ into shared memory, the bonus sums
    {
      if (tid < kL) {
        float sum = 0.f;
#pragma unroll
        for (int w = 0; w < 8; ++w) sum += sm.diag_part[w][tid];
        sm.diag[tid] = sum;
      }
      uint32_t kt[16];
#pragma unroll
      for (int pp = 0; pp < 2; ++pp) {
        uint32_t qk[4];
        ldsm_x4_t(REV ? rawK + offKt - pp * 2048u : rawK + offKt + pp * 2048u, qk);
#pragma unroll
        for (int m = 0; m < 4; ++m) {
          const int i = 2 * pp + (m >> 1), r = m & 1;
          const float2 f = bf2_to_f2(qk[m]);
          const float g = i == 0 ? 1.f : (i == 1 ? fcs[r] : (i == 2 ? fcs[r] * fcs[r] : fcs[r] * fcs[r] * fcs[r]));
          kt[4 * i + 2 * r] = __float_as_uint(f.x * fc0[r][0] * g);
          kt[4 * i + 2 * r + 1] = __float_as_uint(f.y * fc0[r][1] * g);
        }
        issue_first(2 + 2 * pp);
      }
      tmem_st16(tKt + tquar + (uint32_t)(32 * hc), kt);
#pragma unroll
      for (int pp = 0; pp < 2; ++pp) {
        uint32_t qv[4];
        ldsm_x4_t(REV ? rawV + offT - pp * 4096u : rawV + offT + pp * 4096u, qv);
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
      // ΔS = k̃ᵀ v [d][j] needs only this chunk's operands: it runs while the scores are masked
#pragma unroll
      for (int s = 0; s < 8; ++s) umma_tf32_ts(tDS, tKt + 8 * s, smem_desc(&sm.opVt[s * 64], kLbo, kSbo), kIdesc, s);
      umma_commit(&sm.bar_ds);
      // the raw boxes are consumed: load the next chunk while this one computes
      if (c + 1 < nchunk) {
        fence_proxy_async();
        mbar_arrive_expect_tx(&sm.bar_tma, 3 * kRawBytes);
        const int rown = REV ? p.T - (c + 2) * kL : (c + 1) * kL;
        tma_load_3d(sm.raw[0], &mr, &sm.bar_tma, h * kN, rown, b);
        tma_load_3d(sm.raw[1], &mk, &sm.bar_tma, h * kN, rown, b);
        tma_load_3d(sm.raw[2], &mv, &sm.bar_tma, h * kN, rown, b);
      }
    }

    // T2a: causal mask of the scores in tensor memory, in place (ι < τ kept, ι = τ the bonus
    // Σ_d r u k, ι > τ zero): the A operand of A v.
    // .16x128b fragment: rows τ = 16 q4 + t4 + 8 r, columns ι = 32 hc + 4 q + tq  ->  register 2 q + r
    if (!mbar_wait_bounded(&sm.bar_sc, ph, p.ctl)) sm.abort_flag = 1;
    tc_fence_after();
    {
      const int tau0 = 16 * q4 + t4;
      if (hc > (q4 >> 1)) {  // strictly above the diagonal
        float a[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) a[i] = 0.f;
        tmem_st16x128(tSc + tquar + (uint32_t)(32 * hc), a);
      } else {
        float a[16];
        tmem_ld16x128(tSc + tquar + (uint32_t)(32 * hc), a);
        float dg[2] = {0.f, 0.f};
        if ((q4 >> 1) == hc) {  // the fragment holds the diagonal
          dg[0] = sm.diag[tau0];
          dg[1] = sm.diag[tau0 + 8];
        }
#pragma unroll
        for (int q = 0; q < 8; ++q)
#pragma unroll
          for (int r = 0; r < 2; ++r) {
            const int io = 32 * hc + 4 * q + tq, tau = tau0 + 8 * r;
            a[2 * q + r] = io < tau ? a[2 * q + r] : (io == tau ? dg[r] : 0.f);
          }
        tmem_st16x128(tSc + tquar + (uint32_t)(32 * hc), a);
      }
    }
    tc_fence_before();
    __syncthreads();
    if (issuer) {
      tc_fence_after();
      // Y += (masked scores) v, the scores read from tensor memory
#pragma unroll
      for (int s = 0; s < 8; ++s) umma_tf32_ts(tY, tSc + 8 * s, smem_desc(&sm.opVt[s * 64], kLbo, kSbo), kIdesc, 1);
      umma_commit(&sm.bar_av);
    }

    // T2b: S <- e^{cnt λ} S + e^{(cnt-32) λ} ΔS; e^{32λ} Sᵀ into opS for the next chunk (while A v
    // still runs)
    if (!mbar_wait_bounded(&sm.bar_ds, ph, p.ctl)) sm.abort_flag = 1;
    tc_fence_after();
    {
      float ds[16];
      tmem_ld16x128(tDS + tquar + (uint32_t)(32 * hc), ds);
      if (cnt == kL) {
#pragma unroll
        for (int q = 0; q < 8; ++q)
#pragma unroll
          for (int r = 0; r < 2; ++r) {
            const int x = 2 * q + r;
            const float g = e32[r];
            S[x] = g * fmaf(g, S[x], ds[x]);
            sm.opS[op_off(jcol + 4 * q, drow + 8 * r)] = g * S[x];
          }
      } else {  // last, partial chunk: no later chunk reads opS
#pragma unroll
        for (int r = 0; r < 2; ++r) {
          const float rate = expf(om[drow + 8 * r]);
          const float dl = expf(-rate * (float)cnt), gs = expf(-rate * (float)(cnt - 32));
#pragma unroll
          for (int q = 0; q < 8; ++q) S[2 * q + r] = fmaf(dl, S[2 * q + r], gs * ds[2 * q + r]);
        }
      }
    }

    // T3: Y rows -> bf16 -> global (TMEM lanes 0..15 of each quarter hold the rows)
    if (!mbar_wait_bounded(&sm.bar_av, ph, p.ctl)) sm.abort_flag = 1;
    tc_fence_after();
    {
      float yv[32];
      tmem_ld32(tY + tquar + (uint32_t)(32 * hc), yv);
      const int tau = 16 * q4 + lane;
      if (lane < 16 && tau < cnt) {
        const int ty = REV ? p.T - 1 - (t0 + tau) : t0 + tau;
        __nv_bfloat16* yp = p.y + (((size_t)b * p.T + ty) * p.H + h) * kN + 32 * hc;
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
  }

  if (aborted && tid == 0) {
    // a wait gave up at chunk c: the previous chunk's MMA chains (committed last on bar_av) and
    // this chunk's loads must finish before the tensor memory and shared memory are released,
    // each wait bounded again
    if (c >= 1 && !fast) mbar_wait_bounded(&sm.bar_av, (uint32_t)(c - 1) & 1u, p.ctl);
    if (!withheld) mbar_wait_bounded(&sm.bar_tma, (uint32_t)c & 1u, p.ctl);
  }
  if (p.s_out != nullptr) {
#pragma unroll
    for (int q = 0; q < 8; ++q)
#pragma unroll
      for (int r = 0; r < 2; ++r) p.s_out[sbase + (size_t)(drow + 8 * r) * kN + jcol + 4 * q] = S[2 * q + r];
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tbase, kTmemCols);
  }
}

}  // namespace

size_t wkv5_smem_bytes() { return sizeof(Wkv5Smem) + 1024; }  // + alignment slack

cudaError_t launch_wkv5_fwd(const CUtensorMap& mr, const CUtensorMap& mk, const CUtensorMap& mv, const Wkv5Params& p,
                            cudaStream_t st, bool reversed) {
  const size_t smem = wkv5_smem_bytes();
  static unsigned mask_f = 0, mask_r = 0;
  const void* fn = reversed ? reinterpret_cast<const void*>(wkv5_fwd_tc_kernel<true>)
                            : reinterpret_cast<const void*>(wkv5_fwd_tc_kernel<false>);
  cudaError_t e = ensure_smem_attr(fn, (int)smem, reversed ? &mask_r : &mask_f);
  if (e != cudaSuccess) return e;
  if (reversed)
    wkv5_fwd_tc_kernel<true><<<(unsigned)(p.B * p.H), kThreads, smem, st>>>(mr, mk, mv, p);
  else
    wkv5_fwd_tc_kernel<false><<<(unsigned)(p.B * p.H), kThreads, smem, st>>>(mr, mk, mv, p);
  return cudaGetLastError();
}


}  // namespace rwkv
