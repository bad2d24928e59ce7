// Eagle / RWKV-5 WKV backward (sm_100a): the two chunked tensor-core passes
// that give gr, gk and the decay gradient.
//
// "RWKV-5 Eagle과 RWKV-6 Finch", section Eagle, per head:
//   y_t = r_t (s_t + diag(u) k_tᵀ v_t),   s_{t+1} = diag(w) s_t + k_tᵀ v_t,
// s[i][j] indexed (key i, value j).  The pages print no backward; for
// L = Σ gy·y + Σ gs_out ∘ s_T the chain rule gives, with G_{t+1} = ∂L/∂s_{t+1}
// (G_T = gs_out, G_t = diag(w) G_{t+1} + r_tᵀ gy_t):
//   gr_t[d] = Σ_j s_t[d][j] gy_t[j] + u_d k_t[d] (v_t·gy_t)
//   gk_t[d] = Σ_j G_{t+1}[d][j] v_t[j] + u_d r_t[d] (v_t·gy_t)
//   ∂L/∂w_d = Σ_t Σ_j G_{t+1}[d][j] s_t[d][j]
// Both gradients have one shape, a "state read with the decay on the output
// channel": for queries q_t, keys p_i, coefficients c_i and a carried state X
//   out_t[d] = Σ_{i<t} (q_t·p_i) w_d^{t-1-i} c_i[d] + Σ_j w_d^t X_0[d][j] q_t[j]
//              + u_d c_t[d] (q_t·p_t),      X ← diag(w) X + c_tᵀ p_t,
// which is gr for (q, p, c, X_0) = (gy, v, k, s_in) in forward time, and gk for
// (q, p, c, X_0) = (v, gy, r, gs_out) with time reversed.  One kernel runs
// either pass (REV = the reversed one).  The reversed pass reads and writes
// the tensors in their own order: its chunk c is forward chunk nchunk-1-c,
// loaded as usual, with its rows taken bottom up.
//
// Chunked form (chunk of 64 positions, λ_d = -exp(ω_d), c̃_ι = c_ι e^{λ(31-ι)}):
//   A[τ][ι]  = q_τ·p_ι                                 (no decay: a plain product)
//   Xᵀ[d][τ] = Σ_j (e^{32λ} X)[d][j] q_τ[j]             state read
//            + Σ_{ι<τ} c̃ᵀ[d][ι] A[τ][ι]                 intra-chunk term
//   out[τ][d] = e^{λ_d (τ-32)} Xᵀ[d][τ] + u_d c_τ[d] A[τ][τ]
//   X' = e^{64λ} X + e^{32λ} c̃ᵀ p                       (per key row d)
// four tcgen05 chains of eight K = 8 steps (kind::tf32, fp32 accumulators in
// tensor memory): A = q·pᵀ, the state read (A operand e^{32λ}X [d][j], B
// operand q [τ][j]), the intra term (A operand c̃ᵀ from tensor memory, B the
// masked A), the state increment (A c̃ᵀ, B pᵀ).  q and p are bf16 in HBM, so
// their tf32 copies are exact and A is exact up to fp32 accumulation.
//
// The decay gradient.  Per forward chunk (positions σ, ι in 0..n-1, X_c the
// forward state at the chunk start, G its gradient at the chunk end)
//   Σ_τ G_{τ+1}∘s_τ = n w^{n-1} G∘X_c
//                  + Σ_ι (n-1-ι) w^{n-2-ι} k_ι ⊙ (G v_ιᵀ)
//                  + Σ_σ σ w^{σ-1} r_σ ⊙ (X_c gy_σᵀ)
//                  + Σ_{ι<σ} (σ-1-ι) w^{σ-2-ι} (r_σ ⊙ k_ι) (gy_σ·v_ι),
// every term a sum of products with non-negative weights (so no cancellation
// between separately rounded passes).  The reversed pass holds G and reads the
// forward states X_c, which the forward pass writes at every chunk start
// (checkpoints): the first term is elementwise, the second is its own state
// read weighted by position, the third one more chain (X_c · gyᵀ), the last
// one more chain with the masked scores weighted by the lag.  The reversed
// pass's chunks are the forward ones: its first (the partial last forward
// chunk, whose rows past the sequence read as zero) has `lead` empty positions
// before the carried state enters.
//
// Memory: q, p, c arrive as TMA boxes; the epilogue's c and m rows are fetched with 16-byte loads at
// the top of the chunk, parked in shared memory once the first chains have released their operand
// buffer, and the outputs leave through the same rows as 16-byte stores.  The forward pass stores
// each checkpoint in the tf32 operand layout, so the reversed pass brings it in with one bulk copy a
// chunk ahead.
//
// Fast rows.  A key row decaying faster than the factorization takes (exp(ω) > 2:
// factors beyond e^{±64} would push small operands into the subnormal range)
// stays out of the factorized products: its c̃ᵀ row is zero, its state row is
// read unscaled and its output takes e^{λ(τ-lo)}.  Its intra-chunk terms (the
// plain one and, reversed, the lag-weighted one) are summed on the CUDA cores
// over lags 0..15 by all threads, from the masked scores and the staged c rows,
// into operand tiles that are free at that point, and read by that row's
// epilogue; its state increment is summed in the fold over the chunk's last 16
// positions: beyond that e^{λn} < 2^-46 of the lag-0 weight.  Any w in [0, 1]
// is handled.  Heads without fast rows run a second instance of the chunk loop
// that has none of this code.
//
// CTA: one (batch, head), 8 warps.  Forward pass: ~112 KB of shared memory,
// 256 TMEM columns, two CTAs per SM.  Reversed pass: ~146 KB, 512 columns, one
// CTA per SM.  Thread 0 issues the TMA loads and the scores, state-read and
// intra chains; a thread of warp 4 (whose share of the masking is a zero fill)
// issues the state-increment chain and, reversed, the lag-weighted chain.
#include <cstddef>
#include <type_traits>

#include "launch.h"
#include "tc_common.cuh"
#include "wkv_common.cuh"

namespace rwkv {
namespace {

using namespace tc;

constexpr int kN = 64;
constexpr int kL = 64;
constexpr int kThreads = 256;
constexpr uint32_t kRawBytes = kL * kN * 2;
constexpr float kMaxRate = 2.f;  // largest rate the chunked factorization takes
constexpr int kBand = 15;         // lags a fast row keeps: e^{-2 (kBand+1)} < 2^-46
constexpr uint32_t kCkBytes = kN * kN * 4;  // one forward-state checkpoint (fp32, operand layout)

struct Wkv5BwdSmem {
  alignas(1024) __nv_bfloat16 raw[3][kL * kN];  // q, p, c boxes [position][channel] (128-byte swizzle)
  alignas(128) float opQ[64 * 64];   // q [τ][j]: A of the scores, B of the state read
  alignas(128) float opP[64 * 64];   // p [ι][j]: B of the scores (and, reversed, of the X_c read)
  alignas(128) float opX[64 * 64];   // e^{f λ} X [d][j]: A of the state read
  alignas(128) float opPt[64 * 64];  // pᵀ [j][ι]: B of the state increment
  alignas(128) float opAm[64 * 64];  // strictly causal scores [τ][ι]: B of the intra term
  float diag[kL];                    // A[τ][τ] = q_τ·p_τ
  float EB[kBand + 1][kN];           // e^{λ_d n} [n][key row d], n = 0..kBand (fast rows)
  int flist[kN];                     // the fast rows, in order
  int nfl;                           // their count
  alignas(8) uint64_t bar_tma;
  alignas(8) uint64_t bar_sc;        // scores and state read (and the X_c read) done
  alignas(8) uint64_t bar_av;        // intra term (and the lag-weighted term) done
  alignas(8) uint64_t bar_ds;        // state increment done
  alignas(8) uint64_t bar_ck;        // reversed pass: the forward state X_c has arrived in opXc
  uint32_t tmem_base;
  int abort_flag;
  // reversed pass only (not part of the forward pass's shared memory)
  alignas(128) float opXc[64 * 64];  // forward state X_c [d][j]: A of the X_c read (bulk-copied)
  alignas(128) float opAl[64 * 64];  // lag-weighted scores (τ-1-ι) A [τ][ι]: B of the lag term
  double red[kN];                    // per key row: the decay-gradient sum of this CTA
};

// dynamic shared memory = the struct (or its forward-pass prefix) + 1024 bytes of alignment slack;
// an SM has 228 KB, of which each resident CTA also takes 1 KB: two forward-pass CTAs per SM
static_assert(2 * (offsetof(Wkv5BwdSmem, opXc) + 1024 + 1024) <= 228 * 1024, "two CTAs per SM");

size_t bwd_smem_bytes(bool rev) {
  return (rev ? sizeof(Wkv5BwdSmem) : offsetof(Wkv5BwdSmem, opXc)) + 1024;  // + alignment slack
}

// Checkpoint of forward chunk `cf` of (b, h): X_c stored in the tf32 operand layout (op_off), so
// that the reversed pass copies it into shared memory as one contiguous block.
__device__ __forceinline__ float* ckpt_at(const Wkv5BwdParams& p, int b, int h, int nchunk, int cf) {
  return p.ckpt + (((size_t)b * p.H + h) * nchunk + cf) * (kN * kN);
}

// Fast rows' intra-chunk terms over lags 0..kBand, by all threads (thread = position x one quarter
// of the fast rows): BF0[pos][d] = Σ_n A[pos][pos-1-n] c_{pos-1-n}[d] e^{λ_d n} and, reversed,
// BF1[pos][d] = Σ_{n≥1} n A[pos][pos-1-n] c_{pos-1-n}[d] e^{λ_d (n-1)}.  Out of line: it runs only
// for heads with fast rows and keeps the main loop's code as it is for the others.
template <bool REV>
__device__ __noinline__ void fast_band(Wkv5BwdSmem& sm, const __nv_bfloat16* stC, float* BF0, float* BF1, int lo) {
  const int tid = threadIdx.x;
  const int pos = tid >> 2, g = tid & 3;
  float an[kBand + 1];
#pragma unroll
  for (int n = 0; n <= kBand; ++n) {
    const int io = pos - 1 - n;
    an[n] = io >= lo ? sm.opAm[op_off(pos, io)] : 0.f;
  }
  const int nf = sm.nfl;
#pragma unroll 1
  for (int cf = g; cf < nf; cf += 4) {
    const int d = sm.flist[cf];
    float b0 = 0.f, b1 = 0.f;
#pragma unroll
    for (int n = 0; n <= kBand; ++n) {
      const int io = pos - 1 - n;
      const float ac = io >= 0 ? an[n] * __bfloat162float(stC[(REV ? kL - 1 - io : io) * kN + d]) : 0.f;
      b0 = fmaf(ac, sm.EB[n][d], b0);
      if constexpr (REV) {
        if (n >= 1) b1 = fmaf((float)n * ac, sm.EB[n - 1][d], b1);
      }
    }
    BF0[pos * kN + d] = b0;
    if constexpr (REV) BF1[pos * kN + d] = b1;
  }
}

// A fast row's state increment over the chunk's last kBand + 1 positions, Σ_ι c_ι[d] e^{λ(63-ι)}
// p_ι[j] for the thread's eight columns j = jcol + 4 q (its tensor-core increment is zero).
template <bool REV>
__device__ __noinline__ void fast_increment(const Wkv5BwdSmem& sm, const __nv_bfloat16* stC, int d, int jcol, int lo,
                                            float (&dsf)[8]) {
#pragma unroll
  for (int q = 0; q < 8; ++q) dsf[q] = 0.f;
#pragma unroll
  for (int n = 0; n <= kBand; ++n) {
    const int io = kL - 1 - n;
    if (io >= lo) {
      const float cw = __bfloat162float(stC[(REV ? kL - 1 - io : io) * kN + d]) * sm.EB[n][d];
#pragma unroll
      for (int q = 0; q < 8; ++q) dsf[q] = fmaf(cw, sm.opPt[op_off(jcol + 4 * q, io)], dsf[q]);
    }
  }
}

// A fast row's epilogue for 16 positions col.. (z: its state read, unscaled; x3: the X_c read):
// out = e^{λ(pos-lo)} z + BF0 + u c A[pos][pos] into the output rows, and (reversed) the returned
// sum of its decay-gradient terms, m ((pos-lo) e^{λ(pos-1-lo)} z + BF1) + f3 c x3.  Out of line, so
// that heads without fast rows run the main epilogue untouched.
template <bool REV>
__device__ __noinline__ float fast_epilogue(const Wkv5BwdSmem& sm, const __nv_bfloat16* stC,
                                            const __nv_bfloat16* stM, __nv_bfloat16* stO, const float* BF0,
                                            const float* BF1, const float (&z)[16], const float (&x3)[16], int col,
                                            int lo, int cnt, int de, float lam_e, float u_e) {
  float accf = 0.f;
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const int pos = col + i;
    if (pos < lo || pos >= cnt) continue;
    const int so = (REV ? kL - 1 - pos : pos) * kN + de;
    const float cval = __bfloat162float(stC[so]), mval = __bfloat162float(stM[so]);
    const float fr = pos == lo ? 1.f : __expf(lam_e * (float)(pos - lo));
    stO[so] = __float2bfloat16_rn(fmaf(u_e * cval, sm.diag[pos], fmaf(fr, z[i], BF0[pos * kN + de])));
    if constexpr (REV) {
      const float fz = pos > lo ? (float)(pos - lo) * __expf(lam_e * (float)(pos - 1 - lo)) : 0.f;
      const float f3 = pos < kL - 1 ? (float)(kL - 1 - pos) * __expf(lam_e * (float)(kL - 2 - pos)) : 0.f;
      accf = fmaf(mval, fmaf(fz, z[i], BF1[pos * kN + de]), accf);
      accf = fmaf(f3 * cval, x3[i], accf);
    }
  }
  return accf;
}

template <bool REV>
__global__ void __launch_bounds__(kThreads, REV ? 1 : 2) wkv5_bwd_tc_kernel(const __grid_constant__ CUtensorMap mq,
                                                                          const __grid_constant__ CUtensorMap mp,
                                                                          const __grid_constant__ CUtensorMap mc,
                                                                          Wkv5BwdParams p) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  const uint32_t base_s = smem_u32(smem_raw);
  Wkv5BwdSmem& sm = *reinterpret_cast<Wkv5BwdSmem*>(smem_raw + ((1024u - (base_s & 1023u)) & 1023u));
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int t4 = lane >> 2, tq = lane & 3;
  const int q4 = warp & 3, hc = warp >> 2;  // TMEM lane quarter and column half of this warp
  const int b = blockIdx.x / p.H, h = blockIdx.x % p.H;
  const int nchunk = (p.T + p.lead + kL - 1) / kL;
  const float* om = p.omega + h * kN;
  const size_t sbase = ((size_t)b * p.H + h) * kN * kN;

  if (tid == 0) sm.abort_flag = 0;
  if constexpr (REV) {
    if (tid < kN) sm.red[tid] = 0.0;
  }
  // fast rows (rate > 2) stay out of the factorized products (their c̃ᵀ row is zero); their
  // intra-chunk terms and state increment are summed on the CUDA cores over lags 0..kBand
  bool fast_any = false;
  if (tid < kN) {
    const float lam = -expf(om[tid]);
    fast_any = !(-lam <= kMaxRate);
#pragma unroll 1
    for (int n = 0; n <= kBand; ++n) sm.EB[n][tid] = n == 0 ? 1.f : expf(lam * (float)n);
  }
  if (tid == 0) {  // the fast rows in order (once per CTA)
    int nf = 0;
    for (int d = 0; d < kN; ++d)
      if (!(expf(om[d]) <= kMaxRate)) sm.flist[nf++] = d;
    sm.nfl = nf;
  }
  const bool nfast = __syncthreads_or(fast_any) != 0;

  if (warp == 0) tmem_alloc(&sm.tmem_base, REV ? 512u : 256u);
  const bool withheld = tid == 0 && loads_withheld(p.ctl);
  // chunk c covers positions [c*64 - lead, c*64 - lead + 64) of the pass's own time
  // the box of chunk c starts at token 64 c (forward pass) or 64 (nchunk-1-c) (reversed pass)
  if (tid == 0) {
    prefetch_tensormap(&mq);
    prefetch_tensormap(&mp);
    prefetch_tensormap(&mc);
    mbar_init(&sm.bar_tma, 1);
    mbar_init(&sm.bar_sc, 1);
    mbar_init(&sm.bar_av, REV ? 2 : 1);  // reversed: the intra and lag-weighted chains commit apart
    mbar_init(&sm.bar_ds, 1);
    mbar_init(&sm.bar_ck, 1);
    fence_mbar_init();
    mbar_arrive_expect_tx(&sm.bar_tma, 3 * kRawBytes);
    if (!withheld) {
      const int row0 = REV ? kL * (nchunk - 1) : 0;
      tma_load_3d(sm.raw[0], &mq, &sm.bar_tma, h * kN, row0, b);
      tma_load_3d(sm.raw[1], &mp, &sm.bar_tma, h * kN, row0, b);
      tma_load_3d(sm.raw[2], &mc, &sm.bar_tma, h * kN, row0, b);
    }
    if constexpr (REV) {
      mbar_arrive_expect_tx(&sm.bar_ck, kCkBytes);
      if (!withheld) bulk_load(sm.opXc, ckpt_at(p, b, h, nchunk, nchunk - 1), kCkBytes, &sm.bar_ck);
    }
  }

  // ---- q, p (shared memory, unscaled): warp w owns channels 8w..8w+7, lane holds positions
  // 8 ib + rr, channels dR, dR + 1; a half-warp writes one whole core matrix.  Position τ is box
  // row τ, or 63 - τ in the reversed pass.
  const int rr = lane & 7, rp = lane >> 3;
  const int dR = 8 * warp + 2 * rp;
  const int rb = REV ? 7 - rr : rr;
  const uint32_t offRK = (uint32_t)rb * 128u + (uint32_t)((warp ^ rb) << 4) + (uint32_t)rp * 4u;
  const int lrow = lane & 7, lmat = lane >> 3;
  // ---- pᵀ (shared memory): ldmatrix.trans of block column w; lanes whose bit 1 and bit 4 differ
  // trade their pair with lane ^ 18 so that each half-warp covers one core matrix
  const int sw = ((lane >> 1) ^ (lane >> 4)) & 1;
  const int srow = t4 ^ (sw << 2), stq = tq ^ (sw << 1);
  const uint32_t offT = REV ? (uint32_t)(63 - lmat * 8 - lrow) * 128u + (uint32_t)((warp ^ (7 - lrow)) << 4)
                            : (uint32_t)(lmat * 8 + lrow) * 128u + (uint32_t)((warp ^ lrow) << 4);
  // ---- c̃ᵀ (tensor memory, A of the intra term and of the state increment), .16x256b fragment:
  // rows d = 16 q4 + t4 + 8 r, columns ι = 32 hc + 8 i + 2 tq + e  ->  register 4 i + 2 r + e
  float fc0[2][2], fcs[2];
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    const float rate = expf(om[16 * q4 + 8 * r + t4]);
    const bool fr = !(rate <= kMaxRate);  // a fast row: zero, its terms are formed elsewhere
#pragma unroll
    for (int e = 0; e < 2; ++e) fc0[r][e] = fr ? 0.f : expf(-rate * (float)(31 - 32 * hc - 2 * tq - e));
    fcs[r] = fr ? 0.f : expf(8.f * rate);
  }
  const uint32_t offKt =
      REV ? (uint32_t)(63 - (4 * hc + (lmat >> 1)) * 8 - lrow) * 128u + (uint32_t)(((2 * q4 + (lmat & 1)) ^ (7 - lrow)) << 4)
          : (uint32_t)((4 * hc + (lmat >> 1)) * 8 + lrow) * 128u + (uint32_t)(((2 * q4 + (lmat & 1)) ^ lrow) << 4);

  // ---- carried state X[d][j] (fp32) in the .16x128b fragment: d = 16 q4 + t4 + 8 r,
  // j = 32 hc + 4 q + tq  ->  X[2 q + r]
  const int drow = 16 * q4 + t4;
  const int jcol = 32 * hc + tq;
  const uint32_t tquar = (uint32_t)(32 * q4) << 16;
  float lamr[2], e32[2];
  bool fastR[2];
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    lamr[r] = -expf(om[drow + 8 * r]);
    e32[r] = expf(32.f * lamr[r]);
    fastR[r] = !(-lamr[r] <= kMaxRate);
  }
  float X[16];
#pragma unroll
  for (int q = 0; q < 8; ++q)
#pragma unroll
    for (int r = 0; r < 2; ++r)
      X[2 * q + r] = p.x0 ? p.x0[sbase + (size_t)(drow + 8 * r) * kN + jcol + 4 * q] : 0.f;
  // the carried state enters at position `lead` of the first chunk: its read factor is e^{(32-lead)λ}
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    // (a fast row is read unscaled: its factor e^{λ(τ-lo)} is applied to the output)
    const float f0 = fastR[r] ? 1.f : expf((32.f - (float)p.lead) * lamr[r]);
#pragma unroll
    for (int q = 0; q < 8; ++q) sm.opX[op_off(drow + 8 * r, jcol + 4 * q)] = to_tf32(f0 * X[2 * q + r]);
  }

  // ---- epilogue rows: lane < 16 of quarter q4 holds key row de = 16 q4 + lane, positions 32 hc + i
  const int de = 16 * q4 + (lane & 15);
  const float lam_e = -expf(om[de]);
  const bool fast_e = !(-lam_e <= kMaxRate);
  const float u_e = p.u[h * kN + de];
  double acc_e = 0.0;              // forward pass: the gu sum of row de; reversed: its decay-gradient terms
  double acc_t1[2] = {0.0, 0.0};   // reversed pass: the elementwise term of rows drow, drow + 8

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = sm.tmem_base;
  const uint32_t tA = tbase, tZ = tbase + 64, tDS = tbase + 128, tCt = tbase + 192;
  const uint32_t tI = tbase + 256, tX3 = tbase + 320, tX4 = tbase + 384;  // reversed pass only
  const uint32_t rawQ = smem_u32(sm.raw[0]), rawP = smem_u32(sm.raw[1]), rawC = smem_u32(sm.raw[2]);
  // staging rows [token][channel] bf16 of c (then out) and m, in opQ between the first chains and
  // the next chunk's conversion
  __nv_bfloat16* stC = reinterpret_cast<__nv_bfloat16*>(sm.opQ);
  __nv_bfloat16* stM = stC + kL * kN;
  // the output rows, in opP (free from the first chains' end to the next chunk's conversion), so
  // that c stays readable for the fast rows' terms
  __nv_bfloat16* stO = reinterpret_cast<__nv_bfloat16*>(sm.opP);
  const bool issuer = tid == 0;
  const bool ds_issuer = tid == 128;  // warp 4 (q4 = 0, hc = 1): its scores quarter lies above the diagonal

  int c = 0;
  bool aborted = false;
  // the chunk loop, in two instances: heads with fast rows take the one with their extra terms,
  // the others one without a trace of them
  auto chunks = [&](auto fast_tag) {
    constexpr bool FAST = decltype(fast_tag)::value;
    for (; c < nchunk; ++c) {
      const int t0 = c * kL - p.lead;            // pass position of position 0 of this chunk
      const int lo = max(0, -t0);                // positions before the sequence start (first reversed chunk)
      const int cnt = min(kL, p.T - t0);         // positions up to the sequence end (last forward chunk)
      const uint32_t ph = (uint32_t)c & 1u;
      const int cf = nchunk - 1 - c;             // reversed pass: the forward chunk this one mirrors

      // this chunk's box of c and m (tokens tb .. tb + 63, rows past the sequence end zero): two
      // 16-byte loads per tensor and thread, staged in shared memory for the epilogue after the first
      // chains have released opQ
      const int tb = REV ? kL * cf : t0;
      const int nrow = min(kL, p.T - tb);
      uint4 pre[2][2];
  #pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        const int row = 32 * hh + (tid >> 3);
        const size_t off = (((size_t)b * p.T + tb + row) * p.H + h) * kN + 8 * (tid & 7);
        const uint4 z = make_uint4(0u, 0u, 0u, 0u);
        pre[0][hh] = row < nrow ? __ldg(reinterpret_cast<const uint4*>(p.c + off)) : z;
        pre[1][hh] = row < nrow ? __ldg(reinterpret_cast<const uint4*>(p.m + off)) : z;
      }

      // forward pass: the state at this chunk's start is the checkpoint the reversed pass reads
      if constexpr (!REV) {
        float* ck = ckpt_at(p, b, h, nchunk, c);
  #pragma unroll
        for (int q = 0; q < 8; ++q)
  #pragma unroll
          for (int r = 0; r < 2; ++r) ck[op_off(drow + 8 * r, jcol + 4 * q)] = X[2 * q + r];
      } else {
        // X_c (the forward state at the mirrored chunk's start, copied into opXc) and the elementwise
        // term n w^{n-1} Σ_j G∘X_c with n = 64 - lo positions in the chunk
        if (!mbar_wait_bounded(&sm.bar_ck, ph, p.ctl)) sm.abort_flag = 1;
        float part[2] = {0.f, 0.f};
  #pragma unroll
        for (int q = 0; q < 8; ++q)
  #pragma unroll
          for (int r = 0; r < 2; ++r) {
            float& xc = sm.opXc[op_off(drow + 8 * r, jcol + 4 * q)];
            part[r] = fmaf(X[2 * q + r], xc, part[r]);
            xc = to_tf32(xc);  // the X_c read below takes it rounded to nearest
          }
        const float n = (float)(kL - lo);
  #pragma unroll
        for (int r = 0; r < 2; ++r) acc_t1[r] += (double)(n * (n == 1.f ? 1.f : expf((n - 1.f) * lamr[r])) * part[r]);
      }

      if (!mbar_wait_bounded(&sm.bar_tma, ph, p.ctl)) sm.abort_flag = 1;
      // T1a: q, p as fp32 operands (rows outside the sequence hold zeros from the TMA fill)
  #pragma unroll
      for (int ib = 0; ib < 8; ++ib) {
        const int row = 8 * ib + rr;
        const uint32_t ibo = (uint32_t)(REV ? 7 - ib : ib) * 1024u;
        *reinterpret_cast<float2*>(&sm.opQ[op_off(row, dR)]) = bf2_to_f2(lds_u32(rawQ + offRK + ibo));
        *reinterpret_cast<float2*>(&sm.opP[op_off(row, dR)]) = bf2_to_f2(lds_u32(rawP + offRK + ibo));
      }
      fence_proxy_async();
      tc_fence_before();
      __syncthreads();
      if (sm.abort_flag) {
        aborted = true;
        break;
      }
      // scores A = q pᵀ [τ][ι], state read (e^{32λ} X) qᵀ [d][τ], and (reversed) X_c pᵀ [d][ι]; the
      // issuing thread hands the K steps out in groups between its warp's T1b steps
      auto issue_first = [&](int s0) {
        if (issuer) {
          if (s0 == 0) tc_fence_after();
  #pragma unroll
          for (int s = s0; s < s0 + 2; ++s) {
            umma_tf32(tA, smem_desc(&sm.opQ[s * 64], kLbo, kSbo), smem_desc(&sm.opP[s * 64], kLbo, kSbo), kIdesc, s);
            umma_tf32(tZ, smem_desc(&sm.opX[s * 64], kLbo, kSbo), smem_desc(&sm.opQ[s * 64], kLbo, kSbo), kIdesc, s);
            if constexpr (REV)
              umma_tf32(tX3, smem_desc(&sm.opXc[s * 64], kLbo, kSbo), smem_desc(&sm.opP[s * 64], kLbo, kSbo), kIdesc,
                        s);
          }
          if (s0 == 6) umma_commit(&sm.bar_sc);
        }
      };
      issue_first(0);

      // T1b: c̃ᵀ into tensor memory, pᵀ into shared memory
      {
        uint32_t kt[16];
  #pragma unroll
        for (int pp = 0; pp < 2; ++pp) {
          uint32_t qk[4];
          ldsm_x4_t(REV ? rawC + offKt - pp * 2048u : rawC + offKt + pp * 2048u, qk);
  #pragma unroll
          for (int m = 0; m < 4; ++m) {
            const int i = 2 * pp + (m >> 1), r = m & 1;
            const float2 f = bf2_to_f2(qk[m]);
            const float g = i == 0 ? 1.f : (i == 1 ? fcs[r] : (i == 2 ? fcs[r] * fcs[r] : fcs[r] * fcs[r] * fcs[r]));
            kt[4 * i + 2 * r] = __float_as_uint(to_tf32(f.x * fc0[r][0] * g));
            kt[4 * i + 2 * r + 1] = __float_as_uint(to_tf32(f.y * fc0[r][1] * g));
          }
          issue_first(2 + 2 * pp);
        }
        tmem_st16(tCt + tquar + (uint32_t)(32 * hc), kt);
  #pragma unroll
        for (int pp = 0; pp < 2; ++pp) {
          uint32_t qv[4];
          ldsm_x4_t(REV ? rawP + offT - pp * 4096u : rawP + offT + pp * 4096u, qv);
  #pragma unroll
          for (int m = 0; m < 4; ++m) {
            const int ib = 4 * pp + m;
            const uint32_t xv = __shfl_xor_sync(0xffffffffu, qv[m], 18);
            *reinterpret_cast<float2*>(&sm.opPt[op_off(8 * warp + srow, 8 * ib + 2 * stq)]) =
                bf2_to_f2(sw ? xv : qv[m]);
          }
          if (pp == 0) issue_first(6);
        }
      }
      fence_proxy_async();
      tc_fence_before();
      __syncthreads();
      if (ds_issuer) {
        tc_fence_after();
        // state increment c̃ᵀ p [d][j]: needs only this chunk's operands, runs while the scores are
        // masked; issued from warp 4, whose share of the masking is a zero fill
  #pragma unroll
        for (int s = 0; s < 8; ++s) umma_tf32_ts(tDS, tCt + 8 * s, smem_desc(&sm.opPt[s * 64], kLbo, kSbo), kIdesc, s);
        umma_commit(&sm.bar_ds);
      }
      if (issuer) {
        // the raw boxes are consumed: load the next chunk while this one computes
        if (c + 1 < nchunk) {
          fence_proxy_async();
          mbar_arrive_expect_tx(&sm.bar_tma, 3 * kRawBytes);
          const int rown = REV ? kL * (cf - 1) : t0 + kL;
          tma_load_3d(sm.raw[0], &mq, &sm.bar_tma, h * kN, rown, b);
          tma_load_3d(sm.raw[1], &mp, &sm.bar_tma, h * kN, rown, b);
          tma_load_3d(sm.raw[2], &mc, &sm.bar_tma, h * kN, rown, b);
        }
      }

      // T2a: strictly causal scores -> opAm (and, reversed, weighted by the lag -> opAl); the diagonal
      // q_τ·p_τ -> diag.  .16x128b fragment: rows τ = 16 q4 + t4 + 8 r, columns ι = 32 hc + 4 q + tq
      if (!mbar_wait_bounded(&sm.bar_sc, ph, p.ctl)) sm.abort_flag = 1;
      tc_fence_after();
      // the first chains have read opQ, opP and opXc: c and m into the staging rows (opQ), and
      // (reversed) the next chunk's checkpoint into opXc
  #pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        const int row = 32 * hh + (tid >> 3);
        *reinterpret_cast<uint4*>(&stC[row * kN + 8 * (tid & 7)]) = pre[0][hh];
        *reinterpret_cast<uint4*>(&stM[row * kN + 8 * (tid & 7)]) = pre[1][hh];
      }
      if constexpr (REV) {
        if (issuer && c + 1 < nchunk) {
          fence_proxy_async();
          mbar_arrive_expect_tx(&sm.bar_ck, kCkBytes);
          bulk_load(sm.opXc, ckpt_at(p, b, h, nchunk, cf - 1), kCkBytes, &sm.bar_ck);
        }
      }
      {
        const int tau0 = 16 * q4 + t4;
        if (hc > (q4 >> 1)) {  // strictly above the diagonal
  #pragma unroll
          for (int q = 0; q < 8; ++q)
  #pragma unroll
            for (int r = 0; r < 2; ++r) {
              sm.opAm[op_off(tau0 + 8 * r, 32 * hc + 4 * q + tq)] = 0.f;
              if constexpr (REV) sm.opAl[op_off(tau0 + 8 * r, 32 * hc + 4 * q + tq)] = 0.f;
            }
        } else {
          float a[16];
          tmem_ld16x128(tA + tquar + (uint32_t)(32 * hc), a);
  #pragma unroll
          for (int q = 0; q < 8; ++q)
  #pragma unroll
            for (int r = 0; r < 2; ++r) {
              const int io = 32 * hc + 4 * q + tq, tau = tau0 + 8 * r;
              const float am = io < tau ? a[2 * q + r] : 0.f;
              sm.opAm[op_off(tau, io)] = to_tf32(am);
              if constexpr (REV) sm.opAl[op_off(tau, io)] = to_tf32((float)(tau - 1 - io) * am);
              if (io == tau) sm.diag[tau] = a[2 * q + r];
            }
        }
      }
      fence_proxy_async();
      tc_fence_before();
      __syncthreads();
      // intra term: forward pass into the state-read accumulator, reversed pass into its own (the
      // decay gradient weights the state read alone); reversed also the lag-weighted term, from a
      // second thread (bar_av then takes two commits)
      if (issuer) {
        tc_fence_after();
  #pragma unroll
        for (int s = 0; s < 8; ++s) {
          if constexpr (REV)
            umma_tf32_ts(tI, tCt + 8 * s, smem_desc(&sm.opAm[s * 64], kLbo, kSbo), kIdesc, s);
          else
            umma_tf32_ts(tZ, tCt + 8 * s, smem_desc(&sm.opAm[s * 64], kLbo, kSbo), kIdesc, 1);
        }
        umma_commit(&sm.bar_av);
      }
      if constexpr (REV) {
        if (ds_issuer) {
          tc_fence_after();
  #pragma unroll
          for (int s = 0; s < 8; ++s) umma_tf32_ts(tX4, tCt + 8 * s, smem_desc(&sm.opAl[s * 64], kLbo, kSbo), kIdesc, s);
          umma_commit(&sm.bar_av);
        }
      }

      // T2b: X <- e^{nλ} X + e^{32λ} (c̃ᵀ p) with n the positions since the state entered
      // (64 - lead in the first reversed chunk), or the partial last chunk's own form
      if (!mbar_wait_bounded(&sm.bar_ds, ph, p.ctl)) sm.abort_flag = 1;
      tc_fence_after();
      {
        float ds[16];
        tmem_ld16x128(tDS + tquar + (uint32_t)(32 * hc), ds);
        if (cnt == kL) {
  #pragma unroll
          for (int r = 0; r < 2; ++r) {
            const float gx = lo == 0 ? e32[r] * e32[r] : expf((float)(kL - lo) * lamr[r]);
  #pragma unroll
            for (int q = 0; q < 8; ++q) {
              const int x = 2 * q + r;
              X[x] = fmaf(gx, X[x], e32[r] * ds[x]);
              sm.opX[op_off(drow + 8 * r, jcol + 4 * q)] = to_tf32(e32[r] * X[x]);
            }
          }
          if (FAST) {
  #pragma unroll
            for (int r = 0; r < 2; ++r) {  // unrolled: X stays in registers
              if (!fastR[r]) continue;
              // a fast row (its tensor-core increment is zero): Σ_ι c_ι[d] e^{λ(63-ι)} p_ι[j] over the
              // chunk's last kBand + 1 positions, and the row read unscaled
              const int d = drow + 8 * r;
              float dsf[8];
              fast_increment<REV>(sm, stC, d, jcol, lo, dsf);
  #pragma unroll
              for (int q = 0; q < 8; ++q) {
                const int x = 2 * q + r;
                X[x] += dsf[q];
                sm.opX[op_off(d, jcol + 4 * q)] = to_tf32(X[x]);
              }
            }
          }
        } else {  // partial last chunk (forward pass): no later chunk reads opX
  #pragma unroll
          for (int r = 0; r < 2; ++r) {
            const float dl = expf(lamr[r] * (float)cnt), gs = expf(lamr[r] * (float)(cnt - 32));
  #pragma unroll
            for (int q = 0; q < 8; ++q) X[2 * q + r] = fmaf(dl, X[2 * q + r], gs * ds[2 * q + r]);
          }
        }
      }
      // T3: out[τ][de] = e^{λ(τ-32)} (state read + intra)[de][τ] + u c_τ A[τ][τ], and the sums; 16
      // positions at a time (lanes 0..15 of each quarter hold the rows of the M = 64 accumulators)
      if (!mbar_wait_bounded(&sm.bar_av, ph, p.ctl)) sm.abort_flag = 1;
      tc_fence_after();
      // fast rows: their intra-chunk terms over lags 0..kBand, by all threads (thread = position x one
      // quarter of the fast rows) into opPt (free after the fold) and, reversed, the lag-weighted ones
      // into opAl (free after the intra chains): BF0[pos][d] = Σ_n A[pos][pos-1-n] c_{pos-1-n}[d]
      // e^{λ_d n}, BF1[pos][d] = Σ_{n≥1} n A[pos][pos-1-n] c_{pos-1-n}[d] e^{λ_d (n-1)}
      float* BF0 = sm.opPt;
      float* BF1 = REV ? sm.opAl : nullptr;
      if (FAST) {
        __syncthreads();  // every fold has read opPt
        fast_band<REV>(sm, stC, BF0, BF1, lo);
        __syncthreads();
      }
  #pragma unroll 1
      for (int half = 0; half < 2; ++half) {
        const uint32_t col = (uint32_t)(32 * hc + 16 * half);
        float zv[16];
        [[maybe_unused]] float iv[REV ? 16 : 1], x3[REV ? 16 : 1], x4[REV ? 16 : 1];
        tmem_ld32x16(tZ + tquar + col, zv);
        if constexpr (REV) {
          tmem_ld32x16(tI + tquar + col, iv);
          tmem_ld32x16(tX3 + tquar + col, x3);
          tmem_ld32x16(tX4 + tquar + col, x4);
        }
        if (lane < 16) {
          float acc = 0.f;
  #pragma unroll
          for (int i = 0; i < 16; ++i) {
            const int pos = (int)col + i;
            if (pos < lo || pos >= cnt) continue;
            // staging row of this position (the box holds the tokens in forward order)
            const int so = (REV ? kL - 1 - pos : pos) * kN + de;
            const float cval = __bfloat162float(stC[so]), mval = __bfloat162float(stM[so]);
            const float dg = sm.diag[pos];
            const float f = __expf(lam_e * (float)(pos - 32));
            float o;
            if constexpr (REV) o = f * (zv[i] + iv[i]);
            else o = f * zv[i];
            o = fmaf(u_e * cval, dg, o);
            if constexpr (REV) {
              // position-weighted state read, lag-weighted intra term, and the X_c read (for a fast row
              // these are not its sums, which are formed below; its acc is dropped after the loop)
              const float f1 = __expf(lam_e * (float)(pos - 33));
              const float f3 = pos < kL - 1 ? (float)(kL - 1 - pos) * __expf(lam_e * (float)(kL - 2 - pos)) : 0.f;
              acc = fmaf(mval * f1, fmaf((float)(pos - lo), zv[i], x4[i]), acc);
              acc = fmaf(f3 * cval, x3[i], acc);
            } else {
              acc = fmaf(mval * cval, dg, acc);  // gu: r k (v·gy)
            }
            stO[so] = __float2bfloat16_rn(o);
          }
          if (FAST && fast_e) {
            // a fast row: its output and (reversed) its sums, out of line
            float zl[16], xl[16];
  #pragma unroll
            for (int t = 0; t < 16; ++t) {
              zl[t] = zv[t];
              xl[t] = REV ? x3[REV ? t : 0] : 0.f;
            }
            acc_e += (double)fast_epilogue<REV>(sm, stC, stM, stO, BF0, BF1, zl, xl, (int)col, lo, cnt, de, lam_e, u_e);
          }
          if constexpr (REV && FAST) acc_e += fast_e ? 0.0 : (double)acc;  // (the gu sum has no decay factor)
          else acc_e += (double)acc;
        }
      }
      // the chunk's out rows, 16 bytes a thread
      __syncthreads();
  #pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        const int row = 32 * hh + (tid >> 3);
        if (row < nrow)
          *reinterpret_cast<uint4*>(p.out + (((size_t)b * p.T + tb + row) * p.H + h) * kN + 8 * (tid & 7)) =
              *reinterpret_cast<const uint4*>(&stO[row * kN + 8 * (tid & 7)]);
      }

      __syncthreads();  // the staging rows (opQ) are read out before the next chunk converts q into it
    }
  };
  if (nfast)
    chunks(std::true_type{});
  else
    chunks(std::false_type{});

  if (aborted && tid == 0) {
    // a wait gave up at chunk c: the last MMA chains and this chunk's loads must finish before the
    // tensor memory and shared memory are released, each wait bounded again
    if (c >= 1) {  // the last chains of c-1 (bar_av, and bar_ds from the second issuer)
      mbar_wait_bounded(&sm.bar_av, (uint32_t)(c - 1) & 1u, p.ctl);
      mbar_wait_bounded(&sm.bar_ds, (uint32_t)(c - 1) & 1u, p.ctl);
    }
    if (!withheld) {
      mbar_wait_bounded(&sm.bar_tma, (uint32_t)c & 1u, p.ctl);
      if constexpr (REV) mbar_wait_bounded(&sm.bar_ck, (uint32_t)c & 1u, p.ctl);  // checkpoint copy c
    }
  }
  // per-row sums of the CTA: forward gu parts, reversed decay-gradient parts
  double* part = p.part + ((size_t)b * p.H + h) * kN;
  if constexpr (REV) {
    if (lane < 16) atomicAdd(&sm.red[de], acc_e);
    atomicAdd(&sm.red[drow], acc_t1[0]);
    atomicAdd(&sm.red[drow + 8], acc_t1[1]);
    __syncthreads();
    if (tid < kN) part[tid] = sm.red[tid];
  } else {
    // the two column halves (warps hc = 0, 1) of each row: combine through shared memory
    double* red = reinterpret_cast<double*>(sm.opAm);
    if (lane < 16 && hc == 1) red[de] = acc_e;
    __syncthreads();
    if (lane < 16 && hc == 0) part[de] = acc_e + red[de];
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tbase, REV ? 512u : 256u);
  }
}

// gomega[h][d] = Σ_b part_rev[b][h][d] · dw/dω (dw/dω = -e^ω w), gu[h][d] = Σ_b part_fwd[b][h][d], in
// batch order (deterministic).
__global__ void wkv5_reduce_kernel(int B, int H, const double* __restrict__ part_fwd,
                                   const double* __restrict__ part_rev, const float* __restrict__ omega,
                                   float* __restrict__ gomega, float* __restrict__ gu) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= H * kN) return;
  double sw = 0.0, su = 0.0;
  for (int bb = 0; bb < B; ++bb) {
    su += part_fwd[(size_t)bb * H * kN + i];
    sw += part_rev[(size_t)bb * H * kN + i];
  }
  const double e = exp((double)omega[i]);
  gomega[i] = (float)(sw * (-e * exp(-e)));
  gu[i] = (float)su;
}

}  // namespace

size_t wkv5_bwd_smem(bool rev) { return bwd_smem_bytes(rev); }

cudaError_t launch_wkv5_bwd_pass(bool rev, const CUtensorMap& mq, const CUtensorMap& mp, const CUtensorMap& mc,
                                 const Wkv5BwdParams& p, cudaStream_t st) {
  const size_t smem = bwd_smem_bytes(rev);
  static unsigned mask_f = 0, mask_r = 0;
  const void* fn = rev ? reinterpret_cast<const void*>(wkv5_bwd_tc_kernel<true>)
                       : reinterpret_cast<const void*>(wkv5_bwd_tc_kernel<false>);
  cudaError_t e = ensure_smem_attr(fn, (int)smem, rev ? &mask_r : &mask_f);
  if (e != cudaSuccess) return e;
  if (rev)
    wkv5_bwd_tc_kernel<true><<<(unsigned)(p.B * p.H), kThreads, smem, st>>>(mq, mp, mc, p);
  else
    wkv5_bwd_tc_kernel<false><<<(unsigned)(p.B * p.H), kThreads, smem, st>>>(mq, mp, mc, p);
  return cudaGetLastError();
}

cudaError_t launch_wkv5_bwd_reduce(int B, int H, const double* part_fwd, const double* part_rev, const float* omega,
                                   float* gomega, float* gu, cudaStream_t st) {
  wkv5_reduce_kernel<<<(H * kN + 127) / 128, 128, 0, st>>>(B, H, part_fwd, part_rev, omega, gomega, gu);
  return cudaGetLastError();
}

}  // namespace rwkv
