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
// every factor within e^{±32|λ|}: for -λ ≤ 2 (w ≥ 0.135) within e^{±64}, which
// leaves the small operands (a factor e^{-64} times a value down to 1e-10)
// clear of the subnormal range, where a tf32 operand keeps few bits.  A
// faster channel enters the products only where its factor is at most 1: its r̃
// column is r e^{λτ} with e^{λ·0} Sᵀ unscaled in opS (the state read), its k̃
// column is zero (no part in the scores), and its k̃ᵀ row is k e^{λ(cnt-1-ι)}
// (the state increment, folded without a further factor).  Its intra-chunk
// scores Σ_c r_τ[c] k_ι[c] e^{λ_c (τ-1-ι)} are added on the CUDA cores while the
// scores are masked, at lags τ-1-ι ≤ 15: beyond that e^{λn} < 2^-46 of the lag-0
// weight, far below the fp32 rounding of the output rows those terms would join.  Any w in [0, 1] is
// therefore handled on the same path, down to w = 0.
//
// The tensor core takes tf32 operands K-major only, so the operand tiles are
// fp32 [rows][64] in the K-major core-matrix layout without swizzle (8 rows x
// 16 bytes per core matrix); k̃ᵀ and vᵀ are transposed on the way in with
// ldmatrix.trans.  Each tcgen05.mma of these sizes costs its issuing thread
// about 70 cycles whatever M and N are, so the kernel uses the widest shapes
// the data allows (N = 128 for the first chain) and the issuing thread hands
// the first chain out in pairs between the other work of its warp.
//
// Work distribution (slot plan): the heads' chunks, laid end to end, are dealt
// out evenly to two CTAs per SM, so a CTA holds the tail of one head, whole
// heads and the start of another, in the order of a ticket it draws when it
// starts.  A CTA whose chunks end inside a head first scans them for a summary,
// the state they reach from a zero state,
//   Σ_t e^{λ (E-1-t)} k_tᵀ v_t   up to the end E of its chunks,
// accumulated in tensor memory chunk after chunk, and publishes it behind a
// flag; the CTAs holding the rest of that head wait for those flags (bounded)
// and fold the summaries in order into their start state,
//   S <- e^{64 n λ} S + summary  (n chunks per summary), from s_in.
// The reversed instance (the backward's gv pass) runs one whole head per CTA.
//
// CTA: 8 warps, about 113 KB of shared memory and 256 TMEM columns, two CTAs
// per SM.  Thread 0 issues the TMA loads of the raw r, k, v
// tiles (one [64 tokens x 64] bf16 box each, 128-byte swizzle, no multicast),
// the scores chain and the A v chain; a thread of warp 4 (whose share of the
// masking is a zero fill) issues the state-increment chain, so that the time
// that chain holds its issuing thread does not delay the masking barrier.  All
// warps build operands, mask the scores, fold the state and write the output
// rows.
#include <cstddef>

#include "launch.h"
#include "tc_common.cuh"
#include "wkv_common.cuh"

namespace rwkv {
namespace {

using namespace tc;

constexpr int kN = 64;                 // head size
constexpr int kL = 64;                 // tokens per chunk
constexpr int kThreads = 256;
constexpr uint32_t kRawBytes = kL * kN * 2;    // one bf16 [64 x 64] box
constexpr float kMaxRate = 2.f;        // largest -λ the chunked factorization takes
constexpr int kBand = 15;              // lags a fast channel keeps in the scores: e^{-2 (kBand+1)} < 2^-46
static_assert(kBand == 15, "the band pass gives each thread 4 of the 16 lags of one position");
constexpr uint32_t kTmemCols = 256;
constexpr unsigned int kSlotReady = 1u;   // a slot's summary is published
constexpr unsigned int kSlotGaveUp = 2u;  // a slot's wait gave up: it publishes no summary  // [scores | output rows], state increment, k̃ᵀ (64 columns each)

struct Wkv5Smem {
  alignas(1024) __nv_bfloat16 raw[3][kL * kN];  // r, k, v boxes [token][channel] (128-byte swizzle)
  alignas(128) float opR[64 * 64];   // r̃ = r e^{λ(τ-32)}   [τ][d]: A of the scores and of the state read
  alignas(128) float opK[64 * 64];   // k̃ = k e^{λ(31-ι)}   [ι][d]: B rows 0..63 of the first product
  alignas(128) float opS[64 * 64];   // e^{32λ} ⊙ Sᵀ         [j][d]: B rows 64..127 of the first product
  alignas(128) float opVt[64 * 64];  // vᵀ                   [j][ι]: B of A v and of the state increment
  union {
    float diag_part[8][kL];          // per-warp parts of Σ_d r u k (the bonus term), T1a -> T1b
    float AF[kL][kBand + 1];         // the fast channels' scores [τ][n = τ-1-ι], T1b (after the
  } u;                               // bonus sums) -> T2a
  float diag[kL];                    // Σ_d r u k per token
  // fast channels: r and k as bf16 pairs of fast indices [position][pair], rows padded to 33 words
  // (lanes on different rows meet different banks); KFw's extra row is zero: the k row of a lag
  // that reaches before the chunk
  uint32_t RFw[kL][kN / 2 + 1];
  uint32_t KFw[kL + 1][kN / 2 + 1];
  alignas(16) float E4[kN][4];           // e^{λ n} for n = 0, 4, 8, 12 [fast index][n / 4]
  float E1[kN];                          // e^{λ} [fast index]
  int fidx[kN];                          // fast index of each key channel, -1 for a slow one
  int flist[kN];                         // key channel of each fast index
  unsigned fmask[2];
  alignas(8) uint64_t bar_tma;
  alignas(8) uint64_t bar_sc;        // scores and state read done
  alignas(8) uint64_t bar_av;        // A v done
  alignas(8) uint64_t bar_ds;        // state increment done
  alignas(8) uint64_t bar_scan[3];   // a summary scan's k, v boxes, three stages
  alignas(8) uint64_t bar_scan_ds[4];  // a summary scan's products: [issuer][chunk parity]
  uint32_t tmem_base;
  int nfast;
  int abort_flag;
  int ticket;                        // the CTA's slot (slot plan)
};
// dynamic shared memory = the struct + 1024 bytes of alignment slack; an SM has 228 KB, of which
// each resident CTA also takes 1 KB: two CTAs per SM
static_assert(2 * (sizeof(Wkv5Smem) + 1024 + 1024) <= 228 * 1024, "two CTAs per SM");
static_assert(offsetof(Wkv5Smem, opS) == offsetof(Wkv5Smem, opK) + 64 * 64 * sizeof(float),
              "the first product reads k̃ and e^{32λ} Sᵀ as one 128-row operand");
static_assert(offsetof(Wkv5Smem, opR) % 1024 == 0 && offsetof(Wkv5Smem, opK) % 1024 == 0 && kRawBytes % 1024 == 0,
              "a summary scan loads 128-byte-swizzled boxes into the r̃ and k̃ tiles");

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
  const int nchunk = (p.T + kL - 1) / kL;
  // ---- the CTA's work.  Reversed, or without a slot plan: one whole head (blockIdx).  With a
  // plan, the heads' chunks laid end to end (head-major) are dealt out: slot s takes chunks
  // [F(s), F(s+1)) (F = p.slot_first), the tail of one head, whole heads and the start of
  // another.  s is a ticket drawn in the order the CTAs start, so a CTA only ever waits for slots
  // that are already running.
  const bool slots = !REV && p.nslot > 0;
  auto slot_first = [&](int s) { return (long long)p.slot_first[s]; };  // F(s)
  int slot = 0;
  long long f0 = (long long)blockIdx.x * nchunk, f1 = f0 + nchunk;
  if (slots) {
    if (tid == 0) sm.ticket = (int)atomicAdd(&p.slot_flag[p.nslot], 1u);
    __syncthreads();
    slot = sm.ticket;
    f0 = slot_first(slot);
    f1 = slot_first(slot + 1);
  }
  const int bh_first = (int)(f0 / nchunk);
  const int nseg = (int)((f1 - 1) / nchunk) - bh_first + 1;
  // segment k of the CTA: head bh_first + k, its chunks [cb, ce)
  auto seg_range = [&](int k, int& cb, int& ce) {
    const long long base = (long long)(bh_first + k) * nchunk;
    cb = (int)(max(f0, base) - base);
    ce = (int)(min(f1, base + nchunk) - base);
  };
  // when the last segment ends before its head does, the CTA first scans it for the summary that
  // the slots after it fold into their start states
  int last_cb, last_ce;
  seg_range(nseg - 1, last_cb, last_ce);
  const bool summary = slots && last_ce < nchunk;

  if (tid == 0) sm.abort_flag = 0;
  if (warp == 0) tmem_alloc(&sm.tmem_base, kTmemCols);
  // thread 0 issues every load; with the test hook set it arms the barriers and issues none
  const bool withheld = tid == 0 && loads_withheld(p.ctl);
  if (tid == 0) {
    prefetch_tensormap(&mr);
    prefetch_tensormap(&mk);
    prefetch_tensormap(&mv);
    mbar_init(&sm.bar_tma, 1);
    mbar_init(&sm.bar_sc, 1);
    mbar_init(&sm.bar_av, 1);
    mbar_init(&sm.bar_ds, 1);
    for (int st = 0; st < 3; ++st) mbar_init(&sm.bar_scan[st], 1);
    for (int x = 0; x < 4; ++x) mbar_init(&sm.bar_scan_ds[x], 1);
    fence_mbar_init();
  }

  // ---- r̃, k̃: warp w owns channels 8w..8w+7; lane holds token row 8 ib + rr, channels dR, dR + 1.
  // A half-warp then writes one whole core matrix (eight 16-byte rows): no bank conflicts.
  const int rr = lane & 7, rp = lane >> 3;
  const int dR = 8 * warp + 2 * rp;
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
  // position 32 hc + 8 (lmat >> 1) + lrow (+ 16 per pp); its box row bottom up when REV
  const uint32_t offKt =
      REV ? (uint32_t)(63 - (4 * hc + (lmat >> 1)) * 8 - lrow) * 128u + (uint32_t)(((2 * q4 + (lmat & 1)) ^ (7 - lrow)) << 4)
          : (uint32_t)((4 * hc + (lmat >> 1)) * 8 + lrow) * 128u + (uint32_t)(((2 * q4 + (lmat & 1)) ^ lrow) << 4);
  // ---- state S[d][j] (fp32 master copy) in the .16x128b fragment of warp w:
  // d = 16 q4 + t4 + 8 r, j = 32 hc + 4 q + tq  ->  S[2 q + r]
  const int drow = 16 * q4 + t4;
  const int jcol = 32 * hc + tq;
  const uint32_t tquar = (uint32_t)(32 * q4) << 16;

  // ---- per head: its fast channels and every thread's decay factors
  int b = 0, h = 0, nfast = 0;
  const float* om = p.omega;
  // r̃, k̃ build: a fast channel's r e^{λτ} (read only; its k̃ is zero, so it adds nothing to the scores)
  float fr0[2], frs[2], fk0[2], fks[2], uA[2];
  int fiA[2];
  // k̃ᵀ rows (a fast row's factor is e^{λ(cnt-1-ι)}, formed per chunk)
  float fc0[2][2], fcs[2], lamT[2];
  bool fastT[2];
  int fidxT[2];  // fast index of the row (-1: slow)
  float e32[2];  // e^{32λ} of the state rows
  auto setup_head = [&](int bh) {
    // the previous segment's reads of the tables, of tensor memory and of opS are done
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    b = bh / p.H;
    h = bh % p.H;
    om = p.omega + h * kN;
    // fast channels (-λ > 2): outside the factorization's range.  They enter the tensor-core
    // products only where the factor stays at most 1 (state read e^{λτ}, state increment
    // e^{λ(cnt-1-ι)}); their intra-chunk scores are summed on the CUDA cores over lags 0..kBand.
    for (int i = tid; i < (kL + 1) * (kN / 2 + 1); i += kThreads) {
      if (i < kL * (kN / 2 + 1)) (&sm.RFw[0][0])[i] = 0u;
      (&sm.KFw[0][0])[i] = 0u;
    }
    if (tid < kN) {  // the weights of an odd count's padding channel must read as zero too
#pragma unroll
      for (int g = 0; g < 4; ++g) sm.E4[tid][g] = 0.f;
      sm.E1[tid] = 0.f;
    }
    if (tid < kN) {
      const bool f = !(expf(om[tid]) <= kMaxRate);
      const unsigned m = __ballot_sync(0xffffffffu, f);
      if (lane == 0) sm.fmask[warp] = m;
    }
    __syncthreads();
    if (tid < kN) {
      const unsigned m0 = sm.fmask[0], m1 = sm.fmask[1];
      const bool f = ((tid < 32 ? m0 : m1) >> (tid & 31)) & 1u;
      const int below = tid < 32 ? __popc(m0 & ((1u << tid) - 1u)) : __popc(m0) + __popc(m1 & ((1u << (tid & 31)) - 1u));
      sm.fidx[tid] = f ? below : -1;
      if (f) {
        sm.flist[below] = tid;
        const float lam = -expf(om[tid]);
#pragma unroll
        for (int g = 0; g < 4; ++g) sm.E4[below][g] = g == 0 ? 1.f : expf(lam * (float)(4 * g));
        sm.E1[below] = expf(lam);
      }
      if (tid == 0) sm.nfast = __popc(m0) + __popc(m1);
    }
    __syncthreads();
    nfast = sm.nfast;
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const float rate = expf(om[dR + e]);  // -λ
      fiA[e] = sm.fidx[dR + e];
      fr0[e] = fiA[e] >= 0 ? (rr == 0 ? 1.f : expf(-rate * (float)rr)) : expf(-rate * (float)(rr - 32));
      frs[e] = expf(-8.f * rate);
      fk0[e] = fiA[e] >= 0 ? 0.f : expf(-rate * (float)(31 - rr));
      fks[e] = fiA[e] >= 0 ? 0.f : expf(8.f * rate);
      uA[e] = p.u[h * kN + dR + e];
    }
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      const float rate = expf(om[16 * q4 + 8 * r + t4]);
      lamT[r] = -rate;
      fidxT[r] = sm.fidx[16 * q4 + 8 * r + t4];
      fastT[r] = fidxT[r] >= 0;
#pragma unroll
      for (int e = 0; e < 2; ++e) fc0[r][e] = fastT[r] ? 0.f : expf(-rate * (float)(31 - 32 * hc - 2 * tq - e));
      fcs[r] = fastT[r] ? 0.f : expf(8.f * rate);
      e32[r] = expf(-32.f * expf(om[drow + 8 * r]));
    }
  };
  float S[16];
  auto load_s_in = [&]() {
    const size_t sb = ((size_t)b * p.H + h) * kN * kN;
#pragma unroll
    for (int q = 0; q < 8; ++q)
#pragma unroll
      for (int r = 0; r < 2; ++r) S[2 * q + r] = p.s_in ? p.s_in[sb + (size_t)(drow + 8 * r) * kN + jcol + 4 * q] : 0.f;
  };

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = sm.tmem_base;
  const uint32_t tSc = tbase, tY = tbase + 64, tDS = tbase + 128, tKt = tbase + 192;
  const uint32_t rawR = smem_u32(sm.raw[0]), rawK = smem_u32(sm.raw[1]), rawV = smem_u32(sm.raw[2]);
  const bool issuer = tid == 0;
  const bool ds_issuer = tid == 128;  // warp 4 (q4 = 0, hc = 1): its scores quarter lies above the diagonal
  static_assert(kThreads > 128, "the state-increment chain's issuing thread");

  // k̃ᵀ fragment from the k box at kbox, step pp of two: a slow row's k e^{λ(31-ι)} (a fast row's
  // factor is zero here)
  auto kt_slow = [&](int pp, uint32_t(&kt)[16], uint32_t kbox) {
    uint32_t qk[4];
    ldsm_x4_t(REV ? kbox + offKt - pp * 2048u : kbox + offKt + pp * 2048u, qk);
#pragma unroll
    for (int m = 0; m < 4; ++m) {
      const int i = 2 * pp + (m >> 1), r = m & 1;
      const float2 f = bf2_to_f2(qk[m]);
      const float g = i == 0 ? 1.f : (i == 1 ? fcs[r] : (i == 2 ? fcs[r] * fcs[r] : fcs[r] * fcs[r] * fcs[r]));
      kt[4 * i + 2 * r] = __float_as_uint(f.x * fc0[r][0] * g);
      kt[4 * i + 2 * r + 1] = __float_as_uint(f.y * fc0[r][1] * g);
    }
  };
  // a fast row of k̃ᵀ: k e^{λ(cnt-1-ι)} at the chunk's last kBand + 1 positions, zero past the
  // chunk's tokens; before those positions the weight is below 2^-46 and kt_slow has left the
  // entry at zero, so a warp whose positions (32 hc + 16 pp .. + 15 in step pp) all lie before
  // them skips the step
  auto kt_fast = [&](int cnt, uint32_t(&kt)[16], uint32_t kbox) {
#pragma unroll
    for (int pp = 0; pp < 2; ++pp) {
      if (32 * hc + 16 * pp + 15 < cnt - 1 - kBand) continue;
      uint32_t qk[4];
      ldsm_x4_t(REV ? kbox + offKt - pp * 2048u : kbox + offKt + pp * 2048u, qk);
#pragma unroll
      for (int m = 0; m < 4; ++m) {
        const int i = 2 * pp + (m >> 1), r = m & 1;
        if (fastT[r]) {
          const float2 f = bf2_to_f2(qk[m]);
          const int io = 32 * hc + 8 * i + 2 * tq;
          // e^{λ n}, n = cnt-1-ι: the tabled powers up to n = 15, zero beyond (below 2^-46)
          const int cf = fidxT[r];
          const float e1 = sm.E1[cf];
          auto pw = [&](int n) {
            if (n < 0 || n > kBand) return 0.f;
            const float x = sm.E4[cf][n >> 2];
            const int q = n & 3;
            return q == 0 ? x : (q == 1 ? x * e1 : (q == 2 ? x * e1 * e1 : x * e1 * e1 * e1));
          };
          kt[4 * i + 2 * r] = __float_as_uint(f.x * pw(cnt - 1 - io));
          kt[4 * i + 2 * r + 1] = __float_as_uint(f.y * pw(cnt - 2 - io));
        }
      }
    }
  };
  // vᵀ from the v box at vbox into the tile vt (opVt; a summary scan alternates with opS), step pp of two
  auto vt_step = [&](int pp, uint32_t vbox, float* vt) {
    uint32_t qv[4];
    ldsm_x4_t(REV ? vbox + offT - pp * 4096u : vbox + offT + pp * 4096u, qv);
#pragma unroll
    for (int m = 0; m < 4; ++m) {
      const int ib = 4 * pp + m;
      const uint32_t xv = __shfl_xor_sync(0xffffffffu, qv[m], 18);
      *reinterpret_cast<float2*>(&vt[op_off(8 * warp + srow, 8 * ib + 2 * stq)]) = bf2_to_f2(sw ? xv : qv[m]);
    }
  };

  // counts the abort path needs: output-pass chunks begun, chains committed, load batches armed
  int m_it = 0, n_ds = 0, n_av = 0, tma_armed = 0;
  int scan_loaded = 0;  // chunks of the summary scan whose loads were issued (chunk i in stage i % 3)
  int scan_done = 0;    // chunks of the summary scan whose products were issued
  bool aborted = false;

  if (summary) {
    // ---- the summary of the last segment: the state its chunks reach from a zero state,
    // Σ_t e^{λ(E-1-t)} k_tᵀ v_t up to its end E, accumulated in tensor memory chunk after chunk
    // (no fold).  Its k, v boxes arrive three chunks ahead in the raw k, v boxes and in the r̃, k̃
    // operand tiles, which the scan does not use; k̃ᵀ alternates between two tensor-memory tiles.
    setup_head(bh_first + nseg - 1);
    load_s_in();  // kept through the scan: s_out may be s_in, so it is read before the summary goes out
    const int n = last_ce - last_cb;  // whole chunks: the segment ends before its head does
    // stage st: its k box, its v box 8 KB after it (the raw boxes are adjacent too)
    auto stage_k = [&](int st) {
      return st == 0 ? reinterpret_cast<unsigned char*>(sm.raw[1])
                     : reinterpret_cast<unsigned char*>(st == 1 ? sm.opR : sm.opK);
    };
    static_assert(offsetof(Wkv5Smem, raw) + 3 * kRawBytes == offsetof(Wkv5Smem, opR), "raw boxes, then opR");
    auto scan_load = [&](int i) {  // chunk i of the segment into stage i % 3 (thread 0)
      const int st = i % 3, row = (last_cb + i) * kL;
      fence_proxy_async();
      mbar_arrive_expect_tx(&sm.bar_scan[st], 2 * kRawBytes);
      if (!withheld) {
        tma_load_3d(stage_k(st), &mk, &sm.bar_scan[st], h * kN, row, b);
        tma_load_3d(stage_k(st) + kRawBytes, &mv, &sm.bar_scan[st], h * kN, row, b);
      }
    };
    for (; scan_loaded < min(3, n); ++scan_loaded)
      if (issuer) scan_load(scan_loaded);
    // Chunk i's k̃ᵀ and vᵀ go to tile pair i & 1 ((tKt, opVt) or (tSc, opS)), so that a chunk is
    // built while the one before it is multiplied.  The eight K steps are split between two
    // issuing threads with an accumulator each (steps 0..3 by thread 0 into tY, 4..7 by warp 4's
    // into tDS, added at the end): each MMA holds its issuing thread ~70 cycles, and neither
    // warp then falls far behind the others' share of the next build.  Each issuer commits to
    // the barrier of its chunk parity, bar_scan_ds[2 x + (i & 1)], once per two chunks.
    auto scan_bar = [&](int x, int i) { return &sm.bar_scan_ds[2 * x + (i & 1)]; };
    for (int i = 0; i < n; ++i) {
      const int st = i % 3;
      const uint32_t tk = (i & 1) ? tSc : tKt;
      float* const vt = (i & 1) ? sm.opS : sm.opVt;
      if (!mbar_wait_bounded(&sm.bar_scan[st], (uint32_t)(i / 3) & 1u, p.ctl)) sm.abort_flag = 1;
      if (i >= 2) {  // chunk i - 2's products have read this tile pair
        const uint32_t par = (uint32_t)((i - 2) >> 1) & 1u;
        if (!mbar_wait_bounded(scan_bar(0, i), par, p.ctl) || !mbar_wait_bounded(scan_bar(1, i), par, p.ctl))
          sm.abort_flag = 1;
      }
      {
        uint32_t kt[16];
        const uint32_t kbox = smem_u32(stage_k(st));
        kt_slow(0, kt, kbox);
        kt_slow(1, kt, kbox);
        // a slow row's k e^{λ(31-ι)} times e^{λ(32 + 64 (n-1-i))}: the weight e^{λ(E-1-t)}
        const float rest = (float)(32 + kL * (n - 1 - i));
#pragma unroll
        for (int r = 0; r < 2; ++r) {
          const float sc = expf(lamT[r] * rest);
#pragma unroll
          for (int x = 0; x < 4; ++x)
#pragma unroll
            for (int e = 0; e < 2; ++e)
              kt[4 * x + 2 * r + e] = __float_as_uint(__uint_as_float(kt[4 * x + 2 * r + e]) * sc);
        }
        // a fast row keeps the last 16 positions only (beyond, its weight is below 2^-46)
        if (nfast > 0 && i == n - 1) kt_fast(kL, kt, kbox);
        tmem_st16(tk + tquar + (uint32_t)(32 * hc), kt);
      }
      vt_step(0, smem_u32(stage_k(st)) + kRawBytes, vt);
      vt_step(1, smem_u32(stage_k(st)) + kRawBytes, vt);
      fence_proxy_async();
      tc_fence_before();
      __syncthreads();
      if (sm.abort_flag) {
        aborted = true;
        break;
      }
      if (issuer || ds_issuer) {
        tc_fence_after();
        const int x = issuer ? 0 : 1;
        const uint32_t acc = issuer ? tY : tDS;
#pragma unroll
        for (int s4 = 0; s4 < 4; ++s4) {
          const int s = 4 * x + s4;
          umma_tf32_ts(acc, tk + 8 * s, smem_desc(&vt[s * 64], kLbo, kSbo), kIdesc, (i > 0 || s4 > 0) ? 1u : 0u);
        }
        umma_commit(scan_bar(x, i));
      }
      ++scan_done;
      if (scan_loaded < n) {  // stage st is consumed: chunk i + 3 into it
        if (issuer) scan_load(scan_loaded);
        ++scan_loaded;
      }
    }
    if (!aborted) {
      const uint32_t par = (uint32_t)((n - 1) >> 1) & 1u;  // the last chunk's commits cover every earlier product
      if (!mbar_wait_bounded(scan_bar(0, n - 1), par, p.ctl) || !mbar_wait_bounded(scan_bar(1, n - 1), par, p.ctl))
        sm.abort_flag = 1;
      tc_fence_after();
      float sum[16], sum2[16];
      tmem_ld16x128(tDS + tquar + (uint32_t)(32 * hc), sum);
      tmem_ld16x128(tY + tquar + (uint32_t)(32 * hc), sum2);
      tc_fence_before();
      __syncthreads();
      aborted = sm.abort_flag != 0;
      if (!aborted) {
        // in the fragment order (thread tid's 16 entries S[0..15] at [tid][16]), which only this
        // kernel reads: four 16-byte stores here, four 16-byte loads for each fold
        float4* dst = reinterpret_cast<float4*>(p.slot_sum + (size_t)slot * kN * kN) + 4 * tid;
#pragma unroll
        for (int x = 0; x < 4; ++x)
          dst[x] = make_float4(sum[4 * x] + sum2[4 * x], sum[4 * x + 1] + sum2[4 * x + 1],
                               sum[4 * x + 2] + sum2[4 * x + 2], sum[4 * x + 3] + sum2[4 * x + 3]);
      }
    }
    // publish it, or that this slot gave up (the slots waiting for it then stop at once)
    __syncthreads();
    if (tid == 0) {
      __threadfence();
      flag_release(&p.slot_flag[slot], aborted ? kSlotGaveUp : kSlotReady);
    }
  }

  // ---- the outputs, segment by segment: the scanned one first (its s_in is already in S), then
  // the others in order
  for (int j = 0; j < nseg && !aborted; ++j) {
    const int k = summary ? (j == 0 ? nseg - 1 : j - 1) : j;
    int cb, ce;
    seg_range(k, cb, ce);
    const int bh = bh_first + k;
    if (summary && j == 0) {
      tc_fence_before();
      __syncthreads();
      tc_fence_after();
    } else {
      setup_head(bh);
      load_s_in();
    }
    if (cb > 0) {
      // the start state: s_in carried over the head's earlier chunks, which the slots before this
      // one have summarized.  Wait (bounded) for their flags, warp 0's lanes polling 32 at once.
      const long long hb = (long long)bh * nchunk;
      int s_lo = slot;  // the slot that holds the head's first chunk hb
      while (slot_first(s_lo) > hb) --s_lo;
      if (warp == 0) {
        bool ok = true;
        for (int s0 = s_lo; s0 < slot && ok; s0 += 32) {
          unsigned int fl = kSlotReady;
          if (s0 + lane < slot) fl = flag_wait_bounded(&p.slot_flag[s0 + lane], p.ctl);
          ok = __all_sync(0xffffffffu, fl == kSlotReady);
        }
        if (!ok && lane == 0) sm.abort_flag = 1;
      }
      __syncthreads();
      if (sm.abort_flag) {
        aborted = true;
        break;
      }
      // two summaries' loads in flight at once (a head spread over many CTAs folds many)
#pragma unroll 2
      for (int s2 = s_lo; s2 < slot; ++s2) {
        const long long a0 = max(slot_first(s2), hb), a1 = slot_first(s2 + 1);
        const float len = (float)((a1 - a0) * kL);
        const float4* src = reinterpret_cast<const float4*>(p.slot_sum + (size_t)s2 * kN * kN) + 4 * tid;
        float x[16];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float4 v = __ldcg(src + i);
          x[4 * i] = v.x;
          x[4 * i + 1] = v.y;
          x[4 * i + 2] = v.z;
          x[4 * i + 3] = v.w;
        }
#pragma unroll
        for (int r = 0; r < 2; ++r) {
          const float d = expf(lamT[r] * len);
#pragma unroll
          for (int q = 0; q < 8; ++q) S[2 * q + r] = fmaf(d, S[2 * q + r], x[2 * q + r]);
        }
      }
    }
    // e^{32λ} Sᵀ into opS for the first state read (a fast row's unscaled)
#pragma unroll
    for (int q = 0; q < 8; ++q)
#pragma unroll
      for (int r = 0; r < 2; ++r) sm.opS[op_off(jcol + 4 * q, drow + 8 * r)] = (fastT[r] ? 1.f : e32[r]) * S[2 * q + r];
    if (issuer) {
      mbar_arrive_expect_tx(&sm.bar_tma, 3 * kRawBytes);
      if (!withheld) {
        const int row0 = REV ? p.T - kL : cb * kL;
        tma_load_3d(sm.raw[0], &mr, &sm.bar_tma, h * kN, row0, b);
        tma_load_3d(sm.raw[1], &mk, &sm.bar_tma, h * kN, row0, b);
        tma_load_3d(sm.raw[2], &mv, &sm.bar_tma, h * kN, row0, b);
      }
    }
    ++tma_armed;

    for (int c = cb; c < ce; ++c, ++m_it) {
      const int t0 = c * kL;
      const int cnt = min(kL, p.T - t0);
      const uint32_t ph = (uint32_t)m_it & 1u;  // bar_tma, bar_sc, bar_av: the output pass's chunks
      const uint32_t pg = (uint32_t)n_ds & 1u;  // bar_ds: the output pass's state increments
      if (!mbar_wait_bounded(&sm.bar_tma, ph, p.ctl)) sm.abort_flag = 1;

      // T1a: r̃, k̃ and the bonus parts (rows past the sequence end hold zeros from the TMA fill).
      // r̃ and k̃ are rounded to nearest tf32: the tensor core would truncate both, and the two
      // biases toward zero add in every score.
      {
        float fr[2] = {fr0[0], fr0[1]}, fk[2] = {fk0[0], fk0[1]};
#pragma unroll
        for (int ib = 0; ib < 8; ++ib) {
          const uint32_t ibo = (uint32_t)(REV ? 7 - ib : ib) * 1024u;
          const float2 rv = bf2_to_f2(lds_u32(rawR + offRK + ibo));
          const float2 kv = bf2_to_f2(lds_u32(rawK + offRK + ibo));
          const int row = 8 * ib + rr;
          *reinterpret_cast<float2*>(&sm.opR[op_off(row, dR)]) = make_float2(to_tf32(rv.x * fr[0]), to_tf32(rv.y * fr[1]));
          *reinterpret_cast<float2*>(&sm.opK[op_off(row, dR)]) = make_float2(to_tf32(kv.x * fk[0]), to_tf32(kv.y * fk[1]));
          float part = fmaf(rv.x * uA[0], kv.x, rv.y * uA[1] * kv.y);
          part += __shfl_xor_sync(0xffffffffu, part, 8);
          part += __shfl_xor_sync(0xffffffffu, part, 16);
          if (rp == 0) sm.u.diag_part[warp][row] = part;
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            fr[e] *= frs[e];
            fk[e] *= fks[e];
          }
        }
      }
      if (nfast > 0) {  // the fast channels' r and k into the compact rows (bf16 as loaded)
#pragma unroll
        for (int ib = 0; ib < 8; ++ib) {
          const uint32_t ibo = (uint32_t)(REV ? 7 - ib : ib) * 1024u;
          const uint32_t rw = lds_u32(rawR + offRK + ibo), kw = lds_u32(rawK + offRK + ibo);
          const int row = 8 * ib + rr;
#pragma unroll
          for (int e = 0; e < 2; ++e)
            if (fiA[e] >= 0) {
              const int col = fiA[e] >> 1;
              unsigned short* rh = reinterpret_cast<unsigned short*>(&sm.RFw[row][col]) + (fiA[e] & 1);
              unsigned short* kh = reinterpret_cast<unsigned short*>(&sm.KFw[row][col]) + (fiA[e] & 1);
              *rh = (unsigned short)(e ? rw >> 16 : rw & 0xFFFFu);
              *kh = (unsigned short)(e ? kw >> 16 : kw & 0xFFFFu);
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
          for (int w = 0; w < 8; ++w) sum += sm.u.diag_part[w][tid];
          sm.diag[tid] = sum;
        }
        uint32_t kt[16];
#pragma unroll
        for (int pp = 0; pp < 2; ++pp) {
          kt_slow(pp, kt, rawK);
          issue_first(2 + 2 * pp);
        }
        if (nfast > 0) {
          // the fast channels' scores at lags n = 0..kBand, Σ_c r_τ[c] k_{τ-1-n}[c] e^{λ_c n}: thread
          // (τ, 4 lags), every CTA thread busy; AF overlays the bonus parts, summed above
          __syncthreads();
          const int tau = tid >> 2, g4 = tid & 3, n0 = 4 * g4;
          // k rows of the four lags (a lag reaching before the chunk reads the zero row)
          const uint32_t* kp[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int io = tau - 1 - (n0 + e);
            kp[e] = &sm.KFw[io < 0 ? kL : io][0];
          }
          const uint32_t* rp = &sm.RFw[tau][0];
          float acc[4] = {0.f, 0.f, 0.f, 0.f};
          const int npair = (nfast + 1) >> 1;
#pragma unroll 2
          for (int w = 0; w < npair; ++w) {
            const float2 rv = bf2_to_f2(rp[w]);
            float ew[2][4];
#pragma unroll
            for (int h2 = 0; h2 < 2; ++h2) {
              const int cfi = 2 * w + h2;
              const float e1 = sm.E1[cfi];
              ew[h2][0] = sm.E4[cfi][g4];
              ew[h2][1] = ew[h2][0] * e1;
              ew[h2][2] = ew[h2][1] * e1;
              ew[h2][3] = ew[h2][2] * e1;
            }
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const float2 kv = bf2_to_f2(kp[e][w]);
              acc[e] = fmaf(rv.x * kv.x, ew[0][e], acc[e]);
              acc[e] = fmaf(rv.y * kv.y, ew[1][e], acc[e]);
            }
          }
#pragma unroll
          for (int e = 0; e < 4; ++e) sm.u.AF[tau][n0 + e] = acc[e];
        }
        if (nfast > 0) kt_fast(cnt, kt, rawK);
        tmem_st16(tKt + tquar + (uint32_t)(32 * hc), kt);
#pragma unroll
        for (int pp = 0; pp < 2; ++pp) {
          vt_step(pp, rawV, sm.opVt);
          if (pp == 0) issue_first(6);
        }
      }
      fence_proxy_async();
      tc_fence_before();
      __syncthreads();
      if (ds_issuer) {
        tc_fence_after();
        // ΔS = k̃ᵀ v [d][j] needs only this chunk's operands: it runs while the scores are masked.
        // Issued from warp 4, whose share of the masking is a zero fill, so that the ≈ 0.9k cycles
        // the chain holds its issuing thread do not delay the masking barrier.
#pragma unroll
        for (int s = 0; s < 8; ++s) umma_tf32_ts(tDS, tKt + 8 * s, smem_desc(&sm.opVt[s * 64], kLbo, kSbo), kIdesc, s);
        umma_commit(&sm.bar_ds);
      }
      ++n_ds;
      if (issuer) {
        // the raw boxes are consumed: load the next chunk while this one computes
        if (c + 1 < ce) {
          fence_proxy_async();
          mbar_arrive_expect_tx(&sm.bar_tma, 3 * kRawBytes);
          const int rown = REV ? p.T - (c + 2) * kL : (c + 1) * kL;
          tma_load_3d(sm.raw[0], &mr, &sm.bar_tma, h * kN, rown, b);
          tma_load_3d(sm.raw[1], &mk, &sm.bar_tma, h * kN, rown, b);
          tma_load_3d(sm.raw[2], &mv, &sm.bar_tma, h * kN, rown, b);
        }
      }
      if (c + 1 < ce) ++tma_armed;

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
          if (nfast > 0) {  // the fast channels' scores at lags 0..kBand (formed in T1b)
#pragma unroll
            for (int q = 0; q < 8; ++q)
#pragma unroll
              for (int r = 0; r < 2; ++r) {
                const int io = 32 * hc + 4 * q + tq, tau = tau0 + 8 * r, n = tau - 1 - io;
                if (n >= 0 && n <= kBand) a[2 * q + r] += sm.u.AF[tau][n];
              }
          }
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
      ++n_av;

      // T2b: S <- e^{cnt λ} S + e^{(cnt-32) λ} ΔS; e^{32λ} Sᵀ into opS for the next chunk (while A v
      // still runs).  A fast row's ΔS already carries e^{λ(cnt-1-ι)}, and its opS row is S itself.
      if (!mbar_wait_bounded(&sm.bar_ds, pg, p.ctl)) sm.abort_flag = 1;
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
              if (fastT[r]) {
                S[x] = fmaf(g * g, S[x], ds[x]);
                sm.opS[op_off(jcol + 4 * q, drow + 8 * r)] = S[x];
              } else {
                S[x] = g * fmaf(g, S[x], ds[x]);
                sm.opS[op_off(jcol + 4 * q, drow + 8 * r)] = g * S[x];
              }
            }
        } else {  // last, partial chunk: no later chunk reads opS
#pragma unroll
          for (int r = 0; r < 2; ++r) {
            const float rate = expf(om[drow + 8 * r]);
            const float dl = expf(-rate * (float)cnt), gs = fastT[r] ? 1.f : expf(-rate * (float)(cnt - 32));
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
    if (aborted) break;
    if (ce == nchunk && p.s_out != nullptr) {  // the head's last chunk: its final state
      const size_t sb = ((size_t)b * p.H + h) * kN * kN;
#pragma unroll
      for (int q = 0; q < 8; ++q)
#pragma unroll
        for (int r = 0; r < 2; ++r) p.s_out[sb + (size_t)(drow + 8 * r) * kN + jcol + 4 * q] = S[2 * q + r];
    }
  }

  if (aborted && tid == 0) {
    // a wait gave up: what was issued before it must finish before the tensor memory and shared
    // memory are released, each wait bounded again: the last A v and state-increment chains (a
    // commit covers every earlier chain of its issuing thread), the last batch of output-pass
    // loads and each scan stage's last loads
    if (n_av > 0) mbar_wait_bounded(&sm.bar_av, (uint32_t)(n_av - 1) & 1u, p.ctl);
    if (n_ds > 0) mbar_wait_bounded(&sm.bar_ds, (uint32_t)(n_ds - 1) & 1u, p.ctl);
    for (int x = 0; x < 4; ++x) {  // the scan's products: commits on bar_scan_ds[x], one per chunk of parity x & 1
      const int uses = (scan_done + 1 - (x & 1)) / 2;
      if (uses > 0) mbar_wait_bounded(&sm.bar_scan_ds[x], (uint32_t)(uses - 1) & 1u, p.ctl);
    }
    if (!withheld) {
      if (tma_armed > 0) mbar_wait_bounded(&sm.bar_tma, (uint32_t)(tma_armed - 1) & 1u, p.ctl);
      for (int st = 0; st < min(3, scan_loaded); ++st)  // stage st's last load: its ((scan_loaded - 1 - st) / 3)-th
        mbar_wait_bounded(&sm.bar_scan[st], (uint32_t)((scan_loaded - 1 - st) / 3) & 1u, p.ctl);
    }
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
  // one CTA per slot, or per head
  const long long nblk = p.nslot > 0 && !reversed ? (long long)p.nslot : (long long)p.B * p.H;
  if (reversed)
    wkv5_fwd_tc_kernel<true><<<(unsigned)nblk, kThreads, smem, st>>>(mr, mk, mv, p);
  else
    wkv5_fwd_tc_kernel<false><<<(unsigned)nblk, kThreads, smem, st>>>(mr, mk, mv, p);
  return cudaGetLastError();
}


}  // namespace rwkv
