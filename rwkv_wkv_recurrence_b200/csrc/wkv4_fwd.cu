// RWKV-4 WKV forward kernels (sm_100a).
//
// Operator: "RWKV - Transformer 시대에 RNN을 재발명하다", Method / (2) Time-mixing
// (WKV), time-parallel formula and its recurrent form; identical formula in
// "RWKV: Reinventing RNNs for the Transformer Era" (flashpapers), 3. How It
// Works / The WKV Operator.  The time-parallel form is a decayed prefix sum of
// numerator and denominator, and "exp decay + sum" is associative: that is
// what lets each warp below scan its own 16 steps independently and have the
// pieces joined by a fold.
//
// Kernel shape.  A CTA owns 32 consecutive channels of one batch row (one
// thread per channel lane in each warp) over a range of time, processed in
// tiles of 64 steps.  The 4 warps split a tile into four 16-step segments:
//   1. each warp scans its segment from a zero state (segment summary),
//   2. each warp folds the CTA's running state with the summaries before its
//      segment (and all four, for the next tile),
//   3. each warp rescans its segment from that state and writes y (and, at
//      segment starts, the checkpoints the backward reads).
// k and v arrive in [64 x 32] boxes through a multi-stage TMA pipeline
// without multicast, so every input element is read from HBM once.
//
// Receptance gate (GATE).  The time-mixing output of the same page is
// o_t = W_o (σ(r_t) ⊙ WKV_t) ((2) and (4) Receptance Gating); W_o is a GEMM
// outside the operator, σ(r) ⊙ WKV is fused here: r arrives as a third box
// per stage and the rescan writes σ(r_t) WKV_t instead of WKV_t, so the gate
// costs one more input stream instead of a separate pass over y and r.
//
// Precision.  Steps inside a segment run in fp32 with the decay applied as
// e^{-w} = lh + ll (hi and lo fp32 parts), one power-of-two scale per segment;
// the running state carried from segment to segment is fp64.  So fp32 rounding
// accumulates over 16 steps at most, never over the whole sequence, which the
// backward's cancelling gradient terms would not tolerate.
#include "launch.h"
#include "wkv_common.cuh"

namespace rwkv {
namespace {

constexpr int kW = 4;           // warps per CTA = segments per tile
constexpr int kL = 16;          // steps per segment (= checkpoint interval)
constexpr int kTile = kW * kL;  // steps per tile

struct Summ {  // a segment scanned from a zero state, at scale 2^p
  float a, b, p, pad;
};

// Phase 1 of one segment: scan from a zero state at scale 2^p1, where p1 is
// at least every k log2 e of the segment (so all weights are <= 1).  Keeps
// the token weights for phase 3.
template <typename T, bool FULL>
__device__ __forceinline__ void seg_summary(const T* ks, const T* vs, int cnt, float lh, float ll, float& kmax,
                                            int& p1, float& la, float& lb, float (&E)[kL]) {
  float kk[kL];
  kmax = -INFINITY;
#pragma unroll
  for (int j = 0; j < kL; ++j) {
    if (FULL || j < cnt) {
      kk[j] = IO<T>::to_f(ks[j * 32]);
      kmax = fmaxf(kmax, kk[j] * kL2eHi);
    }
  }
  p1 = clamp_scale((int)fminf(fmaxf(ceilf(kmax), -(float)kScaleMax), (float)kScaleMax));
  const float p1f = (float)p1;
  la = 0.f;
  lb = 0.f;
#pragma unroll
  for (int j = 0; j < kL; ++j) {
    if (FULL || j < cnt) {
      const float e = tok_weight(kk[j], p1f);
      E[j] = e;
      la = decay_add(la, e * IO<T>::to_f(vs[j * 32]), lh, ll);
      lb = decay_add(lb, e, lh, ll);
    }
  }
}

// Phase 3 of one segment: rescan from the true state (a, b) at the segment's
// scale, weights E * f, writing y_j to ys[j * 32] (the segment's k rows in
// shared memory, which phase 1 has consumed).
// With GATE, rs holds the segment's r rows and y_j is multiplied by σ(r_j).
template <typename T, bool FULL, bool GATE>
__device__ __forceinline__ void seg_output(const T* vs, const T* rs, int cnt, const float (&E)[kL], float f,
                                           float U, float a, float b, float lh, float ll, T* ys) {
#pragma unroll
  for (int j = 0; j < kL; ++j) {
    if (FULL || j < cnt) {
      const float e = E[j] * f;
      const float eu = e * U;
      const float vj = IO<T>::to_f(vs[j * 32]);
      const float d = b + eu;
      const float n = fmaf(eu, vj, a);
      float y = !(d < kMinDen) ? n * rcp_approx(d) : vj;  // a NaN d propagates
      if constexpr (GATE) y *= sigmoid(IO<T>::to_f(rs[j * 32]));
      ys[j * 32] = IO<T>::from_f(y);
      a = decay_add(a, e * vj, lh, ll);
      b = decay_add(b, e, lh, ll);
    }
  }
}

struct CarrySlot {  // CTA running state at a tile boundary, per lane
  double a, b;
  int p, pad;
};

// e^{-w len} in fp64: 16-step powers and the remainder, as the carry pass forms them.
__device__ __forceinline__ double lam_len(double lam, double lam16, int len) {
  double r = lam_pow(lam, len & 15);
  for (int q = 0; q < (len >> 4); ++q) r *= lam16;
  return r;
}

constexpr unsigned int kFlagAggregate = 1u;  // the segment's own summary is published

// LB: the chunked schedule in one launch (p.lb_* set; TMA, every tile of the segment resident in
// the pipeline's stages).  The CTA scans its resident tiles once from a zero state for its
// segment's summary and publishes it; it then waits (bounded) until every earlier segment of its
// lanes has published its own, folds them in order from the sequence's start state into its own
// start state (the flags polled, and the summaries loaded, by all lanes at once: no chain of
// round trips), and scans the same tiles again from that state for the outputs.  Every CTA of a
// launch is resident at once (the schedule keeps to four CTAs per SM).
template <typename T, bool GATE, bool TMA, bool LB>
__global__ void __launch_bounds__(kW * 32, 4) wkv4_fwd_kernel(const __grid_constant__ CUtensorMap mk,
                                                              const __grid_constant__ CUtensorMap mv,
                                                              const __grid_constant__ CUtensorMap my,
                                                              const __grid_constant__ CUtensorMap mr,
                                                              const Fwd4Params p) {
  extern __shared__ __align__(128) unsigned char smem_raw[];
  constexpr uint32_t kBoxElems = kTile * 32;
  constexpr uint32_t kBoxBytes = kBoxElems * sizeof(T);
  constexpr int kNB = GATE ? 3 : 2;  // boxes per stage: k, v (, r)
  T* tiles = reinterpret_cast<T*>(smem_raw);  // [stages][k|v(|r)][kTile][32]
  Summ* summ = reinterpret_cast<Summ*>(smem_raw + (size_t)p.stages * kNB * kBoxBytes);  // [2][kW][32]
  // [2][32]; LB: [3][32], the third the sequence's start state
  CarrySlot* cslot = reinterpret_cast<CarrySlot*>(summ + 2 * kW * 32);
  uint64_t* bars = reinterpret_cast<uint64_t*>(cslot + (LB ? 3 : 2) * 32);  // [stages]
  int* abort_flag = reinterpret_cast<int*>(bars + p.stages);

  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  int blk = blockIdx.x;
  const int ct = blk % p.ctiles;
  blk /= p.ctiles;
  const int bb = blk % p.B;
  const int seg = blk / p.B;
  const int c = ct * 32 + lane;
  const bool valid = c < p.C;
  const int t0 = seg * p.seg_len;
  const int t1 = min(p.T, t0 + p.seg_len);
  const int ntile = (t1 - t0 + kTile - 1) / kTile;

  // thread 0 issues every load; with the test hook set it arms the barriers and issues none
  if (!TMA && threadIdx.x == 0) *abort_flag = 0;
  if (TMA && threadIdx.x == 0) {
    const bool withheld = loads_withheld(p.ctl);
    const int pre = min(p.stages, ntile);
    *abort_flag = 0;
    prefetch_tensormap(&mk);
    prefetch_tensormap(&mv);
    if constexpr (GATE) prefetch_tensormap(&mr);
    for (int s = 0; s < p.stages; ++s) mbar_init(&bars[s], 1);
    fence_mbar_init();
    for (int s = 0; s < pre; ++s) {
      mbar_arrive_expect_tx(&bars[s], kNB * kBoxBytes);
      if (withheld) continue;
      tma_load_3d(tiles + (size_t)(kNB * s) * kBoxElems, &mk, &bars[s], ct * 32, t0 + s * kTile, bb);
      tma_load_3d(tiles + (size_t)(kNB * s + 1) * kBoxElems, &mv, &bars[s], ct * 32, t0 + s * kTile, bb);
      if constexpr (GATE)
        tma_load_3d(tiles + (size_t)(kNB * s + 2) * kBoxElems, &mr, &bars[s], ct * 32, t0 + s * kTile, bb);
    }
  }

  const float w = valid ? p.w[c] : 0.f;
  const float u = valid ? p.u[c] : 0.f;
  const double lam = exp(-(double)w);
  const double lam16 = lam_pow(lam, kL);
  const float lh = (float)lam, ll = (float)(lam - (double)lh);
  const float U = expf(u);
  const size_t plane = (size_t)p.B * p.C;
  const size_t lane_off = (size_t)bb * p.C + c;

  if (warp == kW - 1) {  // running state entering the first tile
    State s0{0.0, 0.0, 0};
    if (p.start != nullptr && valid) {
      const float* sp = p.start + (size_t)seg * p.start_seg_stride;
      s0 = load_state(sp[lane_off], sp[plane + lane_off], sp[2 * plane + lane_off]);
    }
    cslot[32 + lane] = CarrySlot{s0.a, s0.b, s0.p, 0};  // slot of "tile -1"
    if constexpr (LB) {
      // read before this CTA publishes its summary: state_out may be state_in, and the last
      // segment overwrites it as soon as every summary is out
      State si{0.0, 0.0, 0};
      if (p.lb_in != nullptr && valid)
        si = load_state(p.lb_in[lane_off], p.lb_in[plane + lane_off], p.lb_in[2 * plane + lane_off]);
      cslot[64 + lane] = CarrySlot{si.a, si.b, si.p, 0};
    }
  }
  __syncthreads();

  const bool write_y = p.y != nullptr;
  State total{0.0, 0.0, 0};

  int i = 0;
  for (int pass = 0; pass < (LB ? 2 : 1); ++pass) {
  // LB: the first pass only sums the segment (from the zero state set above)
  const bool rescan = (!LB || pass == 1) && ((p.y != nullptr) || (p.ckpt != nullptr));
  for (i = 0; i < ntile; ++i) {
    const int s = i % p.stages;
    const uint32_t ph = (uint32_t)(i / p.stages) & 1u;
    if constexpr (TMA) {
      if (!mbar_wait_bounded(&bars[s], ph, p.ctl)) *abort_flag = 1;
    }
    const int tb = t0 + i * kTile;
    const int ts = tb + warp * kL;
    const int cnt = max(0, min(kL, t1 - ts));
    const T* ks = tiles + (size_t)(kNB * s) * kBoxElems + warp * kL * 32 + lane;
    const T* vs = ks + kBoxElems;
    const T* rs = vs + kBoxElems;  // the r rows (GATE only)
    if constexpr (!TMA) {  // this warp's own rows, by plain loads (nothing else reads them)
      T* kw = const_cast<T*>(ks) - lane;
      warp_rows_in<T, kL>(kw, static_cast<const T*>(p.k), bb, p.T, p.C, ts, cnt, c, valid, lane, kTile);
      warp_rows_in<T, kL>(kw + kBoxElems, static_cast<const T*>(p.v), bb, p.T, p.C, ts, cnt, c, valid, lane, kTile);
      if constexpr (GATE)
        warp_rows_in<T, kL>(kw + 2 * kBoxElems, static_cast<const T*>(p.r), bb, p.T, p.C, ts, cnt, c, valid, lane,
                        kTile);
      __syncwarp();
    }

    // 1. this warp's segment from a zero state
    float E[kL], kmax = -INFINITY, la = 0.f, lb = 0.f;
    int p1 = 0;
    if (cnt == kL)
      seg_summary<T, true>(ks, vs, cnt, lh, ll, kmax, p1, la, lb, E);
    else if (cnt > 0)
      seg_summary<T, false>(ks, vs, cnt, lh, ll, kmax, p1, la, lb, E);
    Summ* sb = summ + (i & 1) * kW * 32;
    sb[warp * 32 + lane] = Summ{la, lb, (float)p1, 0.f};
    // the previous tile's y box must be out of shared memory before its stage is refilled below
    if (lane == 0) bulk_wait_read();
    __syncthreads();
    if (*abort_flag) break;
    // every warp is done with tile i-1: refill its stage
    if (TMA && threadIdx.x == 0 && i >= 1 && i - 1 + p.stages < ntile) {
      const int sp = (i - 1) % p.stages;
      const int tn = t0 + (i - 1 + p.stages) * kTile;
      fence_proxy_async();
      mbar_arrive_expect_tx(&bars[sp], kNB * kBoxBytes);
      // (never reached with the loads withheld: the first wait gives up)
      tma_load_3d(tiles + (size_t)(kNB * sp) * kBoxElems, &mk, &bars[sp], ct * 32, tn, bb);
      tma_load_3d(tiles + (size_t)(kNB * sp + 1) * kBoxElems, &mv, &bars[sp], ct * 32, tn, bb);
      if constexpr (GATE) tma_load_3d(tiles + (size_t)(kNB * sp + 2) * kBoxElems, &mr, &bars[sp], ct * 32, tn, bb);
    }

    // 2. fold: the state at this warp's segment start is the running state
    //    folded with the summaries of the segments before it; the last warp
    //    also folds its own, giving the running state for the next tile.
    const CarrySlot cs = cslot[((i + 1) & 1) * 32 + lane];
    State mine{cs.a, cs.b, cs.p};
    for (int j = 0; j < warp; ++j) {
      const int cj = max(0, min(kL, t1 - (tb + j * kL)));
      if (cj > 0) {
        const Summ x = sb[j * 32 + lane];
        mine = fold(mine, cj == kL ? lam16 : lam_pow(lam, cj), State{(double)x.a, (double)x.b, (int)x.p});
      }
    }
    if (warp == kW - 1) {
      total = mine;
      if (cnt > 0) total = fold(mine, cnt == kL ? lam16 : lam_pow(lam, cnt), State{(double)la, (double)lb, p1});
      cslot[(i & 1) * 32 + lane] = CarrySlot{total.a, total.b, total.p, 0};
    }

    // 3. rescan from the true state: outputs and checkpoints
    if (cnt > 0 && rescan) {
      // the segment's scale: at least every k log2 e of the segment and above the state's b
      const int q = segment_scale(kmax, mine);
      const State sc = rescale(mine, q);
      if (p.ckpt != nullptr && valid && (ts % p.ckpt_len) == 0) {
        // checkpoints are written at that scale (b < 1), so the backward takes q from them
        float* ck = p.ckpt + (size_t)(ts / p.ckpt_len) * 3 * plane + lane_off;
        ck[0] = (float)sc.a;
        ck[plane] = (float)sc.b;
        ck[2 * plane] = (float)q;
      }
      if (write_y) {
        const float f = pow2f_neg(p1 - q);
        T* const yw = const_cast<T*>(ks) - lane;  // this warp's [16][32] k rows
        if (cnt == kL)
          seg_output<T, true, GATE>(vs, rs, cnt, E, f, U, (float)sc.a, (float)sc.b, lh, ll, yw + lane);
        else
          seg_output<T, false, GATE>(vs, rs, cnt, E, f, U, (float)sc.a, (float)sc.b, lh, ll, yw + lane);
        if constexpr (TMA) {
          // y of the segment as one [16 x 32] box (rows past T and channels past C are clipped)
          fence_proxy_async();
          __syncwarp();
          if (lane == 0) {
            tma_store_3d(&my, yw, ct * 32, ts, bb);
            bulk_commit();
          }
        } else if (valid) {  // each lane stores its own channel's outputs
          T* yg = static_cast<T*>(p.y) + ((size_t)bb * p.T + ts) * p.C + c;
          for (int j = 0; j < cnt; ++j) yg[(size_t)j * p.C] = yw[j * 32 + lane];
        }
      }
    }
  }
  if constexpr (LB) {
    if (pass == 0) {
      __syncthreads();
      if (*abort_flag) break;
      if (warp == kW - 1) {
        // the segment's summary (total, from the zero state) out; the state before it in
        const size_t ncta = (size_t)p.ctiles * p.B;
        const size_t cta = (size_t)ct + (size_t)p.ctiles * bb;
        const size_t me = ((size_t)seg * plane + lane_off) * 3;
        if (valid) {
          p.lb_agg[me] = total.a;
          p.lb_agg[me + 1] = total.b;
          p.lb_agg[me + 2] = (double)total.p;
        }
        __syncwarp();
        if (lane == 0) {
          __threadfence();
          flag_release(&p.lb_flag[(size_t)seg * ncta + cta], kFlagAggregate);
        }
        // wait until every earlier segment has published its summary: the lanes poll up to 32
        // flags at once (segment seg - 1 - lane, then 32 further back, ...)
        bool failed = false;
        for (int j0 = 0; j0 < seg && !failed; j0 += 32) {
          const int j = seg - 1 - (j0 + lane);
          unsigned int f = 1u;
          if (j0 + lane < seg) f = flag_wait_bounded(&p.lb_flag[(size_t)j * ncta + cta], p.ctl);
          failed = __any_sync(0xffffffffu, f == 0u);
        }
        // each lane reads after the acquires and the barrier, bypassing L1
        __syncwarp();
        if (failed) {
          if (lane == 0) *abort_flag = 1;
        } else {
          State st{cslot[64 + lane].a, cslot[64 + lane].b, cslot[64 + lane].p};
          if (valid) {
            const double lam_seg = lam_len(lam, lam16, p.seg_len);  // every earlier segment is whole
            // the earlier summaries in order, eight at a time, their loads in flight together
            constexpr int kBatch = 8;
            for (int m0 = 0; m0 < seg; m0 += kBatch) {
              double ag[kBatch][3];
#pragma unroll
              for (int e = 0; e < kBatch; ++e) {
                if (m0 + e < seg) {
                  const size_t o = ((size_t)(m0 + e) * plane + lane_off) * 3;
                  ag[e][0] = __ldcg(&p.lb_agg[o]);
                  ag[e][1] = __ldcg(&p.lb_agg[o + 1]);
                  ag[e][2] = __ldcg(&p.lb_agg[o + 2]);
                }
              }
#pragma unroll
              for (int e = 0; e < kBatch; ++e)
                if (m0 + e < seg) st = fold(st, lam_seg, State{ag[e][0], ag[e][1], (int)ag[e][2]});
            }
          }
          cslot[32 + lane] = CarrySlot{st.a, st.b, st.p, 0};  // the second pass starts from it
        }
      }
      __syncthreads();
      if (*abort_flag) break;
    }
  }
  }
  if (TMA && threadIdx.x == 0 && *abort_flag) drain_loads(bars, p.stages, i, ntile, p.ctl);  // a wait gave up
  if (lane == 0) bulk_wait_all();

  if (p.end != nullptr && valid && warp == kW - 1 && !*abort_flag && (!LB || seg == p.nseg - 1)) {
    float* e = p.end + (size_t)seg * p.end_seg_stride;
    store_state(total, &e[lane_off], &e[plane + lane_off], &e[2 * plane + lane_off]);
  }
}

// Carry pass of the multi-CTA (chunked) forward: turns per-segment summaries
// (each the state reached from a zero state over that segment alone) into the
// state at the start of every segment, in place, by the associative fold
//   S_{<=j} = e^{-w len_j} S_{<=j-1}  (+)  summary_j,
// and writes the final state.  One thread per lane (b, c), fp64 arithmetic.
__global__ void wkv4_carry_kernel(int B, int C, int T, int nseg, int seg_len, const float* __restrict__ w,
                                  const float* state_in, float* __restrict__ ws,
                                  float* state_out) {  // state_out may be state_in
  const size_t plane = (size_t)B * C;
  const size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= plane) return;
  const int c = (int)(i % C);
  State st{0.0, 0.0, 0};
  if (state_in != nullptr) st = load_state(state_in[i], state_in[plane + i], state_in[2 * plane + i]);
  const double lam = exp(-(double)w[c]);
  const double lam16 = lam_pow(lam, 16);
  for (int j = 0; j < nseg; ++j) {
    float* sj = ws + (size_t)j * 3 * plane + i;
    const State x = load_state(sj[0], sj[plane], sj[2 * plane]);
    store_state(st, &sj[0], &sj[plane], &sj[2 * plane]);
    // e^{-w len} as the product of len factors e^{-w}, len = 16 q + r
    const int len = min(seg_len, T - j * seg_len);
    double lamL = lam_pow(lam, len & 15);
    for (int q = 0; q < (len >> 4); ++q) lamL *= lam16;
    st = fold(st, lamL, x);
  }
  if (state_out != nullptr) store_state(st, &state_out[i], &state_out[plane + i], &state_out[2 * plane + i]);
}

template <typename T, bool GATE, bool LB = false>
size_t fwd_smem_bytes(int stages) {  // also the plain path's (one stage)
  return (size_t)stages * (GATE ? 3 : 2) * kTile * 32 * sizeof(T) + 2 * kW * 32 * sizeof(Summ) +
         (LB ? 3 : 2) * 32 * sizeof(CarrySlot) + (size_t)stages * 8 + 16;
}

template <typename T, bool GATE, bool TMA, bool LB = false>
cudaError_t launch_fwd_tt(const CUtensorMap& mk, const CUtensorMap& mv, const CUtensorMap& my, const CUtensorMap& mr,
                          const Fwd4Params& p, cudaStream_t st) {
  const size_t smem = fwd_smem_bytes<T, GATE, LB>(p.stages);
  static unsigned device_mask = 0;
  cudaError_t e =
      ensure_smem_attr(reinterpret_cast<const void*>(wkv4_fwd_kernel<T, GATE, TMA, LB>), (int)smem, &device_mask);
  if (e != cudaSuccess) return e;
  const long long nblk = (long long)p.ctiles * p.B * p.nseg;
  wkv4_fwd_kernel<T, GATE, TMA, LB><<<(unsigned)nblk, kW * 32, smem, st>>>(mk, mv, my, mr, p);
  return cudaGetLastError();
}

template <typename T, bool GATE>
cudaError_t launch_fwd_t(const CUtensorMap& mk, const CUtensorMap& mv, const CUtensorMap& my, const CUtensorMap& mr,
                         const Fwd4Params& p, cudaStream_t st) {
  return p.tma ? launch_fwd_tt<T, GATE, true>(mk, mv, my, mr, p, st)
               : launch_fwd_tt<T, GATE, false>(mk, mv, my, mr, p, st);
}

}  // namespace

int fwd_tile_steps() { return kTile; }

int fwd_store_steps() { return kL; }

int fwd_stages(bool bf16, int seg_len, bool gate, bool tma) {
  if (!tma) return 1;  // the plain path reads each warp's rows into one buffer, no pipeline
  // three stages of fp32 k, v boxes (48 KB) keep four CTAs per SM; bf16 boxes are half as big; with the
  // gate's r box, two stages (fp32) or four (bf16) stay within the same 48 KB
  const int want = gate ? (bf16 ? 4 : 2) : (bf16 ? 6 : 3);
  const int ntile = (seg_len + kTile - 1) / kTile;
  return max(2, min(want, ntile));
}

cudaError_t launch_wkv4_fwd(bool bf16, const CUtensorMap& mk, const CUtensorMap& mv, const CUtensorMap& my,
                            const Fwd4Params& p, cudaStream_t st) {
  return bf16 ? launch_fwd_t<__nv_bfloat16, false>(mk, mv, my, mk, p, st)
              : launch_fwd_t<float, false>(mk, mv, my, mk, p, st);
}

cudaError_t launch_wkv4_fwd_lookback(bool bf16, const CUtensorMap& mk, const CUtensorMap& mv, const CUtensorMap& my,
                                     const Fwd4Params& p, cudaStream_t st) {
  return bf16 ? launch_fwd_tt<__nv_bfloat16, false, true, true>(mk, mv, my, mk, p, st)
              : launch_fwd_tt<float, false, true, true>(mk, mv, my, mk, p, st);
}

cudaError_t launch_wkv4_fwd_gated(bool bf16, const CUtensorMap& mk, const CUtensorMap& mv, const CUtensorMap& my,
                                  const CUtensorMap& mr, const Fwd4Params& p, cudaStream_t st) {
  return bf16 ? launch_fwd_t<__nv_bfloat16, true>(mk, mv, my, mr, p, st)
              : launch_fwd_t<float, true>(mk, mv, my, mr, p, st);
}

cudaError_t launch_wkv4_carry(int B, int C, int T, int nseg, int seg_len, const float* w, const float* state_in,
                              float* ws, float* state_out, cudaStream_t st) {
  const size_t n = (size_t)B * C;
  const unsigned grid = (unsigned)((n + 255) / 256);
  wkv4_carry_kernel<<<grid, 256, 0, st>>>(B, C, T, nseg, seg_len, w, state_in, ws, state_out);
  return cudaGetLastError();
}

}  // namespace rwkv
