// RWKV-4 WKV backward kernels (sm_100a).
//
// The pages print no backward; this is the chain rule through the recurrent
// form of "RWKV - Transformer 시대에 RNN을 재발명하다", Method / (2) Time-mixing
// (WKV), for L = Σ gy_t WKV_t.  With D_t = B_{t-1} + e^{u+k_t},
// g_t = gy_t / D_t, h_t = gy_t WKV_t / D_t and the reverse sums
//   α_t = Σ_{s>t} e^{-(s-t-1)w} g_s,   β_t = -Σ_{s>t} e^{-(s-t-1)w} h_s
// (the gradients of L with respect to the state A_t, B_t):
//   gv_t = e^{k_t} (e^u g_t + α_t)
//   gk_t = e^{k_t} (e^u (g_t v_t - h_t) + α_t v_t + β_t)
//   gu   = Σ e^{u+k_t} (g_t v_t - h_t)
//   gw   = -e^{-w} Σ (α_t A_{t-1} + β_t B_{t-1})          (summed over b and t)
// α and β obey α_{t-1} = g_t + e^{-w} α_t (likewise β with -h_t), a linear
// reverse recurrence: the same associativity as the forward lets the four
// 16-step chunks of a tile run their reverse walks in parallel once each has
// its carry, and the carries come from folding each chunk's local sums.
//
// Scaling.  Inside a chunk everything is measured against one power of two
// 2^q, the exponent the forward wrote the chunk's checkpoint at (q is at least
// every k log2 e of the chunk, so no weight exceeds 1, and above the state's
// b): e_t = e^{k_t} 2^{-q}, d_t = D_t 2^{-q}, G_t = gy_t / d_t, and the
// carries are kept as α~ = α 2^q; then e^{k_t} α_t = e_t α~_t and
// α_t A_{t-1} = α~_t a_{t-1}, so the scale cancels from every gradient.
// Precision.  The gradient terms cancel each other (α_t v_t + β_t is small
// when the state's mean is close to v_t), so fp32 sums over thousands of steps
// would not hold 1e-4 relative accuracy.  Steps inside a chunk run in fp32 with
// the decay e^{-w} = lh + ll split into fp32 hi and lo parts; the carries
// folded from chunk to chunk and the per-lane gw, gu sums are fp64, so fp32
// rounding accumulates over 16 steps at most.
//
// Kernel shape.  A CTA owns 32 channels of one batch row over all of T,
// processed in 64-step tiles from the last to the first; warp w takes the
// tile's w-th 16-step chunk: it recomputes that chunk's forward from the
// forward pass's checkpoint, keeps e_t, G_t, y_t and b_{t-1} in registers,
// sums its local reverse carries, folds the carries of the chunks after it,
// then walks the chunk backwards.  k, v, gy arrive by TMA (no multicast); the
// walk writes gk and gv over the chunk's consumed k and v rows in shared
// memory and the warp sends its two [16 x 32] boxes out with TMA stores, so
// each element is read once and each gradient written once, without
// per-element address arithmetic.  A tile's checkpoints (three floats per
// lane) are loaded into registers while the tile before it is processed, and
// the next tile's are prefetched into L2, so no tile waits on DRAM for them
// (waiting cost 11 % of the kernel's time).  Per-lane gw, gu partials are reduced over
// the batch by a second kernel.
//
// Receptance gate (GATE): gradients of L = Σ go_t σ(r_t) WKV_t (the gated
// output of the same page's time mixing).  go takes gy's place as the third
// box of a stage, so the gated kernel keeps the plain one's shared memory and
// all of a training shape's CTAs resident (a fourth box would leave three CTAs
// per SM and a second wave).  r is read with plain loads (a warp reads one
// 128-byte row per step; the rows of the next tile are prefetched into L2),
// the recompute phase forms gy_t = σ(r_t) go_t and
// gr_t = go_t WKV_t σ(r_t) (1 - σ(r_t)) from the WKV_t it recomputes anyway,
// and gr leaves with plain coalesced stores.
#include "launch.h"
#include "wkv_common.cuh"

namespace rwkv {
namespace {

constexpr int kW = 4;
constexpr int kL = 16;
constexpr int kTile = kW * kL;

struct RSumm {  // a chunk's own reverse sums from a zero carry, at scale 2^q
  float la;  // α~ carried out of the chunk (into the step before its first)
  float lg;  // γ at the chunk's first step
  float ys;  // y at the chunk's first step
  float ye;  // y at the chunk's last step
  float q;
  float pad;  // 24 bytes: two stages of boxes plus these still fit four CTAs per SM
};

// Phase A: forward recompute of one chunk from its checkpoint state (a, b) at
// scale 2^q, keeping e_t, G_t = gy_t / d_t, y_t and b_{t-1}.  gs holds the gy
// rows, or with GATE the go rows: then gy_t = σ(r_t) go_t with r_t read from
// rg[t * C], and gr_t is stored to grg[t * C].
// The state recurrence runs in fp64 (lam = e^{-w}); d_t and the numerator are
// formed in fp32 from it.  A large term that persists in the state (an outlier
// key) would otherwise be re-rounded at every fp32 step: over 16 steps that
// drift in y_t and b_t moved gw by up to 5e-4 relative, against the 1e-4 bound.
// With GATE the chunk's r values are loaded eight steps at a time (their rows
// were prefetched into L2 a tile ahead), which keeps the kernel in 128
// registers without spills.
template <typename T, bool FULL, bool GATE>
__device__ __forceinline__ void chunk_recompute(const T* ks, const T* vs, const T* gs, const T* rg, T* grg,
                                                int C, int cnt, float qf, float U, double lam, double a, double b,
                                                float (&E)[kL], float (&G)[kL], float (&Y)[kL], float (&BP)[kL]) {
  constexpr int kHalf = kL / 2;
  float rv[GATE ? kHalf : 1];
#pragma unroll
  for (int j = 0; j < kL; ++j) {
    if constexpr (GATE) {
      if (j % kHalf == 0) {
#pragma unroll
        for (int i = 0; i < kHalf; ++i)
          rv[i] = (rg != nullptr && (FULL || j + i < cnt)) ? IO<T>::load(rg + (size_t)(j + i) * C) : 0.f;
      }
    }
    if (FULL || j < cnt) {
      const float e = tok_weight(IO<T>::to_f(ks[j * 32]), qf);
      const float eu = e * U;
      const float vj = IO<T>::to_f(vs[j * 32]);
      const float bf = (float)b;
      const float d = bf + eu;
      const float rd = rcp_approx(d);
      const bool ok = !(d < kMinDen);  // else no history and e^{u+k} underflowed: WKV = v locally (NaN: ok)
      Y[j] = ok ? fmaf(eu, vj, (float)a) * rd : vj;
      float gy;
      if constexpr (GATE) {
        const float sg = sigmoid(rv[j % kHalf]);
        const float go = IO<T>::to_f(gs[j * 32]);
        gy = sg * go;
        if (grg != nullptr) grg[(size_t)j * C] = IO<T>::from_f(go * Y[j] * (sg - sg * sg));
      } else {
        gy = IO<T>::to_f(gs[j * 32]);
      }
      G[j] = ok ? gy * rd : 0.f;
      E[j] = e;
      BP[j] = bf;
      a = fma(lam, a, (double)(e * vj));
      b = fma(lam, b, (double)e);
    }
  }
}

// Phase B: the chunk's own reverse sums from a zero carry at its end.
template <bool FULL>
__device__ __forceinline__ void chunk_local_sums(int cnt, const float (&G)[kL], const float (&Y)[kL], float lh,
                                                 float ll, float& la, float& lg, float& ye) {
  la = 0.f;
  lg = 0.f;
  ye = FULL ? Y[kL - 1] : 0.f;
#pragma unroll
  for (int j = kL - 1; j >= 0; --j) {
    if (FULL || j < cnt) {
      if (!FULL && j == cnt - 1) ye = Y[j];
      la = decay_add(la, G[j], lh, ll);
      if (j > 0) lg = decay_add(lg, (Y[j - 1] - Y[j]) * la, lh, ll);
    }
  }
}

// Phase D: the reverse walk of one chunk from its carry (al, ga) at the last
// step, writing gk_j over k_j (ks[j * 32]) and gv_j over v_j (vs[j * 32]).
template <typename T, bool FULL>
__device__ __forceinline__ void chunk_walk(T* ks, T* vs, int cnt, const float (&E)[kL], const float (&G)[kL],
                                           const float (&Y)[kL], const float (&BP)[kL], float U, float lh,
                                           float ll, float al, float ga, float& gws, float& gus) {
#pragma unroll
  for (int j = kL - 1; j >= 0; --j) {
    if (FULL || j < cnt) {
      const float vj = IO<T>::to_f(vs[j * 32]);
      const float ug = U * G[j];
      const float dv = vj - Y[j];
      const float eu = E[j] * U;
      const float gvt = E[j] * (ug + al);
      const float gkt = fmaf(dv, gvt, E[j] * ga);
      // α~ a_{t-1} + β~ b_{t-1} = b_{t-1} γ_t - α~ e^u e_t (v_t - y_t)
      gws = fmaf(BP[j], ga, fmaf(-al * eu, dv, gws));
      gus = fmaf(ug * E[j], dv, gus);
      al = decay_add(al, G[j], lh, ll);
      if (j > 0) ga = decay_add(ga, (Y[j - 1] - Y[j]) * al, lh, ll);
      ks[j * 32] = IO<T>::from_f(gkt);
      vs[j * 32] = IO<T>::from_f(gvt);
    }
  }
}

struct RCarry {  // reverse carry at a chunk boundary, per lane (see phase C)
  double a, g;
  float y;
  int p;
};

// mg: gy boxes, or with GATE go boxes.
template <typename T, bool GATE, bool TMA>
__global__ void __launch_bounds__(kW * 32, 4) wkv4_bwd_kernel(const __grid_constant__ CUtensorMap mk,
                                                              const __grid_constant__ CUtensorMap mv,
                                                              const __grid_constant__ CUtensorMap mg,
                                                              const __grid_constant__ CUtensorMap mgk,
                                                              const __grid_constant__ CUtensorMap mgv,
                                                              const Bwd4Params p) {
  extern __shared__ __align__(128) unsigned char smem_raw[];
  constexpr uint32_t kBoxElems = kTile * 32;
  constexpr uint32_t kBoxBytes = kBoxElems * sizeof(T);
  constexpr int kNB = 3;  // boxes per stage: k, v, and gy (or go)
  T* tiles = reinterpret_cast<T*>(smem_raw);  // [stages][k|v|gy][kTile][32]
  RSumm* rs = reinterpret_cast<RSumm*>(smem_raw + (size_t)p.stages * kNB * kBoxBytes);  // [2][kW][32]
  RCarry* cslot = reinterpret_cast<RCarry*>(rs + 2 * kW * 32);                        // [2][32]
  uint64_t* bars = reinterpret_cast<uint64_t*>(cslot + 2 * 32);
  int* abort_flag = reinterpret_cast<int*>(bars + p.stages);

  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int ct = blockIdx.x % p.ctiles;
  const int bb = blockIdx.x / p.ctiles;
  const int c = ct * 32 + lane;
  const bool valid = c < p.C;
  const int ntile = (p.T + kTile - 1) / kTile;

  // thread 0 issues every load; with the test hook set it arms the barriers and issues none
  if (!TMA && threadIdx.x == 0) *abort_flag = 0;
  if (TMA && threadIdx.x == 0) {
    const bool withheld = loads_withheld(p.ctl);
    const int pre = min(p.stages, ntile);
    *abort_flag = 0;
    prefetch_tensormap(&mk);
    prefetch_tensormap(&mv);
    prefetch_tensormap(&mg);
    for (int s = 0; s < p.stages; ++s) mbar_init(&bars[s], 1);
    fence_mbar_init();
    for (int s = 0; s < pre; ++s) {
      const int tc = (ntile - 1 - s) * kTile;
      mbar_arrive_expect_tx(&bars[s], kNB * kBoxBytes);
      if (withheld) continue;
      tma_load_3d(tiles + (size_t)(kNB * s) * kBoxElems, &mk, &bars[s], ct * 32, tc, bb);
      tma_load_3d(tiles + (size_t)(kNB * s + 1) * kBoxElems, &mv, &bars[s], ct * 32, tc, bb);
      tma_load_3d(tiles + (size_t)(kNB * s + 2) * kBoxElems, &mg, &bars[s], ct * 32, tc, bb);
    }
  }
  if (warp == 0) cslot[32 + lane] = RCarry{0.0, 0.0, 0.f, 0};  // nothing flows back from after the end
  __syncthreads();

  const float w = valid ? p.w[c] : 0.f;
  const float u = valid ? p.u[c] : 0.f;
  const double lam = exp(-(double)w);
  const double lam15 = lam_pow(lam, kL - 1);
  const float lh = (float)lam, ll = (float)(lam - (double)lh);
  const float U = expf(u);
  const size_t plane = (size_t)p.B * p.C;
  const size_t lane_off = (size_t)bb * p.C + c;

  double gw_acc = 0.0, gu_acc = 0.0;
  float cka = 0.f, ckb = 0.f, ckp = 0.f;  // checkpoint of the tile about to be processed
  {
    const int ts0 = (ntile - 1) * kTile + warp * kL;
    if (valid && ts0 < p.T) {
      const float* ck = p.ckpt + (size_t)(ts0 / kL) * 3 * plane + lane_off;
      cka = ck[0];
      ckb = ck[plane];
      ckp = ck[2 * plane];
    }
  }

  int i = 0;
  for (; i < ntile; ++i) {
    const int tile = ntile - 1 - i;
    const int s = i % p.stages;
    const uint32_t ph = (uint32_t)(i / p.stages) & 1u;
    const int tb = tile * kTile;
    const int ts = tb + warp * kL;
    const int cnt = max(0, min(kL, p.T - ts));
    // checkpoint of this chunk (independent of the pipeline)
    State st{0.0, 0.0, 0};
    if (cnt > 0 && valid) st = load_state(cka, ckb, ckp);
    {  // the next tile's checkpoint, one tile ahead of its use
      const int tsn = (tile - 1) * kTile + warp * kL;
      if (tile >= 1 && valid && tsn < p.T) {
        const float* ck = p.ckpt + (size_t)(tsn / kL) * 3 * plane + lane_off;
        cka = ck[0];
        ckb = ck[plane];
        ckp = ck[2 * plane];
      }
      if constexpr (GATE) {  // the next tile's r rows into L2: lane j < 16 one 32-channel row of this warp's chunk
        if (tile >= 1 && lane < kL && tsn + lane < p.T) {
          const T* rrow = static_cast<const T*>(p.r) + ((size_t)bb * p.T + tsn + lane) * p.C + (size_t)ct * 32;
          asm volatile("prefetch.global.L2 [%0];" ::"l"(rrow) : "memory");
        }
      }
      if (tile >= 2 && valid) {  // and the one after it into L2
        const float* ck2 = p.ckpt + (size_t)((tsn - kTile) / kL) * 3 * plane + lane_off;
        asm volatile("prefetch.global.L2 [%0];" ::"l"(ck2) : "memory");
        asm volatile("prefetch.global.L2 [%0];" ::"l"(ck2 + plane) : "memory");
        asm volatile("prefetch.global.L2 [%0];" ::"l"(ck2 + 2 * plane) : "memory");
      }
    }
    if constexpr (TMA) {
      if (!mbar_wait_bounded(&bars[s], ph, p.ctl)) *abort_flag = 1;
    }
    T* const kw = tiles + (size_t)(kNB * s) * kBoxElems + warp * kL * 32;  // this warp's [16][32] rows
    T* const vw = kw + kBoxElems;
    T* const ks = kw + lane;
    T* const vs = vw + lane;
    const T* gs = vs + kBoxElems;  // gy rows (go with GATE)
    if constexpr (!TMA) {  // this warp's own rows, by plain loads (nothing else reads them)
      warp_rows_in<T, kL>(kw, static_cast<const T*>(p.k), bb, p.T, p.C, ts, cnt, c, valid, lane, -kTile);
      warp_rows_in<T, kL>(vw, static_cast<const T*>(p.v), bb, p.T, p.C, ts, cnt, c, valid, lane, -kTile);
      warp_rows_in<T, kL>(vw + kBoxElems, static_cast<const T*>(p.g), bb, p.T, p.C, ts, cnt, c, valid, lane,
                          -kTile);
      __syncwarp();
    }
    // GATE: this lane's r and gr of the chunk, token stride C
    const size_t tok0 = ((size_t)bb * p.T + (size_t)max(ts, 0)) * p.C + (size_t)c;
    const T* rg = (GATE && valid) ? static_cast<const T*>(p.r) + tok0 : nullptr;  // lanes past C: no access
    T* grg = (GATE && valid) ? static_cast<T*>(p.gr) + tok0 : nullptr;

    // A. forward recompute of the chunk at one scale 2^q: the forward wrote the
    //    checkpoint at the chunk's scale (at least every k log2 e of the chunk,
    //    and b < 1), so q is the checkpoint's exponent
    float E[kL], G[kL], Y[kL], BP[kL];
    const int q = st.p;
    if (cnt == kL)
      chunk_recompute<T, true, GATE>(ks, vs, gs, rg, grg, p.C, cnt, (float)q, U, lam, st.a, st.b, E, G, Y, BP);
    else if (cnt > 0)
      chunk_recompute<T, false, GATE>(ks, vs, gs, rg, grg, p.C, cnt, (float)q, U, lam, st.a, st.b, E, G, Y, BP);

    // B. the chunk's own reverse sums
    float la = 0.f, lg = 0.f, ye = 0.f;
    if (cnt == kL)
      chunk_local_sums<true>(cnt, G, Y, lh, ll, la, lg, ye);
    else if (cnt > 0)
      chunk_local_sums<false>(cnt, G, Y, lh, ll, la, lg, ye);
    RSumm* sb = rs + (i & 1) * kW * 32;
    sb[warp * 32 + lane] = RSumm{la, lg, cnt > 0 ? Y[0] : 0.f, ye, (float)q, 0.f};
    // the previous tile's gradient boxes must be out of shared memory before its stage is refilled below
    if (lane == 0) bulk_wait_read();
    __syncthreads();
    if (*abort_flag) break;
    // (never reached with the loads withheld: the first wait gives up)
    if (TMA && threadIdx.x == 0 && i >= 1 && i - 1 + p.stages < ntile) {
      const int sp = (i - 1) % p.stages;
      const int tc = (ntile - 1 - (i - 1 + p.stages)) * kTile;
      fence_proxy_async();
      mbar_arrive_expect_tx(&bars[sp], kNB * kBoxBytes);
      tma_load_3d(tiles + (size_t)(kNB * sp) * kBoxElems, &mk, &bars[sp], ct * 32, tc, bb);
      tma_load_3d(tiles + (size_t)(kNB * sp + 1) * kBoxElems, &mv, &bars[sp], ct * 32, tc, bb);
      tma_load_3d(tiles + (size_t)(kNB * sp + 2) * kBoxElems, &mg, &bars[sp], ct * 32, tc, bb);
    }

    // C. fold the carries of the later chunks.  A carry is (α~ out of a chunk,
    //    γ at that chunk's first step, y there) at scale 2^kp.  Entering a
    //    chunk with last step e:   α~_e = α~,  γ_e = e^{-w} γ + (y_e - y) α~_e;
    //    leaving it (n steps, first step s):
    //      α~ = e^{-wn} α~_e + La,  γ_s = e^{-w(n-1)} (γ_e + (y_s - y_e) α~_e) + Lg.
    //    Warp 0 folds all four chunks, giving the carry into the next tile.
    const RCarry cin = cslot[((i + 1) & 1) * 32 + lane];
    double ka = cin.a, kg = cin.g;
    float ky = cin.y;
    int kp = cin.p;
    double ae = 0.0, ge = 0.0;  // this chunk's (α~_e, γ_e)
    for (int j = kW - 1; j >= warp; --j) {
      const int cj = max(0, min(kL, p.T - (tb + j * kL)));
      if (cj == 0) continue;
      const RSumm x = sb[j * 32 + lane];
      // carries scale inversely to the state: α~ = α 2^q, so moving from 2^kp to 2^q multiplies by 2^(q - kp)
      const double f = pow2d((int)x.q - kp);
      const double a_e = ka * f;
      const double g_e = fma(lam, kg * f, (double)(x.ye - ky) * a_e);
      if (j == warp) {
        ae = a_e;
        ge = g_e;
        if (warp != 0) break;
      }
      const double lamN1 = cj == kL ? lam15 : lam_pow(lam, cj - 1);
      ka = fma(lamN1 * lam, a_e, (double)x.la);
      kg = fma(lamN1, fma(a_e, (double)(x.ys - x.ye), g_e), (double)x.lg);
      ky = x.ys;
      kp = (int)x.q;
    }
    if (warp == 0) cslot[(i & 1) * 32 + lane] = RCarry{ka, kg, ky, kp};

    // D. reverse walk with the true carry.  Besides α~ it carries
    //   γ_t = y_t α~_t + β~_t = Σ_{s>t} e^{-(s-t-1)w} G_s (y_t - y_s),
    // built from small increments (y_{t-1} - y_t) α~_{t-1}, so that
    //   gk_t = (v_t - y_t) gv_t + e_t γ_t
    // never subtracts two large nearly equal fp32 numbers.
    if (cnt > 0) {
      float gws = 0.f, gus = 0.f;
      if (cnt == kL)
        chunk_walk<T, true>(ks, vs, cnt, E, G, Y, BP, U, lh, ll, (float)ae, (float)ge, gws, gus);
      else
        chunk_walk<T, false>(ks, vs, cnt, E, G, Y, BP, U, lh, ll, (float)ae, (float)ge, gws, gus);
      gw_acc += (double)gws;
      gu_acc += (double)gus;
      if constexpr (TMA) {
        // gk, gv of the chunk: one [16 x 32] box each (rows past T and channels past C are clipped)
        fence_proxy_async();
        __syncwarp();
        if (lane == 0) {
          tma_store_3d(&mgk, kw, ct * 32, ts, bb);
          tma_store_3d(&mgv, vw, ct * 32, ts, bb);
          bulk_commit();
        }
      } else if (valid) {  // each lane stores its own channel's gradients
        const size_t o = ((size_t)bb * p.T + ts) * p.C + c;
        T* gkg = static_cast<T*>(p.gk) + o;
        T* gvg = static_cast<T*>(p.gv) + o;
        for (int j = 0; j < cnt; ++j) {
          gkg[(size_t)j * p.C] = ks[j * 32];
          gvg[(size_t)j * p.C] = vs[j * 32];
        }
      }
    }
  }
  if (TMA && threadIdx.x == 0 && *abort_flag) drain_loads(bars, p.stages, i, ntile, p.ctl);  // a wait gave up
  if (lane == 0) bulk_wait_all();

  // reduce the four warps' gw, gu partials of each lane
  __syncthreads();
  double2* red = reinterpret_cast<double2*>(rs);
  red[warp * 32 + lane] = make_double2(gw_acc, gu_acc);
  __syncthreads();
  if (warp == 0 && valid) {
    double sw = 0.0, su = 0.0;
#pragma unroll
    for (int j = 0; j < kW; ++j) {
      sw += red[j * 32 + lane].x;
      su += red[j * 32 + lane].y;
    }
    p.part[lane_off] = -lam * sw;
    p.part[plane + lane_off] = su;
  }
}

// gw[c] = Σ_b part[0][b][c], gu[c] = Σ_b part[1][b][c], fp64, in batch order.
__global__ void wkv4_reduce_wu_kernel(int B, int C, const double* __restrict__ part, float* __restrict__ gw,
                                      float* __restrict__ gu) {
  const int c = blockIdx.x * blockDim.x + threadIdx.x;
  if (c >= C) return;
  const size_t plane = (size_t)B * C;
  double sw = 0.0, su = 0.0;
  for (int b = 0; b < B; ++b) {
    sw += part[(size_t)b * C + c];
    su += part[plane + (size_t)b * C + c];
  }
  gw[c] = (float)sw;
  gu[c] = (float)su;
}

template <typename T>
size_t bwd_smem_bytes(int stages) {
  return (size_t)stages * 3 * kTile * 32 * sizeof(T) + 2 * kW * 32 * sizeof(RSumm) + 2 * 32 * sizeof(RCarry) +
         (size_t)stages * 8 + 16;
}

template <typename T, bool GATE, bool TMA>
cudaError_t launch_bwd_tt(const CUtensorMap& mk, const CUtensorMap& mv, const CUtensorMap& mg, const CUtensorMap& mgk,
                          const CUtensorMap& mgv, const Bwd4Params& p, cudaStream_t st) {
  const size_t smem = bwd_smem_bytes<T>(p.stages);
  static unsigned device_mask = 0;
  cudaError_t e =
      ensure_smem_attr(reinterpret_cast<const void*>(wkv4_bwd_kernel<T, GATE, TMA>), (int)smem, &device_mask);
  if (e != cudaSuccess) return e;
  const long long nblk = (long long)p.ctiles * p.B;
  wkv4_bwd_kernel<T, GATE, TMA><<<(unsigned)nblk, kW * 32, smem, st>>>(mk, mv, mg, mgk, mgv, p);
  return cudaGetLastError();
}

template <typename T, bool GATE>
cudaError_t launch_bwd_t(const CUtensorMap& mk, const CUtensorMap& mv, const CUtensorMap& mg, const CUtensorMap& mgk,
                         const CUtensorMap& mgv, const Bwd4Params& p, cudaStream_t st) {
  return p.tma ? launch_bwd_tt<T, GATE, true>(mk, mv, mg, mgk, mgv, p, st)
               : launch_bwd_tt<T, GATE, false>(mk, mv, mg, mgk, mgv, p, st);
}

}  // namespace

int bwd_tile_steps() { return kTile; }

int bwd_store_steps() { return kL; }

int bwd_stages(bool bf16, int T, bool gate, bool tma) {
  (void)gate;  // the gated kernel streams the same three boxes (k, v, go)
  if (!tma) return 1;  // the plain path reads each warp's rows into one buffer, no pipeline
  const int want = bf16 ? 4 : 2;  // 48 KB of boxes keeps four CTAs per SM
  const int ntile = (T + kTile - 1) / kTile;
  return max(2, min(want, ntile));
}

cudaError_t launch_wkv4_bwd(bool bf16, const CUtensorMap& mk, const CUtensorMap& mv, const CUtensorMap& mg,
                            const CUtensorMap& mgk, const CUtensorMap& mgv, const Bwd4Params& p, cudaStream_t st) {
  return bf16 ? launch_bwd_t<__nv_bfloat16, false>(mk, mv, mg, mgk, mgv, p, st)
              : launch_bwd_t<float, false>(mk, mv, mg, mgk, mgv, p, st);
}

cudaError_t launch_wkv4_bwd_gated(bool bf16, const CUtensorMap& mk, const CUtensorMap& mv, const CUtensorMap& mo,
                                  const CUtensorMap& mgk, const CUtensorMap& mgv, const Bwd4Params& p,
                                  cudaStream_t st) {
  return bf16 ? launch_bwd_t<__nv_bfloat16, true>(mk, mv, mo, mgk, mgv, p, st)
              : launch_bwd_t<float, true>(mk, mv, mo, mgk, mgv, p, st);
}

cudaError_t launch_wkv4_reduce_wu(int B, int C, const double* part, float* gw, float* gu, cudaStream_t st) {
  wkv4_reduce_wu_kernel<<<(C + 127) / 128, 128, 0, st>>>(B, C, part, gw, gu);
  return cudaGetLastError();
}

}  // namespace rwkv
