/*
 * fp64 CPU oracle for the RWKV WKV operator.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the plain, slow, obviously correct
 * statement of what the WKV operator computes, in double precision, with no
 * blocking, fusion or reordering beyond the formulas themselves.  Only the
 * test-suite, the package's smoke check and the benchmark's CPU-baseline leg
 * may load it; the CUDA library never calls it and shares no code with it.
 *
 * Sources (page title, section):
 *  [P1] "RWKV - Transformer 시대에 RNN을 재발명하다" (digest of "RWKV: Reinventing
 *       RNNs for the Transformer Era"), Method / (2) Time-mixing (WKV): the
 *       time-parallel WKV_t formula and the recurrent form with the state
 *       (a_t, b_t).
 *  [P4] "RWKV: Reinventing RNNs for the Transformer Era" (flashpapers
 *       explainer), 3. How It Works / The WKV Operator: the same formula with
 *       per-channel (elementwise) products.
 *  [P3] "RWKV-5 Eagle과 RWKV-6 Finch", section "Eagle: 벡터 기억을 행렬 기억으로
 *       확장": s' = diag(w) s + k^T v, wkv' = s + diag(u) k^T v, w = exp(-exp(ω)),
 *       receptance reads the state like a query.
 *  [P1] also (2) output line o_t = W_o (σ(r_t) ⊙ WKV_t) and (4) Receptance
 *       Gating: σ(r_t) decides per channel how much of the aggregate passes.
 *  [P3] also, section "Finch: recurrence를 입력에 반응시키기": Finch keeps the
 *       Eagle update and makes the decay data dependent (a per-token decay
 *       vector, corrected from the input through a LoRA).
 *  [P5] "RWKV-7 \"Goose\" 아키텍처 분석", the per-token state-update pseudo-code:
 *       kv[d,e] = k_d v_e and out_e = Σ_d r_d state[d,e] (rows = key index,
 *       columns = value index).
 *
 * Readings where the pages leave a step open:
 *  - w is the positive decay RATE: the weight of a past token i seen from t is
 *    exp(-(t-1-i) w + k_i) [P1 (2)]; P1 says the raw parameter is usually
 *    mapped through -exp(.) to fix this sign, and the API takes the mapped
 *    (positive) value.
 *  - The most recent past token (i = t-1) has lag 0, i.e. weight exp(k_i),
 *    which is what makes the time-parallel and recurrent forms of [P1] agree.
 *  - The WKV-4 backward is not printed on the pages.  It is the derivative of
 *    the time-parallel formula: oracle_wkv4_backward_bruteforce writes that
 *    derivative out term by term; oracle_wkv4_backward is the same chain rule
 *    taken through the recurrent form.  gw and gu are summed over batch and time.
 *  - Eagle reads the state before the current token's k^T v is added, and
 *    diag(w), diag(u) scale the key (row) index; w is a multiplicative factor in
 *    (0, 1), unlike RWKV-4's rate.
 *  - The Eagle and Finch backward are not printed either: oracle_wkv5_backward and
 *    oracle_wkv6_backward take the chain rule through the recurrence, with the
 *    gradient of L = Σ gy·y + Σ gs_out·s_out; gomega and gu are summed over
 *    batch (and over time for Eagle's per-channel omega).
 *  - Finch's data-dependent decay is read as omega_t [B, T, H, N], one omega
 *    per token and channel with w_t = exp(-exp(omega_t)) as in Eagle, and the
 *    decay of token t multiplies the state when token t's k^T v is added (the
 *    Eagle update with w replaced by w_t), so token t reads a state in which
 *    token i < t has been decayed by w_{i+1} ... w_{t-1}.
 *
 * Layouts: WKV-4 k, v, y, gy, gk, gv are [B, T, C] (C fastest); w, u, gw, gu
 * are [C]; the fp64 state is [2, B, C] = (numerator A, denominator B) without
 * any rescaling.  WKV-5 r, k, v, y are [B, T, H, N]; omega, u are [H, N]; the
 * state is [B, H, N, N] with s[b, h, i, j], i = key index, j = value index.
 * Finch takes the same tensors with omega [B, T, H, N].
 *
 * Every function returns the number of non-finite outputs it produced (0 on
 * a healthy run), so a test can tell an overflow from a mismatch.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

int oracle_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* Sets the OpenMP thread count of later calls (n >= 1); returns the count in force. */
int oracle_set_num_threads(int n)
{
#ifdef _OPENMP
    if (n >= 1) omp_set_num_threads(n);
    return omp_get_max_threads();
#else
    (void)n;
    return 1;
#endif
}

#define IDX3(b, t, c) ((((int64_t)(b)) * T + (t)) * C + (c))

/*
 * WKV-4 forward, recurrent form [P1 (2)]:
 *   WKV_t = (a_{t-1} + e^{u+k_t} v_t) / (b_{t-1} + e^{u+k_t}),
 *   a_t = e^{-w} a_{t-1} + e^{k_t} v_t,   b_t = e^{-w} b_{t-1} + e^{k_t},
 * with a_0 = b_0 = 0 unless state_in [2,B,C] = (a_0, b_0) is given.
 * state_out, if given, receives (a_T, b_T).
 */
int64_t oracle_wkv4_forward(int64_t B, int64_t T, int64_t C,
                            const double *w, const double *u,
                            const double *k, const double *v,
                            const double *state_in, double *y, double *state_out)
{
    int64_t bad = 0;
#pragma omp parallel for collapse(2) schedule(static) reduction(+ : bad)
    for (int64_t b = 0; b < B; ++b) {
        for (int64_t c = 0; c < C; ++c) {
            double num = state_in ? state_in[(0 * B + b) * C + c] : 0.0;
            double den = state_in ? state_in[(1 * B + b) * C + c] : 0.0;
            const double decay = exp(-w[c]);
            for (int64_t t = 0; t < T; ++t) {
                const double kt = k[IDX3(b, t, c)], vt = v[IDX3(b, t, c)];
                const double cur = exp(u[c] + kt);
                const double out = (num + cur * vt) / (den + cur);
                if (!isfinite(out)) ++bad;
                if (y) y[IDX3(b, t, c)] = out;
                const double ek = exp(kt);
                num = decay * num + ek * vt;
                den = decay * den + ek;
            }
            if (state_out) {
                state_out[(0 * B + b) * C + c] = num;
                state_out[(1 * B + b) * C + c] = den;
            }
        }
    }
    return bad;
}

/*
 * WKV-4 forward, time-parallel form [P1 (2), P4 The WKV Operator], evaluated
 * term by term in O(T^2) per channel from a zero state:
 *   WKV_t = (Σ_{i<t} e^{-(t-1-i)w + k_i} v_i + e^{u+k_t} v_t)
 *         / (Σ_{i<t} e^{-(t-1-i)w + k_i}     + e^{u+k_t}).
 * The exponents of one output are shifted by their maximum before exp (the
 * ratio is unchanged), so heavy-tailed keys stay in range.
 */
int64_t oracle_wkv4_forward_bruteforce(int64_t B, int64_t T, int64_t C,
                                       const double *w, const double *u,
                                       const double *k, const double *v, double *y)
{
    int64_t bad = 0;
#pragma omp parallel for collapse(2) schedule(static) reduction(+ : bad)
    for (int64_t b = 0; b < B; ++b) {
        for (int64_t c = 0; c < C; ++c) {
            for (int64_t t = 0; t < T; ++t) {
                double m = u[c] + k[IDX3(b, t, c)];
                for (int64_t i = 0; i < t; ++i) {
                    const double ex = -(double)(t - 1 - i) * w[c] + k[IDX3(b, i, c)];
                    if (ex > m) m = ex;
                }
                double num = 0.0, den = 0.0;
                for (int64_t i = 0; i < t; ++i) {
                    const double wt = exp(-(double)(t - 1 - i) * w[c] + k[IDX3(b, i, c)] - m);
                    num += wt * v[IDX3(b, i, c)];
                    den += wt;
                }
                const double cur = exp(u[c] + k[IDX3(b, t, c)] - m);
                num += cur * v[IDX3(b, t, c)];
                den += cur;
                const double out = num / den;
                if (!isfinite(out)) ++bad;
                y[IDX3(b, t, c)] = out;
            }
        }
    }
    return bad;
}

/*
 * WKV-4 backward through the recurrent form [P1 (2)].  With L = Σ gy_t WKV_t,
 * D_t = b_{t-1} + e^{u+k_t}, g_t = gy_t / D_t and h_t = gy_t WKV_t / D_t:
 *   dL/da_{t-1} = g_t + e^{-w} dL/da_t,   dL/db_{t-1} = -h_t + e^{-w} dL/db_t,
 *   gv_t = e^{u+k_t} g_t + e^{k_t} dL/da_t,
 *   gk_t = e^{u+k_t} (g_t v_t - h_t) + e^{k_t} (v_t dL/da_t + dL/db_t),
 *   gu  += e^{u+k_t} (g_t v_t - h_t),
 *   gw  += -e^{-w} (a_{t-1} dL/da_t + b_{t-1} dL/db_t),
 * with dL/da_T = dL/db_T = 0.  gw, gu [C] are summed over batch and time
 * (overwritten, not accumulated).  state_in as in oracle_wkv4_forward.
 */
int64_t oracle_wkv4_backward(int64_t B, int64_t T, int64_t C,
                             const double *w, const double *u,
                             const double *k, const double *v, const double *gy,
                             const double *state_in,
                             double *gk, double *gv, double *gw, double *gu)
{
    int64_t bad = 0;
    double *pw = (double *)calloc((size_t)(B * C), sizeof(double));
    double *pu = (double *)calloc((size_t)(B * C), sizeof(double));
#pragma omp parallel reduction(+ : bad)
    {
        double *aprev = (double *)malloc((size_t)T * sizeof(double));
        double *bprev = (double *)malloc((size_t)T * sizeof(double));
        double *den = (double *)malloc((size_t)T * sizeof(double));
        double *out = (double *)malloc((size_t)T * sizeof(double));
#pragma omp for collapse(2) schedule(static)
        for (int64_t b = 0; b < B; ++b) {
            for (int64_t c = 0; c < C; ++c) {
                const double decay = exp(-w[c]);
                double num = state_in ? state_in[(0 * B + b) * C + c] : 0.0;
                double dd = state_in ? state_in[(1 * B + b) * C + c] : 0.0;
                for (int64_t t = 0; t < T; ++t) {
                    const double kt = k[IDX3(b, t, c)], vt = v[IDX3(b, t, c)];
                    const double cur = exp(u[c] + kt);
                    aprev[t] = num;
                    bprev[t] = dd;
                    den[t] = dd + cur;
                    out[t] = (num + cur * vt) / den[t];
                    const double ek = exp(kt);
                    num = decay * num + ek * vt;
                    dd = decay * dd + ek;
                }
                double da = 0.0, db = 0.0, sw = 0.0, su = 0.0;
                for (int64_t t = T - 1; t >= 0; --t) {
                    const double kt = k[IDX3(b, t, c)], vt = v[IDX3(b, t, c)];
                    const double g = gy[IDX3(b, t, c)] / den[t];
                    const double h = gy[IDX3(b, t, c)] * out[t] / den[t];
                    const double ek = exp(kt), cur = exp(u[c] + kt);
                    const double gvt = cur * g + ek * da;
                    const double gkt = cur * (g * vt - h) + ek * (vt * da + db);
                    if (!isfinite(gvt)) ++bad;
                    if (!isfinite(gkt)) ++bad;
                    gv[IDX3(b, t, c)] = gvt;
                    gk[IDX3(b, t, c)] = gkt;
                    su += cur * (g * vt - h);
                    sw += -decay * (aprev[t] * da + bprev[t] * db);
                    da = g + decay * da;
                    db = -h + decay * db;
                }
                pw[b * C + c] = sw;
                pu[b * C + c] = su;
            }
        }
        free(aprev);
        free(bprev);
        free(den);
        free(out);
    }
    for (int64_t c = 0; c < C; ++c) {
        double sw = 0.0, su = 0.0;
        for (int64_t b = 0; b < B; ++b) {
            sw += pw[b * C + c];
            su += pu[b * C + c];
        }
        gw[c] = sw;
        gu[c] = su;
        if (!isfinite(sw)) ++bad;
        if (!isfinite(su)) ++bad;
    }
    free(pw);
    free(pu);
    return bad;
}

/*
 * WKV-4 backward written out from the time-parallel form, term by term, in
 * O(T^2) per channel, zero initial state.  With weights
 *   q_{t,i} = e^{-(t-1-i)w + k_i} (i < t),  q_{t,t} = e^{u+k_t},
 *   D_t = Σ_{i<=t} q_{t,i},  WKV_t = Σ_{i<=t} q_{t,i} v_i / D_t:
 *   dWKV_t/dv_i = q_{t,i}/D_t,
 *   dWKV_t/dk_i = q_{t,i} (v_i - WKV_t)/D_t,
 *   dWKV_t/du   = q_{t,t} (v_t - WKV_t)/D_t,
 *   dWKV_t/dw   = -Σ_{i<t} (t-1-i) q_{t,i} (v_i - WKV_t)/D_t,
 * contracted with gy.  Each output's weights are shifted by their maximum.
 */
int64_t oracle_wkv4_backward_bruteforce(int64_t B, int64_t T, int64_t C,
                                        const double *w, const double *u,
                                        const double *k, const double *v, const double *gy,
                                        double *gk, double *gv, double *gw, double *gu)
{
    int64_t bad = 0;
    double *pw = (double *)calloc((size_t)(B * C), sizeof(double));
    double *pu = (double *)calloc((size_t)(B * C), sizeof(double));
#pragma omp parallel reduction(+ : bad)
    {
        double *q = (double *)malloc((size_t)T * sizeof(double));
#pragma omp for collapse(2) schedule(static)
        for (int64_t b = 0; b < B; ++b) {
            for (int64_t c = 0; c < C; ++c) {
                for (int64_t i = 0; i < T; ++i) {
                    gk[IDX3(b, i, c)] = 0.0;
                    gv[IDX3(b, i, c)] = 0.0;
                }
                double sw = 0.0, su = 0.0;
                for (int64_t t = 0; t < T; ++t) {
                    double m = u[c] + k[IDX3(b, t, c)];
                    for (int64_t i = 0; i < t; ++i) {
                        const double ex = -(double)(t - 1 - i) * w[c] + k[IDX3(b, i, c)];
                        if (ex > m) m = ex;
                    }
                    double den = 0.0, num = 0.0;
                    for (int64_t i = 0; i <= t; ++i) {
                        q[i] = (i < t) ? exp(-(double)(t - 1 - i) * w[c] + k[IDX3(b, i, c)] - m)
                                       : exp(u[c] + k[IDX3(b, t, c)] - m);
                        den += q[i];
                        num += q[i] * v[IDX3(b, i, c)];
                    }
                    const double out = num / den;
                    const double gyt = gy[IDX3(b, t, c)];
                    for (int64_t i = 0; i <= t; ++i) {
                        const double vi = v[IDX3(b, i, c)];
                        gv[IDX3(b, i, c)] += gyt * q[i] / den;
                        gk[IDX3(b, i, c)] += gyt * q[i] * (vi - out) / den;
                        if (i < t) sw += -gyt * (double)(t - 1 - i) * q[i] * (vi - out) / den;
                    }
                    su += gyt * q[t] * (v[IDX3(b, t, c)] - out) / den;
                }
                for (int64_t i = 0; i < T; ++i) {
                    if (!isfinite(gk[IDX3(b, i, c)])) ++bad;
                    if (!isfinite(gv[IDX3(b, i, c)])) ++bad;
                }
                pw[b * C + c] = sw;
                pu[b * C + c] = su;
            }
        }
        free(q);
    }
    for (int64_t c = 0; c < C; ++c) {
        double sw = 0.0, su = 0.0;
        for (int64_t b = 0; b < B; ++b) {
            sw += pw[b * C + c];
            su += pu[b * C + c];
        }
        gw[c] = sw;
        gu[c] = su;
    }
    free(pw);
    free(pu);
    return bad;
}

/*
 * One recurrent WKV-4 step for every (stream b, channel c) [P1 (2)]:
 * reads (a, b) from state [2, B, C], writes WKV into y [B, C] and the updated
 * state back into state.  k, v are [B, C].
 */
int64_t oracle_wkv4_step(int64_t B, int64_t C, const double *w, const double *u,
                         const double *k, const double *v, double *state, double *y)
{
    int64_t bad = 0;
#pragma omp parallel for collapse(2) schedule(static) reduction(+ : bad)
    for (int64_t b = 0; b < B; ++b) {
        for (int64_t c = 0; c < C; ++c) {
            double *num = &state[(0 * B + b) * C + c];
            double *den = &state[(1 * B + b) * C + c];
            const double kt = k[b * C + c], vt = v[b * C + c];
            const double cur = exp(u[c] + kt);
            const double out = (*num + cur * vt) / (*den + cur);
            if (!isfinite(out)) ++bad;
            y[b * C + c] = out;
            const double decay = exp(-w[c]), ek = exp(kt);
            *num = decay * *num + ek * vt;
            *den = decay * *den + ek;
        }
    }
    return bad;
}

#define IDX4(b, t, h, n) (((((int64_t)(b)) * T + (t)) * H + (h)) * N + (n))

/*
 * Eagle / RWKV-5 WKV forward, per (batch b, head h) [P3 Eagle; P5 layout]:
 *   y_t[j] = Σ_i r_t[i] (s[i][j] + u_i k_t[i] v_t[j]),
 *   s[i][j] <- w_i s[i][j] + k_t[i] v_t[j],   w_i = exp(-exp(omega_i)),
 * starting from s_in [B,H,N,N] (or zero); s_out receives the final state.
 */
int64_t oracle_wkv5_forward(int64_t B, int64_t T, int64_t H, int64_t N,
                            const double *r, const double *k, const double *v,
                            const double *omega, const double *u,
                            const double *s_in, double *y, double *s_out)
{
    int64_t bad = 0;
#pragma omp parallel reduction(+ : bad)
    {
        double *s = (double *)malloc((size_t)(N * N) * sizeof(double));
        double *wdec = (double *)malloc((size_t)N * sizeof(double));
#pragma omp for collapse(2) schedule(static)
        for (int64_t b = 0; b < B; ++b) {
            for (int64_t h = 0; h < H; ++h) {
                for (int64_t i = 0; i < N; ++i) wdec[i] = exp(-exp(omega[h * N + i]));
                for (int64_t ij = 0; ij < N * N; ++ij)
                    s[ij] = s_in ? s_in[((b * H + h) * N) * N + ij] : 0.0;
                for (int64_t t = 0; t < T; ++t) {
                    for (int64_t j = 0; j < N; ++j) {
                        double acc = 0.0;
                        for (int64_t i = 0; i < N; ++i)
                            acc += r[IDX4(b, t, h, i)] *
                                   (s[i * N + j] + u[h * N + i] * k[IDX4(b, t, h, i)] * v[IDX4(b, t, h, j)]);
                        if (!isfinite(acc)) ++bad;
                        y[IDX4(b, t, h, j)] = acc;
                    }
                    for (int64_t i = 0; i < N; ++i)
                        for (int64_t j = 0; j < N; ++j)
                            s[i * N + j] = wdec[i] * s[i * N + j] + k[IDX4(b, t, h, i)] * v[IDX4(b, t, h, j)];
                }
                if (s_out)
                    for (int64_t ij = 0; ij < N * N; ++ij) s_out[((b * H + h) * N) * N + ij] = s[ij];
            }
        }
        free(s);
        free(wdec);
    }
    return bad;
}

/*
 * Eagle / RWKV-5 WKV forward unrolled into its sum over past tokens, O(T^2 N^2)
 * per (b, h), zero initial state:
 *   y_t[j] = Σ_{i<t} Σ_d r_t[d] w_d^{t-1-i} k_i[d] v_i[j] + Σ_d r_t[d] u_d k_t[d] v_t[j],
 * with w_d^n = exp(-n exp(omega_d)).
 */
int64_t oracle_wkv5_forward_bruteforce(int64_t B, int64_t T, int64_t H, int64_t N,
                                       const double *r, const double *k, const double *v,
                                       const double *omega, const double *u, double *y)
{
    int64_t bad = 0;
#pragma omp parallel for collapse(3) schedule(static) reduction(+ : bad)
    for (int64_t b = 0; b < B; ++b) {
        for (int64_t h = 0; h < H; ++h) {
            for (int64_t t = 0; t < T; ++t) {
                for (int64_t j = 0; j < N; ++j) {
                    double acc = 0.0;
                    for (int64_t i = 0; i < t; ++i) {
                        double att = 0.0;
                        for (int64_t d = 0; d < N; ++d)
                            att += r[IDX4(b, t, h, d)] * exp(-(double)(t - 1 - i) * exp(omega[h * N + d])) *
                                   k[IDX4(b, i, h, d)];
                        acc += att * v[IDX4(b, i, h, j)];
                    }
                    double bonus = 0.0;
                    for (int64_t d = 0; d < N; ++d)
                        bonus += r[IDX4(b, t, h, d)] * u[h * N + d] * k[IDX4(b, t, h, d)];
                    acc += bonus * v[IDX4(b, t, h, j)];
                    if (!isfinite(acc)) ++bad;
                    y[IDX4(b, t, h, j)] = acc;
                }
            }
        }
    }
    return bad;
}

/*
 * Finch / RWKV-6 WKV forward [P3 Finch: the decay of the Eagle update becomes
 * data dependent, one decay vector per token], per (batch b, head h):
 *   y_t[j] = Σ_i r_t[i] (s[i][j] + u_i k_t[i] v_t[j]),
 *   s[i][j] <- w_t[i] s[i][j] + k_t[i] v_t[j],   w_t[i] = exp(-exp(omega_t[i])),
 * i.e. the Eagle recurrence above with omega [B,T,H,N] read at the current
 * token; starts from s_in [B,H,N,N] (or zero), s_out receives the final state.
 */
int64_t oracle_wkv6_forward(int64_t B, int64_t T, int64_t H, int64_t N,
                            const double *r, const double *k, const double *v,
                            const double *omega, const double *u,
                            const double *s_in, double *y, double *s_out)
{
    int64_t bad = 0;
#pragma omp parallel reduction(+ : bad)
    {
        double *s = (double *)malloc((size_t)(N * N) * sizeof(double));
#pragma omp for collapse(2) schedule(static)
        for (int64_t b = 0; b < B; ++b) {
            for (int64_t h = 0; h < H; ++h) {
                for (int64_t ij = 0; ij < N * N; ++ij)
                    s[ij] = s_in ? s_in[((b * H + h) * N) * N + ij] : 0.0;
                for (int64_t t = 0; t < T; ++t) {
                    for (int64_t j = 0; j < N; ++j) {
                        double acc = 0.0;
                        for (int64_t i = 0; i < N; ++i)
                            acc += r[IDX4(b, t, h, i)] *
                                   (s[i * N + j] + u[h * N + i] * k[IDX4(b, t, h, i)] * v[IDX4(b, t, h, j)]);
                        if (!isfinite(acc)) ++bad;
                        y[IDX4(b, t, h, j)] = acc;
                    }
                    for (int64_t i = 0; i < N; ++i) {
                        const double wt = exp(-exp(omega[IDX4(b, t, h, i)]));
                        for (int64_t j = 0; j < N; ++j)
                            s[i * N + j] = wt * s[i * N + j] + k[IDX4(b, t, h, i)] * v[IDX4(b, t, h, j)];
                    }
                }
                if (s_out)
                    for (int64_t ij = 0; ij < N * N; ++ij) s_out[((b * H + h) * N) * N + ij] = s[ij];
            }
        }
        free(s);
    }
    return bad;
}

/*
 * Finch / RWKV-6 WKV forward unrolled into its sum over past tokens, zero
 * initial state: token i's k_i^T v_i enters the state after token i and is
 * then multiplied by the decay of every later token up to t-1, so
 *   y_t[j] = Σ_{i<t} Σ_d r_t[d] (Π_{m=i+1}^{t-1} w_m[d]) k_i[d] v_i[j]
 *          + Σ_d r_t[d] u_d k_t[d] v_t[j],      w_m[d] = exp(-exp(omega_m[d])).
 * The product is formed term by term (O(T^3 N^2) per head: tiny inputs only).
 */
int64_t oracle_wkv6_forward_bruteforce(int64_t B, int64_t T, int64_t H, int64_t N,
                                       const double *r, const double *k, const double *v,
                                       const double *omega, const double *u, double *y)
{
    int64_t bad = 0;
#pragma omp parallel for collapse(3) schedule(static) reduction(+ : bad)
    for (int64_t b = 0; b < B; ++b) {
        for (int64_t h = 0; h < H; ++h) {
            for (int64_t t = 0; t < T; ++t) {
                for (int64_t j = 0; j < N; ++j) {
                    double acc = 0.0;
                    for (int64_t i = 0; i < t; ++i) {
                        double att = 0.0;
                        for (int64_t d = 0; d < N; ++d) {
                            double decay = 1.0;
                            for (int64_t m = i + 1; m < t; ++m) decay *= exp(-exp(omega[IDX4(b, m, h, d)]));
                            att += r[IDX4(b, t, h, d)] * decay * k[IDX4(b, i, h, d)];
                        }
                        acc += att * v[IDX4(b, i, h, j)];
                    }
                    double bonus = 0.0;
                    for (int64_t d = 0; d < N; ++d)
                        bonus += r[IDX4(b, t, h, d)] * u[h * N + d] * k[IDX4(b, t, h, d)];
                    acc += bonus * v[IDX4(b, t, h, j)];
                    if (!isfinite(acc)) ++bad;
                    y[IDX4(b, t, h, j)] = acc;
                }
            }
        }
    }
    return bad;
}

/*
 * Receptance-gated WKV-4 forward [P1 (2) output line o_t = W_o (σ(r_t) ⊙ WKV_t)
 * and (4) Receptance Gating; the projection W_o is not part of the operator]:
 *   o_t = σ(r_t) WKV_t,   σ(x) = 1 / (1 + e^{-x}),
 * with WKV_t from oracle_wkv4_forward (same state conventions).
 */
int64_t oracle_wkv4_gated_forward(int64_t B, int64_t T, int64_t C,
                                  const double *w, const double *u,
                                  const double *k, const double *v, const double *r,
                                  const double *state_in, double *o, double *state_out)
{
    const int64_t bad = oracle_wkv4_forward(B, T, C, w, u, k, v, state_in, o, state_out);
    for (int64_t i = 0; i < B * T * C; ++i) o[i] *= 1.0 / (1.0 + exp(-r[i]));
    return bad;
}

/*
 * Gradients of L = Σ go_t o_t for the gated forward above, by the chain rule:
 * L depends on WKV through gy_t = σ(r_t) go_t, so gk, gv, gw, gu are
 * oracle_wkv4_backward with that gy, and
 *   gr_t = go_t WKV_t σ(r_t) (1 - σ(r_t)).
 */
int64_t oracle_wkv4_gated_backward(int64_t B, int64_t T, int64_t C,
                                   const double *w, const double *u,
                                   const double *k, const double *v, const double *r,
                                   const double *go, const double *state_in,
                                   double *gk, double *gv, double *gr, double *gw, double *gu)
{
    const int64_t n = B * T * C;
    double *wkv = (double *)malloc((size_t)n * sizeof(double));
    double *gy = (double *)malloc((size_t)n * sizeof(double));
    int64_t bad = oracle_wkv4_forward(B, T, C, w, u, k, v, state_in, wkv, NULL);
    for (int64_t i = 0; i < n; ++i) {
        const double s = 1.0 / (1.0 + exp(-r[i]));
        gy[i] = s * go[i];
        gr[i] = go[i] * wkv[i] * s * (1.0 - s);
    }
    bad += oracle_wkv4_backward(B, T, C, w, u, k, v, gy, state_in, gk, gv, gw, gu);
    free(wkv);
    free(gy);
    return bad;
}

/*
 * Backward of the Eagle / RWKV-5 forward above (and, with omega_per_token, of the
 * Finch / RWKV-6 forward): gradients of
 *   L = Σ_t Σ_j gy_t[j] y_t[j] + Σ_{i,j} gs_out[i][j] s_out[i][j]
 * by the chain rule through the recurrence (the pages print no backward).  With
 * S_t the state before token t and G the gradient of L with respect to S_{t+1},
 * walking t = T-1 .. 0:
 *   gr_t[i] = Σ_j gy_t[j] (S_t[i][j] + u_i k_t[i] v_t[j])
 *   gk_t[i] = Σ_j G[i][j] v_t[j] + u_i r_t[i] Σ_j gy_t[j] v_t[j]
 *   gv_t[j] = Σ_i G[i][j] k_t[i] + (Σ_i r_t[i] u_i k_t[i]) gy_t[j]
 *   gu[i]  += r_t[i] k_t[i] Σ_j gy_t[j] v_t[j]
 *   gw_t[i] = Σ_j G[i][j] S_t[i][j]                (S_{t+1} = diag(w_t) S_t + k_t^T v_t)
 *   G      <- diag(w_t) G + r_t^T gy_t              (then G is the gradient for S_t)
 * gomega = gw * dw/domega = gw * (-exp(omega)) * w, per token for Finch, summed over
 * tokens and batch for Eagle; gu is summed over batch; gs_in = G after the walk.
 * gy [B,T,H,N]; gs_out [B,H,N,N] or NULL; outputs gr, gk, gv [B,T,H,N], gomega [H,N]
 * (Eagle) or [B,T,H,N] (Finch), gu [H,N], gs_in [B,H,N,N] (or NULL).  The states of
 * every token are recomputed and kept per head (O(T N^2) memory: small inputs).
 */
static int64_t wkv56_backward(int64_t B, int64_t T, int64_t H, int64_t N, const double *r, const double *k,
                              const double *v, const double *omega, int omega_per_token, const double *u,
                              const double *s_in, const double *gy, const double *gs_out, double *gr, double *gk,
                              double *gv, double *gomega, double *gu, double *gs_in)
{
    int64_t bad = 0;
    const int64_t nomega = omega_per_token ? B * T * H * N : H * N;
    for (int64_t i = 0; i < nomega; ++i) gomega[i] = 0.0;
    for (int64_t i = 0; i < H * N; ++i) gu[i] = 0.0;
    double *S = (double *)malloc((size_t)((T + 1) * N * N) * sizeof(double));
    double *G = (double *)malloc((size_t)(N * N) * sizeof(double));
    double *wt = (double *)malloc((size_t)N * sizeof(double));
    for (int64_t b = 0; b < B; ++b) {
        for (int64_t h = 0; h < H; ++h) {
            /* forward: S[t] = state before token t, S[T] = s_out */
            for (int64_t ij = 0; ij < N * N; ++ij) S[ij] = s_in ? s_in[((b * H + h) * N) * N + ij] : 0.0;
            for (int64_t t = 0; t < T; ++t) {
                for (int64_t i = 0; i < N; ++i)
                    wt[i] = exp(-exp(omega_per_token ? omega[IDX4(b, t, h, i)] : omega[h * N + i]));
                for (int64_t i = 0; i < N; ++i)
                    for (int64_t j = 0; j < N; ++j)
                        S[(t + 1) * N * N + i * N + j] =
                            wt[i] * S[t * N * N + i * N + j] + k[IDX4(b, t, h, i)] * v[IDX4(b, t, h, j)];
            }
            for (int64_t ij = 0; ij < N * N; ++ij) G[ij] = gs_out ? gs_out[((b * H + h) * N) * N + ij] : 0.0;
            for (int64_t t = T - 1; t >= 0; --t) {
                const double *St = S + t * N * N;
                double gyv = 0.0, ruk = 0.0;
                for (int64_t j = 0; j < N; ++j) gyv += gy[IDX4(b, t, h, j)] * v[IDX4(b, t, h, j)];
                for (int64_t i = 0; i < N; ++i) ruk += r[IDX4(b, t, h, i)] * u[h * N + i] * k[IDX4(b, t, h, i)];
                for (int64_t i = 0; i < N; ++i) {
                    const double ui = u[h * N + i], ri = r[IDX4(b, t, h, i)], ki = k[IDX4(b, t, h, i)];
                    double a = 0.0, c = 0.0, gw = 0.0;
                    for (int64_t j = 0; j < N; ++j) {
                        a += gy[IDX4(b, t, h, j)] * (St[i * N + j] + ui * ki * v[IDX4(b, t, h, j)]);
                        c += G[i * N + j] * v[IDX4(b, t, h, j)];
                        gw += G[i * N + j] * St[i * N + j];
                    }
                    gr[IDX4(b, t, h, i)] = a;
                    gk[IDX4(b, t, h, i)] = c + ui * ri * gyv;
                    gu[h * N + i] += ri * ki * gyv;
                    const double om = omega_per_token ? omega[IDX4(b, t, h, i)] : omega[h * N + i];
                    const double dw = -exp(om) * exp(-exp(om));
                    if (omega_per_token) gomega[IDX4(b, t, h, i)] = gw * dw;
                    else gomega[h * N + i] += gw * dw;
                    if (!isfinite(a) || !isfinite(c)) ++bad;
                }
                for (int64_t j = 0; j < N; ++j) {
                    double a = 0.0;
                    for (int64_t i = 0; i < N; ++i) a += G[i * N + j] * k[IDX4(b, t, h, i)];
                    gv[IDX4(b, t, h, j)] = a + ruk * gy[IDX4(b, t, h, j)];
                }
                for (int64_t i = 0; i < N; ++i) {
                    const double w_i = exp(-exp(omega_per_token ? omega[IDX4(b, t, h, i)] : omega[h * N + i]));
                    for (int64_t j = 0; j < N; ++j)
                        G[i * N + j] = w_i * G[i * N + j] + r[IDX4(b, t, h, i)] * gy[IDX4(b, t, h, j)];
                }
            }
            if (gs_in)
                for (int64_t ij = 0; ij < N * N; ++ij) gs_in[((b * H + h) * N) * N + ij] = G[ij];
        }
    }
    free(S);
    free(G);
    free(wt);
    return bad;
}

int64_t oracle_wkv5_backward(int64_t B, int64_t T, int64_t H, int64_t N, const double *r, const double *k,
                             const double *v, const double *omega, const double *u, const double *s_in,
                             const double *gy, const double *gs_out, double *gr, double *gk, double *gv,
                             double *gomega, double *gu, double *gs_in)
{
    return wkv56_backward(B, T, H, N, r, k, v, omega, 0, u, s_in, gy, gs_out, gr, gk, gv, gomega, gu, gs_in);
}

int64_t oracle_wkv6_backward(int64_t B, int64_t T, int64_t H, int64_t N, const double *r, const double *k,
                             const double *v, const double *omega, const double *u, const double *s_in,
                             const double *gy, const double *gs_out, double *gr, double *gk, double *gv,
                             double *gomega, double *gu, double *gs_in)
{
    return wkv56_backward(B, T, H, N, r, k, v, omega, 1, u, s_in, gy, gs_out, gr, gk, gv, gomega, gu, gs_in);
}
