/*
 * rwkv_wkv.h — C ABI of the B200 (sm_100a) WKV operator library.
 *
 * The operator is RWKV's WKV:
 *
 *   RWKV-4 ("RWKV - Transformer 시대에 RNN을 재발명하다", Method / (2) Time-mixing
 *   (WKV); same formula in "RWKV: Reinventing RNNs for the Transformer Era",
 *   3. How It Works / The WKV Operator), per channel c:
 *
 *     wkv_t = ( Σ_{i<t} e^{-(t-1-i) w + k_i} v_i + e^{u + k_t} v_t )
 *           / ( Σ_{i<t} e^{-(t-1-i) w + k_i}     + e^{u + k_t} )
 *
 *   and its recurrent form with state (a_t, b_t):
 *     wkv_t = (a_{t-1} + e^{u+k_t} v_t) / (b_{t-1} + e^{u+k_t}),
 *     a_t = e^{-w} a_{t-1} + e^{k_t} v_t,   b_t = e^{-w} b_{t-1} + e^{k_t}.
 *
 *   Eagle / RWKV-5 ("RWKV-5 Eagle과 RWKV-6 Finch", section Eagle), per head:
 *     y_t = r_t · (s + diag(u) k_tᵀ v_t),   s ← diag(w) s + k_tᵀ v_t,
 *     w = exp(-exp(ω)),  s[i][j] with i = key index (row), j = value index.
 *
 *   Finch / RWKV-6 (same page, section Finch): the Eagle update with a
 *   data-dependent decay, w_t = exp(-exp(ω_t)) for every token t:
 *     y_t = r_t · (s + diag(u) k_tᵀ v_t),   s ← diag(w_t) s + k_tᵀ v_t.
 *
 * Conventions for every call
 *   - All tensor arguments are DEVICE pointers owned by the caller, on the
 *     current CUDA device; the library never allocates, frees or keeps them.
 *     Work is enqueued on `stream` (NULL = the legacy default stream) and the
 *     call returns without synchronising.  Inputs must stay valid and outputs
 *     untouched until the stream has run the work.
 *   - Layouts are dense row-major: WKV-4 k, v, y, gy, gk, gv are [B, T, C]
 *     (C fastest); w, u, gw, gu are [C] fp32.  WKV-5 r, k, v, y are
 *     [B, T, H, N] bf16; omega, u are [H, N] fp32; s is [B, H, N, N] fp32.
 *     Finch takes the same with omega [B, T, H, N] fp32 (step: [B, H, N]).
 *   - `w` (WKV-4) is the positive decay RATE of the formula above (the raw
 *     parameter mapped through -exp(.) by the model), not a factor.
 *   - WKV-4 state: [3, B, C] fp32 planes (a, b, p) meaning A = a·2^p,
 *     B = b·2^p (p an exponent of two).  A zero state is a = b = 0 (any p).
 *     Any finite (A, B) with A, B within fp32 range may be passed as (A, B, 0).
 *     The representation is not unique: compare states through a/b and
 *     log2(b) + p.
 *   - Returns RWKV_OK or an error status; nothing throws or aborts.
 *     Negative sizes or a NULL required pointer give RWKV_ERR_INVALID_ARG
 *     before anything is enqueued.  A launch failure gives RWKV_ERR_CUDA.
 *     Zero-sized problems are a successful no-op (T = 0 copies the state).
 *   - Values are data: no range validation; NaN and Inf propagate.
 *   - Alignment.  WKV-4 [B,T,C] tensors (k, v, y, gy, gk, gv, r, o, go, gr)
 *     whose bases are all 16-byte aligned, with C·sizeof(element) a multiple
 *     of 16, move through TMA; any other element-aligned bases or C take the
 *     plain-access instances of the same kernels (same results, fewer bytes
 *     in flight).  A pointer not aligned to its element size (4 bytes fp32,
 *     2 bytes bf16) gives RWKV_ERR_UNSUPPORTED.  The WKV-5/6 tensors r, k, v,
 *     y (and Finch's omega) must be 16-byte aligned (their rows are whole
 *     heads of 64), else RWKV_ERR_UNSUPPORTED; rwkv_wkv4_backward_noalloc
 *     keeps to the TMA conditions.
 */
#ifndef RWKV_WKV_H
#define RWKV_WKV_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define RWKV_API __attribute__((visibility("default")))
#else
#define RWKV_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t. */
typedef struct CUstream_st *rwkv_stream_t;

typedef enum {
    RWKV_OK = 0,
    RWKV_ERR_INVALID_ARG = 1,    /* bad size, NULL required pointer, bad enum */
    RWKV_ERR_UNSUPPORTED = 2,    /* valid request this build does not handle */
    RWKV_ERR_WORKSPACE = 3,      /* workspace NULL or smaller than the query */
    RWKV_ERR_CUDA = 4,           /* a CUDA runtime call or launch failed */
    RWKV_ERR_DEVICE_TIMEOUT = 5  /* a kernel's bounded wait gave up */
} rwkv_status;

/* Element type of WKV-4 k, v, y, gy, gk, gv (arithmetic is fp32 either way). */
typedef enum { RWKV_F32 = 0, RWKV_BF16 = 1 } rwkv_dtype;

/* WKV-4 forward schedule.  SEQUENTIAL: one thread scans one channel over all
 * of T.  CHUNKED: time is cut into segments scanned in parallel from a zero
 * state, joined by an associative carry pass, then rescanned for outputs
 * (for problems with too few channels to fill the GPU).  AUTO picks. */
typedef enum { RWKV_ALGO_AUTO = 0, RWKV_ALGO_SEQUENTIAL = 1, RWKV_ALGO_CHUNKED = 2 } rwkv_algo;

/* Human-readable name of a status code (static string). */
RWKV_API const char *rwkv_status_string(rwkv_status s);

/* Library ABI version, (major << 16) | minor. */
RWKV_API int rwkv_version(void);

/* Number of WKV-4 checkpoints for T steps at interval chunk_len:
 * ceil(T / chunk_len); -1 if chunk_len is not a positive multiple of 16. */
RWKV_API int64_t rwkv_wkv4_num_checkpoints(int64_t T, int64_t chunk_len);

/* Workspace bytes rwkv_wkv4_forward needs for this shape and algo (0 if none). */
RWKV_API size_t rwkv_wkv4_forward_workspace_bytes(int64_t B, int64_t T, int64_t C, int algo);

/*
 * WKV-4 forward (time-parallel training form; the recurrent form gives the
 * same values).
 *   k, v      [B,T,C] dtype, read.           y [B,T,C] dtype, written.
 *   w, u      [C] fp32, read.
 *   state_in  [3,B,C] or NULL (zero state).  state_out [3,B,C] or NULL:
 *             the state after the last token; may equal state_in.
 *   ckpt      [num_checkpoints(T, chunk_len), 3, B, C] or NULL: ckpt[j] is
 *             the state before token j·chunk_len (ckpt[0] = state_in), in
 *             the state format, with p chosen at least ceil(k·log2 e) for
 *             every key of that chunk and b < 1; rwkv_wkv4_backward reads it
 *             and relies on that choice.  chunk_len must be 16 today.
 *   algo      rwkv_algo.   workspace: device scratch of
 *             rwkv_wkv4_forward_workspace_bytes() bytes (may be NULL if 0).
 */
RWKV_API rwkv_status rwkv_wkv4_forward(int64_t B, int64_t T, int64_t C, rwkv_dtype dtype,
                              const float *w, const float *u, const void *k, const void *v, void *y,
                              const float *state_in, float *state_out, float *ckpt, int64_t chunk_len,
                              int algo, void *workspace, size_t workspace_bytes, rwkv_stream_t stream);

/*
 * Receptance-gated WKV-4 forward: the time-mixing output of the same page,
 * o_t = W_o (σ(r_t) ⊙ WKV_t) ((2) and (4) Receptance Gating), without the
 * projection W_o (a GEMM outside the operator):
 *   o = σ(r) ⊙ WKV,   σ(x) = 1 / (1 + e^{-x}),
 * in one pass: the same arguments as rwkv_wkv4_forward plus
 *   r         [B,T,C] dtype, read (required);
 *   o         [B,T,C] dtype, written (required; replaces y).
 * state_out and ckpt are those of the ungated forward over the same k, v (the
 * gate does not enter the recurrence), so rwkv_wkv4_backward_gated reads the
 * same checkpoints.  Workspace: rwkv_wkv4_forward_workspace_bytes().
 */
RWKV_API rwkv_status rwkv_wkv4_forward_gated(int64_t B, int64_t T, int64_t C, rwkv_dtype dtype,
                                    const float *w, const float *u, const void *k, const void *v,
                                    const void *r, void *o, const float *state_in, float *state_out,
                                    float *ckpt, int64_t chunk_len, int algo, void *workspace,
                                    size_t workspace_bytes, rwkv_stream_t stream);

/* Workspace bytes rwkv_wkv4_backward needs; have_ckpt = 0 adds room to
 * recompute the checkpoints. */
RWKV_API size_t rwkv_wkv4_backward_workspace_bytes(int64_t B, int64_t T, int64_t C, int64_t chunk_len, int have_ckpt);

/*
 * WKV-4 backward: gradients of L = Σ gy·y with respect to k, v, w, u.
 * The pages print no backward; this is the derivative of the formula above.
 *   k, v, gy  [B,T,C] dtype, read.          gk, gv [B,T,C] dtype, written.
 *   gw, gu    [C] fp32, OVERWRITTEN with the sum over batch and time.
 *   state_in  the forward's initial state, or NULL (zero); used only when
 *             ckpt is NULL.
 *   ckpt      the checkpoints written by rwkv_wkv4_forward with the same
 *             inputs and chunk_len (16), or NULL to recompute them into the
 *             workspace.
 *   Deterministic: the same inputs give bit-identical outputs.
 */
RWKV_API rwkv_status rwkv_wkv4_backward(int64_t B, int64_t T, int64_t C, rwkv_dtype dtype,
                               const float *w, const float *u, const void *k, const void *v,
                               const void *gy, const float *state_in, const float *ckpt,
                               int64_t chunk_len, void *gk, void *gv, float *gw, float *gu,
                               void *workspace, size_t workspace_bytes, rwkv_stream_t stream);

/*
 * Backward of the receptance-gated forward: gradients of L = Σ go·o with
 * o = σ(r) ⊙ WKV.  The same arguments as rwkv_wkv4_backward with gy replaced
 * by r and go, plus gr:
 *   r, go     [B,T,C] dtype, read (required).
 *   gr        [B,T,C] dtype, written: go · WKV · σ(r)(1 - σ(r)).
 *   gk, gv, gw, gu as rwkv_wkv4_backward with gy = σ(r) ⊙ go.
 * Workspace: rwkv_wkv4_backward_workspace_bytes().  Deterministic.
 */
RWKV_API rwkv_status rwkv_wkv4_backward_gated(int64_t B, int64_t T, int64_t C, rwkv_dtype dtype,
                                     const float *w, const float *u, const void *k, const void *v,
                                     const void *r, const void *go, const float *state_in,
                                     const float *ckpt, int64_t chunk_len, void *gk, void *gv, void *gr,
                                     float *gw, float *gu, void *workspace, size_t workspace_bytes,
                                     rwkv_stream_t stream);

/*
 * WKV-4 recurrent decode: one token for each of B independent streams.
 *   k, v, y   [B,C] dtype.   w, u [C] fp32.
 *   state_in  [3,B,C] or NULL (zero).  state_out [3,B,C]; may equal
 *             state_in (in-place update).
 */
RWKV_API rwkv_status rwkv_wkv4_step(int64_t B, int64_t C, rwkv_dtype dtype, const float *w, const float *u,
                           const void *k, const void *v, void *y, const float *state_in,
                           float *state_out, rwkv_stream_t stream);

/* Workspace bytes rwkv_wkv5_forward needs (0 if none): with two or more 64-token chunks per head,
 * a 64 x 64 fp32 summary and a flag for each of up to 296 CTAs (the heads' chunks are dealt out
 * evenly to two CTAs per SM; a CTA whose chunks end inside a head publishes the state they reach
 * from a zero state, and the CTAs holding the rest of that head fold it into their start). */
RWKV_API size_t rwkv_wkv5_forward_workspace_bytes(int64_t B, int64_t T, int64_t H, int64_t N);

/*
 * Eagle / RWKV-5 multi-head matrix-state WKV forward.
 *   r, k, v   [B,T,H,N] bf16, read.      y [B,T,H,N] bf16, written.
 *   omega, u  [H,N] fp32 (w = exp(-exp(omega)) is formed inside).
 *   s_in      [B,H,N,N] fp32 or NULL (zero).  s_out [B,H,N,N] fp32 or NULL;
 *             may equal s_in.
 *   workspace device scratch of rwkv_wkv5_forward_workspace_bytes() bytes, 16-byte aligned
 *             (RWKV_ERR_WORKSPACE if NULL or smaller, RWKV_ERR_UNSUPPORTED if misaligned;
 *             may be NULL if the query gives 0).  Calls that share one workspace must be
 *             ordered (the same stream): it holds flags the kernel waits on.
 *   N must be 64 (RWKV_ERR_UNSUPPORTED otherwise).
 */
RWKV_API rwkv_status rwkv_wkv5_forward(int64_t B, int64_t T, int64_t H, int64_t N,
                              const void *r, const void *k, const void *v,
                              const float *omega, const float *u, void *y,
                              const float *s_in, float *s_out,
                              void *workspace, size_t workspace_bytes, rwkv_stream_t stream);

/* Workspace bytes rwkv_wkv5_backward needs (0 for an empty problem or N != 64). */
RWKV_API size_t rwkv_wkv5_backward_workspace_bytes(int64_t B, int64_t T, int64_t H, int64_t N);

/*
 * Eagle / RWKV-5 backward: gradients of L = Σ gy·y + Σ gs_out ∘ s_out for the
 * forward above ("RWKV-5 Eagle과 RWKV-6 Finch", section Eagle; the pages print
 * no backward, this is the chain rule through its recurrence).  With
 * G_T = gs_out and G_t = diag(w) G_{t+1} + r_tᵀ gy_t (the gradient of the
 * state after token t-1):
 *   gr_t = s_t gy_tᵀ + u ⊙ k_t (v_t·gy_t),   gk_t = G_{t+1} v_tᵀ + u ⊙ r_t (v_t·gy_t),
 *   gv_t = G_{t+1}ᵀ k_t + (Σ r_t u k_t) gy_t,  gs_in = G_0,
 *   gomega_d = Σ_{b,t} (Σ_j G_{t+1}[d][j] s_t[d][j]) · dw_d/dω_d,  gu_d = Σ_{b,t} r_t[d] k_t[d] (v_t·gy_t).
 *   r, k, v, gy   [B,T,H,N] bf16, read.      gr, gk, gv [B,T,H,N] bf16, written.
 *   omega, u      [H,N] fp32, read.          gomega, gu [H,N] fp32, OVERWRITTEN with the sums over
 *                                            batch and time.
 *   s_in          [B,H,N,N] fp32, the forward's initial state, or NULL (zero).
 *   gs_out        [B,H,N,N] fp32, the gradient of the final state, or NULL (zero).
 *   gs_in         [B,H,N,N] fp32, written with the gradient of s_in, or NULL (not wanted).
 *   workspace     device scratch of rwkv_wkv5_backward_workspace_bytes() bytes (the forward
 *                 states at every 64th token, per-row sums).
 *   N must be 64; the [B,T,H,N] tensors 16-byte aligned (RWKV_ERR_UNSUPPORTED otherwise).
 *   Any decay w in [0, 1]: channels decaying faster than exp(omega) = 2
 *   (w < 0.135) are summed over lags up to 15 where the rest stays on the
 *   chunked tensor-core form.  The reversed forward pass (gv, gs_in) runs on an
 *   internal non-blocking stream per device, ordered after and before the
 *   caller's stream with events (capture-safe once a first call has made it).
 *   Deterministic.
 */
RWKV_API rwkv_status rwkv_wkv5_backward(int64_t B, int64_t T, int64_t H, int64_t N, const void *r, const void *k,
                               const void *v, const float *omega, const float *u, const float *s_in,
                               const void *gy, const float *gs_out, void *gr, void *gk, void *gv,
                               float *gomega, float *gu, float *gs_in, void *workspace, size_t workspace_bytes,
                               rwkv_stream_t stream);

/*
 * Eagle / RWKV-5 recurrent decode: one token for each of B independent
 * streams ("RWKV-5 Eagle과 RWKV-6 Finch", section Eagle): per head,
 *   y = r·(s + diag(u)·kᵀv),   then   s <- diag(w)·s + kᵀv,  w = exp(-exp(ω)),
 * which is rwkv_wkv5_forward with T = 1.
 *   r, k, v, y  [B,H,N] bf16 (the token of every stream and head).
 *   omega, u    [H,N] fp32.
 *   s_in        [B,H,N,N] fp32, or NULL (zero state).
 *   s_out       [B,H,N,N] fp32, required; may equal s_in (in-place update).
 *   N must be 64 (RWKV_ERR_UNSUPPORTED otherwise); s_in and s_out must be
 *   16-byte aligned (RWKV_ERR_UNSUPPORTED otherwise).
 */
RWKV_API rwkv_status rwkv_wkv5_step(int64_t B, int64_t H, int64_t N, const void *r, const void *k,
                           const void *v, const float *omega, const float *u, void *y,
                           const float *s_in, float *s_out, rwkv_stream_t stream);

/* Workspace bytes rwkv_wkv6_forward needs (0 if none). */
RWKV_API size_t rwkv_wkv6_forward_workspace_bytes(int64_t B, int64_t T, int64_t H, int64_t N);

/*
 * Finch / RWKV-6 multi-head matrix-state WKV forward with a per-token decay
 * ("RWKV-5 Eagle과 RWKV-6 Finch", section Finch: Eagle's recurrence with the
 * decay made data dependent).  Per head, for t = 0 .. T-1:
 *   y_t = r_t · (s + diag(u) k_tᵀ v_t),   then   s <- diag(w_t) s + k_tᵀ v_t,
 *   w_t = exp(-exp(omega_t)),
 * so token i < t reaches token t decayed by w_{i+1} ⋯ w_{t-1}.
 *   r, k, v   [B,T,H,N] bf16, read.      y [B,T,H,N] bf16, written.
 *   omega     [B,T,H,N] fp32 (one value per token and channel), read.
 *   u         [H,N] fp32.
 *   s_in      [B,H,N,N] fp32 or NULL (zero).  s_out [B,H,N,N] fp32 or NULL;
 *             may equal s_in.
 *   N must be 64 (RWKV_ERR_UNSUPPORTED otherwise); omega follows the
 *   alignment rule of the [B,T,.] tensors.
 */
RWKV_API rwkv_status rwkv_wkv6_forward(int64_t B, int64_t T, int64_t H, int64_t N,
                              const void *r, const void *k, const void *v,
                              const float *omega, const float *u, void *y,
                              const float *s_in, float *s_out,
                              void *workspace, size_t workspace_bytes, rwkv_stream_t stream);

/*
 * Finch / RWKV-6 recurrent decode: one token for each of B independent
 * streams, rwkv_wkv6_forward with T = 1.
 *   r, k, v, y  [B,H,N] bf16.   omega [B,H,N] fp32 (this token's decay).
 *   u           [H,N] fp32.
 *   s_in        [B,H,N,N] fp32, or NULL (zero state).
 *   s_out       [B,H,N,N] fp32, required; may equal s_in (in-place update).
 *   N must be 64; s_in and s_out must be 16-byte aligned
 *   (RWKV_ERR_UNSUPPORTED otherwise).
 */
RWKV_API rwkv_status rwkv_wkv6_step(int64_t B, int64_t H, int64_t N, const void *r, const void *k,
                           const void *v, const float *omega, const float *u, void *y,
                           const float *s_in, float *s_out, rwkv_stream_t stream);

/* Workspace bytes rwkv_wkv6_backward needs (0 for an empty problem or N != 64). */
RWKV_API size_t rwkv_wkv6_backward_workspace_bytes(int64_t B, int64_t T, int64_t H, int64_t N);

/*
 * Finch / RWKV-6 backward: gradients of L = Σ gy·y + Σ gs_out ∘ s_out for
 * rwkv_wkv6_forward ("RWKV-5 Eagle과 RWKV-6 Finch", section Finch; the pages
 * print no backward, this is the chain rule through its recurrence).  With s_t
 * the state before token t, G_T = gs_out and G_t = diag(w_t) G_{t+1} + r_tᵀ gy_t:
 *   gr_t = s_t gy_tᵀ + u ⊙ k_t (v_t·gy_t),   gk_t = G_{t+1} v_tᵀ + u ⊙ r_t (v_t·gy_t),
 *   gv_t = G_{t+1}ᵀ k_t + (Σ r_t u k_t) gy_t,  gs_in = G_0,
 *   gomega_t[d] = (Σ_j G_{t+1}[d][j] s_t[d][j]) · dw_t[d]/dω_t[d]   (dw/dω = -e^ω w),
 *   gu_d = Σ_{b,t} r_t[d] k_t[d] (v_t·gy_t).
 *   r, k, v, gy   [B,T,H,N] bf16, read.      gr, gk, gv [B,T,H,N] bf16, written.
 *   omega         [B,T,H,N] fp32, read.      gomega [B,T,H,N] fp32, written (one value per
 *                                            token and channel, as omega).
 *   u             [H,N] fp32, read.          gu [H,N] fp32, OVERWRITTEN with the sum over
 *                                            batch and time.
 *   s_in          [B,H,N,N] fp32, the forward's initial state, or NULL (zero).
 *   gs_out        [B,H,N,N] fp32, the gradient of the final state, or NULL (zero).
 *   gs_in         [B,H,N,N] fp32, written with the gradient of s_in, or NULL (not wanted).
 *   workspace     device scratch of rwkv_wkv6_backward_workspace_bytes() bytes (the forward
 *                 states at every 64th token, per-CTA scratch, the gu parts);
 *                 RWKV_ERR_WORKSPACE if smaller.
 *   N must be 64 and every tensor 16-byte aligned, and B·H·ceil(T/64) (one CTA per
 *   64-token chunk) and 2·B·H (two per head for the boundary scans) at most 2^31 - 1
 *   (RWKV_ERR_UNSUPPORTED otherwise).
 *   Any decay w in [0, 1]: the recurrence runs token by token on the CUDA cores,
 *   so no factorization range applies.  Deterministic (gu is reduced in a fixed
 *   order).  Runs on `stream` only; allocates nothing.
 */
RWKV_API rwkv_status rwkv_wkv6_backward(int64_t B, int64_t T, int64_t H, int64_t N, const void *r, const void *k,
                               const void *v, const float *omega, const float *u, const float *s_in,
                               const void *gy, const float *gs_out, void *gr, void *gk, void *gv,
                               float *gomega, float *gu, float *gs_in, void *workspace, size_t workspace_bytes,
                               rwkv_stream_t stream);

/* Largest B * C that rwkv_wkv4_backward_noalloc accepts. */
#define RWKV_NOALLOC_MAX_LANES 262144

/*
 * WKV-4 backward that allocates nothing and needs no workspace.
 * The pages have no counterpart: this is a library convenience for callers
 * that cannot allocate device memory where they run the backward (device
 * memory owned in full by another allocator, latency-critical loops that
 * must not pay cudaMalloc's implicit synchronisation, systems that allocate
 * only at start-up).  Same arguments and results as rwkv_wkv4_backward with
 * ckpt required (the forward's checkpoints), no workspace, and the TMA
 * alignment (16-byte bases, C·sizeof(element) a multiple of 16; else
 * RWKV_ERR_UNSUPPORTED); the per-lane
 * scratch lives in a fixed array inside the library (RWKV_NOALLOC_MAX_LANES
 * lanes, 4 MiB, held on every GPU that loads the library until exit).
 *   - B * C > RWKV_NOALLOC_MAX_LANES returns RWKV_ERR_WORKSPACE (too big for
 *     the fixed scratch); ckpt == NULL returns RWKV_ERR_INVALID_ARG.
 *   - The first call on each device looks up the array's device address
 *     (cudaGetSymbolAddress) with that device current and caches it for the
 *     device's current context; the first call after that context is
 *     replaced (cudaDeviceReset) looks it up again.  Make the first call on
 *     a device before any stream capture.
 *   - All calls share the array: calls whose GPU work overlaps (other
 *     streams, other threads) race and must be ordered by the caller.
 *   - Calls no cudaMalloc, cudaFree or allocating library routine.
 */
RWKV_API rwkv_status rwkv_wkv4_backward_noalloc(int64_t B, int64_t T, int64_t C, rwkv_dtype dtype,
                                                const float *w, const float *u, const void *k,
                                                const void *v, const void *gy, const float *ckpt,
                                                int64_t chunk_len, void *gk, void *gv, float *gw,
                                                float *gu, rwkv_stream_t stream);

/*
 * Synchronises `stream`, then reports and clears the device error word that
 * kernels set when a bounded wait gives up (RWKV_ERR_DEVICE_TIMEOUT), or
 * RWKV_ERR_CUDA if the stream itself failed.
 * The error word is one per device and process, shared by every call on that
 * device whatever its stream or host thread: a timeout in work on one stream
 * is reported to (and cleared by) the first caller that checks, on any
 * stream.  Callers that run the library from several streams and need to
 * know which call timed out must check after each call, in stream order.
 */
RWKV_API rwkv_status rwkv_check_device_error(rwkv_stream_t stream);

/*
 * Test hooks for the failure path of the bounded waits (the pages have no
 * counterpart; they exist so that a test can watch a wait give up without
 * faulting or hanging the GPU).  Both act on the current device, synchronise
 * it first, and hold until changed; they are not meant for production use.
 *
 * rwkv_debug_set_wait_limit_ns: how long every bounded wait of the library's
 *   kernels polls before giving up (it then sets RWKV_ERR_DEVICE_TIMEOUT in
 *   the device error word and the CTA leaves at its next barrier, after
 *   waiting, bounded again, for the copies and MMAs it had issued).  ns = 0
 *   restores the default of one second.
 * rwkv_debug_withhold_loads: on != 0 makes the thread that issues a kernel's
 *   TMA loads arm its barrier and issue none, so the first wait of every CTA
 *   runs out with nothing in flight; on = 0 restores normal operation.
 *   Calls return RWKV_OK meanwhile and their outputs are undefined.
 */
RWKV_API rwkv_status rwkv_debug_set_wait_limit_ns(uint64_t ns);
RWKV_API rwkv_status rwkv_debug_withhold_loads(int on);

#ifdef __cplusplus
}
#endif

#endif /* RWKV_WKV_H */
