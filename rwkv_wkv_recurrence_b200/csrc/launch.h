// Internal launch interface between the C-ABI layer (api.cu) and the kernel
// translation units.  Not part of the public header.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

namespace rwkv {

struct DevCtl;  // the device control block (wkv_common.cuh)

// Parameters of the WKV-4 forward kernel.  A CTA owns 32 channels of one
// batch row over one time segment [seg*seg_len, min(T, (seg+1)*seg_len)).
struct Fwd4Params {
  int B, T, C;
  int ctiles;   // ceil(C / 32)
  int seg_len;  // time steps per segment (multiple of the 64-step tile)
  int nseg;
  int stages;   // TMA pipeline depth
  const float* w;
  const float* u;
  void* y;                        // [B,T,C] or null (state-only pass)
  const float* start;             // start state per segment, or null = zero
  long long start_seg_stride;     // floats between consecutive segments' start states
  float* end;                     // end state per segment, or null
  long long end_seg_stride;
  float* ckpt;                    // [nck,3,B,C] states before tokens 0, L, 2L, ... or null
  int ckpt_len;                   // L (multiple of 16) when ckpt != null
  int tma;                        // 1: k, v (, r) arrive by TMA and y leaves by TMA stores; 0: plain
                                  // element loads and stores (any element-aligned base, any C)
  const void* k;                  // [B,T,C] (read directly when tma == 0)
  const void* v;
  const void* r;                  // [B,T,C] receptance of the gated forward (tma == 0), else null
  DevCtl* ctl;                    // device control block (error word, wait limit)
  // the one-launch chunked schedule (launch_wkv4_fwd_lookback): per segment and lane the summary as
  // (a, b, p) doubles, one flag per (segment, CTA) zeroed before the launch, and the sequence's
  // start state (or null = zero)
  double* lb_agg;                 // [nseg][B*C][3]
  unsigned int* lb_flag;          // [nseg][ctiles*B]
  const float* lb_in;             // [3,B,C] or null
};

struct Bwd4Params {
  int B, T, C;
  int ctiles;
  int stages;
  const float* w;
  const float* u;
  const float* ckpt;  // [ceil(T/16),3,B,C], interval 16
  void* gk;
  void* gv;
  double* part;       // [2,B,C] per-lane gw, gu partial sums
  DevCtl* ctl;        // device control block
  const void* r;      // [B,T,C] receptance (gated backward only)
  void* gr;           // [B,T,C] its gradient (gated backward only)
  int tma;            // 1: k, v, gy (go) by TMA, gk, gv by TMA stores; 0: plain element accesses
  const void* k;      // [B,T,C] (read directly when tma == 0)
  const void* v;
  const void* g;      // gy, or go with the gate (tma == 0)
};

struct Wkv5StepParams {
  int B, H;
  const __nv_bfloat16* r;  // [B,H,64]
  const __nv_bfloat16* k;
  const __nv_bfloat16* v;
  const float* omega;      // [H,64], or [B,H,64] when omega_per_stream
  int omega_per_stream;    // 1: one decay per stream and head (Finch), 0: per head (Eagle)
  const float* u;          // [H,64]
  __nv_bfloat16* y;        // [B,H,64]
  const float* s_in;       // [B,H,64,64] or null (zero state)
  float* s_out;            // [B,H,64,64]; may equal s_in
};

constexpr int kWkv5MaxSlots = 296;  // Eagle forward CTAs: two per SM of a 148-SM part

struct Wkv5Params {
  int B, T, H;
  const __nv_bfloat16* r;
  const __nv_bfloat16* k;
  const __nv_bfloat16* v;
  const float* omega;   // [H,64]
  const float* u;       // [H,64]
  __nv_bfloat16* y;
  const float* s_in;    // [B,H,64,64] or null
  float* s_out;         // [B,H,64,64] or null
  DevCtl* ctl;
  // Slot plan (forward only; nslot = 0: one CTA per head).  The heads' 64-token chunks, laid end
  // to end, are dealt out to nslot CTAs in the order they start: slot s takes chunks
  // [slot_first[s], slot_first[s + 1]).
  int nslot;
  int slot_first[kWkv5MaxSlots + 1];
  float* slot_sum;          // [nslot][256 threads][16]: a slot's last segment from a zero state
  unsigned int* slot_flag;  // [nslot] flags, then the ticket counter; zeroed before the launch
};

struct Wkv6Params {
  int B, T, H;
  const __nv_bfloat16* r;
  const __nv_bfloat16* k;
  const __nv_bfloat16* v;
  const float* omega;   // [B,T,H,64]: one decay per token and channel
  const float* u;       // [H,64]
  __nv_bfloat16* y;
  const float* s_in;    // [B,H,64,64] or null
  float* s_out;         // [B,H,64,64] or null
  DevCtl* ctl;
};

// One pass of the Eagle backward (wkv5_bwd.cu): for queries q, keys p (both through TMA maps),
// coefficients c and multipliers m (read directly), the state read with the decay on the output
// channel.  Forward pass: gr, the state checkpoints and the gu sums; reversed pass (time reversed
// inside the kernel, the tensors read and written in their own order, chunks those of the forward
// pass, the first `lead` positions empty): gk and the decay-gradient sums.
struct Wkv5BwdParams {
  int B, T, H;
  int lead;                  // positions the first chunk starts before the sequence (reversed pass)
  const __nv_bfloat16* m;    // [B,T,H,64]: r (forward pass) or k (reversed)
  const __nv_bfloat16* c;    // [B,T,H,64]: k (forward pass) or r (reversed)
  const float* omega;        // [H,64]
  const float* u;            // [H,64]
  const float* x0;           // [B,H,64,64] carried state at the start, or null (zero)
  __nv_bfloat16* out;        // [B,T,H,64]: gr (forward pass) or gk (reversed)
  float* ckpt;               // [B,H,nchunk,64,64] forward states at chunk starts (written / read)
  double* part;              // [B,H,64] per-row sums (gu parts / decay-gradient parts)
  DevCtl* ctl;
};

// Finch backward (wkv6_bwd.cu), chunk-parallel: per 64-token chunk the state and gradient increments
// and the decay product (xs, xg, dec); per (batch row, head) the state entering and the gradient
// leaving every chunk (in place over xs, xg) and gs_in; per chunk gr, gk, gv, gomega and the gu
// parts; the gu parts summed over batch rows and chunks.
struct Wkv6BwdParams {
  int B, T, H;
  const __nv_bfloat16* r;
  const __nv_bfloat16* k;
  const __nv_bfloat16* v;
  const __nv_bfloat16* gy;
  const float* omega;    // [B,T,H,64]
  const float* u;        // [H,64]
  const float* s_in;     // [B,H,64,64] or null (zero)
  const float* gs_out;   // [B,H,64,64] or null (zero)
  __nv_bfloat16* gr;
  __nv_bfloat16* gk;
  __nv_bfloat16* gv;
  float* gomega;         // [B,T,H,64]
  float* gu;             // [H,64]
  float* gs_in;          // [B,H,64,64] or null (not wanted)
  float* xs;             // wkv6_bwd_block_floats() floats of workspace
  float* xg;             // wkv6_bwd_block_floats() floats
  float* dec;            // wkv6_bwd_row_floats() floats
  float* part;           // wkv6_bwd_row_floats() floats (gu parts)
};
size_t wkv6_bwd_block_floats(int B, int T, int H);
size_t wkv6_bwd_row_floats(int B, int T, int H);
cudaError_t launch_wkv6_bwd(const Wkv6BwdParams& p, cudaStream_t st);

int fwd_tile_steps();
int fwd_store_steps();
// Stage count of the forward's input pipeline (1 on the plain-access path, which has no pipeline).
int fwd_stages(bool bf16, int seg_len, bool gate = false, bool tma = true);
int bwd_tile_steps();
int bwd_store_steps();
int bwd_stages(bool bf16, int T, bool gate = false, bool tma = true);
// mk, mv: [fwd_tile_steps() x 32] boxes over k, v; my: [fwd_store_steps() x 32] boxes over y
// (TMA stores; any valid map when p.y is null).  With p.tma == 0 the maps are not read (any value).
cudaError_t launch_wkv4_fwd(bool bf16, const CUtensorMap& mk, const CUtensorMap& mv, const CUtensorMap& my,
                            const Fwd4Params& p, cudaStream_t st);
// The chunked schedule in one launch (TMA only, every tile of a segment resident in the stages,
// p.start null, p.end the final state written by the last segment, p.lb_* set).
cudaError_t launch_wkv4_fwd_lookback(bool bf16, const CUtensorMap& mk, const CUtensorMap& mv, const CUtensorMap& my,
                                     const Fwd4Params& p, cudaStream_t st);
// The receptance-gated forward: also reads r ([fwd_tile_steps() x 32] boxes) and writes σ(r) ⊙ WKV.
cudaError_t launch_wkv4_fwd_gated(bool bf16, const CUtensorMap& mk, const CUtensorMap& mv, const CUtensorMap& my,
                                  const CUtensorMap& mr, const Fwd4Params& p, cudaStream_t st);
cudaError_t launch_wkv4_carry(int B, int C, int T, int nseg, int seg_len, const float* w, const float* state_in,
                              float* ws, float* state_out, cudaStream_t st);
// mk, mv, mgy: [bwd_tile_steps() x 32] boxes over k, v, gy; mgk, mgv: [bwd_store_steps() x 32]
// boxes over gk, gv (written by TMA stores).
cudaError_t launch_wkv4_bwd(bool bf16, const CUtensorMap& mk, const CUtensorMap& mv, const CUtensorMap& mgy,
                            const CUtensorMap& mgk, const CUtensorMap& mgv, const Bwd4Params& p, cudaStream_t st);
// The receptance-gated backward: mo are [bwd_tile_steps() x 32] boxes over go; p.r is read and p.gr
// written with plain coalesced accesses.
cudaError_t launch_wkv4_bwd_gated(bool bf16, const CUtensorMap& mk, const CUtensorMap& mv, const CUtensorMap& mo,
                                  const CUtensorMap& mgk, const CUtensorMap& mgv, const Bwd4Params& p,
                                  cudaStream_t st);
cudaError_t launch_wkv4_reduce_wu(int B, int C, const double* part, float* gw, float* gu, cudaStream_t st);
cudaError_t launch_wkv4_step(bool bf16, int B, int C, const float* w, const float* u, const void* k, const void* v,
                             void* y, const float* state_in, float* state_out, bool vec4, cudaStream_t st);
cudaError_t launch_copy_state(int B, int C, const float* state_in, float* state_out, cudaStream_t st);

// Tensor map over a dense [B, T, C] tensor with boxes of [1, box_t, 32].
bool make_btc_map(CUtensorMap* m, const void* base, bool bf16, int B, int T, int C, int box_t);
// Tensor map over a bf16 [B, T, W] tensor with [1, 64, 64] boxes and the 128-byte swizzle.
bool make_bf16_box64_map(CUtensorMap* m, const void* base, int B, int T, int W);
cudaError_t launch_wkv5_step(const Wkv5StepParams& p, cudaStream_t st);
// reversed: the operator over reversed time on tensors kept in their own order (token t of the
// reversed problem is token T-1-t of r, k, v and y).
cudaError_t launch_wkv5_fwd(const CUtensorMap& mr, const CUtensorMap& mk, const CUtensorMap& mv, const Wkv5Params& p,
                            cudaStream_t st, bool reversed = false);
// mw: [1, 64, 32] fp32 boxes (128-byte swizzle) over omega [B, T, H*64].
cudaError_t launch_wkv6_fwd(const CUtensorMap& mr, const CUtensorMap& mk, const CUtensorMap& mv,
                            const CUtensorMap& mw, const Wkv6Params& p, cudaStream_t st);
// Eagle backward passes (maps over q, p, c: [1, 64, 64] bf16 boxes, 128-byte swizzle) and the batch
// reduction of the passes' per-row sums into gomega and gu.
cudaError_t launch_wkv5_bwd_pass(bool rev, const CUtensorMap& mq, const CUtensorMap& mp, const CUtensorMap& mc,
                                 const Wkv5BwdParams& p, cudaStream_t st);
cudaError_t launch_wkv5_bwd_reduce(int B, int H, const double* part_fwd, const double* part_rev, const float* omega,
                                   float* gomega, float* gu, cudaStream_t st);
// Tensor map over an fp32 [B, T, W] tensor with [1, 64, 32] boxes and the 128-byte swizzle.
bool make_f32_box32_map(CUtensorMap* m, const void* base, int B, int T, int W);
// Device address of the library's control block on the current device (null on failure).
DevCtl* device_ctl();

// Sets the dynamic shared-memory limit of `func` once per device.
cudaError_t ensure_smem_attr(const void* func, int bytes, unsigned* device_mask);

// Unique id of the context current on this thread; 0 if there is none or the driver cannot say.
unsigned long long current_context_id();

}  // namespace rwkv
