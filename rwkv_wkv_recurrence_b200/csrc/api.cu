// C-ABI layer: argument validation, workspace planning, TMA descriptors and
// kernel dispatch for the calls declared in include/rwkv_wkv.h.
#include <algorithm>
#include <climits>
#include <cstddef>
#include <cstring>
#include <initializer_list>
#include <mutex>

#include "../../include/rwkv_wkv.h"
#include "launch.h"
#include "wkv_common.cuh"

namespace rwkv {

// The library's device control block (one per device that loads the library):
// error word, load-withholding test hook, bounded-wait limit.
__device__ DevCtl g_ctl = {0u, 0u, kDefaultWaitLimitNs};

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// Tensor map over a dense [B, T, C] tensor, box = [1, box_t, 32] (C innermost).
bool make_btc_map(CUtensorMap* m, const void* base, bool bf16, int B, int T, int C, int box_t) {
  EncodeTiledFn enc = encode_fn();
  if (enc == nullptr) return false;
  const size_t esz = bf16 ? 2 : 4;
  cuuint64_t dims[3] = {(cuuint64_t)C, (cuuint64_t)T, (cuuint64_t)B};
  cuuint64_t strides[2] = {(cuuint64_t)C * esz, (cuuint64_t)C * T * esz};
  cuuint32_t box[3] = {32u, (cuuint32_t)box_t, 1u};
  cuuint32_t estr[3] = {1u, 1u, 1u};
  std::memset(m, 0, sizeof(*m));
  CUresult r = enc(m, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3,
                   const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                   CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool make_bf16_box64_map(CUtensorMap* m, const void* base, int B, int T, int W) {
  EncodeTiledFn enc = encode_fn();
  if (enc == nullptr) return false;
  cuuint64_t dims[3] = {(cuuint64_t)W, (cuuint64_t)T, (cuuint64_t)B};
  cuuint64_t strides[2] = {(cuuint64_t)W * 2, (cuuint64_t)W * T * 2};
  cuuint32_t box[3] = {64u, 64u, 1u};
  cuuint32_t estr[3] = {1u, 1u, 1u};
  std::memset(m, 0, sizeof(*m));
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool make_f32_box32_map(CUtensorMap* m, const void* base, int B, int T, int W) {
  EncodeTiledFn enc = encode_fn();
  if (enc == nullptr) return false;
  cuuint64_t dims[3] = {(cuuint64_t)W, (cuuint64_t)T, (cuuint64_t)B};
  cuuint64_t strides[2] = {(cuuint64_t)W * 4, (cuuint64_t)W * T * 4};
  cuuint32_t box[3] = {32u, 64u, 1u};
  cuuint32_t estr[3] = {1u, 1u, 1u};
  std::memset(m, 0, sizeof(*m));
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

DevCtl* device_ctl() {
  DevCtl* p = nullptr;
  if (cudaGetSymbolAddress(reinterpret_cast<void**>(&p), g_ctl) != cudaSuccess) return nullptr;
  return p;
}

namespace {

constexpr int kDesignSMs = 148;  // B200 SM count the schedules are planned for
constexpr int kCtasPerSM = 4;    // resident WKV-4 forward CTAs per SM (registers and 48 KB of boxes)
constexpr int kCkLen = 16;       // checkpoint interval the backward reads

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Element alignment (4 bytes for fp32, 2 for bf16): the least the kernels' plain accesses need.
bool elem_aligned(const void* p, bool bf16) { return (reinterpret_cast<uintptr_t>(p) & (bf16 ? 1u : 3u)) == 0; }

// The WKV-4 [B,T,C] tensors go through TMA when every base is 16-byte aligned and the row pitch
// C * sizeof(element) is a multiple of 16 bytes; otherwise the same kernels use plain element
// loads and stores (null entries are skipped).
bool tma_ok(int64_t C, bool bf16, std::initializer_list<const void*> ptrs) {
  if ((C * (bf16 ? 2 : 4)) % 16 != 0) return false;
  for (const void* q : ptrs)
    if (q != nullptr && !aligned16(q)) return false;
  return true;
}

bool all_elem_aligned(bool bf16, std::initializer_list<const void*> ptrs) {
  for (const void* q : ptrs)
    if (q != nullptr && !elem_aligned(q, bf16)) return false;
  return true;
}

bool fits_int(int64_t x) { return x >= 0 && x <= INT_MAX; }

struct FwdPlan {
  int algo;      // RWKV_ALGO_SEQUENTIAL or RWKV_ALGO_CHUNKED
  int seg_len;
  int nseg;
  size_t ws_bytes;
};

// Workspace of the one-launch chunked forward: [nseg][B*C][3] doubles, then the flags.
struct LookbackWs {
  size_t agg, flag, flag_bytes, total;
};
LookbackWs lookback_ws(int64_t nseg, int64_t B, int64_t C) {
  auto up = [](size_t x) { return (x + 255) & ~(size_t)255; };
  LookbackWs w{};
  const size_t states = (size_t)nseg * B * C * 3 * sizeof(double);
  w.agg = 0;
  w.flag = up(states);
  w.flag_bytes = (size_t)nseg * ((C + 31) / 32) * B * sizeof(unsigned int);
  w.total = w.flag + up(w.flag_bytes);
  return w;
}

FwdPlan plan_forward(int64_t B, int64_t T, int64_t C, int algo) {
  FwdPlan pl{RWKV_ALGO_SEQUENTIAL, 0, 1, 0};
  const int tt = fwd_tile_steps();
  const int64_t lane_tiles = B * ((C + 31) / 32);
  int a = algo;
  // AUTO cuts time into segments only when one 32-channel tile per SM or fewer would run alone: at
  // 8 x 1024 x 768 (192 tiles) the chunked schedule measured 42 us against 33 us sequential (its
  // two passes share the SMs four CTAs at a time), at 1 x 4096 x 768 (24 tiles) it wins
  if (a == RWKV_ALGO_AUTO) a = (lane_tiles < kDesignSMs && T >= 512) ? RWKV_ALGO_CHUNKED : RWKV_ALGO_SEQUENTIAL;
  if (a == RWKV_ALGO_CHUNKED && T > 0 && lane_tiles > 0) {
    // as many time segments as keep every CTA of a pass resident at once (four per SM): a
    // second wave would cost a whole segment's latency again
    const int64_t want = std::max<int64_t>(1, (int64_t)(kCtasPerSM * kDesignSMs) / lane_tiles);
    int64_t seg = (T + want - 1) / want;
    seg = ((seg + tt - 1) / tt) * tt;
    if (seg < 64) seg = 64;
    const int64_t nseg = (T + seg - 1) / seg;
    if (nseg > 1) {
      pl.algo = RWKV_ALGO_CHUNKED;
      pl.seg_len = (int)seg;
      pl.nseg = (int)nseg;
      // the one-launch form's per-segment summaries ((a, b, p) doubles) and flags; the three-launch
      // form's fp32 states ([nseg][3][B*C]) fit in the same bytes
      pl.ws_bytes = lookback_ws(nseg, B, C).total;
      return pl;
    }
  }
  pl.seg_len = (int)(((T + tt - 1) / tt) * tt);
  if (pl.seg_len == 0) pl.seg_len = tt;
  return pl;
}

// Eagle forward: a head's chunks form a chain (each reads the state the one before leaves), and
// one CTA per head leaves the call as long as one head's chain however many SMs are idle, or
// twice that when a few heads are over two per SM.  The slot plan deals the heads' chunks, laid
// end to end, out evenly to two CTAs per SM; a CTA whose chunks end inside a head first scans them
// for a summary (the state they reach from a zero state) that the CTAs holding the rest of that
// head fold into their start states.  (A deal that balanced a modelled cost, giving fewer chunks
// to a CTA that also scans, measured no faster.)
constexpr int kEagleSlotsPerSM = 2;  // resident CTAs per SM (shared memory)
static_assert(kEagleSlotsPerSM * kDesignSMs == kWkv5MaxSlots, "slot bound of the kernel parameters");

struct Wkv5Slots {
  int nslot = 0;
  int first[kWkv5MaxSlots + 1] = {};  // chunk boundaries: slot s takes [first[s], first[s + 1])
  size_t sum = 0, flag = 0, flag_bytes = 0, total = 0;  // workspace offsets and bytes
};

// The Eagle forward's plan: slot s takes chunks [floor(s N / nslot), floor((s + 1) N / nslot)) of
// the N = B H ceil(T / 64) chunks, with a 64 x 64 fp32 summary and a flag per slot and the ticket
// counter in the workspace.
Wkv5Slots plan_wkv5_slots(int64_t B, int64_t T, int64_t H) {
  Wkv5Slots pl;
  const int64_t nchunk = (T + 63) / 64, nflat = B * H * nchunk;
  // one chunk per head: nothing to split; the boundaries are ints
  if (nchunk < 2 || nflat > INT_MAX) return pl;
  const int64_t nslot = std::min<int64_t>(kWkv5MaxSlots, nflat);
  for (int64_t s = 0; s <= nslot; ++s) pl.first[s] = (int)(s * nflat / nslot);
  auto up = [](size_t x) { return (x + 255) & ~(size_t)255; };
  pl.nslot = (int)nslot;
  pl.sum = 0;
  pl.flag = up((size_t)nslot * 64 * 64 * sizeof(float));
  pl.flag_bytes = ((size_t)nslot + 1) * sizeof(unsigned int);
  pl.total = pl.flag + up(pl.flag_bytes);
  return pl;
}

// Runs the forward pass (outputs optional) on already-validated arguments.  With r, the
// output pass writes σ(r) ⊙ WKV (the receptance-gated kernel) instead of WKV.
rwkv_status run_forward(int B, int T, int C, bool bf16, const float* w, const float* u, const void* k,
                        const void* v, void* y, const float* state_in, float* state_out, float* ckpt, int ckpt_len,
                        const FwdPlan& pl, void* ws, cudaStream_t st, const void* r = nullptr) {
  DevCtl* ctl = device_ctl();
  if (ctl == nullptr) return RWKV_ERR_CUDA;
  const int tt = fwd_tile_steps();
  const bool gate = r != nullptr && y != nullptr;
  const bool tma = tma_ok(C, bf16, {k, v, y, gate ? r : nullptr});
  CUtensorMap mk, mv, my, mr;
  std::memset(&mk, 0, sizeof(mk));  // the plain-access path reads no map
  mv = my = mr = mk;
  if (tma) {
    if (!make_btc_map(&mk, k, bf16, B, T, C, tt) || !make_btc_map(&mv, v, bf16, B, T, C, tt)) return RWKV_ERR_CUDA;
    if (gate && !make_btc_map(&mr, r, bf16, B, T, C, tt)) return RWKV_ERR_CUDA;
    if (y != nullptr) {
      if (!make_btc_map(&my, y, bf16, B, T, C, fwd_store_steps())) return RWKV_ERR_CUDA;
    } else {
      my = mk;  // not read without y
    }
  }
  auto launch_out = [&](const Fwd4Params& q) {  // the pass that writes the outputs
    return gate ? launch_wkv4_fwd_gated(bf16, mk, mv, my, mr, q, st) : launch_wkv4_fwd(bf16, mk, mv, my, q, st);
  };
  Fwd4Params p{};
  p.tma = tma ? 1 : 0;
  p.k = k;
  p.v = v;
  p.r = gate ? r : nullptr;
  p.B = B;
  p.T = T;
  p.C = C;
  p.ctiles = (C + 31) / 32;
  p.w = w;
  p.u = u;
  p.ctl = ctl;
  p.ckpt_len = ckpt_len;
  const long long seg_stride = 3LL * B * C;
  if (pl.algo == RWKV_ALGO_SEQUENTIAL) {
    p.seg_len = pl.seg_len;
    p.nseg = 1;
    p.stages = fwd_stages(bf16, pl.seg_len, gate, tma);
    p.y = y;
    p.start = state_in;
    p.end = state_out;
    p.ckpt = ckpt;
    if (launch_out(p) != cudaSuccess) return RWKV_ERR_CUDA;
    return RWKV_OK;
  }
  // one launch when every tile of a segment stays resident in the pipeline: summaries, look-back
  // across segments, outputs
  const int lb_stages = fwd_stages(bf16, pl.seg_len, false, tma);
  if (tma && !gate && (pl.seg_len + tt - 1) / tt <= lb_stages) {
    const LookbackWs L = lookback_ws(pl.nseg, B, C);
    char* wsc = static_cast<char*>(ws);
    if (cudaMemsetAsync(wsc + L.flag, 0, L.flag_bytes, st) != cudaSuccess) return RWKV_ERR_CUDA;
    p.seg_len = pl.seg_len;
    p.nseg = pl.nseg;
    p.stages = lb_stages;
    p.y = y;
    p.start = nullptr;  // the first pass runs from a zero state
    p.end = state_out;  // written by the last segment
    p.end_seg_stride = 0;
    p.ckpt = ckpt;
    p.lb_agg = reinterpret_cast<double*>(wsc + L.agg);
    p.lb_flag = reinterpret_cast<unsigned int*>(wsc + L.flag);
    p.lb_in = state_in;
    if (launch_wkv4_fwd_lookback(bf16, mk, mv, my, p, st) != cudaSuccess) return RWKV_ERR_CUDA;
    return RWKV_OK;
  }
  float* wsf = static_cast<float*>(ws);
  // 1) segment summaries from a zero state
  p.seg_len = pl.seg_len;
  p.nseg = pl.nseg;
  p.stages = fwd_stages(bf16, pl.seg_len, false, tma);
  p.y = nullptr;
  p.start = nullptr;
  p.end = wsf;
  p.end_seg_stride = seg_stride;
  p.ckpt = nullptr;
  if (launch_wkv4_fwd(bf16, mk, mv, my, p, st) != cudaSuccess) return RWKV_ERR_CUDA;
  // 2) carries (in place) and the final state
  if (launch_wkv4_carry(B, C, T, pl.nseg, pl.seg_len, w, state_in, wsf, state_out, st) != cudaSuccess)
    return RWKV_ERR_CUDA;
  // 3) outputs and checkpoints from each segment's carry
  p.y = y;
  p.start = wsf;
  p.start_seg_stride = seg_stride;
  p.end = nullptr;
  p.ckpt = ckpt;
  p.stages = fwd_stages(bf16, pl.seg_len, gate, tma);
  if (launch_out(p) != cudaSuccess) return RWKV_ERR_CUDA;
  return RWKV_OK;
}

}  // namespace
}  // namespace rwkv

using namespace rwkv;

extern "C" {

const char* rwkv_status_string(rwkv_status s) {
  switch (s) {
    case RWKV_OK: return "ok";
    case RWKV_ERR_INVALID_ARG: return "invalid argument";
    case RWKV_ERR_UNSUPPORTED: return "unsupported shape, alignment or option";
    case RWKV_ERR_WORKSPACE: return "workspace missing or too small";
    case RWKV_ERR_CUDA: return "CUDA runtime or launch error";
    case RWKV_ERR_DEVICE_TIMEOUT: return "a kernel's bounded wait timed out";
  }
  return "unknown status";
}

int rwkv_version(void) { return (1 << 16) | 2; }

int64_t rwkv_wkv4_num_checkpoints(int64_t T, int64_t chunk_len) {
  if (chunk_len <= 0 || chunk_len % 16 != 0 || T < 0) return -1;
  return (T + chunk_len - 1) / chunk_len;
}

size_t rwkv_wkv4_forward_workspace_bytes(int64_t B, int64_t T, int64_t C, int algo) {
  if (B <= 0 || T <= 0 || C <= 0) return 0;
  return plan_forward(B, T, C, algo).ws_bytes;
}

rwkv_status rwkv_wkv4_forward(int64_t B, int64_t T, int64_t C, rwkv_dtype dtype, const float* w, const float* u,
                              const void* k, const void* v, void* y, const float* state_in, float* state_out,
                              float* ckpt, int64_t chunk_len, int algo, void* workspace, size_t workspace_bytes,
                              rwkv_stream_t stream) {
  if (!fits_int(B) || !fits_int(T) || !fits_int(C)) return RWKV_ERR_INVALID_ARG;
  if (dtype != RWKV_F32 && dtype != RWKV_BF16) return RWKV_ERR_INVALID_ARG;
  if (algo < RWKV_ALGO_AUTO || algo > RWKV_ALGO_CHUNKED) return RWKV_ERR_INVALID_ARG;
  if (ckpt != nullptr && (chunk_len <= 0 || chunk_len % 16 != 0)) return RWKV_ERR_INVALID_ARG;
  if (ckpt != nullptr && chunk_len != kCkLen) return RWKV_ERR_UNSUPPORTED;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (B == 0 || C == 0) return RWKV_OK;
  if (w == nullptr || u == nullptr) return RWKV_ERR_INVALID_ARG;
  if (T == 0) {
    if (state_out != nullptr && launch_copy_state((int)B, (int)C, state_in, state_out, st) != cudaSuccess)
      return RWKV_ERR_CUDA;
    return RWKV_OK;
  }
  if (k == nullptr || v == nullptr) return RWKV_ERR_INVALID_ARG;
  if (y == nullptr && state_out == nullptr && ckpt == nullptr) return RWKV_ERR_INVALID_ARG;
  const bool bf16 = dtype == RWKV_BF16;
  if (!all_elem_aligned(bf16, {k, v, y})) return RWKV_ERR_UNSUPPORTED;
  const FwdPlan pl = plan_forward(B, T, C, algo);
  if (pl.ws_bytes > 0 && (workspace == nullptr || workspace_bytes < pl.ws_bytes)) return RWKV_ERR_WORKSPACE;
  return run_forward((int)B, (int)T, (int)C, bf16, w, u, k, v, y, state_in, state_out, ckpt, (int)chunk_len, pl,
                     workspace, st);
}

rwkv_status rwkv_wkv4_forward_gated(int64_t B, int64_t T, int64_t C, rwkv_dtype dtype, const float* w,
                                    const float* u, const void* k, const void* v, const void* r, void* o,
                                    const float* state_in, float* state_out, float* ckpt, int64_t chunk_len, int algo,
                                    void* workspace, size_t workspace_bytes, rwkv_stream_t stream) {
  if (!fits_int(B) || !fits_int(T) || !fits_int(C)) return RWKV_ERR_INVALID_ARG;
  if (dtype != RWKV_F32 && dtype != RWKV_BF16) return RWKV_ERR_INVALID_ARG;
  if (algo < RWKV_ALGO_AUTO || algo > RWKV_ALGO_CHUNKED) return RWKV_ERR_INVALID_ARG;
  if (ckpt != nullptr && (chunk_len <= 0 || chunk_len % 16 != 0)) return RWKV_ERR_INVALID_ARG;
  if (ckpt != nullptr && chunk_len != kCkLen) return RWKV_ERR_UNSUPPORTED;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (B == 0 || C == 0) return RWKV_OK;
  if (w == nullptr || u == nullptr) return RWKV_ERR_INVALID_ARG;
  if (T == 0) {
    if (state_out != nullptr && launch_copy_state((int)B, (int)C, state_in, state_out, st) != cudaSuccess)
      return RWKV_ERR_CUDA;
    return RWKV_OK;
  }
  if (k == nullptr || v == nullptr || r == nullptr || o == nullptr) return RWKV_ERR_INVALID_ARG;
  const bool bf16 = dtype == RWKV_BF16;
  if (!all_elem_aligned(bf16, {k, v, r, o})) return RWKV_ERR_UNSUPPORTED;
  const FwdPlan pl = plan_forward(B, T, C, algo);
  if (pl.ws_bytes > 0 && (workspace == nullptr || workspace_bytes < pl.ws_bytes)) return RWKV_ERR_WORKSPACE;
  return run_forward((int)B, (int)T, (int)C, bf16, w, u, k, v, o, state_in, state_out, ckpt, (int)chunk_len, pl,
                     workspace, st, r);
}

size_t rwkv_wkv4_backward_workspace_bytes(int64_t B, int64_t T, int64_t C, int64_t chunk_len, int have_ckpt) {
  if (B <= 0 || T <= 0 || C <= 0) return 0;
  if (chunk_len <= 0) chunk_len = kCkLen;
  size_t bytes = (size_t)2 * B * C * sizeof(double);  // per-lane gw, gu partial sums
  if (!have_ckpt) bytes += (size_t)((T + chunk_len - 1) / chunk_len) * 3 * B * C * sizeof(float);
  return bytes;
}

}  // extern "C"

namespace rwkv {
namespace {

// The WKV-4 backward, plain (gy given) or receptance-gated (r and go given instead, gr written).
rwkv_status backward_impl(bool gate, int64_t B, int64_t T, int64_t C, rwkv_dtype dtype, const float* w,
                          const float* u, const void* k, const void* v, const void* gy, const void* r, const void* go,
                          const float* state_in, const float* ckpt, int64_t chunk_len, void* gk, void* gv, void* gr,
                          float* gw, float* gu, void* workspace, size_t workspace_bytes, rwkv_stream_t stream) {
  if (!fits_int(B) || !fits_int(T) || !fits_int(C)) return RWKV_ERR_INVALID_ARG;
  if (dtype != RWKV_F32 && dtype != RWKV_BF16) return RWKV_ERR_INVALID_ARG;
  if (chunk_len <= 0 || chunk_len % 16 != 0) return RWKV_ERR_INVALID_ARG;
  if (chunk_len != kCkLen) return RWKV_ERR_UNSUPPORTED;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (C == 0) return RWKV_OK;
  if (gw == nullptr || gu == nullptr || w == nullptr || u == nullptr) return RWKV_ERR_INVALID_ARG;
  if (B == 0 || T == 0) {  // empty sums: gradients of w and u are zero
    if (cudaMemsetAsync(gw, 0, C * sizeof(float), st) != cudaSuccess) return RWKV_ERR_CUDA;
    if (cudaMemsetAsync(gu, 0, C * sizeof(float), st) != cudaSuccess) return RWKV_ERR_CUDA;
    return RWKV_OK;
  }
  if (k == nullptr || v == nullptr || gk == nullptr || gv == nullptr) return RWKV_ERR_INVALID_ARG;
  if (gate ? (r == nullptr || go == nullptr || gr == nullptr) : gy == nullptr) return RWKV_ERR_INVALID_ARG;
  const bool bf16 = dtype == RWKV_BF16;
  if (!all_elem_aligned(bf16, {k, v, gy, r, go, gr, gk, gv})) return RWKV_ERR_UNSUPPORTED;
  // r and gr are read and written with plain accesses on either path
  const bool tma = tma_ok(C, bf16, {k, v, gate ? go : gy, gk, gv});
  const size_t need = rwkv_wkv4_backward_workspace_bytes(B, T, C, chunk_len, ckpt != nullptr);
  if (workspace == nullptr || workspace_bytes < need) return RWKV_ERR_WORKSPACE;
  const int iB = (int)B, iT = (int)T, iC = (int)C;
  double* part = static_cast<double*>(workspace);
  const float* ck = ckpt;
  if (ck == nullptr) {
    float* ckw = reinterpret_cast<float*>(part + (size_t)2 * B * C);
    const FwdPlan pl = plan_forward(B, T, C, RWKV_ALGO_SEQUENTIAL);
    rwkv_status s = run_forward(iB, iT, iC, bf16, w, u, k, v, nullptr, state_in, nullptr, ckw, kCkLen, pl,
                                nullptr, st);
    if (s != RWKV_OK) return s;
    ck = ckw;
  }
  DevCtl* ctl = device_ctl();
  if (ctl == nullptr) return RWKV_ERR_CUDA;
  const int box_t = bwd_tile_steps();
  CUtensorMap mk, mv, mg, mgk, mgv;
  std::memset(&mk, 0, sizeof(mk));  // the plain-access path reads no map
  mv = mg = mgk = mgv = mk;
  if (tma && (!make_btc_map(&mk, k, bf16, iB, iT, iC, box_t) || !make_btc_map(&mv, v, bf16, iB, iT, iC, box_t) ||
              !make_btc_map(&mg, gate ? go : gy, bf16, iB, iT, iC, box_t) ||
              !make_btc_map(&mgk, gk, bf16, iB, iT, iC, bwd_store_steps()) ||
              !make_btc_map(&mgv, gv, bf16, iB, iT, iC, bwd_store_steps())))
    return RWKV_ERR_CUDA;
  Bwd4Params p{};
  p.B = iB;
  p.T = iT;
  p.C = iC;
  p.ctiles = (iC + 31) / 32;
  p.stages = bwd_stages(bf16, iT, gate, tma);
  p.tma = tma ? 1 : 0;
  p.k = k;
  p.v = v;
  p.g = gate ? go : gy;
  p.w = w;
  p.u = u;
  p.ckpt = ck;
  p.gk = gk;
  p.gv = gv;
  p.part = part;
  p.ctl = ctl;
  p.r = r;
  p.gr = gr;
  const cudaError_t e = gate ? launch_wkv4_bwd_gated(bf16, mk, mv, mg, mgk, mgv, p, st)
                             : launch_wkv4_bwd(bf16, mk, mv, mg, mgk, mgv, p, st);
  if (e != cudaSuccess) return RWKV_ERR_CUDA;
  if (launch_wkv4_reduce_wu(iB, iC, part, gw, gu, st) != cudaSuccess) return RWKV_ERR_CUDA;
  return RWKV_OK;
}

}  // namespace
}  // namespace rwkv

extern "C" {

rwkv_status rwkv_wkv4_backward(int64_t B, int64_t T, int64_t C, rwkv_dtype dtype, const float* w, const float* u,
                               const void* k, const void* v, const void* gy, const float* state_in,
                               const float* ckpt, int64_t chunk_len, void* gk, void* gv, float* gw, float* gu,
                               void* workspace, size_t workspace_bytes, rwkv_stream_t stream) {
  return backward_impl(false, B, T, C, dtype, w, u, k, v, gy, nullptr, nullptr, state_in, ckpt, chunk_len, gk, gv,
                       nullptr, gw, gu, workspace, workspace_bytes, stream);
}

rwkv_status rwkv_wkv4_backward_gated(int64_t B, int64_t T, int64_t C, rwkv_dtype dtype, const float* w,
                                     const float* u, const void* k, const void* v, const void* r, const void* go,
                                     const float* state_in, const float* ckpt, int64_t chunk_len, void* gk, void* gv,
                                     void* gr, float* gw, float* gu, void* workspace, size_t workspace_bytes,
                                     rwkv_stream_t stream) {
  return backward_impl(true, B, T, C, dtype, w, u, k, v, nullptr, r, go, state_in, ckpt, chunk_len, gk, gv, gr, gw,
                       gu, workspace, workspace_bytes, stream);
}

rwkv_status rwkv_wkv4_step(int64_t B, int64_t C, rwkv_dtype dtype, const float* w, const float* u, const void* k,
                           const void* v, void* y, const float* state_in, float* state_out, rwkv_stream_t stream) {
  if (!fits_int(B) || !fits_int(C)) return RWKV_ERR_INVALID_ARG;
  if (dtype != RWKV_F32 && dtype != RWKV_BF16) return RWKV_ERR_INVALID_ARG;
  if (B == 0 || C == 0) return RWKV_OK;
  if (w == nullptr || u == nullptr || k == nullptr || v == nullptr || y == nullptr || state_out == nullptr)
    return RWKV_ERR_INVALID_ARG;
  const bool bf16 = dtype == RWKV_BF16;
  const bool vec4 = !bf16 && C % 4 == 0 && aligned16(k) && aligned16(v) && aligned16(y) &&
                    (state_in == nullptr || aligned16(state_in)) && aligned16(state_out);
  if (launch_wkv4_step(bf16, (int)B, (int)C, w, u, k, v, y, state_in, state_out, vec4,
                       reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
    return RWKV_ERR_CUDA;
  return RWKV_OK;
}

size_t rwkv_wkv5_forward_workspace_bytes(int64_t B, int64_t T, int64_t H, int64_t N) {
  if (N != 64 || B <= 0 || T <= 0 || H <= 0 || !fits_int(B) || !fits_int(H) || !fits_int(B * H)) return 0;
  return plan_wkv5_slots(B, T, H).total;
}

rwkv_status rwkv_wkv5_forward(int64_t B, int64_t T, int64_t H, int64_t N, const void* r, const void* k,
                              const void* v, const float* omega, const float* u, void* y, const float* s_in,
                              float* s_out, void* workspace, size_t workspace_bytes, rwkv_stream_t stream) {
  if (!fits_int(B) || !fits_int(T) || !fits_int(H) || !fits_int(N)) return RWKV_ERR_INVALID_ARG;
  if (N != 64) return RWKV_ERR_UNSUPPORTED;
  if (B == 0 || H == 0) return RWKV_OK;
  if (omega == nullptr || u == nullptr) return RWKV_ERR_INVALID_ARG;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (T == 0) {  // no tokens: the state passes through
    if (s_out != nullptr && s_out != s_in) {
      const size_t n = (size_t)B * H * 64 * 64 * sizeof(float);
      cudaError_t e = s_in ? cudaMemcpyAsync(s_out, s_in, n, cudaMemcpyDeviceToDevice, st)
                           : cudaMemsetAsync(s_out, 0, n, st);
      if (e != cudaSuccess) return RWKV_ERR_CUDA;
    }
    return RWKV_OK;
  }
  if (r == nullptr || k == nullptr || v == nullptr || y == nullptr) return RWKV_ERR_INVALID_ARG;
  if (!aligned16(r) || !aligned16(k) || !aligned16(v) || !aligned16(y)) return RWKV_ERR_UNSUPPORTED;
  if ((int64_t)H * 64 > INT_MAX || (int64_t)B * H > INT_MAX) return RWKV_ERR_UNSUPPORTED;
  const Wkv5Slots plan = plan_wkv5_slots(B, T, H);
  if (plan.nslot > 0 && (workspace == nullptr || workspace_bytes < plan.total)) return RWKV_ERR_WORKSPACE;
  if (plan.nslot > 0 && !aligned16(workspace)) return RWKV_ERR_UNSUPPORTED;
  DevCtl* ctl = device_ctl();
  if (ctl == nullptr) return RWKV_ERR_CUDA;
  const int iB = (int)B, iT = (int)T, iH = (int)H;
  CUtensorMap mr, mk, mv;
  if (!make_bf16_box64_map(&mr, r, iB, iT, iH * 64) || !make_bf16_box64_map(&mk, k, iB, iT, iH * 64) ||
      !make_bf16_box64_map(&mv, v, iB, iT, iH * 64))
    return RWKV_ERR_CUDA;
  Wkv5Params p{};
  p.B = iB;
  p.T = iT;
  p.H = iH;
  p.r = static_cast<const __nv_bfloat16*>(r);
  p.k = static_cast<const __nv_bfloat16*>(k);
  p.v = static_cast<const __nv_bfloat16*>(v);
  p.omega = omega;
  p.u = u;
  p.y = static_cast<__nv_bfloat16*>(y);
  p.s_in = s_in;
  p.s_out = s_out;
  p.ctl = ctl;
  if (plan.nslot > 0) {
    char* ws = static_cast<char*>(workspace);
    if (cudaMemsetAsync(ws + plan.flag, 0, plan.flag_bytes, st) != cudaSuccess) return RWKV_ERR_CUDA;
    p.nslot = plan.nslot;
    std::copy(plan.first, plan.first + plan.nslot + 1, p.slot_first);
    p.slot_sum = reinterpret_cast<float*>(ws + plan.sum);
    p.slot_flag = reinterpret_cast<unsigned int*>(ws + plan.flag);
  }
  if (launch_wkv5_fwd(mr, mk, mv, p, st) != cudaSuccess) return RWKV_ERR_CUDA;
  return RWKV_OK;
}

rwkv_status rwkv_wkv5_step(int64_t B, int64_t H, int64_t N, const void* r, const void* k, const void* v,
                           const float* omega, const float* u, void* y, const float* s_in, float* s_out,
                           rwkv_stream_t stream) {
  if (!fits_int(B) || !fits_int(H) || !fits_int(N)) return RWKV_ERR_INVALID_ARG;
  if (N != 64) return RWKV_ERR_UNSUPPORTED;
  if (B == 0 || H == 0) return RWKV_OK;
  if (r == nullptr || k == nullptr || v == nullptr || omega == nullptr || u == nullptr || y == nullptr ||
      s_out == nullptr)
    return RWKV_ERR_INVALID_ARG;
  if ((s_in != nullptr && !aligned16(s_in)) || !aligned16(s_out)) return RWKV_ERR_UNSUPPORTED;
  if ((int64_t)B * H > INT_MAX) return RWKV_ERR_UNSUPPORTED;
  Wkv5StepParams p{};
  p.B = (int)B;
  p.H = (int)H;
  p.r = static_cast<const __nv_bfloat16*>(r);
  p.k = static_cast<const __nv_bfloat16*>(k);
  p.v = static_cast<const __nv_bfloat16*>(v);
  p.omega = omega;
  p.omega_per_stream = 0;
  p.u = u;
  p.y = static_cast<__nv_bfloat16*>(y);
  p.s_in = s_in;
  p.s_out = s_out;
  if (launch_wkv5_step(p, reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess) return RWKV_ERR_CUDA;
  return RWKV_OK;
}

size_t rwkv_wkv6_forward_workspace_bytes(int64_t B, int64_t T, int64_t H, int64_t N) {
  (void)B;
  (void)T;
  (void)H;
  (void)N;
  return 0;
}

rwkv_status rwkv_wkv6_forward(int64_t B, int64_t T, int64_t H, int64_t N, const void* r, const void* k,
                              const void* v, const float* omega, const float* u, void* y, const float* s_in,
                              float* s_out, void* workspace, size_t workspace_bytes, rwkv_stream_t stream) {
  (void)workspace;
  (void)workspace_bytes;
  if (!fits_int(B) || !fits_int(T) || !fits_int(H) || !fits_int(N)) return RWKV_ERR_INVALID_ARG;
  if (N != 64) return RWKV_ERR_UNSUPPORTED;
  if (B == 0 || H == 0) return RWKV_OK;
  if (u == nullptr) return RWKV_ERR_INVALID_ARG;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (T == 0) {  // no tokens: the state passes through
    if (s_out != nullptr && s_out != s_in) {
      const size_t n = (size_t)B * H * 64 * 64 * sizeof(float);
      cudaError_t e = s_in ? cudaMemcpyAsync(s_out, s_in, n, cudaMemcpyDeviceToDevice, st)
                           : cudaMemsetAsync(s_out, 0, n, st);
      if (e != cudaSuccess) return RWKV_ERR_CUDA;
    }
    return RWKV_OK;
  }
  if (r == nullptr || k == nullptr || v == nullptr || omega == nullptr || y == nullptr) return RWKV_ERR_INVALID_ARG;
  if (!aligned16(r) || !aligned16(k) || !aligned16(v) || !aligned16(y) || !aligned16(omega))
    return RWKV_ERR_UNSUPPORTED;
  if ((int64_t)H * 64 > INT_MAX || (int64_t)B * H > INT_MAX) return RWKV_ERR_UNSUPPORTED;
  DevCtl* ctl = device_ctl();
  if (ctl == nullptr) return RWKV_ERR_CUDA;
  const int iB = (int)B, iT = (int)T, iH = (int)H;
  CUtensorMap mr, mk, mv, mw;
  if (!make_bf16_box64_map(&mr, r, iB, iT, iH * 64) || !make_bf16_box64_map(&mk, k, iB, iT, iH * 64) ||
      !make_bf16_box64_map(&mv, v, iB, iT, iH * 64) || !make_f32_box32_map(&mw, omega, iB, iT, iH * 64))
    return RWKV_ERR_CUDA;
  Wkv6Params p{};
  p.B = iB;
  p.T = iT;
  p.H = iH;
  p.r = static_cast<const __nv_bfloat16*>(r);
  p.k = static_cast<const __nv_bfloat16*>(k);
  p.v = static_cast<const __nv_bfloat16*>(v);
  p.omega = omega;
  p.u = u;
  p.y = static_cast<__nv_bfloat16*>(y);
  p.s_in = s_in;
  p.s_out = s_out;
  p.ctl = ctl;
  if (launch_wkv6_fwd(mr, mk, mv, mw, p, st) != cudaSuccess) return RWKV_ERR_CUDA;
  return RWKV_OK;
}

rwkv_status rwkv_wkv6_step(int64_t B, int64_t H, int64_t N, const void* r, const void* k, const void* v,
                           const float* omega, const float* u, void* y, const float* s_in, float* s_out,
                           rwkv_stream_t stream) {
  if (!fits_int(B) || !fits_int(H) || !fits_int(N)) return RWKV_ERR_INVALID_ARG;
  if (N != 64) return RWKV_ERR_UNSUPPORTED;
  if (B == 0 || H == 0) return RWKV_OK;
  if (r == nullptr || k == nullptr || v == nullptr || omega == nullptr || u == nullptr || y == nullptr ||
      s_out == nullptr)
    return RWKV_ERR_INVALID_ARG;
  if ((s_in != nullptr && !aligned16(s_in)) || !aligned16(s_out)) return RWKV_ERR_UNSUPPORTED;
  if ((int64_t)B * H > INT_MAX) return RWKV_ERR_UNSUPPORTED;
  Wkv5StepParams p{};
  p.B = (int)B;
  p.H = (int)H;
  p.r = static_cast<const __nv_bfloat16*>(r);
  p.k = static_cast<const __nv_bfloat16*>(k);
  p.v = static_cast<const __nv_bfloat16*>(v);
  p.omega = omega;
  p.omega_per_stream = 1;
  p.u = u;
  p.y = static_cast<__nv_bfloat16*>(y);
  p.s_in = s_in;
  p.s_out = s_out;
  if (launch_wkv5_step(p, reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess) return RWKV_ERR_CUDA;
  return RWKV_OK;
}

}  // extern "C"

namespace rwkv {
namespace {

// Byte layout of the Eagle backward's workspace (every region 256-byte aligned).
struct Wkv5BwdWs {
  size_t ckpt;            // fp32 [B,H,nchunk,64,64]: forward states at chunk starts
  size_t part_f, part_r;  // fp64 [B,H,64]: per-row sums of the two passes
  size_t total;
};

Wkv5BwdWs wkv5_bwd_ws(int64_t B, int64_t T, int64_t H) {
  auto up = [](size_t x) { return (x + 255) & ~(size_t)255; };
  Wkv5BwdWs w{};
  size_t o = 0;
  w.ckpt = o;
  o += up((size_t)B * H * ((T + 63) / 64) * 64 * 64 * 4);
  w.part_f = o;
  o += up((size_t)B * H * 64 * 8);
  w.part_r = o;
  o += up((size_t)B * H * 64 * 8);
  w.total = o;
  return w;
}

}  // namespace
}  // namespace rwkv

extern "C" {

size_t rwkv_wkv5_backward_workspace_bytes(int64_t B, int64_t T, int64_t H, int64_t N) {
  if (B <= 0 || T <= 0 || H <= 0 || N != 64) return 0;
  return wkv5_bwd_ws(B, T, H).total;
}

}  // extern "C"

namespace rwkv {
namespace {
// One non-blocking stream per (device, context), made on first use: the Eagle backward runs its
// reversed forward pass there, next to the reversed gradient pass (whose last CTAs leave most SMs
// idle).  Each call orders it against the caller's stream with its own pair of events.  Returns
// nullptr (run everything on the caller's stream) when no stream can be had: no context id, the
// caller's stream is being captured before the side stream exists, or a CUDA error.
cudaStream_t side_stream(cudaStream_t caller) {
  constexpr int kMaxDev = 64;
  struct Slot {
    cudaStream_t s;
    unsigned long long ctx;
  };
  static std::mutex mu;
  static Slot slots[kMaxDev] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDev) return nullptr;
  const unsigned long long id = current_context_id();
  if (id == 0) return nullptr;
  std::lock_guard<std::mutex> lock(mu);
  Slot& sl = slots[dev];
  if (sl.s != nullptr && sl.ctx == id) return sl.s;
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(caller, &cs) != cudaSuccess || cs != cudaStreamCaptureStatusNone) return nullptr;
  cudaStream_t s = nullptr;
  if (cudaStreamCreateWithFlags(&s, cudaStreamNonBlocking) != cudaSuccess) return nullptr;
  sl.s = s;
  sl.ctx = id;
  return s;
}
}  // namespace
}  // namespace rwkv

extern "C" {

rwkv_status rwkv_wkv5_backward(int64_t B, int64_t T, int64_t H, int64_t N, const void* r, const void* k,
                               const void* v, const float* omega, const float* u, const float* s_in, const void* gy,
                               const float* gs_out, void* gr, void* gk, void* gv, float* gomega, float* gu,
                               float* gs_in, void* workspace, size_t workspace_bytes, rwkv_stream_t stream) {
  if (!fits_int(B) || !fits_int(T) || !fits_int(H) || !fits_int(N)) return RWKV_ERR_INVALID_ARG;
  if (N != 64) return RWKV_ERR_UNSUPPORTED;
  if (B == 0 || H == 0) return RWKV_OK;
  if (omega == nullptr || u == nullptr || gomega == nullptr || gu == nullptr) return RWKV_ERR_INVALID_ARG;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (T == 0) {  // no tokens: the sums are empty and the state gradient passes through
    if (cudaMemsetAsync(gomega, 0, H * 64 * sizeof(float), st) != cudaSuccess) return RWKV_ERR_CUDA;
    if (cudaMemsetAsync(gu, 0, H * 64 * sizeof(float), st) != cudaSuccess) return RWKV_ERR_CUDA;
    if (gs_in != nullptr) {
      const size_t n = (size_t)B * H * 64 * 64 * sizeof(float);
      cudaError_t e = gs_out ? cudaMemcpyAsync(gs_in, gs_out, n, cudaMemcpyDeviceToDevice, st)
                             : cudaMemsetAsync(gs_in, 0, n, st);
      if (e != cudaSuccess) return RWKV_ERR_CUDA;
    }
    return RWKV_OK;
  }
  if (r == nullptr || k == nullptr || v == nullptr || gy == nullptr || gr == nullptr || gk == nullptr ||
      gv == nullptr)
    return RWKV_ERR_INVALID_ARG;
  if (!aligned16(r) || !aligned16(k) || !aligned16(v) || !aligned16(gy) || !aligned16(gr) || !aligned16(gk) ||
      !aligned16(gv))
    return RWKV_ERR_UNSUPPORTED;
  if ((int64_t)H * 64 > INT_MAX || (int64_t)B * H > INT_MAX || (int64_t)T + 64 > INT_MAX) return RWKV_ERR_UNSUPPORTED;
  const Wkv5BwdWs L = wkv5_bwd_ws(B, T, H);
  if (workspace == nullptr || workspace_bytes < L.total) return RWKV_ERR_WORKSPACE;
  DevCtl* ctl = device_ctl();
  if (ctl == nullptr) return RWKV_ERR_CUDA;
  const int iB = (int)B, iT = (int)T, iH = (int)H, W = iH * 64;
  char* ws = static_cast<char*>(workspace);
  float* ckpt = reinterpret_cast<float*>(ws + L.ckpt);
  double* part_f = reinterpret_cast<double*>(ws + L.part_f);
  double* part_r = reinterpret_cast<double*>(ws + L.part_r);
  CUtensorMap mr, mk, mv, mg;
  if (!make_bf16_box64_map(&mr, r, iB, iT, W) || !make_bf16_box64_map(&mk, k, iB, iT, W) ||
      !make_bf16_box64_map(&mv, v, iB, iT, W) || !make_bf16_box64_map(&mg, gy, iB, iT, W))
    return RWKV_ERR_CUDA;

  const int nchunk = (iT + 63) / 64;
  // gr, the forward states at chunk starts, the gu sums: (q, p, c, m) = (gy, v, k, r)
  {
    Wkv5BwdParams p{};
    p.B = iB;
    p.T = iT;
    p.H = iH;
    p.lead = 0;
    p.m = static_cast<const __nv_bfloat16*>(r);
    p.c = static_cast<const __nv_bfloat16*>(k);
    p.omega = omega;
    p.u = u;
    p.x0 = s_in;
    p.out = static_cast<__nv_bfloat16*>(gr);
    p.ckpt = ckpt;
    p.part = part_f;
    p.ctl = ctl;
    if (launch_wkv5_bwd_pass(false, mg, mv, mk, p, st) != cudaSuccess) return RWKV_ERR_CUDA;
  }
  // the reversed forward pass below needs nothing from the two gradient passes: it runs on a side
  // stream, ordered after the forward-time pass so that the reversed pass is dispatched first
  cudaStream_t side = side_stream(st);
  cudaEvent_t ev_fork = nullptr, ev_join = nullptr;
  if (side != nullptr) {
    if (cudaEventCreateWithFlags(&ev_fork, cudaEventDisableTiming) != cudaSuccess ||
        cudaEventCreateWithFlags(&ev_join, cudaEventDisableTiming) != cudaSuccess ||
        cudaEventRecord(ev_fork, st) != cudaSuccess || cudaStreamWaitEvent(side, ev_fork, 0) != cudaSuccess) {
      if (ev_fork) cudaEventDestroy(ev_fork);
      if (ev_join) cudaEventDestroy(ev_join);
      return RWKV_ERR_CUDA;
    }
  }
  auto release = [&]() {
    if (ev_fork) cudaEventDestroy(ev_fork);
    if (ev_join) cudaEventDestroy(ev_join);
  };
  // gk and the decay-gradient sums: (q, p, c, m) = (v, gy, r, k) over reversed time, chunks aligned
  // with the forward pass's
  {
    Wkv5BwdParams p{};
    p.B = iB;
    p.T = iT;
    p.H = iH;
    p.lead = 64 * nchunk - iT;
    p.m = static_cast<const __nv_bfloat16*>(k);
    p.c = static_cast<const __nv_bfloat16*>(r);
    p.omega = omega;
    p.u = u;
    p.x0 = gs_out;
    p.out = static_cast<__nv_bfloat16*>(gk);
    p.ckpt = ckpt;
    p.part = part_r;
    p.ctl = ctl;
    if (launch_wkv5_bwd_pass(true, mv, mg, mr, p, st) != cudaSuccess) {
      release();
      return RWKV_ERR_CUDA;
    }
  }
  // gv and the initial-state gradient: the forward operator over reversed time with r and k
  // swapped and gy as the value, started from gs_out (time reversed inside the kernel)
  {
    Wkv5Params p{};
    p.B = iB;
    p.T = iT;
    p.H = iH;
    p.r = static_cast<const __nv_bfloat16*>(k);
    p.k = static_cast<const __nv_bfloat16*>(r);
    p.v = static_cast<const __nv_bfloat16*>(gy);
    p.omega = omega;
    p.u = u;
    p.y = static_cast<__nv_bfloat16*>(gv);
    p.s_in = gs_out;
    p.s_out = gs_in;
    p.ctl = ctl;
    if (launch_wkv5_fwd(mk, mr, mg, p, side != nullptr ? side : st, true) != cudaSuccess) {
      release();
      return RWKV_ERR_CUDA;
    }
  }
  if (side != nullptr) {
    if (cudaEventRecord(ev_join, side) != cudaSuccess || cudaStreamWaitEvent(st, ev_join, 0) != cudaSuccess) {
      release();
      return RWKV_ERR_CUDA;
    }
  }
  release();
  if (launch_wkv5_bwd_reduce(iB, iH, part_f, part_r, omega, gomega, gu, st) != cudaSuccess) return RWKV_ERR_CUDA;
  return RWKV_OK;
}

size_t rwkv_wkv6_backward_workspace_bytes(int64_t B, int64_t T, int64_t H, int64_t N) {
  if (B <= 0 || T <= 0 || H <= 0 || N != 64) return 0;
  if (!fits_int(B) || !fits_int(T) || !fits_int(H)) return 0;
  auto up = [](size_t x) { return (x + 255) & ~(size_t)255; };
  return 2 * up(wkv6_bwd_block_floats((int)B, (int)T, (int)H) * 4) +
         2 * up(wkv6_bwd_row_floats((int)B, (int)T, (int)H) * 4);
}

rwkv_status rwkv_wkv6_backward(int64_t B, int64_t T, int64_t H, int64_t N, const void* r, const void* k,
                               const void* v, const float* omega, const float* u, const float* s_in, const void* gy,
                               const float* gs_out, void* gr, void* gk, void* gv, float* gomega, float* gu,
                               float* gs_in, void* workspace, size_t workspace_bytes, rwkv_stream_t stream) {
  if (!fits_int(B) || !fits_int(T) || !fits_int(H) || !fits_int(N)) return RWKV_ERR_INVALID_ARG;
  if (N != 64) return RWKV_ERR_UNSUPPORTED;
  if (B == 0 || H == 0) return RWKV_OK;
  if (u == nullptr || gu == nullptr) return RWKV_ERR_INVALID_ARG;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (T == 0) {  // no tokens: gu is an empty sum and the state gradient passes through
    if (cudaMemsetAsync(gu, 0, H * 64 * sizeof(float), st) != cudaSuccess) return RWKV_ERR_CUDA;
    if (gs_in != nullptr) {
      const size_t n = (size_t)B * H * 64 * 64 * sizeof(float);
      cudaError_t e = gs_out ? cudaMemcpyAsync(gs_in, gs_out, n, cudaMemcpyDeviceToDevice, st)
                             : cudaMemsetAsync(gs_in, 0, n, st);
      if (e != cudaSuccess) return RWKV_ERR_CUDA;
    }
    return RWKV_OK;
  }
  if (r == nullptr || k == nullptr || v == nullptr || gy == nullptr || omega == nullptr || gr == nullptr ||
      gk == nullptr || gv == nullptr || gomega == nullptr)
    return RWKV_ERR_INVALID_ARG;
  if (!aligned16(r) || !aligned16(k) || !aligned16(v) || !aligned16(gy) || !aligned16(omega) || !aligned16(gr) ||
      !aligned16(gk) || !aligned16(gv) || !aligned16(gomega) || (s_in && !aligned16(s_in)) ||
      (gs_out && !aligned16(gs_out)) || (gs_in && !aligned16(gs_in)))
    return RWKV_ERR_UNSUPPORTED;
  if ((int64_t)H * 64 > INT_MAX || (int64_t)B * H > INT_MAX || (int64_t)T + 64 > INT_MAX) return RWKV_ERR_UNSUPPORTED;
  // one CTA per 64-token chunk, and two per (batch row, head) for the boundary scans
  if ((int64_t)B * H * ((T + 63) / 64) > INT_MAX || 2 * (int64_t)B * H > INT_MAX) return RWKV_ERR_UNSUPPORTED;
  const size_t need = rwkv_wkv6_backward_workspace_bytes(B, T, H, N);
  if (workspace == nullptr || workspace_bytes < need) return RWKV_ERR_WORKSPACE;
  auto up = [](size_t x) { return (x + 255) & ~(size_t)255; };
  char* ws = static_cast<char*>(workspace);
  Wkv6BwdParams p{};
  p.B = (int)B;
  p.T = (int)T;
  p.H = (int)H;
  p.r = static_cast<const __nv_bfloat16*>(r);
  p.k = static_cast<const __nv_bfloat16*>(k);
  p.v = static_cast<const __nv_bfloat16*>(v);
  p.gy = static_cast<const __nv_bfloat16*>(gy);
  p.omega = omega;
  p.u = u;
  p.s_in = s_in;
  p.gs_out = gs_out;
  p.gr = static_cast<__nv_bfloat16*>(gr);
  p.gk = static_cast<__nv_bfloat16*>(gk);
  p.gv = static_cast<__nv_bfloat16*>(gv);
  p.gomega = gomega;
  p.gu = gu;
  p.gs_in = gs_in;
  const size_t blk_bytes = up(wkv6_bwd_block_floats(p.B, p.T, p.H) * 4);
  const size_t row_bytes = up(wkv6_bwd_row_floats(p.B, p.T, p.H) * 4);
  p.xs = reinterpret_cast<float*>(ws);
  p.xg = reinterpret_cast<float*>(ws + blk_bytes);
  p.dec = reinterpret_cast<float*>(ws + 2 * blk_bytes);
  p.part = reinterpret_cast<float*>(ws + 2 * blk_bytes + row_bytes);
  if (launch_wkv6_bwd(p, st) != cudaSuccess) return RWKV_ERR_CUDA;
  return RWKV_OK;
}

rwkv_status rwkv_check_device_error(rwkv_stream_t stream) {
  if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess) return RWKV_ERR_CUDA;
  unsigned int v = 0;
  if (cudaMemcpyFromSymbol(&v, g_ctl, sizeof(v), offsetof(DevCtl, err)) != cudaSuccess) return RWKV_ERR_CUDA;
  if (v != 0) {
    const unsigned int zero = 0;
    if (cudaMemcpyToSymbol(g_ctl, &zero, sizeof(zero), offsetof(DevCtl, err)) != cudaSuccess) return RWKV_ERR_CUDA;
    return RWKV_ERR_DEVICE_TIMEOUT;  // the one condition a kernel reports there
  }
  return RWKV_OK;
}

rwkv_status rwkv_debug_set_wait_limit_ns(uint64_t ns) {
  const unsigned long long v = ns == 0 ? kDefaultWaitLimitNs : (unsigned long long)ns;
  if (cudaDeviceSynchronize() != cudaSuccess) return RWKV_ERR_CUDA;
  if (cudaMemcpyToSymbol(g_ctl, &v, sizeof(v), offsetof(DevCtl, wait_limit_ns)) != cudaSuccess) return RWKV_ERR_CUDA;
  return RWKV_OK;
}

rwkv_status rwkv_debug_withhold_loads(int on) {
  const unsigned int v = on ? 1u : 0u;
  if (cudaDeviceSynchronize() != cudaSuccess) return RWKV_ERR_CUDA;
  if (cudaMemcpyToSymbol(g_ctl, &v, sizeof(v), offsetof(DevCtl, withhold)) != cudaSuccess) return RWKV_ERR_CUDA;
  return RWKV_OK;
}

}  // extern "C"
