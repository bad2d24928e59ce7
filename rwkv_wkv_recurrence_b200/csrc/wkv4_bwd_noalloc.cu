// rwkv_wkv4_backward_noalloc: the WKV-4 backward without a caller-provided
// workspace and without any device allocation.
//
// Why it exists.  rwkv_wkv4_backward needs scratch for one fp64 gw and gu
// partial per (batch, channel) lane, which the caller allocates.  Some callers
// cannot allocate device memory at the point where they run the backward:
// code whose device memory is owned in full by another allocator (a framework
// pool that has reserved the card), code that must not pay cudaMalloc's
// implicit synchronisation in a latency-critical loop, or systems that permit
// allocation only at start-up.  This entry point takes the same inputs and
// outputs and keeps the partials in a fixed array that lives in the library
// itself.
//
// The array.  g_bwd_scratch below is a file-scope __device__ array of
// kNoAllocMaxLanes lanes x 2 doubles (4 MiB).  Every GPU that loads the
// library holds it until the process exits.  In host code its name is only a
// host-side stand-in, so its device address is looked up with
// cudaGetSymbolAddress, with the device current, on the first call made in
// that device's context, and cached together with the context's unique id.
// A context created later for the same device (after cudaDeviceReset, say)
// has another id, so the next call looks the address up again instead of
// handing the kernel a stale one.  All calls share the array and it keeps the
// last call's contents; the backward writes every partial it later reads
// within the same call, so nothing needs clearing between calls.  Two calls
// whose work overlaps on the GPU (different streams, or different host
// threads without ordering) race on the array.
#include <mutex>

#include "../../include/rwkv_wkv.h"
#include "launch.h"

namespace rwkv {
using CtxGetCurrentFn = CUresult (*)(CUcontext*);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long*);

// Unique id of the context current on this thread (driver entry points looked
// up once); 0 if there is none or the driver cannot say.
unsigned long long current_context_id() {
  static CtxGetCurrentFn get_current = nullptr;
  static CtxGetIdFn get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<CtxGetCurrentFn>(p);
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<CtxGetIdFn>(p);
  });
  if (get_current == nullptr || get_id == nullptr) return 0;
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr) return 0;
  if (get_id(ctx, &id) != CUDA_SUCCESS) return 0;
  return id;
}

namespace {

constexpr int64_t kNoAllocMaxLanes = RWKV_NOALLOC_MAX_LANES;
constexpr int kMaxDevices = 64;

// Per-lane gw, gu partial sums of the backward: [2][kNoAllocMaxLanes] fp64.
static __device__ __align__(256) double g_bwd_scratch[2 * kNoAllocMaxLanes];

struct ScratchAddr {
  unsigned long long ctx_id;  // context the address belongs to (0: none yet)
  double* ptr;
};

std::mutex g_setup_mutex;
ScratchAddr g_scratch[kMaxDevices] = {};

// Device address of g_bwd_scratch in the current device's context, looked up
// once per context.
cudaError_t scratch_for_current_device(double** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_setup_mutex);
  ScratchAddr& slot = g_scratch[dev];
  const unsigned long long id = current_context_id();
  if (slot.ptr == nullptr || id == 0 || id != slot.ctx_id) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_bwd_scratch);  // makes the device's primary context current if needed
    if (e != cudaSuccess) return e;
    slot.ptr = static_cast<double*>(p);
    slot.ctx_id = current_context_id();
  }
  *out = slot.ptr;
  return cudaSuccess;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace
}  // namespace rwkv

using namespace rwkv;

extern "C" rwkv_status rwkv_wkv4_backward_noalloc(int64_t B, int64_t T, int64_t C, rwkv_dtype dtype, const float* w,
                                                  const float* u, const void* k, const void* v, const void* gy,
                                                  const float* ckpt, int64_t chunk_len, void* gk, void* gv,
                                                  float* gw, float* gu, rwkv_stream_t stream) {
  if (B < 0 || T < 0 || C < 0 || B > INT32_MAX || T > INT32_MAX || C > INT32_MAX) return RWKV_ERR_INVALID_ARG;
  if (dtype != RWKV_F32 && dtype != RWKV_BF16) return RWKV_ERR_INVALID_ARG;
  if (chunk_len <= 0 || chunk_len % 16 != 0) return RWKV_ERR_INVALID_ARG;
  if (chunk_len != 16) return RWKV_ERR_UNSUPPORTED;
  if (B * C > kNoAllocMaxLanes) return RWKV_ERR_WORKSPACE;  // beyond the fixed scratch capacity
  if (C == 0) return RWKV_OK;
  if (gw == nullptr || gu == nullptr || w == nullptr || u == nullptr) return RWKV_ERR_INVALID_ARG;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (B == 0 || T == 0) {  // empty sums: gradients of w and u are zero
    if (cudaMemsetAsync(gw, 0, C * sizeof(float), st) != cudaSuccess) return RWKV_ERR_CUDA;
    if (cudaMemsetAsync(gu, 0, C * sizeof(float), st) != cudaSuccess) return RWKV_ERR_CUDA;
    return RWKV_OK;
  }
  if (k == nullptr || v == nullptr || gy == nullptr || ckpt == nullptr || gk == nullptr || gv == nullptr)
    return RWKV_ERR_INVALID_ARG;
  const bool bf16 = dtype == RWKV_BF16;
  if (!aligned16(k) || !aligned16(v) || !aligned16(gy) || !aligned16(gk) || !aligned16(gv) ||
      (C * (bf16 ? 2 : 4)) % 16 != 0)
    return RWKV_ERR_UNSUPPORTED;  // this entry point keeps to the TMA path
  double* scratch = nullptr;
  if (scratch_for_current_device(&scratch) != cudaSuccess) return RWKV_ERR_CUDA;
  DevCtl* ctl = device_ctl();
  if (ctl == nullptr) return RWKV_ERR_CUDA;
  const int iB = (int)B, iT = (int)T, iC = (int)C;
  const int box_t = bwd_tile_steps();
  CUtensorMap mk, mv, mg, mgk, mgv;
  if (!make_btc_map(&mk, k, bf16, iB, iT, iC, box_t) || !make_btc_map(&mv, v, bf16, iB, iT, iC, box_t) ||
      !make_btc_map(&mg, gy, bf16, iB, iT, iC, box_t) ||
      !make_btc_map(&mgk, gk, bf16, iB, iT, iC, bwd_store_steps()) ||
      !make_btc_map(&mgv, gv, bf16, iB, iT, iC, bwd_store_steps()))
    return RWKV_ERR_CUDA;
  Bwd4Params p{};
  p.B = iB;
  p.T = iT;
  p.C = iC;
  p.ctiles = (iC + 31) / 32;
  p.stages = bwd_stages(bf16, iT);
  p.tma = 1;
  p.w = w;
  p.u = u;
  p.ckpt = ckpt;
  p.gk = gk;
  p.gv = gv;
  p.part = scratch;  // [2][B*C] within the fixed array
  p.ctl = ctl;
  if (launch_wkv4_bwd(bf16, mk, mv, mg, mgk, mgv, p, st) != cudaSuccess) return RWKV_ERR_CUDA;
  if (launch_wkv4_reduce_wu(iB, iC, scratch, gw, gu, st) != cudaSuccess) return RWKV_ERR_CUDA;
  return RWKV_OK;
}
