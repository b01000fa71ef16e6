// attn_bwd_noalloc: the reverse pass for callers that cannot allocate device
// memory. Its scratch space is a fixed array in the library's own device
// memory instead of a caller-provided workspace.
#include <mutex>

#include <cuda.h>
#include <cuda_runtime.h>

#include "../../include/attn.h"
#include "launchers.h"

namespace {

// Largest scratch the entry point can use: 64 MiB. Every GPU that loads the
// library holds this array until the process exits.
constexpr size_t kNoAllocScratchBytes = size_t(64) << 20;

// One copy per device. Host code must not pass `g_scratch` itself to a kernel:
// on the host the name is only a stand-in for the device symbol. Its device
// address is looked up with cudaGetSymbolAddress, once per device and context.
static __device__ __align__(256) unsigned char g_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;

// The address found for each device, with the id of the context it was found
// in: a context torn down and created again (cudaDeviceReset, or a framework
// resetting the device) gets a new id, and the address is looked up anew.
struct Slot {
  unsigned long long ctx_id = 0;
  void* addr = nullptr;
};
std::mutex g_mu;
Slot g_slot[kMaxDevices];

using CtxGetCurrentFn = CUresult (*)(CUcontext*);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long*);

// Unique id of the calling thread's current context (0 when there is none or
// the driver cannot say).
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
    p = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<CtxGetIdFn>(p);
  });
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (!get_current || !get_id || get_current(&ctx) != CUDA_SUCCESS || !ctx || get_id(ctx, &id) != CUDA_SUCCESS)
    return 0;
  return id;
}

// Device address of g_scratch on the current device. The set-up (the symbol
// lookup, which may load the library's device code) runs on the first call
// per device and context, with that device current; it is refused while
// `stream` is being captured into a graph, since the lookup cannot be part
// of a capture.
attn_status scratch_address(cudaStream_t stream, void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return ATTN_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return ATTN_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_mu);
  Slot& s = g_slot[dev];
  const unsigned long long id = current_context_id();
  if (s.addr && id != 0 && id == s.ctx_id) {
    *out = s.addr;
    return ATTN_OK;
  }
  cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(stream, &cap) != cudaSuccess) return ATTN_ERR_CUDA;
  if (cap != cudaStreamCaptureStatusNone) return ATTN_ERR_UNSUPPORTED;
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_scratch) != cudaSuccess || !p) return ATTN_ERR_CUDA;
  s.addr = p;
  s.ctx_id = current_context_id();  // the lookup made the device's context current
  *out = p;
  return ATTN_OK;
}

}  // namespace

namespace attn {

void* noalloc_status_word(cudaStream_t stream, attn_status* st) {
  void* p = nullptr;
  *st = scratch_address(stream, &p);
  return *st == ATTN_OK ? p : nullptr;
}

}  // namespace attn

#pragma GCC visibility push(default)
extern "C" attn_status attn_bwd_noalloc(const attn_tensor* q, const attn_tensor* k, const attn_tensor* v,
                                        const attn_tensor* o, const attn_tensor* do_, const attn_tensor* lse,
                                        const attn_mask* mask, float scale, attn_tensor* dq, attn_tensor* dk,
                                        attn_tensor* dv, float* dsink, void* stream) {
  const size_t need = attn_bwd_workspace_size(q, k, v, mask);
  if (need > kNoAllocScratchBytes) return ATTN_ERR_WORKSPACE;
  void* scratch = nullptr;
  const attn_status st = scratch_address(static_cast<cudaStream_t>(stream), &scratch);
  if (st != ATTN_OK) return st;
  // attn_bwd itself zeroes every part of the scratch that must start at zero
  // (status word, dQ accumulator, top-k dKV accumulator) on `stream`.
  return attn_bwd(q, k, v, o, do_, lse, mask, scale, dq, dk, dv, dsink, scratch, kNoAllocScratchBytes, stream);
}
#pragma GCC visibility pop
