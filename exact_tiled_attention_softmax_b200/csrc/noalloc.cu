// attn_bwd_noalloc: the reverse pass for callers that cannot allocate device
// memory. Its scratch space is a fixed array in the library's own device
// memory instead of a caller-provided workspace.
#include <atomic>

#include <cuda_runtime.h>

#include "../../include/attn.h"

namespace {

// Largest scratch the entry point can use: 64 MiB. Every GPU that loads the
// library holds this array until the process exits.
constexpr size_t kNoAllocScratchBytes = size_t(64) << 20;

// One copy per device. Host code must not pass `g_scratch` itself to a kernel:
// on the host the name is only a stand-in for the device symbol. Its device
// address is looked up with cudaGetSymbolAddress, once per device.
static __device__ __align__(256) unsigned char g_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
std::atomic<void*> g_scratch_addr[kMaxDevices];

// Device address of g_scratch on the current device; looked up on the first
// call per device, with that device current.
attn_status scratch_address(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return ATTN_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return ATTN_ERR_UNSUPPORTED;
  void* p = g_scratch_addr[dev].load(std::memory_order_acquire);
  if (!p) {
    if (cudaGetSymbolAddress(&p, g_scratch) != cudaSuccess || !p) return ATTN_ERR_CUDA;
    g_scratch_addr[dev].store(p, std::memory_order_release);
  }
  *out = p;
  return ATTN_OK;
}

}  // namespace

#pragma GCC visibility push(default)
extern "C" attn_status attn_bwd_noalloc(const attn_tensor* q, const attn_tensor* k, const attn_tensor* v,
                                        const attn_tensor* o, const attn_tensor* do_, const attn_tensor* lse,
                                        const attn_mask* mask, float scale, attn_tensor* dq, attn_tensor* dk,
                                        attn_tensor* dv, float* dsink, void* stream) {
  const size_t need = attn_bwd_workspace_size(q, k, v, mask);
  if (need > kNoAllocScratchBytes) return ATTN_ERR_WORKSPACE;
  void* scratch = nullptr;
  const attn_status st = scratch_address(&scratch);
  if (st != ATTN_OK) return st;
  // attn_bwd itself zeroes every part of the scratch that must start at zero
  // (status word, dQ accumulator, fixed-point dKV accumulator) on `stream`.
  return attn_bwd(q, k, v, o, do_, lse, mask, scale, dq, dk, dv, dsink, scratch, kNoAllocScratchBytes, stream);
}
#pragma GCC visibility pop
