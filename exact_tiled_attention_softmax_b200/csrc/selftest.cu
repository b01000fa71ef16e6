// Failure-detection self-test: one CTA whose threads wait, through the same
// bounded mbarrier wait every tensor-core pipeline stage uses, on a barrier
// phase that no thread ever completes. The wait runs out after its limit,
// raises the CTA's abort flag and the ATTN_DEVERR_TIMEOUT status bit, and
// every thread returns, so the context stays usable and the host reads the
// bit through the status word. No attention arithmetic runs here.
#include "launchers.h"
#include "sm100_ptx.cuh"

namespace attn {
namespace {

constexpr int kProbeThreads = 64;

__global__ void __launch_bounds__(kProbeThreads, 1) wait_timeout_kernel(uint32_t* status) {
  __shared__ alignas(8) uint64_t bar;
  __shared__ uint32_t abort_flag;
  if (threadIdx.x == 0) {
    sm100::mbar_init(sm100::smem_u32(&bar), 1);  // one arrival would complete phase 0; none comes
    abort_flag = 0;
    sm100::fence_barrier_init();
  }
  __syncthreads();
  // Every thread waits on phase 0. The first to reach the limit sets the
  // abort flag and the status bit; the others see the flag and leave too.
  (void)sm100::wait_bar(sm100::smem_u32(&bar), 0, &abort_flag, status);
}

}  // namespace

cudaError_t launch_wait_timeout_probe(uint32_t* status, cudaStream_t st) {
  wait_timeout_kernel<<<1, kProbeThreads, 0, st>>>(status);
  return cudaGetLastError();
}

}  // namespace attn
