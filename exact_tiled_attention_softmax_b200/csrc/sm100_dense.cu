// Placeholder: the tensor-core path is not wired in yet.
#include "sm100_dense.h"

namespace attn {

size_t sm100_fwd_workspace_bytes(int, int, int, const attn_mask*) { return 0; }
size_t sm100_bwd_extra_workspace_bytes(int, int, int, int, const attn_mask*) { return 0; }
bool sm100_dense_supported(const DenseP&, const attn_tensor*, const attn_tensor*, const attn_tensor*,
                           const attn_tensor*) {
  return false;
}
bool sm100_dense_bwd_supported(const DenseP&, const attn_tensor*, const attn_tensor*, const attn_tensor*,
                               const attn_tensor*) {
  return false;
}
cudaError_t sm100_dense_fwd(const DenseP&, void*, const int64_t[3], float*, const int64_t[3], void*, uint32_t*,
                            cudaStream_t) {
  return cudaErrorNotSupported;
}
cudaError_t sm100_dense_bwd(const DenseP&, const void*, const int64_t[3], const void*, const int64_t[3],
                            const float*, const int64_t[3], float*, float*, void*, const int64_t[3], void*,
                            const int64_t[3], void*, const int64_t[3], void*, uint32_t*, cudaStream_t) {
  return cudaErrorNotSupported;
}

}  // namespace attn
