// Tensor-core (tcgen05 / TMEM / TMA gather4) path for the top-k forward with a
// shared KV: bf16, 64 heads, Dqk = 576, Dv = 512, on sm_100a (internal; not
// part of the ABI).
#pragma once

#include <cuda_runtime.h>

#include "common.cuh"

namespace attn {

bool sm100_topk_supported(const TopkP& p, const attn_tensor* q, const attn_tensor* kv, const attn_tensor* o);
cudaError_t sm100_topk_fwd(const TopkP& p, void* o, int64_t so_t, int64_t so_h, float* lse, int64_t sl_t,
                           int64_t sl_h, uint32_t* status, cudaStream_t st);

}  // namespace attn
