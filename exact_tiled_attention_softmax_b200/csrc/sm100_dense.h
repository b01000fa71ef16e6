// Tensor-core (tcgen05 / TMEM / TMA) path for dense bf16 attention with
// d = dv = 128 on sm_100a (internal; not part of the ABI).
#pragma once

#include <cuda_runtime.h>

#include "common.cuh"

namespace attn {

size_t sm100_fwd_workspace_bytes(int B, int Hq, int Tq, int Tk, const attn_mask* m);
size_t sm100_bwd_extra_workspace_bytes(int B, int Hq, int Hkv, int Tq, int Tk, const attn_mask* m);
bool sm100_dense_supported(const DenseP& p, const attn_tensor* q, const attn_tensor* k, const attn_tensor* v,
                           const attn_tensor* o);
bool sm100_dense_bwd_supported(const DenseP& p, const attn_tensor* do_, const attn_tensor* dq,
                               const attn_tensor* dk, const attn_tensor* dv);
cudaError_t sm100_dense_fwd(const DenseP& p, void* o, const int64_t so[3], float* lse, const int64_t sl[3],
                            void* ws, uint32_t* status, cudaStream_t st);
cudaError_t sm100_dense_bwd(const DenseP& p, const void* o, const int64_t so[3], const void* g,
                            const int64_t sg[3], const float* lse, const int64_t sl[3], float* delta,
                            float* dq_acc, void* dq, const int64_t sdq[3], void* dk, const int64_t sdk[3],
                            void* dv, const int64_t sdv[3], void* ws_extra, uint32_t* status, cudaStream_t st);

}  // namespace attn
