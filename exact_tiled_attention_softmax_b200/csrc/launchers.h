// Host-side launchers of the device kernels (internal; not part of the ABI).
#pragma once

#include <cuda_runtime.h>

#include "common.cuh"

namespace attn {

// Row-wise kernels (any dtype, head width <= 576, every allowed-set kind).
template <typename T>
cudaError_t launch_dense_fwd_rows(const DenseP& p, void* o, const int64_t so[3], float* lse,
                                  const int64_t sl[3], cudaStream_t st);
template <typename T>
cudaError_t launch_topk_fwd_rows(const TopkP& p, void* o, int64_t so_t, int64_t so_h, float* lse,
                                 int64_t sl_t, int64_t sl_h, uint32_t* status, cudaStream_t st);
template <typename T>
cudaError_t launch_rows_delta(const void* o, const void* g, int64_t n_outer, int64_t n_mid,
                              int64_t n_inner, const int64_t so[3], const int64_t sg[3], int dv,
                              float* delta, cudaStream_t st);
template <typename T>
cudaError_t launch_dense_bwd_rows(const DenseP& p, const void* g, const int64_t sg[3], const float* lse,
                                  const int64_t sl[3], const float* delta, void* dq, const int64_t sdq[3],
                                  void* dk, const int64_t sdk[3], void* dv, const int64_t sdv[3],
                                  cudaStream_t st);
template <typename T>
cudaError_t launch_topk_bwd_rows(const TopkP& p, const void* g, int64_t sg_t, int64_t sg_h,
                                 const float* lse, int64_t sl_t, int64_t sl_h, const float* delta,
                                 void* dq, int64_t sd_t, int64_t sd_h, FixedAcc acc,
                                 void* dkv, int64_t sdkv, uint32_t* status, cudaStream_t st);
// dKV from the fixed-point accumulator, with the per-row range check (sets
// ATTN_DEVERR_OVERFLOW in *status when a row's sum may have wrapped).
template <typename T>
cudaError_t launch_fixed_to_out(FixedAcc acc, int rows, int cols, void* out, int64_t so, uint32_t* status,
                                cudaStream_t st);
// dKV from an fp32 accumulator [rows, cols].
template <typename T>
cudaError_t launch_f32_to_out(const float* acc, int rows, int cols, void* out, int64_t so, cudaStream_t st);
cudaError_t launch_lse_to_total(const float* in, int n0, int n1, int n2, const int64_t s[3], int head_dim,
                                const float* sink, uint32_t fmt, float* out, cudaStream_t st);
cudaError_t launch_dsink(const float* sink, const float* lse, const float* delta, int n_outer, int n_heads,
                         int n_inner, int64_t sl_outer, int64_t sl_head, int64_t sl_inner,
                         bool delta_head_major, float* dsink, cudaStream_t st);
// One CTA that waits on an mbarrier phase nothing completes, until the bounded
// wait gives up and sets the timeout bit in *status.
cudaError_t launch_wait_timeout_probe(uint32_t* status, cudaStream_t st);
// Device address of attn_bwd_noalloc's status word on the current device
// (the start of its fixed scratch array); null with *st set on failure.
void* noalloc_status_word(cudaStream_t stream, attn_status* st);

}  // namespace attn
