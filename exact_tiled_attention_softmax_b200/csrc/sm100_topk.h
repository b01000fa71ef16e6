// Tensor-core (tcgen05 / TMEM, cp.async row gathers) path for the top-k forward and reverse with a
// shared KV: bf16, 64 heads, Dqk = 576, Dv = 512, on sm_100a (internal; not
// part of the ABI).
#pragma once

#include <cuda_runtime.h>

#include "common.cuh"

namespace attn {

bool sm100_topk_supported(const TopkP& p, const attn_tensor* q, const attn_tensor* kv, const attn_tensor* o);
int sm100_topk_pad(int topk_max);
size_t sm100_topk_bwd_scratch_bytes(int Tq, int H, int Dqk, int Dv, int topk_max);
bool sm100_topk_bwd_supported(const TopkP& p, const attn_tensor* q, const attn_tensor* kv, const attn_tensor* o,
                              const attn_tensor* do_, const attn_tensor* dq);
// Reverse on tensor cores: dQ, and dKV added either into the fp32
// accumulator `acc32` [Tkv, Dqk] (when not null; floating-point atomics) or
// into the 32.32 fixed-point accumulator `acc` with its per-row counts and
// largest magnitude (bitwise reproducible); the caller zeroes the one used.
// `scratch` holds the G and P rows (sm100_topk_bwd_scratch_bytes).
cudaError_t sm100_topk_bwd(const TopkP& p, const void* g, int64_t sg_t, int64_t sg_h, const float* lse,
                           int64_t sl_t, int64_t sl_h, const float* delta, void* dq, int64_t sd_t, int64_t sd_h,
                           FixedAcc acc, float* acc32, void* scratch, uint32_t* status, cudaStream_t st);
cudaError_t sm100_topk_fwd(const TopkP& p, void* o, int64_t so_t, int64_t so_h, float* lse, int64_t sl_t,
                           int64_t sl_h, uint32_t* status, cudaStream_t st);

}  // namespace attn
