// Shared device-side definitions: parameter blocks, the allowed-set predicate,
// the Philox4x32-10 dropout generator and dtype-generic loads/stores.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/attn.h"

namespace attn {

// Byte offsets inside every workspace.
constexpr size_t kStatusBytes = 256;  // status word lives at offset 0

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Allowed-set descriptor as the kernels see it.
struct MaskP {
  uint32_t flags;
  int64_t qoff;    // query row i sits at key position i + qoff (Tk - Tq: bottom-right alignment)
  int64_t window;  // W: j > i + qoff - W
  const uint8_t* bm;
  int32_t bq, bk;
  int64_t bm_sb, bm_sh, bm_sq;
  const float* sink;  // [Hq] or null
  int dropout;        // 0/1
  uint32_t keep_thr;  // keep iff philox word >= keep_thr
  float inv_keep;     // 1 / (1 - rho)
  uint32_t seed_lo, seed_hi;
  const int32_t* lengths;  // [B] active cells per batch row, or null
  const int32_t* starts;   // (b, i) at starts[b * st_sb + i]: lowest allowed key, or null
  int64_t st_sb;
  uint32_t lse_fmt;        // ATTN_LSE_* bits of the LSE output
};

// Active length of batch row b, clamped to [0, n] (n when not set).
__device__ __forceinline__ int64_t active_len(const MaskP& m, int b, int64_t n) {
  if (!m.lengths) return n;
  const int64_t L = m.lengths[b];
  return L < 0 ? 0 : (L > n ? n : L);
}

// Lowest allowed key of query row i of batch row b (0 when not set).
__device__ __forceinline__ int64_t row_start(const MaskP& m, int b, int64_t i) {
  return m.starts ? (int64_t)m.starts[b * m.st_sb + i] : 0;
}

// Dense problem: all strides in elements for (b, h, t); innermost stride 1.
struct DenseP {
  const void* q;
  const void* k;
  const void* v;
  int64_t sq[3], sk[3], sv[3];
  int B, Hq, Hkv, Tq, Tk, d, dv;
  int32_t dtype;       // attn_dtype of every tensor
  uint32_t bwd_flags;  // ATTN_BWD_* bits
  float scale;
  MaskP m;
};

// Shared-KV top-k problem.
struct TopkP {
  const void* q;   // [Tq, H, Dqk]
  const void* kv;  // [Tkv, Dqk]; V = first Dv columns
  int64_t sq_t, sq_h, skv;
  const int32_t* idx;
  int64_t idx_stride;
  int32_t topk_max;
  const int32_t* len;  // may be null
  int Tq, Tkv, H, Dqk, Dv;
  int32_t dtype;  // attn_dtype of every tensor
  float scale;
  const float* sink;
  uint32_t lse_fmt;  // ATTN_LSE_* bits of the LSE output
  int32_t check_causal;  // ATTN_MASK_TOPK_CHECK_CAUSAL: flag listed indices past Tkv - Tq + t
};

// The LSE value to store for a row, from base-2 quantities: lse2_total =
// log2 of the sink-inclusive denominator, (m2, l2) = running maximum and
// shifted sum of the allowed scores alone. Default: natural log, sink
// included; ATTN_LSE_KV_ONLY: the sink left out; ATTN_LSE_NEG_LOG2: stored
// as -log2 of the chosen denominator.
__device__ __forceinline__ float stored_lse_log2(uint32_t fmt, float lse2_total, float m2, float l2) {
  constexpr float log2e = 1.4426950408889634f;
  float v = lse2_total;
  if (fmt & ATTN_LSE_KV_ONLY) v = m2 == -INFINITY ? -INFINITY : m2 + log2f(l2);
  return (fmt & ATTN_LSE_NEG_LOG2) ? -v : v / log2e;
}

// The same from natural-log quantities (lse_total, running max m, sum l).
__device__ __forceinline__ float stored_lse_ln(uint32_t fmt, float lse_total, float m, float l) {
  constexpr float log2e = 1.4426950408889634f;
  float v = lse_total;
  if (fmt & ATTN_LSE_KV_ONLY) v = m == -INFINITY ? -INFINITY : m + logf(l);
  return (fmt & ATTN_LSE_NEG_LOG2) ? -v * log2e : v;
}

__device__ __forceinline__ float ld(const float* p) { return *p; }
__device__ __forceinline__ float ld(const __nv_bfloat16* p) { return __bfloat162float(*p); }
__device__ __forceinline__ float ld(const __half* p) { return __half2float(*p); }
__device__ __forceinline__ void st(float* p, float x) { *p = x; }
__device__ __forceinline__ void st(__nv_bfloat16* p, float x) { *p = __float2bfloat16_rn(x); }
__device__ __forceinline__ void st(__half* p, float x) { *p = __float2half_rn(x); }

// The allowed-set predicate A_i (flags intersect).
__device__ __forceinline__ bool allowed(const MaskP& m, int b, int h, int64_t i, int64_t j) {
  const int64_t ip = i + m.qoff;  // the query's key position
  if ((m.flags & ATTN_MASK_CAUSAL) && j > ip) return false;
  if ((m.flags & ATTN_MASK_WINDOW) && j <= ip - m.window) return false;
  if (m.flags & ATTN_MASK_BLOCK) {
    const uint8_t* row = m.bm + b * m.bm_sb + h * m.bm_sh + (i / m.bq) * m.bm_sq;
    if (!row[j / m.bk]) return false;
  }
  if (m.lengths) {
    const int64_t L = active_len(m, b, INT64_MAX);
    if (i >= L || j >= L) return false;
  }
  if (m.starts && j < row_start(m, b, i)) return false;
  return true;
}

// Key range [lo, hi] that can hold allowed keys for query row i.
__device__ __forceinline__ void key_range(const MaskP& m, int b, int64_t i, int64_t n_k,
                                          int64_t& lo, int64_t& hi) {
  const int64_t ip = i + m.qoff;
  lo = 0;
  hi = n_k - 1;
  if (m.flags & ATTN_MASK_CAUSAL) hi = ip < hi ? ip : hi;
  if (m.flags & ATTN_MASK_WINDOW) {
    int64_t w = ip - m.window + 1;
    lo = w > 0 ? w : 0;
  }
  if (m.lengths) {
    const int64_t L = active_len(m, b, n_k);
    if (i >= L) hi = -1;
    if (L - 1 < hi) hi = L - 1;
  }
  if (m.starts) {
    const int64_t s = row_start(m, b, i);
    if (s > lo) lo = s;
  }
}

// Query range [lo, hi] that can hold key j in its allowed set.
__device__ __forceinline__ void query_range(const MaskP& m, int b, int64_t j, int64_t n_q,
                                            int64_t& lo, int64_t& hi) {
  lo = 0;
  hi = n_q - 1;
  if (m.flags & ATTN_MASK_CAUSAL) lo = j - m.qoff > 0 ? j - m.qoff : 0;
  if (m.flags & ATTN_MASK_WINDOW) {
    int64_t w = j + m.window - 1 - m.qoff;
    hi = w < hi ? w : hi;
  }
  if (m.lengths) {  // Tq = Tk here
    const int64_t L = active_len(m, b, n_q);
    if (j >= L) hi = -1;
    if (L - 1 < hi) hi = L - 1;
  }
}

// Philox4x32 with 10 rounds (Salmon, Moraes, Dror, Shaw, "Parallel Random
// Numbers: As Easy as 1, 2, 3", SC'11): two 32x32->64 multiplies per round
// by fixed odd constants, word exchange, key folded into the high halves,
// key advanced by the Weyl increments between rounds.
__device__ __forceinline__ uint4 philox4x32_10(uint4 c, uint32_t k0, uint32_t k1) {
#pragma unroll
  for (int r = 0; r < 10; ++r) {
    if (r) {
      k0 += 0x9E3779B9u;
      k1 += 0xBB67AE85u;
    }
    const uint32_t lo0 = 0xD2511F53u * c.x, hi0 = __umulhi(0xD2511F53u, c.x);
    const uint32_t lo1 = 0xCD9E8D57u * c.z, hi1 = __umulhi(0xCD9E8D57u, c.z);
    c = make_uint4(hi1 ^ c.y ^ k0, lo1, hi0 ^ c.w ^ k1, lo0);
  }
  return c;
}

__device__ __forceinline__ uint32_t uint4_word(const uint4& w, int idx) {
  return idx == 0 ? w.x : idx == 1 ? w.y : idx == 2 ? w.z : w.w;
}

// Keep decision xi for pair (b, h, i, j): counter (j>>2, i, h, b).
__device__ __forceinline__ bool dropout_keep(const MaskP& m, int b, int h, int64_t i, int64_t j) {
  uint4 w = philox4x32_10(make_uint4((uint32_t)(j >> 2), (uint32_t)i, (uint32_t)h, (uint32_t)b),
                          m.seed_lo, m.seed_hi);
  return uint4_word(w, (int)(j & 3)) >= m.keep_thr;
}

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

__device__ __forceinline__ void set_status(uint32_t* status, uint32_t bits) {
  if (status) atomicOr(status, bits);
}

// The debug check of a valid listed index j of token t against the token's
// causal position Tkv - Tq + t (ATTN_MASK_TOPK_CHECK_CAUSAL).
__device__ __forceinline__ void check_topk_causal(int check, int64_t j, int t, int Tq, int Tkv, uint32_t* status) {
  if (check && j > (int64_t)Tkv - Tq + t) set_status(status, ATTN_DEVERR_TOPK_CAUSAL);
}

// The fixed-point dKV accumulator of the top-k reverse: [Tkv, Dqk] signed
// 32.32 integers, then per KV row the number of contributions it received,
// then one word holding the largest contribution magnitude of the call (the
// bit pattern of a non-negative float, ordered like the value). The counts
// and the magnitude bound every row's sum (|sum| <= count * largest), which
// the conversion to the output checks against the accumulator's range.
inline size_t topk_acc_bytes(int Tkv, int Dqk) { return align_up((size_t)Tkv * Dqk * sizeof(unsigned long long), 256); }
inline size_t topk_acc_total_bytes(int Tkv, int Dqk) {
  return topk_acc_bytes(Tkv, Dqk) + align_up(((size_t)Tkv + 1) * sizeof(uint32_t), 256);
}
struct FixedAcc {
  unsigned long long* acc;  // [Tkv, Dqk]
  uint32_t* count;          // [Tkv]
  uint32_t* maxbits;        // one word
};
inline FixedAcc fixed_acc_at(void* base, int Tkv, int Dqk) {
  FixedAcc f;
  f.acc = static_cast<unsigned long long*>(base);
  f.count = reinterpret_cast<uint32_t*>(static_cast<char*>(base) + topk_acc_bytes(Tkv, Dqk));
  f.maxbits = f.count + Tkv;
  return f;
}

// One contribution x to a fixed-point dKV element: clamped to |x| < 2^30
// (flagged), converted to 32.32 and added; *amax keeps the largest |x| seen.
__device__ __forceinline__ void fixed_add(unsigned long long* dst, float x, bool& sat, float& amax) {
  const float lim = 1073741824.f;  // 2^30: |x| 2^32 stays below 2^62
  const float ax = fabsf(x);
  if (!(ax < lim)) {
    sat = true;
    x = x != x ? 0.f : copysignf(lim, x);
  }
  amax = fmaxf(amax, fminf(ax, lim));
  atomicAdd(dst, (unsigned long long)__float2ll_rn(x * 4294967296.f));
}

// The warp's largest contribution magnitude into the call's word (once per
// warp; whole warp, converged).
__device__ __forceinline__ void fixed_publish_max(uint32_t* maxbits, float amax) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  if ((threadIdx.x & 31) == 0 && amax > 0.f) atomicMax(maxbits, __float_as_uint(amax));
}

// Caller-supplied timing events around the main kernel of the next call on
// this host thread (attn_set_kernel_events); no-ops when none is pending.
void main_kernel_begin(cudaStream_t st);
void main_kernel_end(cudaStream_t st);

}  // namespace attn
