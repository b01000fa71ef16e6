/*
 * attn.h -- C ABI of the exact tiled masked softmax attention library.
 *
 * The library computes, on one NVIDIA B200 (sm_100a), exact masked softmax
 * attention with a per-row running summary (m, l, z) carried across key
 * tiles, and its reverse pass, which recomputes the scores tile by tile from
 * the saved log-sum-exp instead of storing the probability grid.
 *
 * Definitions
 *   Forward ("Tiled attention and its recomputed reverse pass are exact",
 *   alphabetamath.cc, proof steps 1.1-2.1; "Accumulate attention without
 *   keeping the full grid", intale.github.io, section "Rescale earlier mass
 *   before adding a new tile"): for query row i with allowed key set A_i,
 *       s_ij = c <Q_i, K_j>,   p_ij = exp(s_ij) / (exp(z_h) + sum_{l in A_i} exp(s_il)),
 *       Y_i  = sum_{j in A_i} p~_ij V_j,  LSE_i = ln(exp(z_h) + sum_{l in A_i} exp(s_il)).
 *   z_h is the optional per-head sink logit ("DeepSeek Sparse Attention
 *   Forward and Backward", icavan.github.io, section 2.2; absent = -inf), and
 *   p~_ij = p_ij xi_ij / (1 - rho) the optional inverted dropout ("A
 *   different dropout mask changes the reverse result", alphabetamath.cc).
 *   Reverse (same proof, steps 4.1-6.1; DSA note, sections 3.1-3.5):
 *       delta_i = <G_i, Y_i>,  gamma_ij = p_ij (xi_ij/(1-rho) <G_i, V_j> - delta_i),
 *       dQ_i = c sum_j gamma_ij K_j,  dK_j = c sum_i gamma_ij Q_i,
 *       dV_j = sum_i p~_ij G_i,       dz_h = -sum_{b,i} exp(z_h - LSE_i) delta_i.
 *   Query head h reads K/V head h / (Hq / Hkv); shared K/V heads sum the
 *   pullbacks of every query head that reads them.
 *
 * Memory and ownership
 *   Every tensor pointer is a DEVICE pointer owned by the caller. The library
 *   allocates no device memory; scratch space is the caller's workspace,
 *   sized by attn_fwd_workspace_size / attn_bwd_workspace_size. All work is
 *   enqueued asynchronously on the caller's stream (a cudaStream_t passed as
 *   void*; NULL = the legacy default stream). Outputs are overwritten, never
 *   accumulated into. The library may cache host-side state per device
 *   (TMA descriptors, kernel attributes).
 *
 * Errors
 *   Every call returns an attn_status synchronously. Argument problems are
 *   found on the host before any launch (ATTN_ERR_INVALID_ARG: shape, stride,
 *   dtype, alignment, Hq % Hkv != 0, a dropout rate outside [0,1), ...).
 *   Conditions only the device can see (a top-k index outside [0, Tkv), a
 *   fixed-point overflow, a pipeline wait that ran out) are written to a
 *   status word at the start of the workspace; read it with attn_get_status
 *   after the stream has reached the call. No call traps the GPU, and on any
 *   error the outputs' contents are unspecified.
 */
#ifndef ATTN_H_
#define ATTN_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define ATTN_VERSION 107 /* major * 100 + minor */

typedef enum attn_status {
  ATTN_OK = 0,
  ATTN_ERR_INVALID_ARG = 1, /* bad shape, stride, dtype, alignment, pointer */
  ATTN_ERR_UNSUPPORTED = 2, /* a valid request with no kernel for it */
  ATTN_ERR_WORKSPACE = 3,   /* workspace NULL or smaller than required */
  ATTN_ERR_CUDA = 4,        /* a CUDA runtime or driver call failed */
  ATTN_ERR_DEVICE = 5       /* the device recorded an error (attn_get_status) */
} attn_status;

/* Device-side error bits reported through attn_get_status. */
#define ATTN_DEVERR_TOPK_INDEX 0x1u  /* a listed index outside [0, Tkv) was skipped */
#define ATTN_DEVERR_OVERFLOW 0x2u    /* the fixed-point dKV sum of a row may not fit (see below) */
#define ATTN_DEVERR_TIMEOUT 0x4u     /* a bounded pipeline wait gave up */
#define ATTN_DEVERR_TOPK_CAUSAL 0x8u /* ATTN_MASK_TOPK_CHECK_CAUSAL: a listed index lies
                                        beyond its token's causal position */
/* ATTN_DEVERR_OVERFLOW: when the top-k reverse pass sums each dKV element in
 * a signed 32.32 fixed-point integer (range +-2^31: the row kernels, and the
 * tensor-core path under ATTN_BWD_DETERMINISTIC), the bit is set when a
 * single contribution was at least 2^30 in magnitude (it is then clamped),
 * and whenever some KV row's number of contributions times the largest
 * contribution magnitude of the call reaches 2^31: a bound on |sum| that
 * every overflow exceeds, so a sum that wrapped always sets the bit (the
 * bound can also set it for sums that did fit). */

typedef enum attn_dtype { ATTN_F32 = 0, ATTN_BF16 = 1, ATTN_F16 = 2 } attn_dtype;

/* A strided tensor view. Strides count elements, not bytes; the innermost
 * dimension must have stride 1. Unused trailing entries are ignored. */
typedef struct attn_tensor {
  void* data;
  int32_t dtype; /* attn_dtype */
  int32_t ndim;
  int64_t shape[4];
  int64_t stride[4];
} attn_tensor;

/* Allowed-set flags. A_i is the intersection of every enabled set. With
 * Tq query rows and Tk keys, query row i sits at key position
 * p(i) = i + Tk - Tq (bottom-right alignment: the last query row sees the
 * last key; p(i) = i when Tq = Tk). */
#define ATTN_MASK_CAUSAL 0x1u /* j <= p(i) */
#define ATTN_MASK_WINDOW 0x2u /* j >  p(i) - window_left */
#define ATTN_MASK_BLOCK 0x4u  /* block_mask[i / block_q][j / block_k] != 0 */
#define ATTN_MASK_TOPK 0x8u   /* j listed in topk_idxs[t][0 : topk_length[t]] */
#define ATTN_MASK_LENGTHS 0x10u /* i < lengths[b] and j < lengths[b] (needs Tq = Tk) */
#define ATTN_MASK_STARTS 0x20u  /* j >= starts[b][i] */
/* Debug check for ATTN_MASK_TOPK (no set of its own): every listed entry
 * inside the token's length is also compared with the token's causal
 * position Tkv - Tq + t; an entry beyond it sets ATTN_DEVERR_TOPK_CAUSAL in
 * the status word. The entry is still used: the lists' causality is the
 * caller's contract, and the check reports a broken one without changing the
 * result. Costs one compare per listed entry. */
#define ATTN_MASK_TOPK_CHECK_CAUSAL 0x40u

/* The allowed-set descriptor ("Tiled attention and its recomputed reverse
 * pass are exact": the fixed allowed sets A_i; causal, windowed and packed
 * intervals from "Accumulate attention without keeping the full grid",
 * section "Change attention evaluation inside the existing model"; the
 * shared-KV index lists of the DSA note, section 1). Pointers are device
 * pointers. */
typedef struct attn_mask {
  uint32_t flags;
  int64_t window_left; /* W >= 1 with ATTN_MASK_WINDOW */
  /* ATTN_MASK_BLOCK: uint8 grid, element (b, h, r, c) at
   * block_mask[b*bm_stride_b + h*bm_stride_h + r*bm_stride_q + c]; a zero
   * stride broadcasts. Rows ceil(Tq/block_q), columns ceil(Tk/block_k). */
  const uint8_t* block_mask;
  int32_t block_q, block_k;
  int64_t bm_stride_b, bm_stride_h, bm_stride_q;
  /* ATTN_MASK_TOPK: int32 [Tq, topk_stride]; entries at positions >=
   * topk_length[t] (or >= topk_max when topk_length is NULL) are ignored.
   * Each listed position counts once. */
  const int32_t* topk_idxs;
  int64_t topk_stride;
  int32_t topk_max;
  const int32_t* topk_length;
  /* Optional per-query-head sink logit z_h, fp32 [Hq]; NULL = no sink. */
  const float* sink;
  /* Optional inverted dropout: rate in [0, 1), 0 = off. The keep decision for
   * pair (b, h, i, j) is word (j & 3) of Philox4x32-10 at counter
   * (j >> 2, i, h, b) and key (seed low 32 bits, seed high 32 bits), kept iff
   * that word >= floor(rate * 2^32). Both passes evaluate it; no mask is
   * stored. */
  float dropout_p;
  uint64_t dropout_seed;
  /* Row-interval layouts ("Accumulate attention without keeping the full
   * grid", section "Change attention evaluation inside the existing model":
   * active lengths and packed-segment boundaries), dense calls only.
   * ATTN_MASK_LENGTHS: int32 [B]; batch row b has lengths[b] active cells
   * (values are clamped to [0, T]); query rows and keys past it belong to no
   * set, so padding rows get the empty-set result. Requires Tq = Tk.
   * ATTN_MASK_STARTS: int32, element (b, i) at starts[b*starts_stride_b + i]
   * for query row i in [0, Tq) (a zero stride broadcasts over the batch);
   * key j is allowed for that row only if j >= the element. With
   * ATTN_MASK_CAUSAL and starts = each row's segment start this is causal
   * attention inside packed segments. */
  const int32_t* lengths;
  const int32_t* starts;
  int64_t starts_stride_b;
  /* Format of the LSE that attn_fwd writes and attn_bwd reads ("DeepSeek
   * Sparse Attention Forward and Backward", section 7): 0 = natural log of
   * the sink-inclusive denominator Z (section 7.1), or a combination of the
   * ATTN_LSE_* bits below. attn_bwd must be given the format attn_fwd wrote. */
  uint32_t lse_format;
  /* Options of attn_bwd: 0 or ATTN_BWD_DETERMINISTIC. */
  uint32_t bwd_flags;
} attn_mask;

/* ATTN_BWD_DETERMINISTIC: every gradient is bitwise reproducible from run to
 * run. Dense dK and dV always are (one CTA per key tile), and so is the
 * top-k dQ (one CTA per query token). With this flag the dense tensor-core
 * path also computes dQ in a query-centric pass (one CTA sums each dQ
 * element over the key tiles in order, recomputing P and gamma) instead of
 * reducing per-key-tile partials with floating-point atomics, at the cost of
 * one extra pass; and the top-k tensor-core path adds the per-token dKV
 * contributions into a signed 32.32 fixed-point accumulator with integer
 * atomics (range check below) instead of fp32 atomics (the DSA note's
 * choice, section 9), at about 1.5 times the reduction traffic. The top-k
 * row kernels (other shapes, fp32 storage) always use the fixed-point
 * accumulator. */
#define ATTN_BWD_DETERMINISTIC 0x1u

/* ATTN_LSE_KV_ONLY: the denominator leaves the sink out, ln sum_j exp(s_j)
 * (section 7.2; -inf for an empty allowed set even with a sink). The reverse
 * pass combines it with the sink logit as logaddexp(LSE_kv, z) before use.
 * ATTN_LSE_NEG_LOG2: the stored value is -log2 of the denominator, the
 * base-2 form of section 7.3 (+inf for an empty row without a sink). */
#define ATTN_LSE_KV_ONLY 0x1u
#define ATTN_LSE_NEG_LOG2 0x2u

/* Layouts
 *   Dense:  q [B,Hq,Tq,d], k [B,Hkv,Tk,d], v [B,Hkv,Tk,dv], o [B,Hq,Tq,dv],
 *           lse fp32 [B,Hq,Tq]; dq, do like q/o, dk, dv like k/v. Tq and Tk
 *           may differ (a query block against a longer key cache); the
 *           block mask grid is [ceil(Tq/block_q)][ceil(Tk/block_k)] indexed
 *           by the query's own row. Any stride order (BHSD, BSHD, ...).
 *   Top-k (ATTN_MASK_TOPK, shared KV): q [Tq,H,Dqk], k = KV [Tkv,Dqk],
 *           v = the view KV[:, :Dv] (same data pointer and row stride as k),
 *           o [Tq,H,Dv], lse fp32 [Tq,H]. dk receives dKV [Tkv,Dqk]; dv is NULL.
 *           Query token t sits at causal position Tkv - Tq + t; the lists
 *           must respect causality themselves.
 *   dtype: all of q, k, v, o (and do, dq, dk, dv) share one dtype, ATTN_F32,
 *   ATTN_BF16 or ATTN_F16 (the DSA note's storage table: BF16 or FP16).
 *   Accumulation is fp32 in every path; the probability and score-gradient
 *   operands of the tensor-core MMAs take the storage type.
 */

/* Workspace bytes attn_fwd needs for these shapes and mask (>= 256). */
size_t attn_fwd_workspace_size(const attn_tensor* q, const attn_tensor* k,
                               const attn_tensor* v, const attn_mask* mask);

/* Workspace bytes attn_bwd needs for these shapes and mask (>= 256). */
size_t attn_bwd_workspace_size(const attn_tensor* q, const attn_tensor* k,
                               const attn_tensor* v, const attn_mask* mask);

/* Forward pass: writes o = Y and lse (natural log, sink-inclusive: DSA note,
 * section 7.1). Rows whose allowed set is empty get Y = 0 and LSE = -inf
 * (or z_h with a sink). scale is c. */
attn_status attn_fwd(const attn_tensor* q, const attn_tensor* k,
                     const attn_tensor* v, const attn_mask* mask, float scale,
                     attn_tensor* o, attn_tensor* lse, void* workspace,
                     size_t workspace_bytes, void* stream);

/* Reverse pass for upstream gradient do_ (= G): recomputes the scores from
 * q, k and the saved lse, forms delta from o and do_, and writes dq, dk, dv
 * (top-k: dk = dKV, dv = NULL) and, when mask->sink is set and dsink is not
 * NULL, dsink fp32 [Hq]. Dense dk and dv, the top-k dq and dsink are
 * deterministic (bitwise identical across runs); the dense dq and the
 * tensor-core top-k dKV are summed with floating-point atomics and are
 * not, unless mask->bwd_flags holds ATTN_BWD_DETERMINISTIC (then every
 * output is). */
attn_status attn_bwd(const attn_tensor* q, const attn_tensor* k,
                     const attn_tensor* v, const attn_tensor* o,
                     const attn_tensor* do_, const attn_tensor* lse,
                     const attn_mask* mask, float scale, attn_tensor* dq,
                     attn_tensor* dk, attn_tensor* dv, float* dsink,
                     void* workspace, size_t workspace_bytes, void* stream);

/* Reverse pass without any device allocation, for callers that cannot call
 * cudaMalloc: a host framework that owns every byte of device memory through
 * its own allocator and budget, a plugin that may not allocate behind that
 * framework's back, or a latency-bound loop where an allocation (which can
 * synchronise the device) is not allowed. The pages have no counterpart to
 * this entry point; it exists only for such callers.
 *
 * Same arguments and results as attn_bwd, minus the workspace: the scratch
 * space is a fixed 64 MiB array inside the library's device memory (one per
 * GPU that loads the library, held until the process exits). A problem whose
 * attn_bwd_workspace_size exceeds 64 MiB is rejected with
 * ATTN_ERR_WORKSPACE before anything is enqueued. The first call on each
 * device looks up the array's device address with that device current (and
 * again after the device's context has been destroyed and re-created, e.g. by
 * cudaDeviceReset); make that first call before any stream capture: made
 * while `stream` is being captured it returns ATTN_ERR_UNSUPPORTED. Every call
 * shares the one array and it keeps the previous call's contents (the pass
 * clears what must start at zero itself), so calls whose GPU work overlaps in
 * time, on different streams or from different threads, race on it:
 * serialise them. The device status word is the first word of that array:
 * read and clear it with attn_get_status(NULL, stream, &bits) with the same
 * device current. */
attn_status attn_bwd_noalloc(const attn_tensor* q, const attn_tensor* k,
                             const attn_tensor* v, const attn_tensor* o,
                             const attn_tensor* do_, const attn_tensor* lse,
                             const attn_mask* mask, float scale, attn_tensor* dq,
                             attn_tensor* dk, attn_tensor* dv, float* dsink,
                             void* stream);

/* Synchronises `stream`, then reads and clears the device status word at the
 * start of `workspace` (workspace NULL: the status word of attn_bwd_noalloc's
 * scratch array on the current device). *device_bits receives the
 * ATTN_DEVERR_* bits (0 when clean). Returns ATTN_ERR_DEVICE when any bit was
 * set. */
attn_status attn_get_status(void* workspace, void* stream, uint32_t* device_bits);

/* Kernel timing without a profiler. `begin` and `end` are cudaEvent_t
 * handles created and owned by the caller. The next attn_fwd or attn_bwd
 * call made from the same host thread records `begin` on its stream just
 * before its main kernel (the tensor-core kernel, or the row-wise kernels
 * that do the attention arithmetic) and `end` just after it, then forgets
 * both, whether or not the call launched anything; the small setup and
 * finishing kernels around it (tile classes, delta, the dq cast) fall
 * outside the pair. NULL, NULL cancels a pending pair. Always ATTN_OK. */
attn_status attn_set_kernel_events(void* begin, void* end);

/* Failure-detection self-test; no attention arithmetic. Clears the status
 * word at the start of `workspace`, then enqueues on `stream` one CTA whose
 * threads wait, through the same bounded mbarrier wait that every stage of
 * the tensor-core pipelines uses, on a barrier phase that nothing completes.
 * When the wait's limit (2 s) runs out the kernel sets ATTN_DEVERR_TIMEOUT in
 * the status word and returns: no trap, and the context stays usable.
 * attn_get_status on the same workspace then returns ATTN_ERR_DEVICE with
 * that bit. workspace: device memory owned by the caller, 256-byte aligned,
 * at least 256 bytes. Returns ATTN_ERR_WORKSPACE for a missing, misaligned
 * or smaller workspace, ATTN_ERR_CUDA when the clear or the launch fails,
 * otherwise ATTN_OK once the work is enqueued. */
attn_status attn_selftest_wait_timeout(void* workspace, size_t workspace_bytes, void* stream);

/* Static, human-readable text for a status code. */
const char* attn_status_string(attn_status status);

/* ATTN_VERSION of the built library. */
int attn_version(void);

#ifdef __cplusplus
}
#endif

#endif /* ATTN_H_ */
