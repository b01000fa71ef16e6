// C ABI of the library: argument validation, workspace layout and dispatch.
// Every check happens on the host before the first launch; device-detected
// conditions go to the status word at workspace offset 0.
#include <math.h>
#include <string.h>

#include "common.cuh"
#include "launchers.h"
#include "sm100_dense.h"
#include "sm100_topk.h"

using namespace attn;

namespace {

struct Dense {
  int B, Hq, Hkv, Tq, Tk, d, dv;
};

bool inner_contiguous(const attn_tensor* t) { return t->ndim >= 1 && t->stride[t->ndim - 1] == 1; }

bool valid_dtype(int32_t dt) { return dt == ATTN_F32 || dt == ATTN_BF16 || dt == ATTN_F16; }

// Calls f with a value of the storage type that dt names.
template <class F>
cudaError_t by_storage(int32_t dt, F&& f) {
  if (dt == ATTN_F32) return f(float());
  if (dt == ATTN_F16) return f(__half());
  return f(__nv_bfloat16());
}

bool dims_fit_int(const attn_tensor* t) {
  for (int i = 0; i < t->ndim; ++i)
    if (t->shape[i] < 0 || t->shape[i] > 0x7fffffffLL) return false;
  return true;
}

bool same_shape(const attn_tensor* t, int ndim, const int64_t* shape) {
  if (t->ndim != ndim) return false;
  for (int i = 0; i < ndim; ++i)
    if (t->shape[i] != shape[i]) return false;
  return true;
}

uint32_t flags_of(const attn_mask* m) { return m ? m->flags : 0u; }

// Validate the mask descriptor itself (not the tensors).
attn_status check_mask(const attn_mask* m) {
  if (!m) return ATTN_OK;
  const uint32_t known = ATTN_MASK_CAUSAL | ATTN_MASK_WINDOW | ATTN_MASK_BLOCK | ATTN_MASK_TOPK |
                         ATTN_MASK_LENGTHS | ATTN_MASK_STARTS | ATTN_MASK_TOPK_CHECK_CAUSAL;
  if (m->flags & ~known) return ATTN_ERR_INVALID_ARG;
  if ((m->flags & ATTN_MASK_TOPK_CHECK_CAUSAL) && !(m->flags & ATTN_MASK_TOPK)) return ATTN_ERR_INVALID_ARG;
  if ((m->flags & ATTN_MASK_WINDOW) && m->window_left < 1) return ATTN_ERR_INVALID_ARG;
  if (m->flags & ATTN_MASK_BLOCK) {
    if (!m->block_mask || m->block_q < 1 || m->block_k < 1) return ATTN_ERR_INVALID_ARG;
    if (m->bm_stride_b < 0 || m->bm_stride_h < 0 || m->bm_stride_q < 0) return ATTN_ERR_INVALID_ARG;
  }
  if (m->flags & ATTN_MASK_TOPK) {
    if (!m->topk_idxs || m->topk_max < 0 || m->topk_stride < m->topk_max) return ATTN_ERR_INVALID_ARG;
    if (m->flags & (ATTN_MASK_CAUSAL | ATTN_MASK_WINDOW | ATTN_MASK_BLOCK | ATTN_MASK_LENGTHS | ATTN_MASK_STARTS))
      return ATTN_ERR_UNSUPPORTED;
    if (m->dropout_p != 0.f) return ATTN_ERR_UNSUPPORTED;
  }
  if (m->lse_format & ~(ATTN_LSE_KV_ONLY | ATTN_LSE_NEG_LOG2)) return ATTN_ERR_INVALID_ARG;
  if (m->bwd_flags & ~ATTN_BWD_DETERMINISTIC) return ATTN_ERR_INVALID_ARG;
  if ((m->flags & ATTN_MASK_LENGTHS) && !m->lengths) return ATTN_ERR_INVALID_ARG;
  if ((m->flags & ATTN_MASK_STARTS) && (!m->starts || m->starts_stride_b < 0)) return ATTN_ERR_INVALID_ARG;
  if (!(m->dropout_p >= 0.f && m->dropout_p < 1.f)) return ATTN_ERR_INVALID_ARG;
  return ATTN_OK;
}

MaskP mask_params(const attn_mask* m) {
  MaskP p;
  memset(&p, 0, sizeof(p));
  if (!m) return p;
  p.flags = m->flags & (ATTN_MASK_CAUSAL | ATTN_MASK_WINDOW | ATTN_MASK_BLOCK | ATTN_MASK_LENGTHS | ATTN_MASK_STARTS);
  p.lengths = (m->flags & ATTN_MASK_LENGTHS) ? m->lengths : nullptr;
  p.starts = (m->flags & ATTN_MASK_STARTS) ? m->starts : nullptr;
  p.st_sb = m->starts_stride_b;
  p.lse_fmt = m->lse_format;
  p.window = m->window_left;
  p.bm = m->block_mask;
  p.bq = m->block_q;
  p.bk = m->block_k;
  p.bm_sb = m->bm_stride_b;
  p.bm_sh = m->bm_stride_h;
  p.bm_sq = m->bm_stride_q;
  p.sink = m->sink;
  if (m->dropout_p > 0.f) {
    p.dropout = 1;
    const double thr = floor((double)m->dropout_p * 4294967296.0);
    p.keep_thr = thr >= 4294967295.0 ? 0xffffffffu : (uint32_t)thr;
    p.inv_keep = (float)(1.0 / (1.0 - (double)m->dropout_p));
    p.seed_lo = (uint32_t)(m->dropout_seed & 0xffffffffu);
    p.seed_hi = (uint32_t)(m->dropout_seed >> 32);
  }
  return p;
}

// Dense layout checks shared by fwd and bwd.
attn_status check_dense(const attn_tensor* q, const attn_tensor* k, const attn_tensor* v, Dense& s) {
  if (!q || !k || !v) return ATTN_ERR_INVALID_ARG;
  if (q->ndim != 4 || k->ndim != 4 || v->ndim != 4) return ATTN_ERR_INVALID_ARG;
  if (!dims_fit_int(q) || !dims_fit_int(k) || !dims_fit_int(v)) return ATTN_ERR_INVALID_ARG;
  s.B = (int)q->shape[0];
  s.Hq = (int)q->shape[1];
  s.Tq = (int)q->shape[2];
  s.Tk = (int)k->shape[2];
  s.d = (int)q->shape[3];
  s.Hkv = (int)k->shape[1];
  s.dv = (int)v->shape[3];
  if (k->shape[0] != s.B || v->shape[0] != s.B || v->shape[2] != s.Tk) return ATTN_ERR_INVALID_ARG;
  if (k->shape[3] != s.d || v->shape[1] != s.Hkv) return ATTN_ERR_INVALID_ARG;
  if (s.Hq < 1 || s.Hkv < 1 || s.Hq % s.Hkv != 0) return ATTN_ERR_INVALID_ARG;
  if (s.d < 1 || s.dv < 1) return ATTN_ERR_INVALID_ARG;
  if (s.d > 576 || s.dv > 576) return ATTN_ERR_UNSUPPORTED;
  if (!q->data || !k->data || !v->data) return (s.B && s.Tq && s.Tk) ? ATTN_ERR_INVALID_ARG : ATTN_OK;
  if (!inner_contiguous(q) || !inner_contiguous(k) || !inner_contiguous(v)) return ATTN_ERR_INVALID_ARG;
  if (!valid_dtype(q->dtype) || k->dtype != q->dtype || v->dtype != q->dtype) return ATTN_ERR_INVALID_ARG;
  return ATTN_OK;
}

struct Topk {
  int Tq, Tkv, H, Dqk, Dv;
};

attn_status check_topk(const attn_tensor* q, const attn_tensor* k, const attn_tensor* v, Topk& s) {
  if (!q || !k || !v) return ATTN_ERR_INVALID_ARG;
  if (q->ndim != 3 || k->ndim != 2 || v->ndim != 2) return ATTN_ERR_INVALID_ARG;
  if (!dims_fit_int(q) || !dims_fit_int(k) || !dims_fit_int(v)) return ATTN_ERR_INVALID_ARG;
  s.Tq = (int)q->shape[0];
  s.H = (int)q->shape[1];
  s.Dqk = (int)q->shape[2];
  s.Tkv = (int)k->shape[0];
  s.Dv = (int)v->shape[1];
  if (k->shape[1] != s.Dqk || v->shape[0] != s.Tkv) return ATTN_ERR_INVALID_ARG;
  if (s.Dv < 1 || s.Dv > s.Dqk || s.H < 1) return ATTN_ERR_INVALID_ARG;
  if (s.Dqk > 576) return ATTN_ERR_UNSUPPORTED;
  // Shared KV: V is the first Dv columns of the same rows.
  if (v->data != k->data || v->stride[0] != k->stride[0]) return ATTN_ERR_INVALID_ARG;
  if (!inner_contiguous(q) || !inner_contiguous(k) || !inner_contiguous(v)) return ATTN_ERR_INVALID_ARG;
  if (!valid_dtype(q->dtype) || k->dtype != q->dtype || v->dtype != q->dtype) return ATTN_ERR_INVALID_ARG;
  if ((s.Tq && !q->data) || (s.Tkv && !k->data)) return ATTN_ERR_INVALID_ARG;
  return ATTN_OK;
}

attn_status cuda_status(cudaError_t e) { return e == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA; }

attn_status check_workspace(void* ws, size_t have, size_t need) {
  if (!ws || have < need) return ATTN_ERR_WORKSPACE;
  if (reinterpret_cast<uintptr_t>(ws) % 256 != 0) return ATTN_ERR_WORKSPACE;
  return ATTN_OK;
}

size_t bwd_dense_bytes(const Dense& s) {
  const size_t rows = (size_t)s.B * s.Hq * s.Tq;
  size_t n = kStatusBytes;
  n += align_up(rows * sizeof(float), 256);                       // delta
  n += align_up(rows * (size_t)s.d * sizeof(float), 256);         // dQ accumulator
  return n;
}

uint32_t lse_format_of(const attn_mask* m) { return m ? m->lse_format : 0u; }

// Room for the reverse pass's natural-log, sink-inclusive copy of an LSE
// given in another format (rows = the LSE's element count).
size_t lse_copy_bytes(const attn_mask* m, size_t rows) {
  return lse_format_of(m) ? align_up(rows * sizeof(float), 256) : 0;
}

size_t bwd_topk_bytes(const Topk& s, const attn_tensor* q, const attn_mask* m) {
  size_t n = kStatusBytes;
  n += align_up((size_t)s.Tq * s.H * sizeof(float), 256);                       // delta
  n += topk_acc_total_bytes(s.Tkv, s.Dqk);  // 32.32 dKV, counts, bound (or, in its first half, an fp32 dKV)
  if (q->dtype != ATTN_F32)                                                     // G, P rows (tensor-core path)
    n += align_up(attn::sm100_topk_bwd_scratch_bytes(s.Tq, s.H, s.Dqk, s.Dv, m->topk_max), 256);
  return n + lse_copy_bytes(m, (size_t)s.Tq * s.H);
}

}  // namespace

namespace attn {

namespace {
thread_local cudaEvent_t g_kernel_ev[2] = {nullptr, nullptr};
}  // namespace

void main_kernel_begin(cudaStream_t st) {
  if (g_kernel_ev[0]) cudaEventRecord(g_kernel_ev[0], st);
}

void main_kernel_end(cudaStream_t st) {
  if (g_kernel_ev[1]) cudaEventRecord(g_kernel_ev[1], st);
  g_kernel_ev[0] = g_kernel_ev[1] = nullptr;
}

// A pending event pair applies to one call only, whichever way it returns.
struct ForgetKernelEvents {
  ~ForgetKernelEvents() { g_kernel_ev[0] = g_kernel_ev[1] = nullptr; }
};

}  // namespace attn

#pragma GCC visibility push(default)
extern "C" {

attn_status attn_set_kernel_events(void* begin, void* end) {
  attn::g_kernel_ev[0] = static_cast<cudaEvent_t>(begin);
  attn::g_kernel_ev[1] = static_cast<cudaEvent_t>(end);
  return ATTN_OK;
}

int attn_version(void) { return ATTN_VERSION; }

const char* attn_status_string(attn_status status) {
  switch (status) {
    case ATTN_OK: return "ok";
    case ATTN_ERR_INVALID_ARG: return "invalid argument (shape, stride, dtype, alignment or pointer)";
    case ATTN_ERR_UNSUPPORTED: return "unsupported combination (no kernel for this request)";
    case ATTN_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
    case ATTN_ERR_CUDA: return "a CUDA call failed";
    case ATTN_ERR_DEVICE: return "the device recorded an error (see attn_get_status bits)";
  }
  return "unknown status";
}

size_t attn_fwd_workspace_size(const attn_tensor* q, const attn_tensor* k, const attn_tensor* v,
                               const attn_mask* mask) {
  (void)mask;
  size_t n = kStatusBytes;
  if (!(flags_of(mask) & ATTN_MASK_TOPK)) {
    Dense s;
    if (check_dense(q, k, v, s) == ATTN_OK) n += sm100_fwd_workspace_bytes(s.B, s.Hq, s.Tq, s.Tk, mask);
  }
  return n;
}

size_t attn_bwd_workspace_size(const attn_tensor* q, const attn_tensor* k, const attn_tensor* v,
                               const attn_mask* mask) {
  if (flags_of(mask) & ATTN_MASK_TOPK) {
    Topk s;
    if (check_topk(q, k, v, s) != ATTN_OK) return kStatusBytes;
    return bwd_topk_bytes(s, q, mask);
  }
  Dense s;
  if (check_dense(q, k, v, s) != ATTN_OK) return kStatusBytes;
  return bwd_dense_bytes(s) + sm100_bwd_extra_workspace_bytes(s.B, s.Hq, s.Hkv, s.Tq, s.Tk, mask) +
         lse_copy_bytes(mask, (size_t)s.B * s.Hq * s.Tq);
}

attn_status attn_fwd(const attn_tensor* q, const attn_tensor* k, const attn_tensor* v,
                     const attn_mask* mask, float scale, attn_tensor* o, attn_tensor* lse,
                     void* workspace, size_t workspace_bytes, void* stream) {
  attn::ForgetKernelEvents forget_events;

  attn_status st = check_mask(mask);
  if (st != ATTN_OK) return st;
  if (!o || !lse || !isfinite(scale)) return ATTN_ERR_INVALID_ARG;
  if (lse->dtype != ATTN_F32 || !dims_fit_int(lse) || !dims_fit_int(o)) return ATTN_ERR_INVALID_ARG;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  uint32_t* status = static_cast<uint32_t*>(workspace);

  if (flags_of(mask) & ATTN_MASK_TOPK) {
    Topk s;
    if ((st = check_topk(q, k, v, s)) != ATTN_OK) return st;
    const int64_t os[3] = {s.Tq, s.H, s.Dv}, ls[2] = {s.Tq, s.H};
    if (!same_shape(o, 3, os) || !same_shape(lse, 2, ls) || o->dtype != q->dtype || !inner_contiguous(o))
      return ATTN_ERR_INVALID_ARG;
    if ((st = check_workspace(workspace, workspace_bytes, kStatusBytes)) != ATTN_OK) return st;
    if (cudaMemsetAsync(status, 0, kStatusBytes, cs) != cudaSuccess) return ATTN_ERR_CUDA;
    if ((int64_t)s.Tq * s.H == 0) return ATTN_OK;
    if ((s.Tq && (!o->data || !lse->data))) return ATTN_ERR_INVALID_ARG;
    TopkP p;
    p.q = q->data;
    p.kv = k->data;
    p.sq_t = q->stride[0];
    p.sq_h = q->stride[1];
    p.skv = k->stride[0];
    p.idx = mask->topk_idxs;
    p.idx_stride = mask->topk_stride;
    p.topk_max = mask->topk_max;
    p.len = mask->topk_length;
    p.Tq = s.Tq;
    p.Tkv = s.Tkv;
    p.H = s.H;
    p.Dqk = s.Dqk;
    p.Dv = s.Dv;
    p.dtype = q->dtype;
    p.scale = scale;
    p.sink = mask->sink;
    p.lse_fmt = mask->lse_format;
    p.check_causal = (mask->flags & ATTN_MASK_TOPK_CHECK_CAUSAL) ? 1 : 0;
    if (sm100_topk_supported(p, q, k, o))
      return cuda_status(sm100_topk_fwd(p, o->data, o->stride[0], o->stride[1], static_cast<float*>(lse->data),
                                        lse->stride[0], lse->stride[1], status, cs));
    main_kernel_begin(cs);
    cudaError_t e = by_storage(q->dtype, [&](auto t) {
      return launch_topk_fwd_rows<decltype(t)>(p, o->data, o->stride[0], o->stride[1],
                                               static_cast<float*>(lse->data), lse->stride[0], lse->stride[1],
                                               status, cs);
    });
    main_kernel_end(cs);
    return cuda_status(e);
  }

  Dense s;
  if ((st = check_dense(q, k, v, s)) != ATTN_OK) return st;
  if ((flags_of(mask) & ATTN_MASK_LENGTHS) && s.Tq != s.Tk) return ATTN_ERR_INVALID_ARG;
  const int64_t os[4] = {s.B, s.Hq, s.Tq, s.dv}, ls[3] = {s.B, s.Hq, s.Tq};
  if (!same_shape(o, 4, os) || !same_shape(lse, 3, ls) || o->dtype != q->dtype || !inner_contiguous(o))
    return ATTN_ERR_INVALID_ARG;
  const size_t need = attn_fwd_workspace_size(q, k, v, mask);
  if ((st = check_workspace(workspace, workspace_bytes, need)) != ATTN_OK) return st;
  if (cudaMemsetAsync(status, 0, kStatusBytes, cs) != cudaSuccess) return ATTN_ERR_CUDA;
  if ((int64_t)s.B * s.Hq * s.Tq == 0) return ATTN_OK;
  if (!o->data || !lse->data) return ATTN_ERR_INVALID_ARG;
  DenseP p;
  p.q = q->data;
  p.k = k->data;
  p.v = v->data;
  for (int i = 0; i < 3; ++i) {
    p.sq[i] = q->stride[i];
    p.sk[i] = k->stride[i];
    p.sv[i] = v->stride[i];
  }
  p.B = s.B;
  p.Hq = s.Hq;
  p.Hkv = s.Hkv;
  p.Tq = s.Tq;
  p.Tk = s.Tk;
  p.d = s.d;
  p.dv = s.dv;
  p.dtype = q->dtype;
  p.bwd_flags = mask ? mask->bwd_flags : 0u;
  p.scale = scale;
  p.m = mask_params(mask);
  p.m.qoff = (int64_t)s.Tk - s.Tq;  // bottom-right alignment of the query rows
  const int64_t so[3] = {o->stride[0], o->stride[1], o->stride[2]};
  const int64_t sl[3] = {lse->stride[0], lse->stride[1], lse->stride[2]};
  float* lsep = static_cast<float*>(lse->data);
  if (sm100_dense_supported(p, q, k, v, o)) {
    return cuda_status(sm100_dense_fwd(p, o->data, so, lsep, sl, static_cast<char*>(workspace) + kStatusBytes,
                                       status, cs));
  }
  main_kernel_begin(cs);
  cudaError_t e = by_storage(q->dtype, [&](auto t) {
    return launch_dense_fwd_rows<decltype(t)>(p, o->data, so, lsep, sl, cs);
  });
  main_kernel_end(cs);
  return cuda_status(e);
}

attn_status attn_bwd(const attn_tensor* q, const attn_tensor* k, const attn_tensor* v, const attn_tensor* o,
                     const attn_tensor* do_, const attn_tensor* lse, const attn_mask* mask, float scale,
                     attn_tensor* dq, attn_tensor* dk, attn_tensor* dv, float* dsink, void* workspace,
                     size_t workspace_bytes, void* stream) {
  attn::ForgetKernelEvents forget_events;

  attn_status st = check_mask(mask);
  if (st != ATTN_OK) return st;
  if (!o || !do_ || !lse || !dq || !dk || !isfinite(scale)) return ATTN_ERR_INVALID_ARG;
  if (lse->dtype != ATTN_F32) return ATTN_ERR_INVALID_ARG;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  uint32_t* status = static_cast<uint32_t*>(workspace);
  char* ws = static_cast<char*>(workspace);
  const bool want_dsink = mask && mask->sink && dsink;

  if (flags_of(mask) & ATTN_MASK_TOPK) {
    Topk s;
    if ((st = check_topk(q, k, v, s)) != ATTN_OK) return st;
    if (dv) return ATTN_ERR_INVALID_ARG;  // tied layout: dKV arrives in dk
    const int64_t os[3] = {s.Tq, s.H, s.Dv}, ls[2] = {s.Tq, s.H}, qs[3] = {s.Tq, s.H, s.Dqk},
                  ks[2] = {s.Tkv, s.Dqk};
    if (!same_shape(o, 3, os) || !same_shape(do_, 3, os) || !same_shape(lse, 2, ls) || !same_shape(dq, 3, qs) ||
        !same_shape(dk, 2, ks))
      return ATTN_ERR_INVALID_ARG;
    if (o->dtype != q->dtype || do_->dtype != q->dtype || dq->dtype != q->dtype || dk->dtype != q->dtype)
      return ATTN_ERR_INVALID_ARG;
    if (!inner_contiguous(o) || !inner_contiguous(do_) || !inner_contiguous(dq) || !inner_contiguous(dk))
      return ATTN_ERR_INVALID_ARG;
    if ((st = check_workspace(workspace, workspace_bytes, bwd_topk_bytes(s, q, mask))) != ATTN_OK) return st;
    if (cudaMemsetAsync(status, 0, kStatusBytes, cs) != cudaSuccess) return ATTN_ERR_CUDA;
    float* delta = reinterpret_cast<float*>(ws + kStatusBytes);
    const FixedAcc acc = fixed_acc_at(ws + kStatusBytes + align_up((size_t)s.Tq * s.H * sizeof(float), 256), s.Tkv,
                                      s.Dqk);
    TopkP p;
    p.q = q->data;
    p.kv = k->data;
    p.sq_t = q->stride[0];
    p.sq_h = q->stride[1];
    p.skv = k->stride[0];
    p.idx = mask->topk_idxs;
    p.idx_stride = mask->topk_stride;
    p.topk_max = mask->topk_max;
    p.len = mask->topk_length;
    p.Tq = s.Tq;
    p.Tkv = s.Tkv;
    p.H = s.H;
    p.Dqk = s.Dqk;
    p.Dv = s.Dv;
    p.dtype = q->dtype;
    p.scale = scale;
    p.sink = mask->sink;
    p.lse_fmt = mask->lse_format;
    p.check_causal = (mask->flags & ATTN_MASK_TOPK_CHECK_CAUSAL) ? 1 : 0;
    const int64_t so[3] = {0, o->stride[0], o->stride[1]}, sg[3] = {0, do_->stride[0], do_->stride[1]};
    cudaError_t e = cudaSuccess;
    const float* lsep = static_cast<const float*>(lse->data);
    int64_t lst = lse->stride[0], lsh = lse->stride[1];
    if (p.lse_fmt) {  // the reverse kernels read the natural-log, sink-inclusive LSE
      const size_t rows = (size_t)s.Tq * s.H;
      float* conv = reinterpret_cast<float*>(ws + bwd_topk_bytes(s, q, mask) - lse_copy_bytes(mask, rows));
      const int64_t st3[3] = {0, lse->stride[0], lse->stride[1]};
      if ((e = launch_lse_to_total(lsep, 1, s.Tq, s.H, st3, 2, mask->sink, p.lse_fmt, conv, cs)) != cudaSuccess)
        return cuda_status(e);
      lsep = conv;
      lst = s.H;
      lsh = 1;
    }
    if (sm100_topk_bwd_supported(p, q, k, o, do_, dq)) {
      // Tensor cores: dQ and the per-token dKV contributions. The accumulator
      // (fp32, or 32.32 fixed point for a bitwise reproducible dKV) starts at
      // zero and is cast to dKV at the end.
      char* scratch = ws + kStatusBytes + align_up((size_t)s.Tq * s.H * sizeof(float), 256) +
                      topk_acc_total_bytes(s.Tkv, s.Dqk);
      const bool fixed = (mask->bwd_flags & ATTN_BWD_DETERMINISTIC) != 0;
      float* acc32 = fixed ? nullptr : reinterpret_cast<float*>(acc.acc);
      e = by_storage(q->dtype, [&](auto t) {
        using T = decltype(t);
        cudaError_t r = launch_rows_delta<T>(o->data, do_->data, 1, s.Tq, s.H, so, sg, s.Dv, delta, cs);
        if (r == cudaSuccess)
          r = cudaMemsetAsync(acc.acc, 0,
                              fixed ? topk_acc_total_bytes(s.Tkv, s.Dqk) : (size_t)s.Tkv * s.Dqk * sizeof(float), cs);
        if (r == cudaSuccess)
          r = sm100_topk_bwd(p, do_->data, do_->stride[0], do_->stride[1], lsep, lst, lsh, delta, dq->data,
                             dq->stride[0], dq->stride[1], acc, acc32, scratch, status, cs);
        if (r == cudaSuccess)
          r = fixed ? launch_fixed_to_out<T>(acc, s.Tkv, s.Dqk, dk->data, dk->stride[0], status, cs)
                    : launch_f32_to_out<T>(acc32, s.Tkv, s.Dqk, dk->data, dk->stride[0], cs);
        return r;
      });
    } else {
      e = by_storage(q->dtype, [&](auto t) {
        using T = decltype(t);
        cudaError_t r = launch_rows_delta<T>(o->data, do_->data, 1, s.Tq, s.H, so, sg, s.Dv, delta, cs);
        main_kernel_begin(cs);
        if (r == cudaSuccess)
          r = launch_topk_bwd_rows<T>(p, do_->data, do_->stride[0], do_->stride[1], lsep, lst, lsh, delta,
                                      dq->data, dq->stride[0], dq->stride[1], acc, dk->data, dk->stride[0],
                                      status, cs);
        main_kernel_end(cs);
        return r;
      });
    }
    if (e == cudaSuccess && want_dsink)
      e = launch_dsink(mask->sink, lsep, delta, s.Tq, s.H, 1, lst, lsh, 0, false, dsink, cs);
    return cuda_status(e);
  }

  Dense s;
  if ((st = check_dense(q, k, v, s)) != ATTN_OK) return st;
  if ((flags_of(mask) & ATTN_MASK_LENGTHS) && s.Tq != s.Tk) return ATTN_ERR_INVALID_ARG;
  if (!dv) return ATTN_ERR_INVALID_ARG;
  const int64_t os[4] = {s.B, s.Hq, s.Tq, s.dv}, ls[3] = {s.B, s.Hq, s.Tq}, qs[4] = {s.B, s.Hq, s.Tq, s.d},
                ks[4] = {s.B, s.Hkv, s.Tk, s.d}, vs[4] = {s.B, s.Hkv, s.Tk, s.dv};
  if (!same_shape(o, 4, os) || !same_shape(do_, 4, os) || !same_shape(lse, 3, ls) || !same_shape(dq, 4, qs) ||
      !same_shape(dk, 4, ks) || !same_shape(dv, 4, vs))
    return ATTN_ERR_INVALID_ARG;
  const attn_tensor* all[5] = {o, do_, dq, dk, dv};
  for (const attn_tensor* t : all)
    if (t->dtype != q->dtype || !inner_contiguous(t)) return ATTN_ERR_INVALID_ARG;
  const size_t need = attn_bwd_workspace_size(q, k, v, mask);
  if ((st = check_workspace(workspace, workspace_bytes, need)) != ATTN_OK) return st;
  if (cudaMemsetAsync(status, 0, kStatusBytes, cs) != cudaSuccess) return ATTN_ERR_CUDA;
  if ((int64_t)s.B * s.Hq * s.Tq == 0) return ATTN_OK;
  float* delta = reinterpret_cast<float*>(ws + kStatusBytes);
  const size_t rows = (size_t)s.B * s.Hq * s.Tq;
  float* dq_acc = reinterpret_cast<float*>(ws + kStatusBytes + align_up(rows * sizeof(float), 256));
  char* extra = ws + bwd_dense_bytes(s);
  DenseP p;
  p.q = q->data;
  p.k = k->data;
  p.v = v->data;
  for (int i = 0; i < 3; ++i) {
    p.sq[i] = q->stride[i];
    p.sk[i] = k->stride[i];
    p.sv[i] = v->stride[i];
  }
  p.B = s.B;
  p.Hq = s.Hq;
  p.Hkv = s.Hkv;
  p.Tq = s.Tq;
  p.Tk = s.Tk;
  p.d = s.d;
  p.dv = s.dv;
  p.dtype = q->dtype;
  p.bwd_flags = mask ? mask->bwd_flags : 0u;
  p.scale = scale;
  p.m = mask_params(mask);
  p.m.qoff = (int64_t)s.Tk - s.Tq;  // bottom-right alignment of the query rows
  const int64_t so[3] = {o->stride[0], o->stride[1], o->stride[2]};
  const int64_t sg[3] = {do_->stride[0], do_->stride[1], do_->stride[2]};
  int64_t sl[3] = {lse->stride[0], lse->stride[1], lse->stride[2]};
  const int64_t sdq[3] = {dq->stride[0], dq->stride[1], dq->stride[2]};
  const int64_t sdk[3] = {dk->stride[0], dk->stride[1], dk->stride[2]};
  const int64_t sdv[3] = {dv->stride[0], dv->stride[1], dv->stride[2]};
  const float* lsep = static_cast<const float*>(lse->data);
  cudaError_t e;
  if (p.m.lse_fmt) {  // the reverse kernels read the natural-log, sink-inclusive LSE
    float* conv = reinterpret_cast<float*>(ws + need - lse_copy_bytes(mask, rows));
    if ((e = launch_lse_to_total(lsep, s.B, s.Hq, s.Tq, sl, 1, mask->sink, p.m.lse_fmt, conv, cs)) != cudaSuccess)
      return cuda_status(e);
    lsep = conv;
    sl[0] = (int64_t)s.Hq * s.Tq;
    sl[1] = s.Tq;
    sl[2] = 1;
  }
  if (sm100_dense_supported(p, q, k, v, o) && sm100_dense_bwd_supported(p, do_, dq, dk, dv)) {
    e = sm100_dense_bwd(p, o->data, so, do_->data, sg, lsep, sl, delta, dq_acc, dq->data, sdq, dk->data, sdk,
                        dv->data, sdv, extra, status, cs);
  } else {
    e = by_storage(q->dtype, [&](auto t) {
      using T = decltype(t);
      cudaError_t r = launch_rows_delta<T>(o->data, do_->data, s.B, s.Hq, s.Tq, so, sg, s.dv, delta, cs);
      main_kernel_begin(cs);
      if (r == cudaSuccess)
        r = launch_dense_bwd_rows<T>(p, do_->data, sg, lsep, sl, delta, dq->data, sdq, dk->data, sdk, dv->data,
                                     sdv, cs);
      main_kernel_end(cs);
      return r;
    });
  }
  if (e == cudaSuccess && want_dsink)
    e = launch_dsink(mask->sink, lsep, delta, s.B, s.Hq, s.Tq, sl[0], sl[1], sl[2], true, dsink, cs);
  return cuda_status(e);
}

attn_status attn_selftest_wait_timeout(void* workspace, size_t workspace_bytes, void* stream) {
  attn_status st;
  if ((st = check_workspace(workspace, workspace_bytes, kStatusBytes)) != ATTN_OK) return st;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  uint32_t* status = static_cast<uint32_t*>(workspace);
  if (cudaMemsetAsync(status, 0, kStatusBytes, cs) != cudaSuccess) return ATTN_ERR_CUDA;
  return cuda_status(launch_wait_timeout_probe(status, cs));
}

attn_status attn_get_status(void* workspace, void* stream, uint32_t* device_bits) {
  if (!device_bits) return ATTN_ERR_INVALID_ARG;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  if (!workspace) {  // the status word of attn_bwd_noalloc's array on the current device
    attn_status st;
    if (!(workspace = attn::noalloc_status_word(cs, &st))) return st;
  }
  if (cudaStreamSynchronize(cs) != cudaSuccess) return ATTN_ERR_CUDA;
  uint32_t bits = 0;
  if (cudaMemcpy(&bits, workspace, sizeof(bits), cudaMemcpyDeviceToHost) != cudaSuccess) return ATTN_ERR_CUDA;
  if (cudaMemset(workspace, 0, sizeof(bits)) != cudaSuccess) return ATTN_ERR_CUDA;
  *device_bits = bits;
  return bits ? ATTN_ERR_DEVICE : ATTN_OK;
}

}  // extern "C"
#pragma GCC visibility pop
