// Row-wise kernels: one warp owns one query row (forward, dQ) or one key row
// (dK/dV). They cover every dtype, head width (<= 576), allowed-set kind,
// sink and dropout, and are the path for fp32 inputs and for shapes the
// tensor-core kernels do not take. Per key the warp forms the score with a
// lane-split dot product and a shuffle reduction, then applies the running
// summary update of "Accumulate attention without keeping the full grid",
// section "Rescale earlier mass before adding a new tile", one key at a time
// (a key block of size 1, which the exactness proof allows).
#include <math.h>

#include "common.cuh"
#include "launchers.h"

namespace attn {

namespace {

constexpr int kWarps = 8;  // warps per block

template <typename T, int N>
__device__ __forceinline__ void load_row(const T* row, int n, int lane, float (&r)[N]) {
#pragma unroll
  for (int c = 0; c < N; ++c) {
    const int idx = lane + 32 * c;
    r[c] = idx < n ? ld(row + idx) : 0.f;
  }
}

template <int N>
__device__ __forceinline__ float dot_lanes(const float (&a)[N], const float (&b)[N]) {
  float s = 0.f;
#pragma unroll
  for (int c = 0; c < N; ++c) s = fmaf(a[c], b[c], s);
  return warp_sum(s);
}

// Finalise a row: fold the sink into the summary and write Y, LSE.
template <typename T, int NV>
__device__ __forceinline__ void finish_row(float m, float l, float (&acc)[NV], float z, bool has_sink,
                                           T* orow, int dv, int lane, float* lse_out, uint32_t lse_fmt) {
  float lse;
  float scale_o;
  if (m == -INFINITY) {  // A_i empty: Y = 0, LSE = -inf or z
    lse = has_sink ? z : -INFINITY;
    scale_o = 0.f;
  } else {
    float M = has_sink ? fmaxf(m, z) : m;
    float tot = l * expf(m - M) + (has_sink ? expf(z - M) : 0.f);
    scale_o = expf(m - M) / tot;
    lse = M + logf(tot);
  }
#pragma unroll
  for (int c = 0; c < NV; ++c) {
    const int idx = lane + 32 * c;
    if (idx < dv) st(orow + idx, acc[c] * scale_o);
  }
  if (lane == 0) *lse_out = stored_lse_ln(lse_fmt, lse, m, l);
}

template <typename T, int NQ, int NV>
__global__ void __launch_bounds__(kWarps * 32)
dense_fwd_rows(DenseP p, T* o, int64_t so0, int64_t so1, int64_t so2, float* lse, int64_t sl0,
               int64_t sl1, int64_t sl2) {
  const int64_t warp = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (warp >= (int64_t)p.B * p.Hq * p.Tq) return;
  const int i = (int)(warp % p.Tq);
  const int h = (int)((warp / p.Tq) % p.Hq);
  const int b = (int)(warp / ((int64_t)p.Tq * p.Hq));
  const int kvh = h / (p.Hq / p.Hkv);
  const T* Q = static_cast<const T*>(p.q) + b * p.sq[0] + h * p.sq[1] + (int64_t)i * p.sq[2];
  const T* Kb = static_cast<const T*>(p.k) + b * p.sk[0] + kvh * p.sk[1];
  const T* Vb = static_cast<const T*>(p.v) + b * p.sv[0] + kvh * p.sv[1];
  float q[NQ], acc[NV];
  load_row(Q, p.d, lane, q);
#pragma unroll
  for (int c = 0; c < NV; ++c) acc[c] = 0.f;
  float m = -INFINITY, l = 0.f;
  int64_t lo, hi;
  key_range(p.m, b, i, p.Tk, lo, hi);
  for (int64_t j = lo; j <= hi; ++j) {
    if (!allowed(p.m, b, h, i, j)) continue;  // empty keys leave the state untouched
    float kr[NQ];
    load_row(Kb + j * p.sk[2], p.d, lane, kr);
    const float s = dot_lanes(q, kr) * p.scale;
    const float mn = fmaxf(m, s);
    const float alpha = expf(m - mn);  // 0 for the first contributing key
    const float e = expf(s - mn);
    l = l * alpha + e;
    float w = e;
    if (p.m.dropout) w = dropout_keep(p.m, b, h, i, j) ? e * p.m.inv_keep : 0.f;
    const T* vr = Vb + j * p.sv[2];
#pragma unroll
    for (int c = 0; c < NV; ++c) {
      const int idx = lane + 32 * c;
      const float vv = idx < p.dv ? ld(vr + idx) : 0.f;
      acc[c] = fmaf(w, vv, acc[c] * alpha);
    }
    m = mn;
  }
  const bool has_sink = p.m.sink != nullptr;
  const float z = has_sink ? p.m.sink[h] : -INFINITY;
  finish_row<T, NV>(m, l, acc, z, has_sink, o + b * so0 + h * so1 + (int64_t)i * so2, p.dv, lane,
                    lse + b * sl0 + h * sl1 + (int64_t)i * sl2, p.m.lse_fmt);
}

template <typename T, int NQ, int NV>
__global__ void __launch_bounds__(kWarps * 32)
topk_fwd_rows(TopkP p, T* o, int64_t so_t, int64_t so_h, float* lse, int64_t sl_t, int64_t sl_h,
              uint32_t* status) {
  const int64_t warp = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (warp >= (int64_t)p.Tq * p.H) return;
  const int h = (int)(warp % p.H);
  const int t = (int)(warp / p.H);
  const T* Q = static_cast<const T*>(p.q) + (int64_t)t * p.sq_t + (int64_t)h * p.sq_h;
  const T* KV = static_cast<const T*>(p.kv);
  float q[NQ], acc[NV];
  load_row(Q, p.Dqk, lane, q);
#pragma unroll
  for (int c = 0; c < NV; ++c) acc[c] = 0.f;
  float m = -INFINITY, l = 0.f;
  const int n = p.len ? min(p.len[t], p.topk_max) : p.topk_max;
  const int32_t* list = p.idx + (int64_t)t * p.idx_stride;
  for (int pos = 0; pos < n; ++pos) {
    const int j = list[pos];
    if (j < 0 || j >= p.Tkv) {
      if (lane == 0) set_status(status, ATTN_DEVERR_TOPK_INDEX);
      continue;
    }
    if (lane == 0) check_topk_causal(p.check_causal, j, t, p.Tq, p.Tkv, status);
    const T* row = KV + (int64_t)j * p.skv;
    float kr[NQ];
    load_row(row, p.Dqk, lane, kr);
    const float s = dot_lanes(q, kr) * p.scale;
    const float mn = fmaxf(m, s);
    const float alpha = expf(m - mn);
    const float e = expf(s - mn);
    l = l * alpha + e;
#pragma unroll
    for (int c = 0; c < NV; ++c) {
      const int idx = lane + 32 * c;
      const float vv = idx < p.Dv ? ld(row + idx) : 0.f;
      acc[c] = fmaf(e, vv, acc[c] * alpha);
    }
    m = mn;
  }
  const bool has_sink = p.sink != nullptr;
  const float z = has_sink ? p.sink[h] : -INFINITY;
  finish_row<T, NV>(m, l, acc, z, has_sink, o + (int64_t)t * so_t + (int64_t)h * so_h, p.Dv, lane,
                    lse + (int64_t)t * sl_t + (int64_t)h * sl_h, p.lse_fmt);
}

// delta_i = <G_i, Y_i> from the stored output, one warp per row. Rows are
// enumerated as (mid, inner) with element offsets mid*s1 + inner*s2; the
// caller folds the outermost dimension.
template <typename T, int NV>
__global__ void __launch_bounds__(kWarps * 32)
rows_delta(const T* o, const T* g, int64_t rows, int inner, int64_t so1, int64_t so2, int64_t sg1,
           int64_t sg2, int dv, float* delta) {
  const int64_t warp = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (warp >= rows) return;
  const int64_t c = warp % inner;
  const int64_t ab = warp / inner;
  float a[NV], bb[NV];
  load_row(o + ab * so1 + c * so2, dv, lane, a);
  load_row(g + ab * sg1 + c * sg2, dv, lane, bb);
  const float s = dot_lanes(a, bb);
  if (lane == 0) delta[warp] = s;
}

template <typename T, int NQ, int NV>
__global__ void __launch_bounds__(kWarps * 32)
dense_dq_rows(DenseP p, const T* g, int64_t sg0, int64_t sg1, int64_t sg2, const float* lse,
              int64_t sl0, int64_t sl1, int64_t sl2, const float* delta, T* dq, int64_t sd0,
              int64_t sd1, int64_t sd2) {
  const int64_t warp = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (warp >= (int64_t)p.B * p.Hq * p.Tq) return;
  const int i = (int)(warp % p.Tq);
  const int h = (int)((warp / p.Tq) % p.Hq);
  const int b = (int)(warp / ((int64_t)p.Tq * p.Hq));
  const int kvh = h / (p.Hq / p.Hkv);
  const T* Kb = static_cast<const T*>(p.k) + b * p.sk[0] + kvh * p.sk[1];
  const T* Vb = static_cast<const T*>(p.v) + b * p.sv[0] + kvh * p.sv[1];
  float q[NQ], gr[NV], acc[NQ];
  load_row(static_cast<const T*>(p.q) + b * p.sq[0] + h * p.sq[1] + (int64_t)i * p.sq[2], p.d, lane, q);
  load_row(g + b * sg0 + h * sg1 + (int64_t)i * sg2, p.dv, lane, gr);
#pragma unroll
  for (int c = 0; c < NQ; ++c) acc[c] = 0.f;
  const float L = lse[b * sl0 + h * sl1 + (int64_t)i * sl2];
  const float dl = delta[warp];
  if (L != -INFINITY) {
    int64_t lo, hi;
    key_range(p.m, b, i, p.Tk, lo, hi);
    for (int64_t j = lo; j <= hi; ++j) {
      if (!allowed(p.m, b, h, i, j)) continue;
      float kr[NQ], vr[NV];
      load_row(Kb + j * p.sk[2], p.d, lane, kr);
      load_row(Vb + j * p.sv[2], p.dv, lane, vr);
      const float s = dot_lanes(q, kr) * p.scale;
      const float pij = expf(s - L);
      float dp = dot_lanes(gr, vr);
      if (p.m.dropout) dp = dropout_keep(p.m, b, h, i, j) ? dp * p.m.inv_keep : 0.f;
      const float gam = pij * (dp - dl);
#pragma unroll
      for (int c = 0; c < NQ; ++c) acc[c] = fmaf(gam, kr[c], acc[c]);
    }
  }
  T* out = dq + b * sd0 + h * sd1 + (int64_t)i * sd2;
#pragma unroll
  for (int c = 0; c < NQ; ++c) {
    const int idx = lane + 32 * c;
    if (idx < p.d) st(out + idx, acc[c] * p.scale);
  }
}

// One warp per (b, kv head, key j): dK_j and dV_j summed over every query head
// of the group and every query row that allows j, in a fixed order.
template <typename T, int NQ, int NV>
__global__ void __launch_bounds__(kWarps * 32)
dense_dkv_rows(DenseP p, const T* g, int64_t sg0, int64_t sg1, int64_t sg2, const float* lse,
               int64_t sl0, int64_t sl1, int64_t sl2, const float* delta, T* dk, int64_t sdk0,
               int64_t sdk1, int64_t sdk2, T* dvp, int64_t sdv0, int64_t sdv1, int64_t sdv2) {
  const int64_t warp = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (warp >= (int64_t)p.B * p.Hkv * p.Tk) return;
  const int j = (int)(warp % p.Tk);
  const int kvh = (int)((warp / p.Tk) % p.Hkv);
  const int b = (int)(warp / ((int64_t)p.Tk * p.Hkv));
  const int group = p.Hq / p.Hkv;
  float kr[NQ], vr[NV], ak[NQ], av[NV];
  load_row(static_cast<const T*>(p.k) + b * p.sk[0] + kvh * p.sk[1] + (int64_t)j * p.sk[2], p.d, lane, kr);
  load_row(static_cast<const T*>(p.v) + b * p.sv[0] + kvh * p.sv[1] + (int64_t)j * p.sv[2], p.dv, lane, vr);
#pragma unroll
  for (int c = 0; c < NQ; ++c) ak[c] = 0.f;
#pragma unroll
  for (int c = 0; c < NV; ++c) av[c] = 0.f;
  int64_t lo, hi;
  query_range(p.m, b, j, p.Tq, lo, hi);
  for (int hh = 0; hh < group; ++hh) {
    const int h = kvh * group + hh;
    const T* Qb = static_cast<const T*>(p.q) + b * p.sq[0] + h * p.sq[1];
    const T* Gb = g + b * sg0 + h * sg1;
    for (int64_t i = lo; i <= hi; ++i) {
      if (!allowed(p.m, b, h, i, j)) continue;
      const float L = lse[b * sl0 + h * sl1 + i * sl2];
      if (L == -INFINITY) continue;
      float q[NQ], gr[NV];
      load_row(Qb + i * p.sq[2], p.d, lane, q);
      load_row(Gb + i * sg2, p.dv, lane, gr);
      const float s = dot_lanes(q, kr) * p.scale;
      const float pij = expf(s - L);
      float dp = dot_lanes(gr, vr);
      float pt = pij;
      if (p.m.dropout) {
        const bool keep = dropout_keep(p.m, b, h, i, j);
        dp = keep ? dp * p.m.inv_keep : 0.f;
        pt = keep ? pij * p.m.inv_keep : 0.f;
      }
      const float gam = pij * (dp - delta[((int64_t)b * p.Hq + h) * p.Tq + i]);
#pragma unroll
      for (int c = 0; c < NQ; ++c) ak[c] = fmaf(gam, q[c], ak[c]);
#pragma unroll
      for (int c = 0; c < NV; ++c) av[c] = fmaf(pt, gr[c], av[c]);
    }
  }
  T* ok = dk + b * sdk0 + kvh * sdk1 + (int64_t)j * sdk2;
  T* ov = dvp + b * sdv0 + kvh * sdv1 + (int64_t)j * sdv2;
#pragma unroll
  for (int c = 0; c < NQ; ++c) {
    const int idx = lane + 32 * c;
    if (idx < p.d) st(ok + idx, ak[c] * p.scale);
  }
#pragma unroll
  for (int c = 0; c < NV; ++c) {
    const int idx = lane + 32 * c;
    if (idx < p.dv) st(ov + idx, av[c]);
  }
}

template <typename T, int NQ, int NV>
__global__ void __launch_bounds__(kWarps * 32)
topk_dq_rows(TopkP p, const T* g, int64_t sg_t, int64_t sg_h, const float* lse, int64_t sl_t,
             int64_t sl_h, const float* delta, T* dq, int64_t sd_t, int64_t sd_h) {
  const int64_t warp = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (warp >= (int64_t)p.Tq * p.H) return;
  const int h = (int)(warp % p.H);
  const int t = (int)(warp / p.H);
  const T* KV = static_cast<const T*>(p.kv);
  float q[NQ], gr[NV], acc[NQ];
  load_row(static_cast<const T*>(p.q) + (int64_t)t * p.sq_t + (int64_t)h * p.sq_h, p.Dqk, lane, q);
  load_row(g + (int64_t)t * sg_t + (int64_t)h * sg_h, p.Dv, lane, gr);
#pragma unroll
  for (int c = 0; c < NQ; ++c) acc[c] = 0.f;
  const float L = lse[(int64_t)t * sl_t + (int64_t)h * sl_h];
  const float dl = delta[warp];
  const int n = p.len ? min(p.len[t], p.topk_max) : p.topk_max;
  const int32_t* list = p.idx + (int64_t)t * p.idx_stride;
  if (L != -INFINITY) {
    for (int pos = 0; pos < n; ++pos) {
      const int j = list[pos];
      if (j < 0 || j >= p.Tkv) continue;
      const T* row = KV + (int64_t)j * p.skv;
      float kr[NQ], vr[NV];
      load_row(row, p.Dqk, lane, kr);
      load_row(row, p.Dv, lane, vr);
      const float s = dot_lanes(q, kr) * p.scale;
      const float pij = expf(s - L);
      const float gam = pij * (dot_lanes(gr, vr) - dl);
#pragma unroll
      for (int c = 0; c < NQ; ++c) acc[c] = fmaf(gam, kr[c], acc[c]);
    }
  }
  T* out = dq + (int64_t)t * sd_t + (int64_t)h * sd_h;
#pragma unroll
  for (int c = 0; c < NQ; ++c) {
    const int idx = lane + 32 * c;
    if (idx < p.Dqk) st(out + idx, acc[c] * p.scale);
  }
}

// One warp per (token t, list position): the tied row contribution
// C_j = sum_h (c gamma_thj Q_th + [p_thj G_th, 0]) added into a signed 32.32
// fixed-point accumulator. Integer addition is associative, so the reduced
// dKV does not depend on the order in which warps arrive. The row's
// contribution count and the largest magnitude feed the range check.
template <typename T, int NQ, int NV>
__global__ void __launch_bounds__(kWarps * 32)
topk_dkv_pairs(TopkP p, const T* g, int64_t sg_t, int64_t sg_h, const float* lse, int64_t sl_t,
               int64_t sl_h, const float* delta, FixedAcc fa, uint32_t* status) {
  const int64_t warp = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (warp >= (int64_t)p.Tq * p.topk_max) return;
  const int pos = (int)(warp % p.topk_max);
  const int t = (int)(warp / p.topk_max);
  const int n = p.len ? min(p.len[t], p.topk_max) : p.topk_max;
  if (pos >= n) return;
  const int j = p.idx[(int64_t)t * p.idx_stride + pos];
  if (j < 0 || j >= p.Tkv) {
    if (lane == 0) set_status(status, ATTN_DEVERR_TOPK_INDEX);
    return;
  }
  if (lane == 0) {
    check_topk_causal(p.check_causal, j, t, p.Tq, p.Tkv, status);
    atomicAdd(fa.count + j, 1u);
  }
  const T* row = static_cast<const T*>(p.kv) + (int64_t)j * p.skv;
  float kr[NQ], vr[NV], ak[NQ], av[NV];
  load_row(row, p.Dqk, lane, kr);
  load_row(row, p.Dv, lane, vr);
#pragma unroll
  for (int c = 0; c < NQ; ++c) ak[c] = 0.f;
#pragma unroll
  for (int c = 0; c < NV; ++c) av[c] = 0.f;
  for (int h = 0; h < p.H; ++h) {
    const float L = lse[(int64_t)t * sl_t + (int64_t)h * sl_h];
    if (L == -INFINITY) continue;
    float q[NQ], gr[NV];
    load_row(static_cast<const T*>(p.q) + (int64_t)t * p.sq_t + (int64_t)h * p.sq_h, p.Dqk, lane, q);
    load_row(g + (int64_t)t * sg_t + (int64_t)h * sg_h, p.Dv, lane, gr);
    const float s = dot_lanes(q, kr) * p.scale;
    const float pij = expf(s - L);
    const float gam = pij * (dot_lanes(gr, vr) - delta[(int64_t)t * p.H + h]) * p.scale;
#pragma unroll
    for (int c = 0; c < NQ; ++c) ak[c] = fmaf(gam, q[c], ak[c]);
#pragma unroll
    for (int c = 0; c < NV; ++c) av[c] = fmaf(pij, gr[c], av[c]);
  }
  unsigned long long* dst = fa.acc + (int64_t)j * p.Dqk;
  bool sat = false;
  float amax = 0.f;
#pragma unroll
  for (int c = 0; c < NQ; ++c) {
    const int idx = lane + 32 * c;
    if (idx < p.Dqk) fixed_add(dst + idx, ak[c] + (c < NV && idx < p.Dv ? av[c] : 0.f), sat, amax);
  }
  fixed_publish_max(fa.maxbits, amax);
  if (__any_sync(0xffffffffu, sat) && lane == 0) set_status(status, ATTN_DEVERR_OVERFLOW);
}

// dKV = the fixed-point sums in the output type. The first element of each
// row also checks the row's bound: count * largest contribution < 2^31 means
// no partial order of additions can have left the 32.32 range, so the
// integer sum is exact; otherwise the row may have wrapped and the overflow
// bit is set.
template <typename T>
__global__ void fixed_to_out(FixedAcc fa, int rows, int cols, T* out, int64_t so, uint32_t* status) {
  const int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= (int64_t)rows * cols) return;
  const int r = (int)(e / cols), c = (int)(e % cols);
  if (c == 0 && (double)fa.count[r] * (double)__uint_as_float(*fa.maxbits) >= 2147483648.0)
    set_status(status, ATTN_DEVERR_OVERFLOW);
  const long long v = (long long)fa.acc[e];
  st(out + (int64_t)r * so + c, (float)((double)v * (1.0 / 4294967296.0)));
}

template <typename T>
__global__ void __launch_bounds__(256) f32_to_out(const float* acc, int rows, int cols, T* out, int64_t so) {
  const int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= (int64_t)rows * cols) return;
  const int r = (int)(e / cols), c = (int)(e % cols);
  st(out + (int64_t)r * so + c, acc[e]);
}

// dz_h = -sum over rows of head h of exp(z_h - LSE_row) delta_row, summed in a
// fixed order by one block per head (deterministic).
__global__ void __launch_bounds__(256)
dsink_reduce(const float* sink, const float* lse, const float* delta, int n_outer, int n_heads,
             int n_inner, int64_t sl_outer, int64_t sl_head, int64_t sl_inner, int delta_head_major,
             float* dsink) {
  const int h = blockIdx.x;
  const float z = sink[h];
  float acc = 0.f;
  const int64_t n = (int64_t)n_outer * n_inner;
  for (int64_t r = threadIdx.x; r < n; r += blockDim.x) {
    const int64_t o = r / n_inner, i = r % n_inner;
    const float L = lse[o * sl_outer + h * sl_head + i * sl_inner];
    const int64_t drow = delta_head_major ? (o * n_heads + h) * n_inner + i : (o * n_inner + i) * n_heads + h;
    if (L != -INFINITY) acc += expf(z - L) * delta[drow];
  }
  __shared__ float red[256];
  red[threadIdx.x] = acc;
  __syncthreads();
  for (int s = blockDim.x / 2; s > 0; s >>= 1) {
    if ((int)threadIdx.x < s) red[threadIdx.x] += red[threadIdx.x + s];
    __syncthreads();
  }
  if (threadIdx.x == 0) dsink[h] = -red[0];
}

inline unsigned blocks_for_warps(int64_t warps) { return (unsigned)((warps + kWarps - 1) / kWarps); }

int width_class(int n) { return n <= 32 ? 1 : n <= 64 ? 2 : n <= 128 ? 4 : n <= 256 ? 8 : 18; }

}  // namespace

#define ATTN_DISPATCH_WIDTH(NQV, ...)                         \
  switch (NQV) {                                              \
    case 1: { constexpr int NQ = 1, NV = 1; (void)NQ; (void)NV; __VA_ARGS__ } break;   \
    case 2: { constexpr int NQ = 2, NV = 2; (void)NQ; (void)NV; __VA_ARGS__ } break;   \
    case 4: { constexpr int NQ = 4, NV = 4; (void)NQ; (void)NV; __VA_ARGS__ } break;   \
    case 8: { constexpr int NQ = 8, NV = 8; (void)NQ; (void)NV; __VA_ARGS__ } break;   \
    default: { constexpr int NQ = 18, NV = 18; (void)NQ; (void)NV; __VA_ARGS__ } break; \
  }

template <typename T>
cudaError_t launch_dense_fwd_rows(const DenseP& p, void* o, const int64_t so[3], float* lse,
                                  const int64_t sl[3], cudaStream_t st) {
  const int64_t rows = (int64_t)p.B * p.Hq * p.Tq;
  if (rows == 0) return cudaSuccess;
  const int w = width_class(p.d > p.dv ? p.d : p.dv);
  ATTN_DISPATCH_WIDTH(w, dense_fwd_rows<T, NQ, NV><<<blocks_for_warps(rows), kWarps * 32, 0, st>>>(
                             p, static_cast<T*>(o), so[0], so[1], so[2], lse, sl[0], sl[1], sl[2]);)
  return cudaGetLastError();
}

template <typename T>
cudaError_t launch_topk_fwd_rows(const TopkP& p, void* o, int64_t so_t, int64_t so_h, float* lse,
                                 int64_t sl_t, int64_t sl_h, uint32_t* status, cudaStream_t st) {
  const int64_t rows = (int64_t)p.Tq * p.H;
  if (rows == 0) return cudaSuccess;
  const int w = width_class(p.Dqk > p.Dv ? p.Dqk : p.Dv);
  ATTN_DISPATCH_WIDTH(w, topk_fwd_rows<T, NQ, NV><<<blocks_for_warps(rows), kWarps * 32, 0, st>>>(
                             p, static_cast<T*>(o), so_t, so_h, lse, sl_t, sl_h, status);)
  return cudaGetLastError();
}

template <typename T>
cudaError_t launch_rows_delta(const void* o, const void* g, int64_t n_outer, int64_t n_mid,
                              int64_t n_inner, const int64_t so[3], const int64_t sg[3], int dv,
                              float* delta, cudaStream_t st) {
  // Rows are (outer, mid, inner); launch one kernel per outer index so that
  // the kernel only folds (mid, inner) with strides (so[1], so[2]).
  const int w = width_class(dv);
  for (int64_t a = 0; a < n_outer; ++a) {
    const T* oa = static_cast<const T*>(o) + a * so[0];
    const T* ga = static_cast<const T*>(g) + a * sg[0];
    const int64_t rows = n_mid * n_inner;
    if (rows == 0) continue;
    ATTN_DISPATCH_WIDTH(w, rows_delta<T, NV><<<blocks_for_warps(rows), kWarps * 32, 0, st>>>(
                               oa, ga, rows, (int)n_inner, so[1], so[2], sg[1], sg[2], dv, delta + a * rows);)
  }
  return cudaGetLastError();
}

template <typename T>
cudaError_t launch_dense_bwd_rows(const DenseP& p, const void* g, const int64_t sg[3], const float* lse,
                                  const int64_t sl[3], const float* delta, void* dq, const int64_t sdq[3],
                                  void* dk, const int64_t sdk[3], void* dv, const int64_t sdv[3],
                                  cudaStream_t st) {
  const int w = width_class(p.d > p.dv ? p.d : p.dv);
  const int64_t qrows = (int64_t)p.B * p.Hq * p.Tq, krows = (int64_t)p.B * p.Hkv * p.Tk;
  if (qrows == 0) return cudaSuccess;
  ATTN_DISPATCH_WIDTH(w,
      dense_dq_rows<T, NQ, NV><<<blocks_for_warps(qrows), kWarps * 32, 0, st>>>(
          p, static_cast<const T*>(g), sg[0], sg[1], sg[2], lse, sl[0], sl[1], sl[2], delta,
          static_cast<T*>(dq), sdq[0], sdq[1], sdq[2]);
      dense_dkv_rows<T, NQ, NV><<<blocks_for_warps(krows), kWarps * 32, 0, st>>>(
          p, static_cast<const T*>(g), sg[0], sg[1], sg[2], lse, sl[0], sl[1], sl[2], delta,
          static_cast<T*>(dk), sdk[0], sdk[1], sdk[2], static_cast<T*>(dv), sdv[0], sdv[1], sdv[2]);)
  return cudaGetLastError();
}

template <typename T>
cudaError_t launch_topk_bwd_rows(const TopkP& p, const void* g, int64_t sg_t, int64_t sg_h,
                                 const float* lse, int64_t sl_t, int64_t sl_h, const float* delta,
                                 void* dq, int64_t sd_t, int64_t sd_h, FixedAcc fa,
                                 void* dkv, int64_t sdkv, uint32_t* status, cudaStream_t st) {
  const int w = width_class(p.Dqk > p.Dv ? p.Dqk : p.Dv);
  const int64_t rows = (int64_t)p.Tq * p.H, pairs = (int64_t)p.Tq * p.topk_max;
  cudaError_t e = cudaMemsetAsync(fa.acc, 0, topk_acc_total_bytes(p.Tkv, p.Dqk), st);
  if (e != cudaSuccess) return e;
  if (rows > 0) {
    ATTN_DISPATCH_WIDTH(w,
        topk_dq_rows<T, NQ, NV><<<blocks_for_warps(rows), kWarps * 32, 0, st>>>(
            p, static_cast<const T*>(g), sg_t, sg_h, lse, sl_t, sl_h, delta, static_cast<T*>(dq), sd_t,
            sd_h);
        if (pairs > 0) topk_dkv_pairs<T, NQ, NV><<<blocks_for_warps(pairs), kWarps * 32, 0, st>>>(
            p, static_cast<const T*>(g), sg_t, sg_h, lse, sl_t, sl_h, delta, fa, status);)
  }
  const int64_t n = (int64_t)p.Tkv * p.Dqk;
  if (n > 0)
    fixed_to_out<T><<<(unsigned)((n + 255) / 256), 256, 0, st>>>(fa, p.Tkv, p.Dqk, static_cast<T*>(dkv), sdkv,
                                                                 status);
  return cudaGetLastError();
}

template <typename T>
cudaError_t launch_fixed_to_out(FixedAcc fa, int rows, int cols, void* out, int64_t so, uint32_t* status,
                                cudaStream_t st) {
  const int64_t n = (int64_t)rows * cols;
  if (n > 0)
    fixed_to_out<T><<<(unsigned)((n + 255) / 256), 256, 0, st>>>(fa, rows, cols, static_cast<T*>(out), so, status);
  return cudaGetLastError();
}

template <typename T>
cudaError_t launch_f32_to_out(const float* acc, int rows, int cols, void* out, int64_t so, cudaStream_t st) {
  const int64_t n = (int64_t)rows * cols;
  if (n > 0) f32_to_out<T><<<(unsigned)((n + 255) / 256), 256, 0, st>>>(acc, rows, cols, static_cast<T*>(out), so);
  return cudaGetLastError();
}

// An LSE in the caller's format -> the natural-log, sink-inclusive LSE that
// the reverse kernels read ("DeepSeek Sparse Attention Forward and
// Backward", sections 7.2-7.3): undo the -log2 scaling, then fold the sink
// logit in as logaddexp(LSE_kv, z). Element (i0, i1, i2) of an
// [n0, n1, n2] view with the given strides goes to out[(i0 n1 + i1) n2 + i2];
// the head index is i1 (head_dim 1) or i2 (head_dim 2).
__global__ void __launch_bounds__(256)
lse_to_total_kernel(const float* in, int n0, int n1, int n2, int64_t s0, int64_t s1, int64_t s2, int head_dim,
                    const float* sink, uint32_t fmt, float* out) {
  constexpr float ln2 = 0.6931471805599453f;
  const int64_t n = (int64_t)n0 * n1 * n2;
  for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < n; e += (int64_t)gridDim.x * blockDim.x) {
    const int i2 = (int)(e % n2);
    const int i1 = (int)((e / n2) % n1);
    const int64_t i0 = e / ((int64_t)n1 * n2);
    float v = in[i0 * s0 + i1 * s1 + i2 * s2];
    if (fmt & ATTN_LSE_NEG_LOG2) v = -v * ln2;
    if ((fmt & ATTN_LSE_KV_ONLY) && sink) {
      const float z = sink[head_dim == 1 ? i1 : i2];
      const float M = fmaxf(v, z);
      v = M == -INFINITY ? -INFINITY : M + logf(expf(v - M) + expf(z - M));
    }
    out[e] = v;
  }
}

cudaError_t launch_lse_to_total(const float* in, int n0, int n1, int n2, const int64_t s[3], int head_dim,
                                const float* sink, uint32_t fmt, float* out, cudaStream_t st) {
  const int64_t n = (int64_t)n0 * n1 * n2;
  if (n == 0) return cudaSuccess;
  const int blocks = (int)((n + 255) / 256 < 4096 ? (n + 255) / 256 : 4096);
  lse_to_total_kernel<<<blocks, 256, 0, st>>>(in, n0, n1, n2, s[0], s[1], s[2], head_dim, sink, fmt, out);
  return cudaGetLastError();
}

cudaError_t launch_dsink(const float* sink, const float* lse, const float* delta, int n_outer, int n_heads,
                         int n_inner, int64_t sl_outer, int64_t sl_head, int64_t sl_inner,
                         bool delta_head_major, float* dsink, cudaStream_t st) {
  if (n_heads == 0) return cudaSuccess;
  dsink_reduce<<<n_heads, 256, 0, st>>>(sink, lse, delta, n_outer, n_heads, n_inner, sl_outer, sl_head,
                                        sl_inner, delta_head_major ? 1 : 0, dsink);
  return cudaGetLastError();
}

#define ATTN_INSTANTIATE(T)                                                                             \
  template cudaError_t launch_dense_fwd_rows<T>(const DenseP&, void*, const int64_t[3], float*,         \
                                                const int64_t[3], cudaStream_t);                        \
  template cudaError_t launch_topk_fwd_rows<T>(const TopkP&, void*, int64_t, int64_t, float*, int64_t,  \
                                               int64_t, uint32_t*, cudaStream_t);                       \
  template cudaError_t launch_rows_delta<T>(const void*, const void*, int64_t, int64_t, int64_t,        \
                                            const int64_t[3], const int64_t[3], int, float*,            \
                                            cudaStream_t);                                              \
  template cudaError_t launch_dense_bwd_rows<T>(const DenseP&, const void*, const int64_t[3],           \
                                                const float*, const int64_t[3], const float*, void*,    \
                                                const int64_t[3], void*, const int64_t[3], void*,       \
                                                const int64_t[3], cudaStream_t);                        \
  template cudaError_t launch_topk_bwd_rows<T>(const TopkP&, const void*, int64_t, int64_t,             \
                                               const float*, int64_t, int64_t, const float*, void*,     \
                                               int64_t, int64_t, FixedAcc, void*, int64_t,              \
                                               uint32_t*, cudaStream_t);                               \
  template cudaError_t launch_fixed_to_out<T>(FixedAcc, int, int, void*, int64_t, uint32_t*, cudaStream_t); \
  template cudaError_t launch_f32_to_out<T>(const float*, int, int, void*, int64_t, cudaStream_t);

ATTN_INSTANTIATE(float)
ATTN_INSTANTIATE(__nv_bfloat16)
ATTN_INSTANTIATE(__half)

}  // namespace attn
