// Tensor-core forward of top-k sparse attention with a shared KV (one KV row
// serves as key and, through its first Dv columns, as value for every head),
// on sm_100a. The method is the DSA note's forward ("DeepSeek Sparse Attention
// Forward and Backward", sections 2-7): per query token t and head h, the
// scores of the listed KV rows, the running summary (m, l, u) over 64-key
// tiles, and the sink-inclusive finish.
//
// One CTA per query token. The 64 heads are the M = 64 rows of every MMA:
// an M = 64 accumulator occupies TMEM lanes 0-15 of each 32-lane quarter (the
// "lower" half) or, addressed at lane 16, lanes 16-31 (the "upper" half).
//   lower half, columns 0-511:   O, 64 heads x 512 fp32
//   upper half, columns 0-127:   two S buffers, 64 heads x 64 keys fp32
//   upper half, columns 128-415: Q as bf16 pairs, the A operand of S = Q K^T
// A warp reads its quarter with 32-lane loads: its upper 16 lanes own the
// S rows (softmax), its lower 16 lanes the O rows of the same heads.
//
// Warp 0 gathers each tile's 64 listed KV rows with TMA gather4 into a
// three-stage ring (9 planes of 64 columns, 128-byte swizzle); warp 1 issues
// the MMAs (S, then O += P V with P staged in shared memory); warps 2-5 run
// the softmax and the epilogue.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <math.h>

#include "sm100_topk.h"
#include "sm100_ptx.cuh"

namespace attn {

using namespace sm100;

namespace {

constexpr int kTH = 64;                        // heads (MMA rows)
constexpr int kTK = 64;                        // listed keys per tile
constexpr int kTD = 576;                       // Dqk
constexpr int kTDV = 512;                      // Dv
constexpr int kTPlanes = kTD / 64;             // 9 planes of 64 columns
constexpr uint32_t kTPlane = kTK * 128;        // 8 KB: 64 rows x 128 bytes
constexpr uint32_t kTTile = kTPlanes * kTPlane;  // 72 KB per KV tile
constexpr int kTStages = 3;
constexpr uint32_t kTKV = 0;
constexpr uint32_t kTP = kTKV + kTStages * kTTile;  // P: 64 heads x 64 keys bf16
constexpr uint32_t kTCtl = kTP + kTH * 128;
constexpr uint32_t kTSmem = kTCtl + 512 + 1024;  // control block + alignment slack
constexpr int kTThreads = 192;                   // producer, MMA issuer, 4 softmax warps
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kRescale = 8.0f;                 // move the running max only past 2^8
constexpr uint32_t kUpper = 16u << 16;           // TMEM lane offset of the upper half
constexpr uint32_t kQCol = 128;                  // first TMEM column of Q (upper half)

struct TopkCtl {
  uint64_t kv_full[kTStages], kv_empty[kTStages];
  uint64_t s_full[2];
  uint64_t p_full, pv_done, q_ready, o_final;
  uint32_t vmask[kTStages][2];  // valid listed keys of the stage: key 2i+e <-> bit i of word e
  uint32_t tmem_base;
  uint32_t abort_flag;
};

struct TopkArgs {
  const __nv_bfloat16* q;
  int64_t sq_t, sq_h;
  const int32_t* idx;
  int64_t idx_stride;
  int32_t topk_max;
  const int32_t* len;
  int Tq, Tkv;
  float scale_log2;
  const float* sink;
  __nv_bfloat16* o;
  int64_t so_t, so_h;
  float* lse;
  int64_t sl_t, sl_h;
  uint32_t* status;
};

__device__ __forceinline__ void gather4(uint32_t dst, const CUtensorMap* map, uint32_t bar, int x, int r0, int r1,
                                        int r2, int r3) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile::gather4.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5, %6, %7}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(x), "r"(r0), "r"(r1), "r"(r2), "r"(r3)
      : "memory");
}

__device__ __forceinline__ bool key_valid(const uint32_t (&vm)[2], int k) { return (vm[k & 1] >> (k >> 1)) & 1u; }

__global__ void __launch_bounds__(kTThreads, 1)
topk_fwd_kernel(const __grid_constant__ CUtensorMap tkv, const TopkArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  TopkCtl* ctl = reinterpret_cast<TopkCtl*>(smem + kTCtl);
  volatile uint32_t* abort_flag = &ctl->abort_flag;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t = blockIdx.x;
  const int n_keys = a.len ? min(max(a.len[t], 0), a.topk_max) : a.topk_max;
  const int ntiles = (n_keys + kTK - 1) / kTK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kTStages; ++s) {
      mbar_init(smem_u32(&ctl->kv_full[s]), 1);
      mbar_init(smem_u32(&ctl->kv_empty[s]), 1);
    }
    for (int b = 0; b < 2; ++b) mbar_init(smem_u32(&ctl->s_full[b]), 1);
    mbar_init(smem_u32(&ctl->p_full), 4);   // one arrival per softmax warp
    mbar_init(smem_u32(&ctl->pv_done), 1);
    mbar_init(smem_u32(&ctl->q_ready), 4);  // one arrival per softmax warp
    mbar_init(smem_u32(&ctl->o_final), 1);
    ctl->abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(&ctl->tmem_base), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ctl->tmem_base;

  if (warp == 0) {
    // ---------------- gather producer (whole warp): lane l holds listed keys
    // 2l and 2l+1 of the tile; lanes 0-15 then gather rows 4g..4g+3 (g = lane)
    // of all nine planes.
    if (lane == 0) tma_prefetch_desc(&tkv);
    const int32_t* list = a.idx + (int64_t)t * a.idx_stride;
    int n = 0;
    for (; n < ntiles; ++n) {
      const int s = n % kTStages;
      if (!__all_sync(0xffffffffu,
                      wait_bar(smem_u32(&ctl->kv_empty[s]), ((n / kTStages) & 1) ^ 1, abort_flag, a.status)))
        break;
      int row[2];
      bool valid[2];
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int pos = n * kTK + 2 * lane + e;
        const int j = pos < n_keys ? list[pos] : -1;
        valid[e] = pos < n_keys && j >= 0 && j < a.Tkv;
        if (pos < n_keys && !valid[e]) set_status(a.status, ATTN_DEVERR_TOPK_INDEX);
        row[e] = valid[e] ? j : 0;  // unlisted and out-of-range keys read row 0 and are masked
      }
      const uint32_t vm0 = __ballot_sync(0xffffffffu, valid[0]), vm1 = __ballot_sync(0xffffffffu, valid[1]);
      const uint32_t kf = smem_u32(&ctl->kv_full[s]);
      if (lane == 0) {
        ctl->vmask[s][0] = vm0;
        ctl->vmask[s][1] = vm1;
        mbar_expect_tx(kf, kTTile);  // its release publishes vmask with the stage
      }
      __syncwarp();
      const int g = lane & 15;
      const int r0 = __shfl_sync(0xffffffffu, row[0], 2 * g), r1 = __shfl_sync(0xffffffffu, row[1], 2 * g);
      const int r2 = __shfl_sync(0xffffffffu, row[0], 2 * g + 1), r3 = __shfl_sync(0xffffffffu, row[1], 2 * g + 1);
      if (lane < 16) {
        const uint32_t dst = sbase + kTKV + s * kTTile + g * 512;
#pragma unroll 1
        for (int c = 0; c < kTPlanes; ++c) gather4(dst + c * kTPlane, &tkv, kf, 64 * c, r0, r1, r2, r3);
      }
    }
    // Leave only after this warp's copies have landed.
    if (lane == 0)
      for (int r = (n > kTStages ? n - kTStages : 0); r < n; ++r)
        wait_bar(smem_u32(&ctl->kv_full[r % kTStages]), (r / kTStages) & 1, abort_flag, nullptr);
  } else if (warp == 1 && lane == 0) {
    // ---------------- MMA issuer: S(n) = Q K(n)^T two tiles ahead of O += P(n) V(n).
    constexpr uint32_t idS = idesc_bf16(64, kTK, 0, 0);
    constexpr uint32_t idPV = idesc_bf16(64, 256, 0, 1);
    const uint64_t dKV0 = smem_desc_sw128(sbase + kTKV, 16, 1024);        // K-major rows of a plane
    const uint64_t dV0 = smem_desc_sw128(sbase + kTKV, kTPlane, 1024);    // MN-major: planes are 64-wide chunks
    const uint64_t dP0 = smem_desc_sw128(sbase + kTP, 16, 1024);
    constexpr uint64_t kStageStep = kTTile >> 4;
    bool ok = wait_bar(smem_u32(&ctl->q_ready), 0, abort_flag, a.status);
    auto issue_s = [&](int m) -> bool {
      const int s = m % kTStages, b = m & 1;
      if (!wait_bar(smem_u32(&ctl->kv_full[s]), (m / kTStages) & 1, abort_flag, a.status)) return false;
      tc_fence_after();
      const uint64_t dk = dKV0 + (uint64_t)s * kStageStep;
#pragma unroll
      for (int kk = 0; kk < kTD / 16; ++kk)  // A = Q from TMEM: 16 columns of Q = 8 packed columns per step
        mma_ts(tmem + kUpper + b * kTK, tmem + kUpper + kQCol + kk * 8,
               dk + (uint64_t)(((kk >> 2) * kTPlane + (kk & 3) * 32) >> 4), idS, kk > 0 ? 1u : 0u);
      mma_commit(smem_u32(&ctl->s_full[b]));
      return true;
    };
    if (ok) tc_fence_after();
    if (ok && ntiles > 0) ok = issue_s(0);
    if (ok && ntiles > 1) ok = issue_s(1);
    for (int n = 0; ok && n < ntiles; ++n) {
      const int s = n % kTStages;
      if (!(ok = wait_bar(smem_u32(&ctl->p_full), n & 1, abort_flag, a.status))) break;
      tc_fence_after();
      const uint64_t dv = dV0 + (uint64_t)s * kStageStep;
#pragma unroll
      for (int nh = 0; nh < 2; ++nh)
#pragma unroll
        for (int kk = 0; kk < kTK / 16; ++kk)  // B = V: planes 4nh..4nh+3, 16 keys (rows) per step
          mma_ss(tmem + nh * 256, dP0 + (uint64_t)(kk * 2),
                 dv + (uint64_t)((4 * nh * kTPlane + kk * 2048) >> 4), idPV, (n > 0 || kk > 0) ? 1u : 0u);
      mma_commit(smem_u32(&ctl->pv_done));
      mma_commit(smem_u32(&ctl->kv_empty[s]));
      if (n + 2 < ntiles) ok = issue_s(n + 2);
    }
    mma_commit(smem_u32(&ctl->o_final));
  } else if (warp >= 2) {
    // ---------------- softmax warps: quarter qt = warp & 3 of TMEM; lane l
    // works on head h = 16 qt + (l & 15): its S row if l >= 16, its O row if l < 16.
    const int qt = warp & 3;
    const bool upper = lane >= 16;
    const int h = 16 * qt + (lane & 15);
    const uint32_t tq = tmem + ((uint32_t)(32 * qt) << 16);  // this warp's lanes, column 0
    // Q row h into TMEM (upper half, columns 128-415) as bf16 pairs. The lower
    // lanes store zeros into O's columns, which the first P V overwrites.
    {
      const uint4* qrow = reinterpret_cast<const uint4*>(a.q + (int64_t)t * a.sq_t + (int64_t)h * a.sq_h);
#pragma unroll 1
      for (int c = 0; c < kTD / 64; ++c) {
        uint32_t r[32];
#pragma unroll
        for (int v = 0; v < 8; ++v) {
          const uint4 x = upper ? qrow[c * 8 + v] : make_uint4(0u, 0u, 0u, 0u);
          r[4 * v] = x.x;
          r[4 * v + 1] = x.y;
          r[4 * v + 2] = x.z;
          r[4 * v + 3] = x.w;
        }
        tmem_st32(tq + kQCol + 32 * c, r);
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&ctl->q_ready));
    }
    float m_run = -INFINITY, l_run = 0.f;  // base-2 running max and sum (upper lanes)
    bool ok = true;
    const uint32_t p_row = sbase + kTP + h * 128;
    for (int n = 0; n < ntiles && ok; ++n) {
      const int b = n & 1, s = n % kTStages;
      ok = __all_sync(0xffffffffu, wait_bar(smem_u32(&ctl->s_full[b]), (n >> 1) & 1, abort_flag, a.status));
      if (ok)  // the stage's valid-key mask comes with its gather
        ok = __all_sync(0xffffffffu,
                        wait_bar(smem_u32(&ctl->kv_full[s]), (n / kTStages) & 1, abort_flag, a.status));
      if (!ok) break;
      tc_fence_after();
      // S(n) row: a 32-lane load of columns 64b..64b+63; the upper lanes hold S.
      uint32_t s0[32], s1[32];
      tmem_ld32(tq + b * kTK, s0);
      tmem_ld32(tq + b * kTK + 32, s1);
      const uint32_t vm[2] = {ctl->vmask[s][0], ctl->vmask[s][1]};
      tmem_wait_ld();
      float mx = -INFINITY;
#pragma unroll
      for (int k = 0; k < 32; ++k) {
        if (key_valid(vm, k)) mx = fmaxf(mx, __uint_as_float(s0[k]) * a.scale_log2);
        if (key_valid(vm, 32 + k)) mx = fmaxf(mx, __uint_as_float(s1[k]) * a.scale_log2);
      }
      float alpha = 1.f;
      if (upper) {
        float m_new = m_run;
        if (mx > -INFINITY && (m_run == -INFINITY || mx > m_run + kRescale)) m_new = fmaxf(mx, m_run);
        alpha = m_new == m_run ? 1.f : ex2(m_run - m_new);
        m_run = m_new;
      }
      const float msub = m_run == -INFINITY ? 0.f : m_run;
      float sum = 0.f;
      uint32_t pk[32];
#pragma unroll
      for (int e = 0; e < 16; ++e) {
        const int k0 = 2 * e, k1 = 2 * e + 1;
        const float p0 = key_valid(vm, k0) ? ex2(__uint_as_float(s0[k0]) * a.scale_log2 - msub) : 0.f;
        const float p1 = key_valid(vm, k1) ? ex2(__uint_as_float(s0[k1]) * a.scale_log2 - msub) : 0.f;
        const float p2 = key_valid(vm, 32 + k0) ? ex2(__uint_as_float(s1[k0]) * a.scale_log2 - msub) : 0.f;
        const float p3 = key_valid(vm, 32 + k1) ? ex2(__uint_as_float(s1[k1]) * a.scale_log2 - msub) : 0.f;
        sum += (p0 + p1) + (p2 + p3);
        pk[e] = pack_bf16(p0, p1);
        pk[16 + e] = pack_bf16(p2, p3);
      }
      l_run = l_run * alpha + sum;
      // The single P buffer is free once P(n-1) V(n-1) has completed; O is
      // then also safe to rescale.
      if (n > 0)
        ok = __all_sync(0xffffffffu, wait_bar(smem_u32(&ctl->pv_done), (n - 1) & 1, abort_flag, a.status));
      if (!ok) break;
      if (upper) {
#pragma unroll
        for (int c = 0; c < 8; ++c)  // 16-byte chunk c = keys 8c..8c+7, 128-byte swizzle
          st_shared_v4(p_row + ((c ^ (h & 7)) << 4), pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
      }
      if (n > 0 && __any_sync(0xffffffffu, alpha != 1.f)) {
        // Rare: the running max moved. No MMA may touch this quarter's TMEM
        // while all 32 lanes rewrite columns 0-511 (the upper lanes write back
        // their own values): S(n+1) must have landed; S(n+2) waits for P(n).
        if (n + 1 < ntiles)
          ok = __all_sync(0xffffffffu,
                          wait_bar(smem_u32(&ctl->s_full[b ^ 1]), ((n + 1) >> 1) & 1, abort_flag, a.status));
        if (!ok) break;
        tc_fence_after();
        const float a_hi = __shfl_sync(0xffffffffu, alpha, (lane + 16) & 31);  // lower lane l <- lane l + 16
        const float fo = upper ? 1.f : a_hi;
#pragma unroll 1
        for (int c = 0; c < kTDV / 32; ++c) {
          uint32_t o[32];
          tmem_ld32(tq + 32 * c, o);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * fo);
          tmem_st32(tq + 32 * c, o);
        }
        tmem_wait_st();
      }
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&ctl->p_full));
    }
    // ---------------- epilogue: Y = u / (l + exp(z - m)), LSE = m + ln(...).
    bool have_o = false;
    if (ok && ntiles > 0) {
      have_o = __all_sync(0xffffffffu, wait_bar(smem_u32(&ctl->o_final), 0, abort_flag, a.status));
      if (have_o) tc_fence_after();
    }
    if (ok) {
      const bool has_sink = a.sink != nullptr;
      const float z2 = has_sink ? a.sink[h] * kLog2e : -INFINITY;
      float lse2 = -INFINITY, oscale = 0.f;
      if (upper) {
        if (m_run == -INFINITY || !have_o) {
          lse2 = has_sink ? z2 : -INFINITY;
        } else {
          const float M = has_sink ? fmaxf(m_run, z2) : m_run;
          const float tot = l_run * exp2f(m_run - M) + (has_sink ? exp2f(z2 - M) : 0.f);
          oscale = exp2f(m_run - M) / tot;
          lse2 = M + log2f(tot);
        }
        a.lse[(int64_t)t * a.sl_t + (int64_t)h * a.sl_h] = lse2 / kLog2e;
      }
      oscale = __shfl_sync(0xffffffffu, oscale, (lane + 16) & 31);  // lower lane l <- upper lane l + 16
      __nv_bfloat16* orow = a.o + (int64_t)t * a.so_t + (int64_t)h * a.so_h;
#pragma unroll 1
      for (int c = 0; c < kTDV / 32; ++c) {
        uint32_t o[32];
        if (have_o) {
          tmem_ld32(tq + 32 * c, o);
          tmem_wait_ld();
        }
        if (!upper) {
#pragma unroll
          for (int c8 = 0; c8 < 4; ++c8) {
            uint32_t pkd[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int idx = c8 * 8 + 2 * e;
              pkd[e] = have_o ? pack_bf16(__uint_as_float(o[idx]) * oscale, __uint_as_float(o[idx + 1]) * oscale) : 0u;
            }
            *reinterpret_cast<uint4*>(orow + c * 32 + c8 * 8) = make_uint4(pkd[0], pkd[1], pkd[2], pkd[3]);
          }
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

PFN_cuTensorMapEncodeTiled_v12000 topk_encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

bool aligned16(const void* p, int64_t stride_elems) {
  return reinterpret_cast<uintptr_t>(p) % 16 == 0 && (stride_elems * 2) % 16 == 0;
}

}  // namespace

bool sm100_topk_supported(const TopkP& p, const attn_tensor* q, const attn_tensor* kv, const attn_tensor* o) {
  if (q->dtype != ATTN_BF16 || kv->dtype != ATTN_BF16 || o->dtype != ATTN_BF16) return false;
  if (p.H != kTH || p.Dqk != kTD || p.Dv != kTDV || p.Tq < 1 || p.Tkv < 1) return false;
  if (!aligned16(p.q, p.sq_t) || !aligned16(p.q, p.sq_h) || !aligned16(p.kv, p.skv)) return false;
  if (!aligned16(o->data, o->stride[0]) || !aligned16(o->data, o->stride[1])) return false;
  if (!topk_encode_fn()) return false;
  int dev = 0, major = 0, minor = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return false;
  cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
  cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
  return major == 10 && minor == 0;
}

cudaError_t sm100_topk_fwd(const TopkP& p, void* o, int64_t so_t, int64_t so_h, float* lse, int64_t sl_t,
                           int64_t sl_h, uint32_t* status, cudaStream_t st) {
  // 2-D map over the KV rows: 64-column boxes one row high (the gather4 form)
  // with 128-byte swizzle, matching the planes the MMAs read.
  CUtensorMap map;
  cuuint64_t dims[2] = {(cuuint64_t)p.Dqk, (cuuint64_t)p.Tkv};
  cuuint64_t strides[1] = {(cuuint64_t)p.skv * 2};
  cuuint32_t box[2] = {64, 1};
  cuuint32_t es[2] = {1, 1};
  if (topk_encode_fn()(&map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(p.kv), dims, strides, box, es,
                       CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                       CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  TopkArgs a;
  a.q = static_cast<const __nv_bfloat16*>(p.q);
  a.sq_t = p.sq_t;
  a.sq_h = p.sq_h;
  a.idx = p.idx;
  a.idx_stride = p.idx_stride;
  a.topk_max = p.topk_max;
  a.len = p.len;
  a.Tq = p.Tq;
  a.Tkv = p.Tkv;
  a.scale_log2 = p.scale * kLog2e;
  a.sink = p.sink;
  a.o = static_cast<__nv_bfloat16*>(o);
  a.so_t = so_t;
  a.so_h = so_h;
  a.lse = lse;
  a.sl_t = sl_t;
  a.sl_h = sl_h;
  a.status = status;
  static bool attr_done[64] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev >= 64 || !attr_done[dev]) {
    e = cudaFuncSetAttribute(reinterpret_cast<const void*>(topk_fwd_kernel),
                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kTSmem);
    if (e != cudaSuccess) return e;
    if (dev < 64) attr_done[dev] = true;
  }
  main_kernel_begin(st);
  topk_fwd_kernel<<<p.Tq, kTThreads, kTSmem, st>>>(map, a);
  main_kernel_end(st);
  return cudaGetLastError();
}

}  // namespace attn
