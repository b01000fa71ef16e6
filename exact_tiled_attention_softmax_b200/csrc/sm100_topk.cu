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
//   upper half, columns 128-415: Q as 16-bit pairs, the A operand of S = Q K^T
// A warp reads its quarter with 32-lane loads: its upper 16 lanes own the
// S rows (softmax), its lower 16 lanes the O rows of the same heads.
//
// Warp 0 publishes each tile's 64 listed KV rows; eight gather warps copy them
// with 16-byte cp.async into a three-stage ring (9 planes of 64 columns,
// 128-byte swizzle); warp 1 issues the MMAs (S, then O += P V with P staged
// in shared memory); warps 2-5 run the softmax and the epilogue.
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
constexpr uint32_t kTP = kTKV + kTStages * kTTile;  // P: 64 heads x 64 keys, 16-bit
constexpr uint32_t kTCtl = kTP + kTH * 128;
constexpr uint32_t kTSmem = kTCtl + 1024 + 1024;  // control block + alignment slack
constexpr int kTFGather = 8;                         // forward gather warps
constexpr int kTFThreads = 192 + 32 * kTFGather;    // row producer, MMA issuer, 4 softmax warps, gather warps
static_assert(kTK * 72 % (32 * kTFGather) == 0, "a tile's 16-byte copies split evenly over the gather warps");
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kRescale = 8.0f;                 // move the running max only past 2^8
constexpr uint32_t kUpper = 16u << 16;           // TMEM lane offset of the upper half
constexpr uint32_t kQCol = 128;                  // first TMEM column of Q (upper half)

struct TopkCtl {
  uint64_t kv_full[kTStages], kv_empty[kTStages], rows_full[kTStages];
  uint64_t s_full[2];
  uint64_t p_full, pv_done, q_ready, o_final;
  uint32_t vmask[kTStages][2];  // valid listed keys of the stage: key 2i+e <-> bit i of word e
  uint32_t tmem_base;
  uint32_t abort_flag;
  int32_t grow[kTStages][kTK];  // forward: the KV row each listed key of the stage reads
};

struct TopkArgs {
  const uint8_t* kv;  // KV rows, skv_bytes apart (the forward's gather source)
  int64_t skv_bytes;
  const uint16_t* q;  // 16-bit storage: bf16 or fp16
  int64_t sq_t, sq_h;
  const int32_t* idx;
  int64_t idx_stride;
  int32_t topk_max;
  const int32_t* len;
  int Tq, Tkv;
  float scale_log2;
  const float* sink;
  uint16_t* o;
  int64_t so_t, so_h;
  float* lse;
  int64_t sl_t, sl_h;
  uint32_t lse_fmt;
  int check_causal;  // ATTN_MASK_TOPK_CHECK_CAUSAL
  uint32_t* status;
};

__device__ __forceinline__ bool key_valid(const uint32_t (&vm)[2], int k) { return (vm[k & 1] >> (k >> 1)) & 1u; }

template <bool kH>
__global__ void __launch_bounds__(kTFThreads, 1)
topk_fwd_kernel(const TopkArgs a) {
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
      mbar_init(smem_u32(&ctl->kv_full[s]), kTFGather);  // one arrival per gather warp
      mbar_init(smem_u32(&ctl->kv_empty[s]), 1);
      mbar_init(smem_u32(&ctl->rows_full[s]), 1);
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
    // ---------------- row producer (whole warp): lane l holds listed keys 2l
    // and 2l+1 of the tile; it publishes the stage's KV rows and valid-key
    // mask to the gather warps.
    const int32_t* list = a.idx + (int64_t)t * a.idx_stride;
    // The listed indices of tile n + 1 are read while tile n's gathers go
    // out, so their latency is not on the producer's path.
    auto read_idx = [&](int m, int e) {
      const int pos = m * kTK + 2 * lane + e;
      return (m < ntiles && pos < n_keys) ? list[pos] : -1;
    };
    int jn[2] = {read_idx(0, 0), read_idx(0, 1)};
    int n = 0;
    for (; n < ntiles; ++n) {
      const int s = n % kTStages;
      if (!__all_sync(0xffffffffu,
                      wait_bar(smem_u32(&ctl->kv_empty[s]), ((n / kTStages) & 1) ^ 1, abort_flag, a.status)))
        break;
      const int jc[2] = {jn[0], jn[1]};
      jn[0] = read_idx(n + 1, 0);
      jn[1] = read_idx(n + 1, 1);
      int row[2];
      bool valid[2];
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int pos = n * kTK + 2 * lane + e;
        const int j = jc[e];
        valid[e] = pos < n_keys && j >= 0 && j < a.Tkv;
        if (pos < n_keys && !valid[e]) set_status(a.status, ATTN_DEVERR_TOPK_INDEX);
        if (valid[e]) check_topk_causal(a.check_causal, j, t, a.Tq, a.Tkv, a.status);
        row[e] = valid[e] ? j : 0;  // unlisted and out-of-range keys read row 0 and are masked
      }
      const uint32_t vm0 = __ballot_sync(0xffffffffu, valid[0]), vm1 = __ballot_sync(0xffffffffu, valid[1]);
      ctl->grow[s][2 * lane] = row[0];
      ctl->grow[s][2 * lane + 1] = row[1];
      if (lane == 0) {
        ctl->vmask[s][0] = vm0;
        ctl->vmask[s][1] = vm1;
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&ctl->rows_full[s]));  // publishes grow and vmask
    }
  } else if (warp >= 6) {
    // ---------------- gather warps: 16-byte asynchronous copies of the 64
    // listed rows (72 chunks of 16 bytes each) into the stage's nine 128-byte-
    // swizzled planes; consecutive threads take consecutive chunks of a row.
    // A stage is signalled when its copies have landed, one stage behind the
    // copies being issued.
    const int gt = threadIdx.x - 192;
    auto signal = [&](int m) {
      fence_proxy_async_smem();  // the MMAs read the stage through the async proxy
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&ctl->kv_full[m % kTStages]));
    };
    int n = 0;
    bool ok = true;
    for (; n < ntiles; ++n) {
      const int s = n % kTStages;
      ok = __all_sync(0xffffffffu, wait_bar(smem_u32(&ctl->rows_full[s]), (n / kTStages) & 1, abort_flag, a.status));
      if (!ok) break;
      const uint32_t dst = sbase + kTKV + s * kTTile;
#pragma unroll 4
      for (int it = 0; it < kTK * 72 / (32 * kTFGather); ++it) {
        const int q = it * (32 * kTFGather) + gt, r = q / 72, c = q - r * 72;
        cp_async_16(dst + (uint32_t)(c >> 3) * kTPlane + sw128_offset(r, (c & 7) * 16),
                    a.kv + (int64_t)ctl->grow[s][r] * a.skv_bytes + c * 16);
      }
      cp_async_commit();
      if (n > 0) {
        cp_async_wait<1>();
        signal(n - 1);
      }
    }
    cp_async_wait<0>();  // nothing stays in flight past the loop
    if (ok && n > 0) signal(n - 1);
  } else if (warp == 1) {
    // ---------------- MMA issuer: S(n) = Q K(n)^T two tiles ahead of O += P(n) V(n).
    // The whole warp runs the loop; one elected lane issues the MMAs.
    const bool leader = elect_one();
    auto wait_all = [&](uint32_t bar, uint32_t par) {
      return __all_sync(0xffffffffu, wait_bar(bar, par, abort_flag, a.status));
    };
    constexpr uint32_t idS = idesc16<kH>(64, kTK, 0, 0);
    constexpr uint32_t idPV = idesc16<kH>(64, 256, 0, 1);
    const uint64_t dKV0 = smem_desc_sw128(sbase + kTKV, 16, 1024);        // K-major rows of a plane
    const uint64_t dV0 = smem_desc_sw128(sbase + kTKV, kTPlane, 1024);    // MN-major: planes are 64-wide chunks
    const uint64_t dP0 = smem_desc_sw128(sbase + kTP, 16, 1024);
    constexpr uint64_t kStageStep = kTTile >> 4;
    bool ok = wait_all(smem_u32(&ctl->q_ready), 0);
    auto issue_s = [&](int m) -> bool {
      const int s = m % kTStages, b = m & 1;
      if (!wait_all(smem_u32(&ctl->kv_full[s]), (m / kTStages) & 1)) return false;
      tc_fence_after();
      const uint64_t dk = dKV0 + (uint64_t)s * kStageStep;
      if (leader) {
#pragma unroll
        for (int kk = 0; kk < kTD / 16; ++kk)  // A = Q from TMEM: 16 columns of Q = 8 packed columns per step
          mma_ts(tmem + kUpper + b * kTK, tmem + kUpper + kQCol + kk * 8,
                 dk + (uint64_t)(((kk >> 2) * kTPlane + (kk & 3) * 32) >> 4), idS, kk > 0 ? 1u : 0u);
        mma_commit(smem_u32(&ctl->s_full[b]));
      }
      __syncwarp();
      return true;
    };
    if (ok) tc_fence_after();
    if (ok && ntiles > 0) ok = issue_s(0);
    if (ok && ntiles > 1) ok = issue_s(1);
    for (int n = 0; ok && n < ntiles; ++n) {
      const int s = n % kTStages;
      if (!(ok = wait_all(smem_u32(&ctl->p_full), n & 1))) break;
      tc_fence_after();
      const uint64_t dv = dV0 + (uint64_t)s * kStageStep;
      if (leader) {
#pragma unroll
        for (int nh = 0; nh < 2; ++nh)
#pragma unroll
          for (int kk = 0; kk < kTK / 16; ++kk)  // B = V: planes 4nh..4nh+3, 16 keys (rows) per step
            mma_ss(tmem + nh * 256, dP0 + (uint64_t)(kk * 2),
                   dv + (uint64_t)((4 * nh * kTPlane + kk * 2048) >> 4), idPV, (n > 0 || kk > 0) ? 1u : 0u);
        mma_commit(smem_u32(&ctl->pv_done));
        mma_commit(smem_u32(&ctl->kv_empty[s]));
      }
      __syncwarp();
      if (n + 2 < ntiles) ok = issue_s(n + 2);
    }
    if (leader) mma_commit(smem_u32(&ctl->o_final));
    __syncwarp();
  } else if (warp >= 2) {
    // ---------------- softmax warps: quarter qt = warp & 3 of TMEM; lane l
    // works on head h = 16 qt + (l & 15): its S row if l >= 16, its O row if l < 16.
    const int qt = warp & 3;
    const bool upper = lane >= 16;
    const int h = 16 * qt + (lane & 15);
    const uint32_t tq = tmem + ((uint32_t)(32 * qt) << 16);  // this warp's lanes, column 0
    // Q row h into TMEM (upper half, columns 128-415) as 16-bit pairs. The lower
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
        pk[e] = pack16<kH>(p0, p1);
        pk[16 + e] = pack16<kH>(p2, p3);
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
        a.lse[(int64_t)t * a.sl_t + (int64_t)h * a.sl_h] = stored_lse_log2(a.lse_fmt, lse2, m_run, l_run);
      }
      oscale = __shfl_sync(0xffffffffu, oscale, (lane + 16) & 31);  // lower lane l <- upper lane l + 16
      uint16_t* orow = a.o + (int64_t)t * a.so_t + (int64_t)h * a.so_h;
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
              pkd[e] = have_o ? pack16<kH>(__uint_as_float(o[idx]) * oscale, __uint_as_float(o[idx + 1]) * oscale) : 0u;
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

// ------------------------------------------------------------- reverse

// Reverse, first kernel (one CTA per query token): recompute S = Q K^T,
// P = 2^(S c log2(e) - LSE2) on the listed keys, dP = dO V^T, and
// G = c P (dP - delta) (DSA note, sections 3.3-3.4, 8); accumulate
// dQ = G K_sel in TMEM over the tiles, and store G and P as 16-bit rows
// [token][head][listed position] for the dKV kernel.
//   upper half: S cols 0-63, dP 64-127, Q 128-415, dQ[:, 512:576] 416-479
//   lower half: dQ[:, 0:512] cols 0-511
constexpr int kBStages = 2;
constexpr uint32_t kBKV = 0;
constexpr uint32_t kBDO = kBKV + kBStages * kTTile;  // dO: 8 planes of 64 heads x 64 columns
constexpr uint32_t kBG = kBDO + 8 * kTPlane;         // G: 64 heads x 64 keys, 16-bit
constexpr uint32_t kBCtl = kBG + kTH * 128;
constexpr uint32_t kBSmem = kBCtl + 1024 + 1024;
constexpr int kBGather = 8;                       // reverse gather warps
constexpr int kBThreads = 192 + 32 * kBGather;    // producer, MMA issuer, 4 compute warps, gather warps
static_assert(kTK * 72 % (32 * kBGather) == 0, "a tile's 16-byte copies split evenly over the gather warps");
constexpr uint32_t kDPCol = 64, kDQHiCol = 416;

struct TopkBwdCtl {
  uint64_t kv_full[kBStages], kv_empty[kBStages], rows_full[kBStages];
  uint64_t do_full, q_ready, st_full, st_empty, g_full, g_free, dq_done;
  uint32_t vmask[kBStages][2];
  uint32_t tmem_base;
  uint32_t abort_flag;
  int32_t grow[kBStages][kTK];  // the KV row each listed key of the stage reads
};

struct TopkBwdArgs {
  const uint8_t* kv;  // KV rows, skv_bytes apart (the gather source)
  int64_t skv_bytes;
  const uint16_t* q;  // 16-bit storage: bf16 or fp16
  int64_t sq_t, sq_h;
  const int32_t* idx;
  int64_t idx_stride;
  int32_t topk_max, topk_pad;
  const int32_t* len;
  int Tq, Tkv;
  float scale, scale_log2;
  const float* lse;
  int64_t sl_t, sl_h;
  const float* delta;  // [Tq, 64]
  uint16_t* dq;
  int64_t sd_t, sd_h;
  uint16_t* g_scr;  // [Tq, 64, topk_pad]
  uint16_t* p_scr;
  int check_causal;  // ATTN_MASK_TOPK_CHECK_CAUSAL
  uint32_t* status;
};

template <bool kH>
__global__ void __launch_bounds__(kBThreads, 1)
topk_bwd_dq_kernel(const __grid_constant__ CUtensorMap tdo,
                   const TopkBwdArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  TopkBwdCtl* ctl = reinterpret_cast<TopkBwdCtl*>(smem + kBCtl);
  volatile uint32_t* abort_flag = &ctl->abort_flag;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t = blockIdx.x;
  const int n_keys = a.len ? min(max(a.len[t], 0), a.topk_max) : a.topk_max;
  const int ntiles = (n_keys + kTK - 1) / kTK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kBStages; ++s) {
      mbar_init(smem_u32(&ctl->kv_full[s]), kBGather);  // one arrival per gather warp
      mbar_init(smem_u32(&ctl->kv_empty[s]), 1);
      mbar_init(smem_u32(&ctl->rows_full[s]), 1);
    }
    mbar_init(smem_u32(&ctl->do_full), 1);
    mbar_init(smem_u32(&ctl->q_ready), 4);
    mbar_init(smem_u32(&ctl->st_full), 1);
    mbar_init(smem_u32(&ctl->st_empty), 4);
    mbar_init(smem_u32(&ctl->g_full), 4);
    mbar_init(smem_u32(&ctl->g_free), 1);
    mbar_init(smem_u32(&ctl->dq_done), 1);
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
    // ---------------- producer: dO once (8 planes), then the KV gathers.
    if (lane == 0) {
      tma_prefetch_desc(&tdo);
      const uint32_t df = smem_u32(&ctl->do_full);
      mbar_expect_tx(df, 8 * kTPlane);
      for (int c = 0; c < 8; ++c) tma_load_3d(sbase + kBDO + c * kTPlane, &tdo, df, 64 * c, 0, t);
    }
    __syncwarp();
    const int32_t* list = a.idx + (int64_t)t * a.idx_stride;
    // The listed indices of tile n + 1 are read while tile n's gathers go
    // out, so their latency is not on the producer's path.
    auto read_idx = [&](int m, int e) {
      const int pos = m * kTK + 2 * lane + e;
      return (m < ntiles && pos < n_keys) ? list[pos] : -1;
    };
    int jn[2] = {read_idx(0, 0), read_idx(0, 1)};
    int n = 0;
    for (; n < ntiles; ++n) {
      const int s = n % kBStages;
      if (!__all_sync(0xffffffffu,
                      wait_bar(smem_u32(&ctl->kv_empty[s]), ((n / kBStages) & 1) ^ 1, abort_flag, a.status)))
        break;
      const int jc[2] = {jn[0], jn[1]};
      jn[0] = read_idx(n + 1, 0);
      jn[1] = read_idx(n + 1, 1);
      int row[2];
      bool valid[2];
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int pos = n * kTK + 2 * lane + e;
        const int j = jc[e];
        valid[e] = pos < n_keys && j >= 0 && j < a.Tkv;
        if (pos < n_keys && !valid[e]) set_status(a.status, ATTN_DEVERR_TOPK_INDEX);
        if (valid[e]) check_topk_causal(a.check_causal, j, t, a.Tq, a.Tkv, a.status);
        row[e] = valid[e] ? j : 0;
      }
      const uint32_t vm0 = __ballot_sync(0xffffffffu, valid[0]), vm1 = __ballot_sync(0xffffffffu, valid[1]);
      ctl->grow[s][2 * lane] = row[0];
      ctl->grow[s][2 * lane + 1] = row[1];
      if (lane == 0) {
        ctl->vmask[s][0] = vm0;
        ctl->vmask[s][1] = vm1;
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&ctl->rows_full[s]));  // publishes grow and vmask
    }
    if (lane == 0) wait_bar(smem_u32(&ctl->do_full), 0, abort_flag, nullptr);
  } else if (warp >= 6) {
    // ---------------- gather warps: 16-byte asynchronous copies of the 64
    // listed rows into the stage's nine 128-byte-swizzled planes (as in the
    // forward); with two stages each one is signalled as soon as its own
    // copies have landed.
    const int gt = threadIdx.x - 192;
    auto signal = [&](int m) {
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&ctl->kv_full[m % kBStages]));
    };
    int n = 0;
    bool ok = true;
    for (; n < ntiles; ++n) {
      const int s = n % kBStages;
      ok = __all_sync(0xffffffffu, wait_bar(smem_u32(&ctl->rows_full[s]), (n / kBStages) & 1, abort_flag, a.status));
      if (!ok) break;
      const uint32_t dst = sbase + kBKV + s * kTTile;
#pragma unroll 4
      for (int it = 0; it < kTK * 72 / (32 * kBGather); ++it) {
        const int q = it * (32 * kBGather) + gt, r = q / 72, c = q - r * 72;
        cp_async_16(dst + (uint32_t)(c >> 3) * kTPlane + sw128_offset(r, (c & 7) * 16),
                    a.kv + (int64_t)ctl->grow[s][r] * a.skv_bytes + c * 16);
      }
      cp_async_commit();
      cp_async_wait<0>();
      signal(n);
    }
    cp_async_wait<0>();
  } else if (warp == 1) {
    // ---------------- MMA issuer: S(n), dP(n) as soon as the compute warps
    // have read S(n-1), dP(n-1) and tile n is gathered; dQ += G(n) K(n) once
    // G(n) is in shared memory, ahead of S(n+1), dP(n+1) when it is ready
    // first.
    // The whole warp runs the loop; one elected lane issues the MMAs.
    const bool leader = elect_one();
    auto wait_all = [&](uint32_t bar, uint32_t par) {
      return __all_sync(0xffffffffu, wait_bar(bar, par, abort_flag, a.status));
    };
    constexpr uint32_t idS = idesc16<kH>(64, kTK, 0, 0);
    constexpr uint32_t idDQ = idesc16<kH>(64, 256, 0, 1);
    constexpr uint32_t idDQ64 = idesc16<kH>(64, 64, 0, 1);
    const uint64_t dKV0 = smem_desc_sw128(sbase + kBKV, 16, 1024);
    const uint64_t dKmn0 = smem_desc_sw128(sbase + kBKV, kTPlane, 1024);
    const uint64_t dDO = smem_desc_sw128(sbase + kBDO, 16, 1024);
    const uint64_t dG = smem_desc_sw128(sbase + kBG, 16, 1024);
    constexpr uint64_t kStageStep = kTTile >> 4;
    bool ok = wait_all(smem_u32(&ctl->q_ready), 0) && wait_all(smem_u32(&ctl->do_full), 0);
    auto issue_sdp = [&](int m) -> bool {
      const int s = m % kBStages;
      if (!wait_all(smem_u32(&ctl->kv_full[s]), (m / kBStages) & 1)) return false;
      if (m > 0 && !wait_all(smem_u32(&ctl->st_empty), (m - 1) & 1)) return false;
      tc_fence_after();
      const uint64_t dk = dKV0 + (uint64_t)s * kStageStep;
      if (leader) {
#pragma unroll
        for (int kk = 0; kk < kTD / 16; ++kk)  // S = Q K^T, A = Q from TMEM
          mma_ts(tmem + kUpper, tmem + kUpper + kQCol + kk * 8,
                 dk + (uint64_t)(((kk >> 2) * kTPlane + (kk & 3) * 32) >> 4), idS, kk > 0 ? 1u : 0u);
#pragma unroll
        for (int kk = 0; kk < kTDV / 16; ++kk) {  // dP = dO V^T, both K-major over the first 8 planes
          const uint32_t off = ((kk >> 2) * kTPlane + (kk & 3) * 32) >> 4;
          mma_ss(tmem + kUpper + kDPCol, dDO + (uint64_t)off, dk + (uint64_t)off, idS, kk > 0 ? 1u : 0u);
        }
        mma_commit(smem_u32(&ctl->st_full));
      }
      __syncwarp();
      return true;
    };
    if (ok && ntiles > 0) ok = issue_sdp(0);
    auto ready = [&](uint32_t bar, uint32_t par) { return __all_sync(0xffffffffu, mbar_try_wait(bar, par)); };
    for (int n = 0; ok && n < ntiles; ++n) {
      const int s = n % kBStages;
      // dQ(n) needs G(n); S/dP(n + 1) needs tile n + 1 gathered and S/dP(n)
      // read. Whichever is ready first is issued first (they touch different
      // TMEM columns; a slow gather then no longer holds dQ(n) back, and with
      // it the release of the stage the next gather fills).
      bool sdp = n + 1 >= ntiles;
      const uint64_t w0 = globaltimer();
      while (!sdp) {
        if (ready(smem_u32(&ctl->g_full), n & 1)) break;
        if (ready(smem_u32(&ctl->kv_full[(n + 1) % kBStages]), ((n + 1) / kBStages) & 1) &&
            ready(smem_u32(&ctl->st_empty), n & 1)) {
          if (!(ok = issue_sdp(n + 1))) break;
          sdp = true;
          break;
        }
        if (*abort_flag) {
          ok = false;
          break;
        }
        if (globaltimer() - w0 > kTimeoutNs) {  // as wait_bar: raise the abort flag and the timeout bit
          if (lane == 0) {
            *abort_flag = 1u;
            atomicOr(a.status, 0x4u);
          }
          ok = false;
          break;
        }
      }
      if (!ok) break;
      if (!(ok = wait_all(smem_u32(&ctl->g_full), n & 1))) break;
      tc_fence_after();
      const uint64_t dk = dKmn0 + (uint64_t)s * kStageStep;
      if (leader) {
#pragma unroll
        for (int kk = 0; kk < kTK / 16; ++kk) {  // dQ += G K: B = K rows as [keys x d], d contiguous
          const uint32_t acc = (n > 0 || kk > 0) ? 1u : 0u;
          mma_ss(tmem, dG + (uint64_t)(kk * 2), dk + (uint64_t)((kk * 2048) >> 4), idDQ, acc);
          mma_ss(tmem + 256, dG + (uint64_t)(kk * 2), dk + (uint64_t)((4 * kTPlane + kk * 2048) >> 4), idDQ, acc);
          mma_ss(tmem + kUpper + kDQHiCol, dG + (uint64_t)(kk * 2), dk + (uint64_t)((8 * kTPlane + kk * 2048) >> 4),
                 idDQ64, acc);
        }
        mma_commit(smem_u32(&ctl->g_free));
        mma_commit(smem_u32(&ctl->kv_empty[s]));
      }
      __syncwarp();
      if (!sdp && !(ok = issue_sdp(n + 1))) break;
    }
    if (leader) mma_commit(smem_u32(&ctl->dq_done));
    __syncwarp();
  } else if (warp >= 2) {
    // ---------------- compute warps: lane l >= 16 of quarter qt owns row
    // h = 16 qt + l - 16 of S, dP and dQ[:, 512:576]; lane l < 16 the same
    // head's dQ[:, 0:512].
    const int qt = warp & 3;
    const bool upper = lane >= 16;
    const int h = 16 * qt + (lane & 15);
    const uint32_t tq = tmem + ((uint32_t)(32 * qt) << 16);
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
    const float L = a.lse[(int64_t)t * a.sl_t + (int64_t)h * a.sl_h];
    const float lse2 = L * kLog2e;
    const float dl = a.delta[(int64_t)t * kTH + h];
    const bool live = L != -INFINITY;
    const uint32_t g_row = sbase + kBG + h * 128;
    uint16_t* gs = a.g_scr + ((int64_t)t * kTH + h) * a.topk_pad;
    uint16_t* ps = a.p_scr + ((int64_t)t * kTH + h) * a.topk_pad;
    bool ok = true;
    for (int n = 0; n < ntiles && ok; ++n) {
      const int s = n % kBStages;
      ok = __all_sync(0xffffffffu, wait_bar(smem_u32(&ctl->st_full), n & 1, abort_flag, a.status));
      if (ok)
        ok = __all_sync(0xffffffffu,
                        wait_bar(smem_u32(&ctl->kv_full[s]), (n / kBStages) & 1, abort_flag, a.status));
      if (!ok) break;
      tc_fence_after();
      uint32_t s0[32], s1[32], d0[32], d1[32];
      tmem_ld32(tq, s0);
      tmem_ld32(tq + 32, s1);
      tmem_ld32(tq + kDPCol, d0);
      tmem_ld32(tq + kDPCol + 32, d1);
      const uint32_t vm[2] = {ctl->vmask[s][0], ctl->vmask[s][1]};
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&ctl->st_empty));  // S and dP may be overwritten
      uint32_t gp[32], pp[32];
#pragma unroll
      for (int e = 0; e < 16; ++e) {
        float pv[4], gv[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int k = (u < 2 ? 2 * e + u : 32 + 2 * e + u - 2);
          const uint32_t sv = u < 2 ? s0[2 * e + u] : s1[2 * e + u - 2];
          const uint32_t dv = u < 2 ? d0[2 * e + u] : d1[2 * e + u - 2];
          const float p = (live && key_valid(vm, k)) ? ex2(__uint_as_float(sv) * a.scale_log2 - lse2) : 0.f;
          pv[u] = p;
          gv[u] = a.scale * p * (__uint_as_float(dv) - dl);
        }
        pp[e] = pack16<kH>(pv[0], pv[1]);
        pp[16 + e] = pack16<kH>(pv[2], pv[3]);
        gp[e] = pack16<kH>(gv[0], gv[1]);
        gp[16 + e] = pack16<kH>(gv[2], gv[3]);
      }
      // G's shared-memory tile is free once dQ += G(n-1) K(n-1) has completed.
      if (n > 0)
        ok = __all_sync(0xffffffffu, wait_bar(smem_u32(&ctl->g_free), (n - 1) & 1, abort_flag, a.status));
      if (!ok) break;
      if (upper) {
#pragma unroll
        for (int c = 0; c < 8; ++c)
          st_shared_v4(g_row + ((c ^ (h & 7)) << 4), gp[4 * c], gp[4 * c + 1], gp[4 * c + 2], gp[4 * c + 3]);
        uint4* gd = reinterpret_cast<uint4*>(gs + n * kTK);
        uint4* pd = reinterpret_cast<uint4*>(ps + n * kTK);
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          gd[c] = make_uint4(gp[4 * c], gp[4 * c + 1], gp[4 * c + 2], gp[4 * c + 3]);
          pd[c] = make_uint4(pp[4 * c], pp[4 * c + 1], pp[4 * c + 2], pp[4 * c + 3]);
        }
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&ctl->g_full));
    }
    // ---------------- epilogue: dQ rows (lower lanes: columns 0-511, upper
    // lanes: 512-575 from the upper half). G already carries the scale c.
    bool have = false;
    if (ok && ntiles > 0) {
      have = __all_sync(0xffffffffu, wait_bar(smem_u32(&ctl->dq_done), 0, abort_flag, a.status));
      if (have) tc_fence_after();
    }
    if (ok) {
      uint16_t* drow = a.dq + (int64_t)t * a.sd_t + (int64_t)h * a.sd_h;
      auto put = [&](const uint32_t (&r)[32], int col0) {
#pragma unroll
        for (int c8 = 0; c8 < 4; ++c8) {
          uint32_t pk[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int idx = c8 * 8 + 2 * e;
            pk[e] = have ? pack16<kH>(__uint_as_float(r[idx]), __uint_as_float(r[idx + 1])) : 0u;
          }
          *reinterpret_cast<uint4*>(drow + col0 + c8 * 8) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
        }
      };
#pragma unroll 1
      for (int c = 0; c < kTDV / 32; ++c) {
        uint32_t r[32];
        if (have) {
          tmem_ld32(tq + 32 * c, r);
          tmem_wait_ld();
        }
        if (!upper) put(r, 32 * c);
      }
#pragma unroll 1
      for (int c = 0; c < 2; ++c) {
        uint32_t r[32];
        if (have) {
          tmem_ld32(tq + kDQHiCol + 32 * c, r);
          tmem_wait_ld();
        }
        if (upper) put(r, kTDV + 32 * c);
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

// Reverse, second kernel (one CTA per query token): the token's
// contribution to dKV for each listed row j (DSA note, sections 8-9),
// C_j = sum_h G[h, j] Q[h, :] + [sum_h P[h, j] dO[h, :], 0], as
// C^T = Q^T G + dO^T P on the tensor cores (M = 128 columns of Dqk per
// chunk, N = 64 listed keys, K = 64 heads), then added into the dKV
// accumulator with global reductions: fp32 atomics as in the note (kFixed
// false; the order of the additions varies from run to run), or 64-bit
// integer atomics into a signed 32.32 fixed-point accumulator (kFixed true:
// integer addition is associative, so dKV is bitwise reproducible).
//   Chunk c = 0..3 covers columns 128c..128c+127 of Dqk, chunk 4 columns
//   512-575 (M = 64, Q part only); a launch takes the chunks [c_lo, c_hi).
//   The CTA's chunks form one sequence (chunk q = nch n + c - c_lo for tile
//   n, nch = c_hi - c_lo) whose accumulators take eight 64-column TMEM slots
//   in turn (slot q mod 8): the MMAs of the next chunks run while the
//   draining warps reduce the previous ones, so the reductions stream.
constexpr int kCStages = 4;  // G/P tiles with their listed rows
constexpr int kCSlots = 8;   // 64-column accumulator slots
constexpr uint32_t kCQ = 0;                                // Q: 9 planes of 64 heads x 64 columns
constexpr uint32_t kCDO = kCQ + kTPlanes * kTPlane;        // dO: 8 planes
constexpr uint32_t kCGP = kCDO + 8 * kTPlane;              // stages x (G, P) tiles of 64 heads x 64 keys
constexpr uint32_t kCRow = kCGP + kCStages * 2 * kTPlane;  // stages x 64 KV rows (-1: not listed / invalid)
constexpr uint32_t kCCtl = kCRow + kCStages * kTK * 4;
constexpr uint32_t kCSmem = kCCtl + 256 + 1024;
constexpr int kCPerQ = 6;                     // draining warps per TMEM lane quarter
constexpr int kCDrain = 4 * kCPerQ;
constexpr int kCThreads = 64 + 32 * kCDrain;  // producer, MMA issuer, draining warps

struct TopkDkvCtl {
  uint64_t qdo_full, gp_full[kCStages], gp_empty[kCStages], c_full[kCSlots], c_empty[kCSlots];
  uint32_t tmem_base;
  uint32_t abort_flag;
};
static_assert(sizeof(TopkDkvCtl) <= 256, "dKV control block");

struct TopkDkvArgs {
  const int32_t* idx;
  int64_t idx_stride;
  int32_t topk_max;
  const int32_t* len;
  int Tq, Tkv, Dqk;
  FixedAcc fa;  // kFixed: [Tkv, Dqk] signed 32.32 fixed point, per-row counts, largest magnitude
  float* acc32;  // otherwise: [Tkv, Dqk] fp32
  uint32_t* status;
  int c_lo, c_hi;  // the launch's column chunks [c_lo, c_hi) of 0..4
};

template <bool kH, bool kFixed>
__global__ void __launch_bounds__(kCThreads, 1)
topk_bwd_dkv_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tdo,
                    const __grid_constant__ CUtensorMap tg, const __grid_constant__ CUtensorMap tp,
                    const TopkDkvArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  TopkDkvCtl* ctl = reinterpret_cast<TopkDkvCtl*>(smem + kCCtl);
  int32_t* krow = reinterpret_cast<int32_t*>(smem + kCRow);
  volatile uint32_t* abort_flag = &ctl->abort_flag;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t = blockIdx.x;
  const int n_keys = a.len ? min(max(a.len[t], 0), a.topk_max) : a.topk_max;
  const int ntiles = (n_keys + kTK - 1) / kTK;
  const int c_lo = kFixed ? a.c_lo : 0, c_hi = kFixed ? a.c_hi : 5;  // the fp32 launch takes every chunk

  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&ctl->qdo_full), 1);
    for (int s = 0; s < kCStages; ++s) {
      mbar_init(smem_u32(&ctl->gp_full[s]), 1);
      mbar_init(smem_u32(&ctl->gp_empty[s]), kCDrain);  // released by the draining warps: krow is theirs too
    }
    for (int i = 0; i < kCSlots; ++i) {
      mbar_init(smem_u32(&ctl->c_full[i]), 1);
      mbar_init(smem_u32(&ctl->c_empty[i]), kCDrain);  // one arrival per draining warp
    }
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
    // ---------------- producer: Q and dO of the token once, then per tile
    // the G and P tiles and the listed rows.
    if (lane == 0 && ntiles > 0) {
      tma_prefetch_desc(&tq);
      tma_prefetch_desc(&tdo);
      tma_prefetch_desc(&tg);
      tma_prefetch_desc(&tp);
      const uint32_t f = smem_u32(&ctl->qdo_full);
      const int p0 = 2 * c_lo, q1 = min(2 * c_hi, kTPlanes), d1 = min(2 * c_hi, 8);
      mbar_expect_tx(f, (q1 - p0 + max(d1 - p0, 0)) * kTPlane);
      for (int c = p0; c < q1; ++c) tma_load_3d(sbase + kCQ + c * kTPlane, &tq, f, 64 * c, 0, t);
      for (int c = p0; c < d1; ++c) tma_load_3d(sbase + kCDO + c * kTPlane, &tdo, f, 64 * c, 0, t);
    }
    __syncwarp();
    const int32_t* list = a.idx + (int64_t)t * a.idx_stride;
    auto read_idx = [&](int m, int e) {  // tile m + 1's indices are read while tile m's rows go out
      const int pos = m * kTK + 2 * lane + e;
      return (m < ntiles && pos < n_keys) ? list[pos] : -1;
    };
    int jn[2] = {read_idx(0, 0), read_idx(0, 1)};
    int n = 0;
    for (; n < ntiles; ++n) {
      const int s = n % kCStages;
      if (!__all_sync(0xffffffffu,
                      wait_bar(smem_u32(&ctl->gp_empty[s]), ((n / kCStages) & 1) ^ 1, abort_flag, a.status)))
        break;
      const int jc[2] = {jn[0], jn[1]};
      jn[0] = read_idx(n + 1, 0);
      jn[1] = read_idx(n + 1, 1);
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int k = 2 * lane + e;
        const int j = jc[e];
        const bool ok_j = j >= 0 && j < a.Tkv;
        krow[s * kTK + k] = ok_j ? j : -1;  // the first kernel flagged invalid entries
        if (kFixed && ok_j && c_lo == 0) atomicAdd(a.fa.count + j, 1u);  // one contribution of this token to row j
      }
      __syncwarp();
      if (lane == 0) {
        const uint32_t f = smem_u32(&ctl->gp_full[s]);
        mbar_expect_tx(f, 2 * kTPlane);  // its release publishes krow with the tiles
        tma_load_3d(sbase + kCGP + (2 * s) * kTPlane, &tg, f, n * kTK, 0, t);
        tma_load_3d(sbase + kCGP + (2 * s + 1) * kTPlane, &tp, f, n * kTK, 0, t);
      }
      __syncwarp();
    }
    if (lane == 0) {  // copies still in flight land before the CTA exits
      for (int r = (n > kCStages ? n - kCStages : 0); r < n; ++r)
        wait_bar(smem_u32(&ctl->gp_full[r % kCStages]), (r / kCStages) & 1, abort_flag, nullptr);
      if (ntiles > 0) wait_bar(smem_u32(&ctl->qdo_full), 0, abort_flag, nullptr);
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer (the warp waits, one elected lane issues):
    // C^T = Q^T G + dO^T P, chunk by chunk into the slot ring.
    constexpr uint32_t id128 = idesc16<kH>(128, kTK, 1, 1);
    constexpr uint32_t id64 = idesc16<kH>(64, kTK, 1, 1);
    const uint64_t dQ0 = smem_desc_sw128(sbase + kCQ, kTPlane, 1024);    // [heads x d], d contiguous
    const uint64_t dDO0 = smem_desc_sw128(sbase + kCDO, kTPlane, 1024);
    const uint64_t dGP0 = smem_desc_sw128(sbase + kCGP, kTPlane, 1024);  // [heads x keys], keys contiguous
    const bool leader = elect_one();
    int issued = 0;  // chunks committed
    bool ok = ntiles == 0 || __all_sync(0xffffffffu, wait_bar(smem_u32(&ctl->qdo_full), 0, abort_flag, a.status));
    for (int n = 0; ok && n < ntiles; ++n) {
      const int s = n % kCStages;
      ok = __all_sync(0xffffffffu, wait_bar(smem_u32(&ctl->gp_full[s]), (n / kCStages) & 1, abort_flag, a.status));
      if (!ok) break;
      tc_fence_after();
      const uint64_t dG = dGP0 + (uint64_t)((2 * s) * (kTPlane >> 4)), dP = dG + (uint64_t)(kTPlane >> 4);
      const int nch = c_hi - c_lo;
#pragma unroll 1
      for (int c = c_lo; c < c_hi; ++c) {
        const int q = nch * n + c - c_lo, slot = q % kCSlots;
        if (q >= kCSlots) {
          ok = __all_sync(0xffffffffu, wait_bar(smem_u32(&ctl->c_empty[slot]), ((q / kCSlots) - 1) & 1,
                                                abort_flag, a.status));
          if (!ok) break;
          tc_fence_after();
        }
        if (leader) {
          const uint32_t d = tmem + 64 * slot;
          if (c < 4) {
#pragma unroll
            for (int kk = 0; kk < kTH / 16; ++kk)  // K = 16 heads = 16 rows of every plane per step
              mma_ss(d, dQ0 + (uint64_t)((2 * c * kTPlane + kk * 2048) >> 4), dG + (uint64_t)(kk * 128), id128,
                     kk > 0 ? 1u : 0u);
#pragma unroll
            for (int kk = 0; kk < kTH / 16; ++kk)
              mma_ss(d, dDO0 + (uint64_t)((2 * c * kTPlane + kk * 2048) >> 4), dP + (uint64_t)(kk * 128), id128,
                     1u);
          } else {
#pragma unroll
            for (int kk = 0; kk < kTH / 16; ++kk)  // columns 512-575: Q part only, M = 64
              mma_ss(d, dQ0 + (uint64_t)((8 * kTPlane + kk * 2048) >> 4), dG + (uint64_t)(kk * 128), id64,
                     kk > 0 ? 1u : 0u);
          }
          mma_commit(smem_u32(&ctl->c_full[slot]));
        }
        __syncwarp();
        issued = q + 1;
      }
    }
    if (issued > 0 && lane == 0)  // the last chunk's MMAs complete before TMEM is released
      wait_bar(smem_u32(&ctl->c_full[(issued - 1) % kCSlots]), ((issued - 1) / kCSlots) & 1, abort_flag, nullptr);
  } else {
    // ---------------- drain: lane l of quarter qt holds column 128 c + 32 qt + l
    // of chunk c (512 + 16 qt + l of chunk 4 when l < 16) for the chunk's 64
    // keys. A quarter's six warps take its 16-key units of the chunk sequence
    // in turn (unit 4 q + g to warp (4 q + g) mod 6), so that the load stays
    // even and many reductions are in flight at once.
    const int qt = warp & 3, kq = (warp - 2) >> 2, nch = c_hi - c_lo;
    const uint32_t tq4 = tmem + ((uint32_t)(32 * qt) << 16);
    bool ok = true, sat = false;
    float amax = 0.f;
    for (int n = 0; n < ntiles && ok; ++n) {
      const int s = n % kCStages;
      // the listed rows come with the stage's tiles
      ok = __all_sync(0xffffffffu, wait_bar(smem_u32(&ctl->gp_full[s]), (n / kCStages) & 1, abort_flag, a.status));
      if (!ok) break;
      const int32_t* rows = krow + s * kTK;
#pragma unroll 1
      for (int c = c_lo; c < c_hi; ++c) {
        const int q = nch * n + c - c_lo, slot = q % kCSlots;
        ok = __all_sync(0xffffffffu, wait_bar(smem_u32(&ctl->c_full[slot]), (q / kCSlots) & 1, abort_flag, a.status));
        if (!ok) break;
        tc_fence_after();
        const int col = c < 4 ? 128 * c + 32 * qt + lane : 512 + 16 * qt + lane;
        const bool live = c < 4 || lane < 16;
#pragma unroll 1
        for (int g = (kq + kCPerQ - (4 * q) % kCPerQ) % kCPerQ; g < 4; g += kCPerQ) {
          uint32_t v[16];
          tmem_ld16(tq4 + 64 * slot + 16 * g, v);
          tmem_wait_ld();
          if (!live) continue;
          const int4* r4 = reinterpret_cast<const int4*>(rows + 16 * g);
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const int4 jj = r4[i];
            const int js[4] = {jj.x, jj.y, jj.z, jj.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              if (js[e] < 0) continue;
              const float x = __uint_as_float(v[4 * i + e]);
              if constexpr (kFixed)
                fixed_add(a.fa.acc + (int64_t)js[e] * a.Dqk + col, x, sat, amax);
              else
                atomicAdd(a.acc32 + (int64_t)js[e] * a.Dqk + col, x);
            }
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&ctl->c_empty[slot]));
      }
      if (!ok) break;
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&ctl->gp_empty[s]));  // c_full of its chunks: the MMAs are done with G and P
    }
    if constexpr (kFixed) {
      fixed_publish_max(a.fa.maxbits, amax);
      if (__any_sync(0xffffffffu, sat) && lane == 0) set_status(a.status, ATTN_DEVERR_OVERFLOW);
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

// 3-D 16-bit map (inner, 64, Tq) with (64, 64, 1) boxes and 128-byte swizzle:
// one token's 64 rows of a 64-column plane per load.
bool make_map3(CUtensorMap* map, const void* base, int64_t inner, int Tq, int64_t s_row, int64_t s_tok, bool f16) {
  cuuint64_t dims[3] = {(cuuint64_t)inner, (cuuint64_t)kTH, (cuuint64_t)Tq};
  cuuint64_t strides[2] = {(cuuint64_t)s_row * 2, (cuuint64_t)s_tok * 2};
  cuuint32_t box[3] = {64, (cuuint32_t)kTH, 1};
  cuuint32_t es[3] = {1, 1, 1};
  return topk_encode_fn()(map, f16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, es,
                          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

cudaError_t raise_smem(const void* fn, uint32_t bytes, int which) {
  static bool done[8][64] = {};  // [kernel instantiation][device]
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 64 && done[which][dev]) return cudaSuccess;
  e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
  if (e == cudaSuccess && dev < 64) done[which][dev] = true;
  return e;
}

}  // namespace

int sm100_topk_pad(int topk_max) { return ((topk_max + kTK - 1) / kTK) * kTK; }

size_t sm100_topk_bwd_scratch_bytes(int Tq, int H, int Dqk, int Dv, int topk_max) {
  if (H != kTH || Dqk != kTD || Dv != kTDV) return 0;
  return 2 * (size_t)Tq * kTH * sm100_topk_pad(topk_max) * sizeof(uint16_t);
}

bool sm100_topk_bwd_supported(const TopkP& p, const attn_tensor* q, const attn_tensor* kv, const attn_tensor* o,
                              const attn_tensor* do_, const attn_tensor* dq) {
  if (!sm100_topk_supported(p, q, kv, o)) return false;
  if (do_->dtype != q->dtype || dq->dtype != q->dtype) return false;
  return aligned16(do_->data, do_->stride[0]) && aligned16(do_->data, do_->stride[1]) &&
         aligned16(dq->data, dq->stride[0]) && aligned16(dq->data, dq->stride[1]);
}

cudaError_t sm100_topk_bwd(const TopkP& p, const void* g, int64_t sg_t, int64_t sg_h, const float* lse,
                           int64_t sl_t, int64_t sl_h, const float* delta, void* dq, int64_t sd_t, int64_t sd_h,
                           FixedAcc acc, float* acc32, void* scratch, uint32_t* status, cudaStream_t st) {
  const int pad = sm100_topk_pad(p.topk_max);
  const bool f16 = p.dtype == ATTN_F16;
  uint16_t* g_scr = static_cast<uint16_t*>(scratch);
  uint16_t* p_scr = g_scr + (size_t)p.Tq * kTH * pad;
  CUtensorMap mdo, mq, mg, mp;
  if (!make_map3(&mdo, g, kTDV, p.Tq, sg_h, sg_t, f16) ||
      !make_map3(&mq, p.q, kTD, p.Tq, p.sq_h, p.sq_t, f16) ||
      !make_map3(&mg, g_scr, pad, p.Tq, pad, (int64_t)kTH * pad, f16) ||
      !make_map3(&mp, p_scr, pad, p.Tq, pad, (int64_t)kTH * pad, f16))
    return cudaErrorInvalidValue;
  TopkBwdArgs a;
  a.kv = static_cast<const uint8_t*>(p.kv);
  a.skv_bytes = p.skv * 2;
  a.q = static_cast<const uint16_t*>(p.q);
  a.sq_t = p.sq_t;
  a.sq_h = p.sq_h;
  a.idx = p.idx;
  a.idx_stride = p.idx_stride;
  a.topk_max = p.topk_max;
  a.topk_pad = pad;
  a.len = p.len;
  a.Tq = p.Tq;
  a.Tkv = p.Tkv;
  a.scale = p.scale;
  a.scale_log2 = p.scale * kLog2e;
  a.lse = lse;
  a.sl_t = sl_t;
  a.sl_h = sl_h;
  a.delta = delta;
  a.dq = static_cast<uint16_t*>(dq);
  a.sd_t = sd_t;
  a.sd_h = sd_h;
  a.g_scr = g_scr;
  a.p_scr = p_scr;
  a.check_causal = p.check_causal;
  a.status = status;
  TopkDkvArgs c;
  c.idx = p.idx;
  c.idx_stride = p.idx_stride;
  c.topk_max = p.topk_max;
  c.len = p.len;
  c.Tq = p.Tq;
  c.Tkv = p.Tkv;
  c.Dqk = p.Dqk;
  c.fa = acc;
  c.acc32 = acc32;
  c.status = status;
  cudaError_t e;
  auto kdq = f16 ? topk_bwd_dq_kernel<true> : topk_bwd_dq_kernel<false>;
  auto kdkv = acc32 ? (f16 ? topk_bwd_dkv_kernel<true, false> : topk_bwd_dkv_kernel<false, false>)
                    : (f16 ? topk_bwd_dkv_kernel<true, true> : topk_bwd_dkv_kernel<false, true>);
  if ((e = raise_smem(reinterpret_cast<const void*>(kdq), kBSmem, f16 ? 4 : 1)) != cudaSuccess) return e;
  if ((e = raise_smem(reinterpret_cast<const void*>(kdkv), kCSmem, acc32 ? (f16 ? 7 : 6) : (f16 ? 5 : 2))) != cudaSuccess)
    return e;
  main_kernel_begin(st);
  kdq<<<p.Tq, kBThreads, kBSmem, st>>>(mdo, a);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  // fp32: one launch over the five column chunks (the 75 MB accumulator fits
  // L2). Fixed point: chunks 0-1, then 2-4, so that each launch's slice of
  // the int64 accumulator (67 and 84 MB of 151 MB) stays in L2 while it is
  // reduced into; the second launch re-reads the G/P rows.
  const int split[3] = {0, acc32 ? 5 : 2, 5};
  for (int i = 0; i < (acc32 ? 1 : 2) && e == cudaSuccess; ++i) {
    c.c_lo = split[i];
    c.c_hi = split[i + 1];
    kdkv<<<p.Tq, kCThreads, kCSmem, st>>>(mq, mdo, mg, mp, c);
    e = cudaGetLastError();
  }
  main_kernel_end(st);
  return cudaGetLastError();
}

bool sm100_topk_supported(const TopkP& p, const attn_tensor* q, const attn_tensor* kv, const attn_tensor* o) {
  if (q->dtype != ATTN_BF16 && q->dtype != ATTN_F16) return false;
  if (kv->dtype != q->dtype || o->dtype != q->dtype) return false;
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
  TopkArgs a;
  a.kv = static_cast<const uint8_t*>(p.kv);
  a.skv_bytes = p.skv * 2;
  a.q = static_cast<const uint16_t*>(p.q);
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
  a.o = static_cast<uint16_t*>(o);
  a.so_t = so_t;
  a.so_h = so_h;
  a.lse = lse;
  a.sl_t = sl_t;
  a.sl_h = sl_h;
  a.lse_fmt = p.lse_fmt;
  a.check_causal = p.check_causal;
  a.status = status;
  const bool f16 = p.dtype == ATTN_F16;
  auto kern = f16 ? topk_fwd_kernel<true> : topk_fwd_kernel<false>;
  cudaError_t e = raise_smem(reinterpret_cast<const void*>(kern), kTSmem, f16 ? 3 : 0);
  if (e != cudaSuccess) return e;
  main_kernel_begin(st);
  kern<<<p.Tq, kTFThreads, kTSmem, st>>>(a);
  main_kernel_end(st);
  return cudaGetLastError();
}

}  // namespace attn
