// Tensor-core path for dense bf16 or fp16 attention with d = dv = 128 on sm_100a.
//
// Forward: one CTA per (256 query rows, query head, batch row), held as two
// 128-row query tiles. A TMA producer warp streams 128-key K/V tiles through
// a two-stage ring; one thread issues tcgen05 MMAs (per query tile, S = Q K^T
// into that tile's TMEM columns and O += P V into its TMEM accumulator, the
// two tiles alternating on the tensor core); two 128-thread softmax
// warpgroups, one per query tile, own one row per thread (TMEM lane = row)
// and apply the running-summary update of
// "Accumulate attention without keeping the full grid", section "Rescale
// earlier mass before adding a new tile": tile maximum, new maximum, the
// rescale factor alpha, shifted exponentials and the running sum, with empty
// tiles skipped without touching the state ("Tiled attention and its
// recomputed reverse pass are exact", proof step 1.1). The maximum is only
// moved when it grows by more than 2^8 (in base-2 units); the output stays
// exact because every stored term shares the same reference maximum.
//
// Reverse: one CTA per (128-key tile, K/V head, batch row) walks every query
// head of its group and every 64-row query tile that can see its keys. Per
// step it recomputes S^T = K Q^T and dP^T = V dO^T, forms
// P = exp(S - LSE) and gamma = P (dP - delta) in registers (DSA note,
// sections 3.3-3.4; exactness proof, step 4.1), and accumulates
// dV += P~^T dO and dK += gamma^T Q in TMEM for the whole CTA (a fixed order,
// hence deterministic), while dQ^T = K^T gamma^T goes to an fp32 buffer by
// bulk reduce-add.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <math.h>

#include "sm100_dense.h"
#include "sm100_ptx.cuh"

namespace attn {

using namespace sm100;

namespace {

constexpr int kD = 128;          // head width handled here (d = dv)
constexpr int kBN = 128;         // keys per tile
constexpr int kBM = 128;         // forward query rows per CTA
constexpr int kBMb = 64;         // reverse query rows per step
constexpr int kStages = 2;       // K/V ring depth (forward), Q/dO ring depth (reverse)
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kRescaleThreshold = 8.0f;  // move the running max only past 2^8
constexpr int kPolyEvery = 4;              // forward: every k-th pair of exponentials on the FMA pipe (0: none)

// Does pair e of a 16-pair chunk take its exponentials on the FMA pipe? Not
// with dropout: there the softmax warps also run Philox4x32-10, whose
// multiplies share the pipe the polynomial would use.
template <bool kDrop>
__host__ __device__ constexpr bool poly_pair(int e) {
  return !kDrop && kPolyEvery > 0 && e % (kPolyEvery > 0 ? kPolyEvery : 1) == kPolyEvery - 1;
}

enum : uint8_t { kEmpty = 0, kFull = 1, kPartial = 2 };

// ------------------------------------------------------------------ masks

// Is every (i, j) of the rectangle [r0, r1] x [c0, c1] inside the
// causal/window band, and is any? Rows are given as key positions (query row
// + qoff). Row i allows [max(c0, i-W+1), min(c1, i)], so some row qualifies
// iff i can be chosen with c0 <= i (causal) and i <= c1 + W - 1 (window).
__device__ __forceinline__ void band_test(const MaskP& m, int64_t r0, int64_t r1, int64_t c0, int64_t c1, bool& any,
                                          bool& all) {
  const bool causal = m.flags & ATTN_MASK_CAUSAL, window = m.flags & ATTN_MASK_WINDOW;
  all = true;
  if (causal && c1 > r0) all = false;
  if (window && c0 < r1 - m.window + 1) all = false;
  int64_t lo = r0, hi = r1;
  if (causal && c0 > lo) lo = c0;
  if (window && c1 + m.window - 1 < hi) hi = c1 + m.window - 1;
  any = c0 <= c1 && lo <= hi;
}

// Class of the (64-row query slice qs, 128-key tile kt) pair.
__device__ uint8_t tile_class(const MaskP& m, int Tq, int Tk, int b, int h, int qs, int kt) {
  const int64_t r0 = (int64_t)qs * kBMb, r1 = (r0 + kBMb < Tq ? r0 + kBMb : Tq) - 1;
  const int64_t c0 = (int64_t)kt * kBN, c1e = c0 + kBN - 1, c1 = (c1e < Tk ? c1e : Tk - 1);
  if (r0 > r1 || c0 > c1) return kEmpty;
  bool any = false, all = c1e <= Tk - 1;
  if (!(m.flags & ATTN_MASK_BLOCK)) {
    bool a, f;
    band_test(m, r0 + m.qoff, r1 + m.qoff, c0, c1, a, f);
    any = a;
    all = all && f;
  } else {
    const uint8_t* base = m.bm + b * m.bm_sb + h * m.bm_sh;
    for (int64_t rb = r0 / m.bq; rb <= r1 / m.bq; ++rb) {
      const int64_t rr0 = rb * m.bq > r0 ? rb * m.bq : r0;
      const int64_t rr1 = rb * m.bq + m.bq - 1 < r1 ? rb * m.bq + m.bq - 1 : r1;
      for (int64_t cb = c0 / m.bk; cb <= c1 / m.bk; ++cb) {
        const int64_t cc0 = cb * m.bk > c0 ? cb * m.bk : c0;
        const int64_t cc1 = cb * m.bk + m.bk - 1 < c1 ? cb * m.bk + m.bk - 1 : c1;
        bool a, f;
        band_test(m, rr0 + m.qoff, rr1 + m.qoff, cc0, cc1, a, f);
        if (base[rb * m.bm_sq + cb]) {
          any = any || a;
          all = all && f;
        } else {
          all = false;
        }
      }
    }
  }
  return any ? (all ? kFull : kPartial) : kEmpty;
}

// tile_class refined by the active lengths and per-row starts. Exact for
// emptiness by length and for "every row's lowest key lies past the tile";
// otherwise conservative (a tile may be marked partial and then masked row
// by row). Only the class-table kernel evaluates it: a table always exists
// when either is set.
__device__ uint8_t tile_class_rows(const MaskP& m, int Tq, int Tk, int b, int h, int qs, int kt) {
  const uint8_t base = tile_class(m, Tq, Tk, b, h, qs, kt);
  if (base == kEmpty || !(m.lengths || m.starts)) return base;
  bool all = base == kFull;
  int64_t r0 = (int64_t)qs * kBMb, ra = (r0 + kBMb < Tq ? r0 + kBMb : Tq) - 1;
  const int64_t c0 = (int64_t)kt * kBN, c1e = c0 + kBN - 1;
  int64_t ca = c1e < Tk ? c1e : Tk - 1;
  if (m.lengths) {
    const int64_t L = active_len(m, b, Tk);
    if (r0 >= L || c0 >= L) return kEmpty;
    if (ra >= L) {
      ra = L - 1;
      all = false;
    }
    if (c1e >= L) all = false;
    if (ca >= L) ca = L - 1;
  }
  if (m.starts) {
    int64_t smin = INT64_MAX, smax = INT64_MIN;
    for (int64_t r = r0; r <= ra; ++r) {
      const int64_t s0 = row_start(m, b, r);
      smin = s0 < smin ? s0 : smin;
      smax = s0 > smax ? s0 : smax;
    }
    if (smin > ca) return kEmpty;
    if (smax > c0) all = false;
  }
  return all ? kFull : kPartial;
}

struct ClassTable {
  const uint8_t* cls;  // null: compute analytically
  int nb, nh;          // slices along batch and head (1 = broadcast)
  int nqs, nkt;
};

__device__ __forceinline__ uint8_t lookup_class(const ClassTable& ct, const MaskP& m, int Tq, int Tk, int b, int h,
                                                int qs, int kt) {
  if ((int64_t)qs * kBMb >= Tq) return kEmpty;  // slices past the last row are not in the table
  if (!ct.cls) return tile_class(m, Tq, Tk, b, h, qs, kt);
  const int sb = ct.nb > 1 ? b : 0, sh = ct.nh > 1 ? h : 0;
  return ct.cls[(((int64_t)sb * ct.nh + sh) * ct.nqs + qs) * ct.nkt + kt];
}

__global__ void classify_kernel(MaskP m, int Tq, int Tk, int B, int Hq, ClassTable ct, uint8_t* out) {
  const int64_t n = (int64_t)ct.nb * ct.nh * ct.nqs * ct.nkt;
  for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < n; e += (int64_t)gridDim.x * blockDim.x) {
    const int kt = (int)(e % ct.nkt);
    const int qs = (int)((e / ct.nkt) % ct.nqs);
    const int sh = (int)((e / ((int64_t)ct.nkt * ct.nqs)) % ct.nh);
    const int sb = (int)(e / ((int64_t)ct.nkt * ct.nqs * ct.nh));
    out[e] = tile_class_rows(m, Tq, Tk, sb, sh, qs, kt);
  }
  (void)B;
  (void)Hq;
}

// Forward tile class for a 128-row query tile: merge its two 64-row slices.
__device__ __forceinline__ uint8_t fwd_class(const ClassTable& ct, const MaskP& m, int Tq, int Tk, int b, int h,
                                             int qt, int kt) {
  const uint8_t a = lookup_class(ct, m, Tq, Tk, b, h, 2 * qt, kt);
  const uint8_t c = (2 * qt + 1) * kBMb < Tq ? lookup_class(ct, m, Tq, Tk, b, h, 2 * qt + 1, kt) : a;
  if (a == kEmpty && c == kEmpty) return kEmpty;
  if (a == kFull && c == kFull) return kFull;
  return kPartial;
}

// ------------------------------------------------------------- forward

struct FwdArgs {
  MaskP m;
  ClassTable ct;
  int B, Hq, Hkv, Tq, Tk;
  int block_aligned;  // block mask constant over every (64-row slice, 128-key tile)
  float scale_log2;   // c * log2(e)
  uint16_t* o;  // 16-bit storage: bf16 or fp16
  int64_t so[3];
  float* lse;
  int64_t sl[3];
  uint32_t* status;
};

// Shared-memory map of the forward kernel (offsets from a 1024-aligned base).
constexpr uint32_t kTileBytes = kBN * kD * 2;  // 32 KB: 128 rows x 128 bf16
constexpr int kFwdRows = 2 * kBM;              // two 128-row query tiles per CTA
constexpr uint32_t kFwdQ = 0;                  // 2 tiles
constexpr uint32_t kFwdK = kFwdQ + 2 * kTileBytes;
constexpr uint32_t kFwdV = kFwdK + kStages * kTileBytes;
constexpr uint32_t kFwdCtl = kFwdV + kStages * kTileBytes;
constexpr uint32_t kFwdSmem = kFwdCtl + 1024 + 1024;  // control block + alignment slack
constexpr int kFwdThreads = 320;  // producer, MMA issuer, softmax warpgroups (warps 2-5, 6-9)
constexpr int kFwdBand = 8;       // (batch row, query head) pairs per scheduling band

struct FwdCtl {
  uint64_t q_full;
  uint64_t k_full[kStages], v_full[kStages], kv_empty[kStages];
  uint64_t s_full[2], p_full[2];  // one pair per softmax warpgroup
  uint64_t o_final;
  uint32_t tmem_base;
  uint32_t abort_flag;
  // Per K/V stage, written by the producer before the stage's loads: bit w =
  // the tile has allowed keys for query tile w, bit 2 = another tile follows.
  uint32_t tinfo[kStages];
};

// Key-tile range that can hold allowed keys for rows [q0, q0 + rows).
__device__ __forceinline__ void fwd_key_tiles(const MaskP& m, int b, int Tq, int Tk, int q0, int rows, int& lo,
                                              int& hi) {
  const int nkt = (Tk + kBN - 1) / kBN;
  lo = 0;
  hi = nkt - 1;
  if (m.flags & ATTN_MASK_CAUSAL) {
    const int64_t last = (int64_t)(q0 + rows - 1 < Tq - 1 ? q0 + rows - 1 : Tq - 1) + m.qoff;  // key position
    if (last < 0)
      hi = -1;
    else if (last / kBN < hi)
      hi = (int)(last / kBN);
  }
  if (m.flags & ATTN_MASK_WINDOW) {
    const int64_t first = (int64_t)q0 + m.qoff - m.window + 1;
    lo = first > 0 ? (int)(first / kBN) : 0;
  }
  if (m.lengths) {  // Tq = Tk here
    const int64_t L = active_len(m, b, Tk);
    if (q0 >= L)
      hi = -1;
    else if ((L - 1) / kBN < hi)
      hi = (int)((L - 1) / kBN);
  }
}

// Class of (128-row query tile qt, key tile kt); tiles past Tq are empty.
__device__ __forceinline__ uint8_t wg_class(const FwdArgs& a, int b, int h, int qt, int kt) {
  if (qt * kBM >= a.Tq) return kEmpty;
  return fwd_class(a.ct, a.m, a.Tq, a.Tk, b, h, qt, kt);
}

// First key tile after `from` (up to kt_hi) with allowed keys for either
// query tile of the CTA (qt0, qt0 + 1); kt_hi + 1 when none. flags: bit w
// set when query tile qt0 + w has allowed keys there.
__device__ __forceinline__ int fwd_next_tile(const FwdArgs& a, int b, int h, int qt0, int kt_hi, int from,
                                             uint32_t& flags) {
  for (int kt = from + 1; kt <= kt_hi; ++kt) {
    flags = (wg_class(a, b, h, qt0, kt) != kEmpty ? 1u : 0u) | (wg_class(a, b, h, qt0 + 1, kt) != kEmpty ? 2u : 0u);
    if (flags) return kt;
  }
  flags = 0;
  return kt_hi + 1;
}

// Bits lo..hi (inclusive, within [0, 63]) of a 64-bit word; 0 when lo > hi.
__device__ __forceinline__ uint64_t range_bits64(int64_t lo, int64_t hi) {
  if (lo > hi || hi < 0 || lo > 63) return 0ull;
  lo = lo < 0 ? 0 : lo;
  hi = hi > 63 ? 63 : hi;
  const uint64_t upto = hi >= 63 ? ~0ull : ((1ull << (hi + 1)) - 1ull);
  return upto & ~((1ull << lo) - 1ull);
}

// Row i's key interval [lo, hi] narrowed by the active length and the row's
// start (lo > hi when nothing is left). Kept out of line, with the few
// fields it reads passed by value: the hot loops that mask partial tiles
// stay as they are when neither is set.
struct KeyInterval {
  int64_t lo, hi;
};

__device__ __noinline__ KeyInterval clip_row_keys(const int32_t* lengths, const int32_t* starts, int64_t st_sb, int b,
                                                  int64_t i, int64_t Tk, int64_t lo, int64_t hi) {
  if (lengths) {
    int64_t L = lengths[b];
    L = L < 0 ? 0 : (L > Tk ? Tk : L);
    if (i >= L) hi = -1;
    hi = L - 1 < hi ? L - 1 : hi;
  }
  if (starts) {
    const int64_t s0 = starts[b * st_sb + i];
    lo = s0 > lo ? s0 : lo;
  }
  return KeyInterval{lo, hi};
}

// Allowed keys of row i inside key tile [j0, j0 + 128) as two 64-bit words
// (bit c <-> key j0 + c). The causal/window conditions give one interval;
// a block mask that is constant over (64-row slice, 128-key tile) blocks is
// already folded into the tile class, otherwise it is looked up per key.
__device__ __forceinline__ void fwd_row_bits(const FwdArgs& a, int b, int h, int64_t i, int64_t j0, uint8_t slice_cls,
                                             uint64_t& w0, uint64_t& w1) {
  w0 = w1 = 0ull;
  if (i >= a.Tq || slice_cls == kEmpty) return;
  const int64_t ip = i + a.m.qoff;  // the row's key position
  int64_t lo = j0, hi = j0 + kBN - 1;
  if (hi > a.Tk - 1) hi = a.Tk - 1;
  if (a.m.flags & ATTN_MASK_CAUSAL) hi = ip < hi ? ip : hi;
  if (a.m.flags & ATTN_MASK_WINDOW) lo = ip - a.m.window + 1 > lo ? ip - a.m.window + 1 : lo;
  if (a.m.flags & (ATTN_MASK_LENGTHS | ATTN_MASK_STARTS)) {
    const KeyInterval iv = clip_row_keys(a.m.lengths, a.m.starts, a.m.st_sb, b, i, a.Tk, lo, hi);
    lo = iv.lo;
    hi = iv.hi;
  }
  if (lo > hi) return;
  w0 = range_bits64(lo - j0, hi - j0);
  w1 = range_bits64(lo - j0 - 64, hi - j0 - 64);
  if ((a.m.flags & ATTN_MASK_BLOCK) && !a.block_aligned) {
    const uint8_t* row = a.m.bm + b * a.m.bm_sb + h * a.m.bm_sh + (i / a.m.bq) * a.m.bm_sq;
    uint64_t b0 = 0, b1 = 0;
#pragma unroll 1
    for (int c = 0; c < 64; ++c) {
      if (j0 + c < a.Tk && row[(j0 + c) / a.m.bk]) b0 |= 1ull << c;
      if (j0 + 64 + c < a.Tk && row[(j0 + 64 + c) / a.m.bk]) b1 |= 1ull << c;
    }
    w0 &= b0;
    w1 &= b1;
  }
}

// Keep bits xi for row i and keys [j0, j0 + 128): 32 Philox blocks of 4 keys.
__device__ __forceinline__ void fwd_keep_bits(const MaskP& m, int b, int h, int64_t i, int64_t j0, uint64_t& k0,
                                              uint64_t& k1) {
  k0 = k1 = 0ull;
#pragma unroll 1
  for (int g = 0; g < 32; ++g) {
    const int64_t j = j0 + 4 * g;
    const uint4 w = philox4x32_10(make_uint4((uint32_t)(j >> 2), (uint32_t)i, (uint32_t)h, (uint32_t)b), m.seed_lo,
                                  m.seed_hi);
    const uint64_t nib = (uint64_t)(w.x >= m.keep_thr) | ((uint64_t)(w.y >= m.keep_thr) << 1) |
                         ((uint64_t)(w.z >= m.keep_thr) << 2) | ((uint64_t)(w.w >= m.keep_thr) << 3);
    if (g < 16)
      k0 |= nib << (4 * g);
    else
      k1 |= nib << (4 * (g - 16));
  }
}

// New running maximum after a tile whose (scaled, base-2) maximum is mx:
// moved only when mx exceeds it by more than the threshold (or on the first
// tile with an allowed key). Returns the factor alpha = 2^(m_old - m_new) that
// rescales the earlier terms (0 when there were none, 1 when m stays).
__device__ __forceinline__ float move_max(float mx, float& m_run) {
  float m_new = m_run;
  if (mx > -INFINITY && (m_run == -INFINITY || mx > m_run + kRescaleThreshold)) m_new = fmaxf(mx, m_run);
  const float alpha = (m_new == m_run) ? 1.f : ex2(m_run - m_new);
  m_run = m_new;
  return alpha;
}

// One S row (128 keys, all allowed, no dropout) of the calling thread's TMEM
// lane -> P (bf16 pairs written over the row's first 64 columns), with the
// running summary (m_run, l_run) updated. The maximum takes two 64-column
// TMEM loads and the exponentials four 32-column reloads, so that no more
// than 64 scores are live at once (the forward then needs no spill slots);
// x = s c log2(e) - m is formed on packed fp32 pairs and every kPolyEvery-th
// pair of exponentials runs on the FMA pipe instead of MUFU. Returns alpha.
template <bool kH, bool kDrop>
__device__ __forceinline__ float softmax_full_tile(uint32_t tS, float scale_log2, float& m_run, float& l_run,
                                                   uint64_t kb0, uint64_t kb1) {
  float mx;
  {
    const bool pos = scale_log2 >= 0.f;
    float e0 = pos ? -INFINITY : INFINITY, e1 = e0, e2 = e0, e3 = e0;
#pragma unroll
    for (int hf = 0; hf < 2; ++hf) {
      uint32_t s0[32], s1[32];
      tmem_ld32(tS + 64 * hf, s0);
      tmem_ld32(tS + 64 * hf + 32, s1);
      tmem_wait_ld();
      if (pos) {
#pragma unroll
        for (int e = 0; e < 32; e += 4) {
          e0 = max3f(e0, __uint_as_float(s0[e]), __uint_as_float(s0[e + 1]));
          e1 = max3f(e1, __uint_as_float(s0[e + 2]), __uint_as_float(s0[e + 3]));
          e2 = max3f(e2, __uint_as_float(s1[e]), __uint_as_float(s1[e + 1]));
          e3 = max3f(e3, __uint_as_float(s1[e + 2]), __uint_as_float(s1[e + 3]));
        }
      } else {
#pragma unroll
        for (int e = 0; e < 32; e += 4) {
          e0 = min3f(e0, __uint_as_float(s0[e]), __uint_as_float(s0[e + 1]));
          e1 = min3f(e1, __uint_as_float(s0[e + 2]), __uint_as_float(s0[e + 3]));
          e2 = min3f(e2, __uint_as_float(s1[e]), __uint_as_float(s1[e + 1]));
          e3 = min3f(e3, __uint_as_float(s1[e + 2]), __uint_as_float(s1[e + 3]));
        }
      }
    }
    mx = (pos ? max3f(e0, e1, fmaxf(e2, e3)) : min3f(e0, e1, fminf(e2, e3))) * scale_log2;
  }
  const float alpha = move_max(mx, m_run);
  const uint64_t sc2 = f2_pack(scale_log2, scale_log2), nm2 = f2_pack(-m_run, -m_run);
  uint64_t acc0 = 0ull, acc1 = 0ull;  // two packed partial sums (pairs of +0.0f)
  auto chunk = [&](const uint32_t (&r)[32], int q) {
    uint32_t pk[16];
#pragma unroll
    for (int e = 0; e < 16; ++e) {
      const uint64_t x = f2_fma(f2_pack(__uint_as_float(r[2 * e]), __uint_as_float(r[2 * e + 1])), sc2, nm2);
      float x0, x1;
      f2_unpack(x, x0, x1);
      const uint64_t pp = poly_pair<kDrop>(e)
                              ? exp2_fma2(f2_pack(fmaxf(x0, -125.f), fmaxf(x1, -125.f)))
                              : f2_pack(ex2(x0), ex2(x1));
      if (e & 1)
        acc1 = f2_add(acc1, pp);
      else
        acc0 = f2_add(acc0, pp);
      float p0, p1;
      f2_unpack(pp, p0, p1);
      if constexpr (kDrop) {  // xi only in the P operand; the sum keeps every term
        const uint64_t kw = q < 2 ? kb0 : kb1;
        const int bit = (q & 1) * 32 + 2 * e;
        p0 = ((kw >> bit) & 1ull) ? p0 : 0.f;
        p1 = ((kw >> (bit + 1)) & 1ull) ? p1 : 0.f;
      }
      pk[e] = pack16<kH>(p0, p1);
    }
    tmem_st16(tS + q * 16, pk);
  };
#pragma unroll 1
  for (int q = 0; q < 4; ++q) {
    uint32_t r[32];
    tmem_ld32(tS + 32 * q, r);
    tmem_wait_ld();
    chunk(r, q);
  }
  float a0, a1, b0, b1;
  f2_unpack(acc0, a0, a1);
  f2_unpack(acc1, b0, b1);
  l_run = l_run * alpha + ((a0 + a1) + (b0 + b1));
  return alpha;
}

// The full row (128 keys, all allowed) with dropout: the row's 128 scores
// loaded from TMEM at once (one wait), the maximum taken over them, then the
// exponentials, every one on MUFU (the softmax warps' FMA pipe also runs
// Philox4x32-10 here). With the keep bits' work in the same warps, the one
// load per row beats re-reading the row in passes.
template <bool kH>
__device__ __forceinline__ float softmax_full_tile_drop(uint32_t tS, float scale_log2, float& m_run, float& l_run,
                                                        uint64_t kb0, uint64_t kb1) {
  uint32_t s0[32], s1[32], s2[32], s3[32];
  tmem_ld32(tS, s0);
  tmem_ld32(tS + 32, s1);
  tmem_ld32(tS + 64, s2);
  tmem_ld32(tS + 96, s3);
  tmem_wait_ld();
  float mx;
  if (scale_log2 >= 0.f) {
    float e0 = -INFINITY, e1 = -INFINITY, e2 = -INFINITY, e3 = -INFINITY;
#pragma unroll
    for (int e = 0; e < 32; e += 2) {
      e0 = max3f(e0, __uint_as_float(s0[e]), __uint_as_float(s0[e + 1]));
      e1 = max3f(e1, __uint_as_float(s1[e]), __uint_as_float(s1[e + 1]));
      e2 = max3f(e2, __uint_as_float(s2[e]), __uint_as_float(s2[e + 1]));
      e3 = max3f(e3, __uint_as_float(s3[e]), __uint_as_float(s3[e + 1]));
    }
    mx = max3f(e0, e1, fmaxf(e2, e3)) * scale_log2;
  } else {
    float e0 = INFINITY, e1 = INFINITY, e2 = INFINITY, e3 = INFINITY;
#pragma unroll
    for (int e = 0; e < 32; e += 2) {
      e0 = min3f(e0, __uint_as_float(s0[e]), __uint_as_float(s0[e + 1]));
      e1 = min3f(e1, __uint_as_float(s1[e]), __uint_as_float(s1[e + 1]));
      e2 = min3f(e2, __uint_as_float(s2[e]), __uint_as_float(s2[e + 1]));
      e3 = min3f(e3, __uint_as_float(s3[e]), __uint_as_float(s3[e + 1]));
    }
    mx = min3f(e0, e1, fminf(e2, e3)) * scale_log2;
  }
  const float alpha = move_max(mx, m_run);
  const uint64_t sc2 = f2_pack(scale_log2, scale_log2), nm2 = f2_pack(-m_run, -m_run);
  uint64_t acc0 = 0ull, acc1 = 0ull;
  auto chunk = [&](const uint32_t (&r)[32], int q) {
    uint32_t pk[16];
    const uint64_t kw = q < 2 ? kb0 : kb1;
#pragma unroll
    for (int e = 0; e < 16; ++e) {
      float x0, x1;
      f2_unpack(f2_fma(f2_pack(__uint_as_float(r[2 * e]), __uint_as_float(r[2 * e + 1])), sc2, nm2), x0, x1);
      const uint64_t pp = f2_pack(ex2(x0), ex2(x1));
      if (e & 1)
        acc1 = f2_add(acc1, pp);
      else
        acc0 = f2_add(acc0, pp);
      float p0, p1;
      f2_unpack(pp, p0, p1);
      const int bit = (q & 1) * 32 + 2 * e;  // xi only in the P operand; the sum keeps every term
      pk[e] = pack16<kH>(((kw >> bit) & 1ull) ? p0 : 0.f, ((kw >> (bit + 1)) & 1ull) ? p1 : 0.f);
    }
    tmem_st16(tS + q * 16, pk);
  };
  chunk(s0, 0);
  chunk(s1, 1);
  chunk(s2, 2);
  chunk(s3, 3);
  float a0, a1, b0, b1;
  f2_unpack(acc0, a0, a1);
  f2_unpack(acc1, b0, b1);
  l_run = l_run * alpha + ((a0 + a1) + (b0 + b1));
  return alpha;
}

// The general row: allowed-key bits (mw0, mw1) and dropout keep bits
// (kb0, kb1) per key; two TMEM passes of 64 columns for the maximum, then 32
// columns per pass for the exponentials. The sum and the maximum use
// every allowed key (undropped); P carries only the kept ones (the 1/(1-rho)
// factor is applied to O in fp32 at the end). Returns alpha.
template <bool kH>
__device__ __forceinline__ float softmax_masked_tile(uint32_t tS, float scale_log2, uint64_t mw0, uint64_t mw1,
                                                     uint64_t kb0, uint64_t kb1, float& m_run, float& l_run) {
  float mx = -INFINITY;
#pragma unroll 1
  for (int hf = 0; hf < 2; ++hf) {
    uint32_t r0[32], r1[32];
    tmem_ld32(tS + hf * 64, r0);
    tmem_ld32(tS + hf * 64 + 32, r1);
    tmem_wait_ld();
    const uint64_t mw = hf ? mw1 : mw0;
#pragma unroll
    for (int e = 0; e < 32; ++e) {
      if ((mw >> e) & 1ull) mx = fmaxf(mx, __uint_as_float(r0[e]) * scale_log2);
      if ((mw >> (32 + e)) & 1ull) mx = fmaxf(mx, __uint_as_float(r1[e]) * scale_log2);
    }
  }
  const float alpha = move_max(mx, m_run);
  const float msub = m_run == -INFINITY ? 0.f : m_run;
  float sum = 0.f;
#pragma unroll 1
  for (int q = 0; q < 4; ++q) {
    uint32_t r[32];
    tmem_ld32(tS + q * 32, r);
    tmem_wait_ld();
    const uint64_t mw = q < 2 ? mw0 : mw1;
    const uint64_t kw = q < 2 ? kb0 : kb1;
    const int base = (q & 1) * 32;
    uint32_t pk[16];
#pragma unroll
    for (int e = 0; e < 16; ++e) {
      const int bit = base + 2 * e;
      const float p0 = ((mw >> bit) & 1ull) ? ex2(__uint_as_float(r[2 * e]) * scale_log2 - msub) : 0.f;
      const float p1 = ((mw >> (bit + 1)) & 1ull) ? ex2(__uint_as_float(r[2 * e + 1]) * scale_log2 - msub) : 0.f;
      sum += p0 + p1;
      pk[e] = pack16<kH>(((kw >> bit) & 1ull) ? p0 : 0.f, ((kw >> (bit + 1)) & 1ull) ? p1 : 0.f);
    }
    tmem_st16(tS + q * 16, pk);
  }
  l_run = l_run * alpha + sum;
  return alpha;
}

// Two query tiles per CTA, one softmax warpgroup each, alternating on the
// tensor core: while one warpgroup turns its S tile into P, the MMA issuer
// runs the other warpgroup's P V and next S. P (bf16 pairs) is written back
// into the warpgroup's own S columns of TMEM and read from there by the PV
// MMA; S of the next tile lands in the same columns only after that PV, in
// issue order.
template <bool kH, bool kDrop>
__global__ void __launch_bounds__(kFwdThreads, 1)
fwd_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
           const __grid_constant__ CUtensorMap tv, const FwdArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  FwdCtl* ctl = reinterpret_cast<FwdCtl*>(smem + kFwdCtl);
  volatile uint32_t* abort_flag = &ctl->abort_flag;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // Bands of kFwdBand (batch row, query head) pairs; within a band the
  // longest query tiles (most keys under a causal mask) go first. The CTAs
  // resident at any time then read the K/V tiles of a few heads (adjacent
  // query heads share their K/V head), which stay in L2 for every query tile
  // that reuses them, and the tail of the launch is made of short tiles.
  const int nct = (a.Tq + kFwdRows - 1) / kFwdRows;
  const int nbh = a.B * a.Hq;
  const int band0 = (int)(blockIdx.x / ((int64_t)kFwdBand * nct)) * kFwdBand;
  const int bw = nbh - band0 < kFwdBand ? nbh - band0 : kFwdBand;
  const int within = (int)(blockIdx.x - (int64_t)band0 * nct);
  const int bh = band0 + within % bw;
  const int ct = nct - 1 - within / bw;
  const int h = bh % a.Hq, b = bh / a.Hq;
  const int kvh = h / (a.Hq / a.Hkv);
  const int q0 = ct * kFwdRows;
  const int qt0 = 2 * ct;
  int kt_lo, kt_hi;
  fwd_key_tiles(a.m, b, a.Tq, a.Tk, q0, kFwdRows, kt_lo, kt_hi);

  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&ctl->q_full), 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(smem_u32(&ctl->k_full[s]), 1);
      mbar_init(smem_u32(&ctl->v_full[s]), 1);
      mbar_init(smem_u32(&ctl->kv_empty[s]), 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(smem_u32(&ctl->s_full[s]), 1);
      mbar_init(smem_u32(&ctl->p_full[s]), 4);  // one arrival per softmax warp
    }
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
  // TMEM columns: S/P of warpgroup w at 128 w, O of warpgroup w at 256 + 128 w.

  if (warp == 0 && lane == 0) {
    // ---------------- TMA producer
    tma_prefetch_desc(&tq);
    tma_prefetch_desc(&tk);
    tma_prefetch_desc(&tv);
    const uint32_t qf = smem_u32(&ctl->q_full);
    mbar_expect_tx(qf, 2 * kTileBytes);
#pragma unroll
    for (int w = 0; w < 2; ++w) {
      tma_load_4d(sbase + kFwdQ + w * kTileBytes, &tq, qf, 0, q0 + w * kBM, h, b);
      tma_load_4d(sbase + kFwdQ + w * kTileBytes + kTileBytes / 2, &tq, qf, 64, q0 + w * kBM, h, b);
    }
    // The tile walk (and its mask classes) runs here, ahead of the MMA
    // issuer, which reads each stage's flags from tinfo.
    int n = 0;
    uint32_t fl;
    for (int kt = fwd_next_tile(a, b, h, qt0, kt_hi, kt_lo - 1, fl); kt <= kt_hi;) {
      uint32_t nfl;
      const int nk = fwd_next_tile(a, b, h, qt0, kt_hi, kt, nfl);
      const int s = n % kStages;
      if (!wait_bar(smem_u32(&ctl->kv_empty[s]), ((n / kStages) & 1) ^ 1, abort_flag, a.status)) break;
      ctl->tinfo[s] = fl | (nk <= kt_hi ? 4u : 0u);  // published by the release of the arrive below
      const uint32_t kf = smem_u32(&ctl->k_full[s]), vf = smem_u32(&ctl->v_full[s]);
      const uint32_t kd = sbase + kFwdK + s * kTileBytes, vd = sbase + kFwdV + s * kTileBytes;
      mbar_expect_tx(kf, kTileBytes);
      tma_load_4d(kd, &tk, kf, 0, kt * kBN, kvh, b);
      tma_load_4d(kd + kTileBytes / 2, &tk, kf, 64, kt * kBN, kvh, b);
      mbar_expect_tx(vf, kTileBytes);
      tma_load_4d(vd, &tv, vf, 0, kt * kBN, kvh, b);
      tma_load_4d(vd + kTileBytes / 2, &tv, vf, 64, kt * kBN, kvh, b);
      ++n;
      kt = nk;
      fl = nfl;
    }
    for (int r = (n > kStages ? n - kStages : 0); r < n; ++r) {
      const int s = r % kStages;
      wait_bar(smem_u32(&ctl->k_full[s]), (r / kStages) & 1, abort_flag, nullptr);
      wait_bar(smem_u32(&ctl->v_full[s]), (r / kStages) & 1, abort_flag, nullptr);
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer: the whole warp runs the loop (warp-uniform
    // waits and descriptor arithmetic), one elected lane issues the MMAs.
    const bool leader = elect_one();
    constexpr uint32_t idS = idesc16<kH>(128, 128, 0, 0);
    constexpr uint32_t idPV = idesc16<kH>(128, 128, 0, 1);
    bool ok = __all_sync(0xffffffffu, wait_bar(smem_u32(&ctl->q_full), 0, abort_flag, a.status));
    // Descriptors of every operand tile, formed once; a K step adds its byte
    // offset >> 4 to the start-address field.
    const uint64_t dQ0 = smem_desc_sw128(sbase + kFwdQ, 16, 1024), dK0 = smem_desc_sw128(sbase + kFwdK, 16, 1024);
    const uint64_t dV0 = smem_desc_sw128(sbase + kFwdV, kTileBytes / 2, 1024);
    constexpr uint64_t kTileStep = kTileBytes >> 4;  // one 32 KB tile further
    auto dQ = [&](int i) { return dQ0 + (uint64_t)i * kTileStep; };
    auto dK = [&](int i) { return dK0 + (uint64_t)i * kTileStep; };
    auto dV = [&](int i) { return dV0 + (uint64_t)i * kTileStep; };
    auto issue_s = [&](int w, int stage) {
      if (leader) {
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t off = ((kk >> 2) * (kTileBytes / 2) + (kk & 3) * 32) >> 4;
          mma_ss(tmem + w * 128, dQ(w) + off, dK(stage) + off, idS, kk > 0);
        }
        mma_commit(smem_u32(&ctl->s_full[w]));
      }
      __syncwarp();
    };
    uint32_t fl0;
    const bool any = fwd_next_tile(a, b, h, qt0, kt_hi, kt_lo - 1, fl0) <= kt_hi;
    uint32_t info = 0;
    int npv[2] = {0, 0};
    int n = 0;
    if (ok && any) {
      ok = __all_sync(0xffffffffu, wait_bar(smem_u32(&ctl->k_full[0]), 0, abort_flag, a.status));
      if (ok) {
        tc_fence_after();
        info = ctl->tinfo[0];
        for (int w = 0; w < 2; ++w)
          if ((info >> w) & 1u) issue_s(w, 0);
      }
    }
    while (ok && any) {
      const int s = n % kStages, s1 = (n + 1) % kStages;
      const bool more = info & 4u;
      uint32_t ninfo = 0;
      for (int w = 0; w < 2 && ok; ++w) {
        if ((info >> w) & 1u) {
          if (!(ok = __all_sync(0xffffffffu, wait_bar(smem_u32(&ctl->p_full[w]), npv[w] & 1, abort_flag, a.status))))
            break;
          if (!(ok = __all_sync(0xffffffffu,
                                wait_bar(smem_u32(&ctl->v_full[s]), (n / kStages) & 1, abort_flag, a.status))))
            break;
          tc_fence_after();
          if (leader) {
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)  // A = P in TMEM: 16 keys = 8 packed columns per step
              mma_ts(tmem + 256 + w * 128, tmem + w * 128 + kk * 8, dV(s) + (uint64_t)(kk * (2048 >> 4)), idPV,
                     (npv[w] > 0 || kk > 0) ? 1u : 0u);
          }
          __syncwarp();
          ++npv[w];
        }
        if (more) {
          if (w == 0) {
            if (!(ok = __all_sync(0xffffffffu,
                                  wait_bar(smem_u32(&ctl->k_full[s1]), ((n + 1) / kStages) & 1, abort_flag, a.status))))
              break;
            tc_fence_after();
            ninfo = ctl->tinfo[s1];
          }
          if ((ninfo >> w) & 1u) issue_s(w, s1);
        }
      }
      if (!ok) break;
      if (leader) mma_commit(smem_u32(&ctl->kv_empty[s]));
      __syncwarp();
      if (!more) break;
      info = ninfo;
      ++n;
    }
    if (leader) mma_commit(smem_u32(&ctl->o_final));
    __syncwarp();
  } else if (warp >= 2) {
    // ---------------- softmax warpgroups: thread t of warpgroup w owns query row
    // q0 + 128 w + t (TMEM lane t of that warpgroup's S/P and O columns).
    const int w = (warp - 2) >> 2;
    const int qt = 2 * ct + w;
    const int t = ((warp & 3) << 5) | lane;
    const int64_t row = (int64_t)q0 + w * kBM + t;
    const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
    const uint32_t tS = tmem + lane_off + w * 128, tO = tmem + lane_off + 256 + w * 128;
    float m_run = -INFINITY, l_run = 0.f;  // base-2 running max and running sum
    int n = 0;
    bool ok = true;
    // Tile classes, 32 key tiles per round: lane l holds tile cbase + l
    // (bits 0-1: this query tile, bits 2-3: this warp's 64-row slice).
    int cbase = kt_lo - 32;
    uint32_t cword = 0;
    for (int kt = kt_lo; kt <= kt_hi && ok; ++kt) {
      if (kt - cbase >= 32) {
        cbase = kt;
        const int mk = kt + lane;
        cword = 0;
        if (mk <= kt_hi) {
          cword = wg_class(a, b, h, qt, mk);
          if (cword == kPartial)
            cword |= ((uint32_t)lookup_class(a.ct, a.m, a.Tq, a.Tk, b, h, 2 * qt + (t >> 6), mk) & 3u) << 2;
        }
      }
      const uint32_t cv = __shfl_sync(0xffffffffu, cword, kt - cbase);
      const uint8_t cls = cv & 3u;
      if (cls == kEmpty) continue;
      uint64_t mw0 = ~0ull, mw1 = ~0ull;
      if (cls == kPartial) {
        mw0 = mw1 = 0ull;
        if (row < a.Tq) fwd_row_bits(a, b, h, row, (int64_t)kt * kBN, (uint8_t)(cv >> 2), mw0, mw1);
      }
      uint64_t kb0 = ~0ull, kb1 = ~0ull;
      if constexpr (kDrop) fwd_keep_bits(a.m, b, h, row, (int64_t)kt * kBN, kb0, kb1);
      ok = __all_sync(0xffffffffu, wait_bar(smem_u32(&ctl->s_full[w]), n & 1, abort_flag, a.status));
      if (!ok) break;
      tc_fence_after();
      float alpha;
      if (cls == kFull)
        alpha = kDrop ? softmax_full_tile_drop<kH>(tS, a.scale_log2, m_run, l_run, kb0, kb1)
                      : softmax_full_tile<kH, kDrop>(tS, a.scale_log2, m_run, l_run, kb0, kb1);
      else
        alpha = softmax_masked_tile<kH>(tS, a.scale_log2, mw0, mw1, kb0, kb1, m_run, l_run);
      // Every earlier P V of this warpgroup has completed (the S commit covers
      // them) and the next one waits for p_full: O can be rescaled in place.
      if (n > 0 && __any_sync(0xffffffffu, alpha != 1.f)) {
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
          uint32_t o[32];
          tmem_ld32(tO + c * 32, o);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
          tmem_st32(tO + c * 32, o);
        }
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&ctl->p_full[w]));
      ++n;
    }
    // ---------------- epilogue: Y = u / (l + exp(z - m)), LSE = m + ln(...)
    bool have_o = false;
    if (ok && n > 0) {
      ok = __all_sync(0xffffffffu, wait_bar(smem_u32(&ctl->o_final), 0, abort_flag, a.status));
      if (ok) tc_fence_after();
      have_o = ok;
    }
    if (ok) {
      const bool has_sink = a.m.sink != nullptr;
      const float z2 = has_sink ? a.m.sink[h] * kLog2e : -INFINITY;
      float lse2, oscale;
      if (m_run == -INFINITY || !have_o) {
        lse2 = has_sink ? z2 : -INFINITY;
        oscale = 0.f;
      } else {
        const float M = has_sink ? fmaxf(m_run, z2) : m_run;
        const float tot = l_run * exp2f(m_run - M) + (has_sink ? exp2f(z2 - M) : 0.f);
        oscale = exp2f(m_run - M) / tot;
        if (a.m.dropout) oscale *= a.m.inv_keep;
        lse2 = M + log2f(tot);
      }
      uint16_t* orow = a.o + b * a.so[0] + h * a.so[1] + row * a.so[2];
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t o[32];
        if (have_o) {
          tmem_ld32(tO + c * 32, o);
          tmem_wait_ld();
        }
        if (row < a.Tq) {
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
      if (row < a.Tq) a.lse[b * a.sl[0] + h * a.sl[1] + row * a.sl[2]] = stored_lse_log2(a.m.lse_fmt, lse2, m_run, l_run);
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

struct BwdArgs {
  MaskP m;
  ClassTable ct;
  int B, Hq, Hkv, Tq, Tk, Tpad;
  int block_aligned;
  float scale_log2;
  const float* lse2;    // [B*Hq, Tpad] minus the base-2 LSE (-inf on rows without keys)
  const float* dpad;    // [B*Hq, Tpad] minus delta, zero on padding rows
  float* dq_acc;        // [B, Hq, Tq, 128] fp32
  uint16_t* dk;  // 16-bit storage: bf16 or fp16
  int64_t sdk[3];
  uint16_t* dv;
  int64_t sdv[3];
  float scale;
  uint32_t* status;
};

constexpr uint32_t kHalfQ = kBMb * 64 * 2;  // 8 KB: 64 rows x 64 bf16
constexpr uint32_t kQTile = kBMb * kD * 2;  // 16 KB: 64 rows x 128 bf16
constexpr uint32_t kPTile = kBN * kBMb * 2; // 16 KB: 128 keys x 64 queries bf16
constexpr uint32_t kBwdK = 0;
constexpr uint32_t kBwdV = kBwdK + kTileBytes;
constexpr int kQStages = 3;                             // Q / dO / LSE / delta ring depth
constexpr int kBwdBand = 8;                             // (b, K/V head) pairs per scheduling band
constexpr bool kBwdDqFirst = true;                      // issue a step's dQ^T product before its dV, dK
constexpr uint32_t kBwdQ = kBwdV + kTileBytes;          // kQStages x 16 KB
constexpr uint32_t kBwdG = kBwdQ + kQStages * kQTile;   // kQStages x 16 KB
constexpr uint32_t kBwdDS = kBwdG + kQStages * kQTile;  // 2 buffers of gamma^T (P^T lives in TMEM)
constexpr uint32_t kBwdDQ = kBwdDS + 2 * kPTile;        // 4 warps x (64 rows x 32 fp32) = 32 KB
constexpr uint32_t kBwdStat = kBwdDQ + 4 * kBMb * 32 * 4;  // kQStages x (64 lse2 + 64 delta) fp32
constexpr uint32_t kBwdCtl = kBwdStat + kQStages * 512;
constexpr uint32_t kBwdSmem = kBwdCtl + 256 + 1024;     // control block + alignment slack
// Warps: 0 TMA producer, 1 MMA issuer, 2-3 idle, 4-7 and 8-11 the two compute
// warpgroups (query columns 0-31 and 32-63 of each step), 12-15 dQ warpgroup.
constexpr int kBwdThreads = 512;

struct BwdCtl {
  uint64_t kv_full;
  uint64_t q_full[kQStages], q_empty[kQStages];
  // Buffer reuse needs no "empty" barriers for S^T/dP^T, P~^T and gamma^T:
  // the MMA issuer writes S^T(n + 2) only after ds_full(n), and st_full(n + 2)
  // commits after the dV, dK, dQ^T products of step n that read them.
  uint64_t st_full[2];
  uint64_t ds_full[2];
  uint64_t dq_full[2], dq_empty[2];
  uint64_t acc_done;
  uint32_t tmem_base;
  uint32_t abort_flag;
  // Per Q/dO stage, written by the producer before the stage's loads:
  // word 0 = query slice | class << 28 | (another step follows) << 30,
  // word 1 = query head within the group.
  uint32_t qinfo[kQStages][2];
};

// Query-slice range [lo, hi] that can hold rows seeing keys [k0, k0 + 128).
__device__ __forceinline__ void bwd_query_slices(const MaskP& m, int b, int Tq, int k0, int& lo, int& hi) {
  const int nqs = (Tq + kBMb - 1) / kBMb;
  lo = 0;
  hi = nqs - 1;
  if (m.flags & ATTN_MASK_CAUSAL) {  // rows whose key position reaches k0
    const int64_t first = (int64_t)k0 - m.qoff;
    if (first > 0) lo = first / kBMb < nqs ? (int)(first / kBMb) : nqs;
  }
  if (m.flags & ATTN_MASK_WINDOW) {  // rows whose window still reaches the tile's last key
    const int64_t last = (int64_t)k0 + kBN - 1 + m.window - 1 - m.qoff;
    if (last < 0)
      hi = -1;
    else if (last < Tq)
      hi = (int)(last / kBMb);
  }
  if (m.lengths) {  // Tq = Tk here
    const int64_t L = active_len(m, b, Tq);
    if (k0 >= L)
      hi = -1;
    else if ((L - 1) / kBMb < hi)
      hi = (int)((L - 1) / kBMb);
  }
}

// The next nonempty (query head in group, query slice) after (hh, qs).
__device__ __forceinline__ bool bwd_next_step(const BwdArgs& a, int b, int kvh, int kt, int group, int qs_lo,
                                              int qs_hi, int& hh, int& qs, uint8_t& cls) {
  if (qs_lo > qs_hi) return false;
  while (true) {
    if (++qs > qs_hi) {
      if (++hh >= group) return false;
      qs = qs_lo;
    }
    cls = lookup_class(a.ct, a.m, a.Tq, a.Tk, b, kvh * group + hh, qs, kt);
    if (cls != kEmpty) return true;
  }
}

// Rows i0..i0+63 that the active length and the per-row starts allow to see
// key j (bit c <-> i0 + c). Out of line, like clip_row_keys.
__device__ __noinline__ uint64_t col_rows_allowed(const int32_t* lengths, const int32_t* starts, int64_t st_sb, int b,
                                                  int64_t i0, int64_t j, int64_t Tq) {
  int64_t hi = i0 + kBMb - 1 < Tq - 1 ? i0 + kBMb - 1 : Tq - 1;
  if (lengths) {
    int64_t L = lengths[b];
    L = L < 0 ? 0 : (L > Tq ? Tq : L);
    if (j >= L) return 0ull;
    hi = L - 1 < hi ? L - 1 : hi;
  }
  uint64_t w = range_bits64(0, hi - i0);
  if (w && starts) {
    uint64_t sb = 0;
#pragma unroll 1
    for (int c = 0; c < kBMb; ++c)
      if (i0 + c <= hi && starts[b * st_sb + i0 + c] <= j) sb |= 1ull << c;
    w &= sb;
  }
  return w;
}

// Allowed query rows i0..i0+63 for key j, as a 64-bit word (bit c <-> i0 + c).
__device__ __forceinline__ uint64_t bwd_col_bits(const BwdArgs& a, int b, int h, int64_t i0, int64_t j) {
  if (j >= a.Tk) return 0ull;
  int64_t lo = i0, hi = i0 + kBMb - 1;
  if (hi > a.Tq - 1) hi = a.Tq - 1;
  if (a.m.flags & ATTN_MASK_CAUSAL) lo = j - a.m.qoff > lo ? j - a.m.qoff : lo;  // row i sees j iff i + qoff >= j
  if (a.m.flags & ATTN_MASK_WINDOW)
    hi = j + a.m.window - 1 - a.m.qoff < hi ? j + a.m.window - 1 - a.m.qoff : hi;
  uint64_t w = range_bits64(lo - i0, hi - i0);
  if (w && (a.m.flags & (ATTN_MASK_LENGTHS | ATTN_MASK_STARTS))) w &= col_rows_allowed(a.m.lengths, a.m.starts, a.m.st_sb, b, i0, j, a.Tq);
  if (w && (a.m.flags & ATTN_MASK_BLOCK) && !a.block_aligned) {
    const uint8_t* base = a.m.bm + b * a.m.bm_sb + h * a.m.bm_sh + j / a.m.bk;
    uint64_t bb = 0;
#pragma unroll 1
    for (int c = 0; c < kBMb; ++c)
      if (i0 + c < a.Tq && base[((i0 + c) / a.m.bq) * a.m.bm_sq]) bb |= 1ull << c;
    w &= bb;
  }
  return w;
}

// Keep bits xi for key j and query rows i0..i0+31 (bit c <-> row i0 + c).
// One Philox block (j >> 2, i, h, b) holds the words of keys 4(j >> 2) .. +3,
// i.e. of the four lanes that share j >> 2 (keys k0 + t with k0 a multiple of
// 4). Those lanes split the 32 rows, 8 blocks each, and trade their keep
// nibbles, so every block is evaluated once. Whole warp, converged.
__device__ __forceinline__ uint32_t bwd_keep_bits(const MaskP& m, int b, int h, int64_t i0, int64_t j) {
  const int lane = threadIdx.x & 31, e = lane & 3;
  uint32_t nib = 0;  // 4 keep bits (keys 4(j >> 2) + 0..3) per row, rows 8e .. 8e+7
#pragma unroll 1
  for (int c = 0; c < 8; ++c) {
    const uint4 w = philox4x32_10(make_uint4((uint32_t)(j >> 2), (uint32_t)(i0 + 8 * e + c), (uint32_t)h, (uint32_t)b),
                                  m.seed_lo, m.seed_hi);
    nib |= ((uint32_t)(w.x >= m.keep_thr) | ((uint32_t)(w.y >= m.keep_thr) << 1) |
            ((uint32_t)(w.z >= m.keep_thr) << 2) | ((uint32_t)(w.w >= m.keep_thr) << 3))
           << (4 * c);
  }
  const int base = lane & ~3, word = (int)(j & 3);
  uint32_t keep = 0;
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const uint32_t nq = __shfl_sync(0xffffffffu, nib, base + q);
#pragma unroll
    for (int c = 0; c < 8; ++c) keep |= ((nq >> (4 * c + word)) & 1u) << (8 * q + c);
  }
  return keep;
}

// Element-wise add of a shared-memory box into global memory through a tensor
// map; boxes reaching past the tensor's extent are clipped.
__device__ __forceinline__ void tma_reduce_add_3d(const CUtensorMap* map, uint32_t ssrc, int c0, int c1, int c2) {
  asm volatile("cp.reduce.async.bulk.tensor.3d.global.shared::cta.add.bulk_group [%0, {%2, %3, %4}], [%1];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(ssrc), "r"(c0), "r"(c1), "r"(c2)
               : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_read0() {
  asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}
__device__ __forceinline__ void bulk_wait0() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

// The element math of one 32-column pass of a reverse step, for the
// calling thread's key row: from S^T and dP^T (rs, rp) and the columns'
// -LSE (base 2) and -delta (nl, nd), P~^T and gamma^T as 16-bit pairs.
// Full tiles: x = s c log2(e) - LSE, p = 2^x, gamma = p (dP - delta) on
// packed fp32 pairs, -LSE and -delta as broadcast 16-byte loads. Partial
// tiles: per column, with the allowed-row bits. With dropout, xi enters the
// P~ operand and dP (p itself stays undropped; dV is scaled by 1/(1-rho) at
// the end).
template <bool kH, bool kDrop>
__device__ __forceinline__ void bwd_chunk_math(const uint32_t (&rs)[32], const uint32_t (&rp)[32], const float* nl,
                                               const float* nd, bool general, uint32_t allow, uint32_t keep,
                                               float scale_log2, float inv_keep, int dropout, uint32_t (&ppk)[16],
                                               uint32_t (&dpk)[16]) {
  if (!general) {
    const uint64_t sc2 = f2_pack(scale_log2, scale_log2);
#pragma unroll
    for (int c4 = 0; c4 < 8; ++c4) {
      const float4 l4 = *reinterpret_cast<const float4*>(nl + 4 * c4);
      const float4 d4 = *reinterpret_cast<const float4*>(nd + 4 * c4);
      const uint64_t lp[2] = {f2_pack(l4.x, l4.y), f2_pack(l4.z, l4.w)};
      const uint64_t dp[2] = {f2_pack(d4.x, d4.y), f2_pack(d4.z, d4.w)};
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int c2 = 2 * c4 + e;
        float x0, x1;
        f2_unpack(f2_fma(f2_pack(__uint_as_float(rs[2 * c2]), __uint_as_float(rs[2 * c2 + 1])), sc2, lp[e]), x0, x1);
        const float p0 = ex2(x0), p1 = ex2(x1);
        uint64_t dv2 = f2_pack(__uint_as_float(rp[2 * c2]), __uint_as_float(rp[2 * c2 + 1]));
        if constexpr (kDrop) {
          const bool k0 = (keep >> (2 * c2)) & 1u, k1 = (keep >> (2 * c2 + 1)) & 1u;
          ppk[c2] = pack16<kH>(k0 ? p0 : 0.f, k1 ? p1 : 0.f);
          dv2 = f2_pack(k0 ? __uint_as_float(rp[2 * c2]) * inv_keep : 0.f,
                        k1 ? __uint_as_float(rp[2 * c2 + 1]) * inv_keep : 0.f);
        } else {
          ppk[c2] = pack16<kH>(p0, p1);
        }
        const uint64_t g = f2_mul(f2_pack(p0, p1), f2_add(dv2, dp[e]));
        float g0, g1;
        f2_unpack(g, g0, g1);
        dpk[c2] = pack16<kH>(g0, g1);
      }
    }
  } else {
    const float inv = dropout ? inv_keep : 1.f;
#pragma unroll
    for (int c2 = 0; c2 < 16; ++c2) {
      float pt[2], ds[2];
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int cc = 2 * c2 + e;
        const float p = ((allow >> cc) & 1u) ? ex2(fmaf(__uint_as_float(rs[cc]), scale_log2, nl[cc])) : 0.f;
        const bool kp = (keep >> cc) & 1u;
        pt[e] = kp ? p : 0.f;
        const float dpv = kp ? __uint_as_float(rp[cc]) * inv : 0.f;
        ds[e] = p * (dpv + nd[cc]);
      }
      ppk[c2] = pack16<kH>(pt[0], pt[1]);
      dpk[c2] = pack16<kH>(ds[0], ds[1]);
    }
  }
}

// kDQ = false (the deterministic mode) leaves dQ to the query-centric pass:
// no dQ^T product, no dQ warpgroup work.
template <bool kH, bool kDQ, bool kDrop>
__global__ void __launch_bounds__(kBwdThreads, 1)
bwd_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
           const __grid_constant__ CUtensorMap tv, const __grid_constant__ CUtensorMap tg,
           const __grid_constant__ CUtensorMap tdq, const BwdArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  BwdCtl* ctl = reinterpret_cast<BwdCtl*>(smem + kBwdCtl);
  volatile uint32_t* abort_flag = &ctl->abort_flag;
  const float* stat = reinterpret_cast<const float*>(smem + kBwdStat);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int group = a.Hq / a.Hkv;
  // Bands of kBwdBand (b, K/V head) pairs: within a band the earliest key tiles
  // (most work under a causal mask) go first; the CTAs resident at any time
  // then share a few heads' dQ accumulator rows and Q/dO in L2.
  const int nkt_all = (a.Tk + kBN - 1) / kBN;
  const int nbkv = a.B * a.Hkv;
  const int band = (int)(blockIdx.x / ((int64_t)kBwdBand * nkt_all));
  const int band0 = band * kBwdBand;
  const int bw = nbkv - band0 < kBwdBand ? nbkv - band0 : kBwdBand;
  const int within = (int)(blockIdx.x - (int64_t)band0 * nkt_all);
  const int kt = within / bw;
  const int bkv = band0 + within % bw;
  const int kvh = bkv % a.Hkv, b = bkv / a.Hkv;
  const int k0 = kt * kBN;
  int qs_lo, qs_hi;
  bwd_query_slices(a.m, b, a.Tq, k0, qs_lo, qs_hi);

  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&ctl->kv_full), 1);
    for (int s = 0; s < kQStages; ++s) {
      mbar_init(smem_u32(&ctl->q_full[s]), 1);
      mbar_init(smem_u32(&ctl->q_empty[s]), 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(smem_u32(&ctl->st_full[s]), 1);
      mbar_init(smem_u32(&ctl->ds_full[s]), kDrop ? 4 : 8);  // one arrival per warp working on the step
      mbar_init(smem_u32(&ctl->dq_full[s]), 1);
      mbar_init(smem_u32(&ctl->dq_empty[s]), 4);  // one arrival per dQ warp
    }
    mbar_init(smem_u32(&ctl->acc_done), 1);
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
  // TMEM columns: two S^T | dP^T buffers (0..127, 128..255). In a step's
  // buffer, P~^T (bf16 pairs) is written over the dP^T half once read, and
  // dQ^T reuses the S^T half. dV 256..383, dK 384..511.
  const uint32_t tDV = tmem + 256, tDK = tmem + 384;

  if (warp == 0 && lane == 0) {
    // ---------------- TMA producer
    tma_prefetch_desc(&tq);
    tma_prefetch_desc(&tk);
    tma_prefetch_desc(&tv);
    tma_prefetch_desc(&tg);
    const uint32_t kvf = smem_u32(&ctl->kv_full);
    mbar_expect_tx(kvf, 2 * kTileBytes);
    tma_load_4d(sbase + kBwdK, &tk, kvf, 0, k0, kvh, b);
    tma_load_4d(sbase + kBwdK + kTileBytes / 2, &tk, kvf, 64, k0, kvh, b);
    tma_load_4d(sbase + kBwdV, &tv, kvf, 0, k0, kvh, b);
    tma_load_4d(sbase + kBwdV + kTileBytes / 2, &tv, kvf, 64, k0, kvh, b);
    // The step walk (query head, query slice, class) runs here, ahead of the
    // MMA issuer and the compute warpgroups, which read it from qinfo.
    int n = 0, hh = 0, qs = qs_lo - 1;
    uint8_t cls, ncls = 0;
    bool have = bwd_next_step(a, b, kvh, kt, group, qs_lo, qs_hi, hh, qs, cls);
    int nh = hh, nq = qs;
    bool next = have && bwd_next_step(a, b, kvh, kt, group, qs_lo, qs_hi, nh, nq, ncls);
    while (have) {
      int mh = nh, mq = nq;
      uint8_t mcls = 0;
      const bool next2 = next && bwd_next_step(a, b, kvh, kt, group, qs_lo, qs_hi, mh, mq, mcls);
      const int h = kvh * group + hh;
      const int s = n % kQStages;
      if (!wait_bar(smem_u32(&ctl->q_empty[s]), ((n / kQStages) & 1) ^ 1, abort_flag, a.status)) break;
      ctl->qinfo[s][0] =
          (uint32_t)qs | ((uint32_t)cls << 28) | (next ? 1u << 30 : 0u) | (next2 ? 1u << 31 : 0u);
      ctl->qinfo[s][1] = (uint32_t)hh;  // both published by the release of the arrive below
      const uint32_t qf = smem_u32(&ctl->q_full[s]);
      mbar_expect_tx(qf, 2 * kQTile + 512);
      const uint32_t qd = sbase + kBwdQ + s * kQTile, gd = sbase + kBwdG + s * kQTile;
      tma_load_4d(qd, &tq, qf, 0, qs * kBMb, h, b);
      tma_load_4d(qd + kHalfQ, &tq, qf, 64, qs * kBMb, h, b);
      tma_load_4d(gd, &tg, qf, 0, qs * kBMb, h, b);
      tma_load_4d(gd + kHalfQ, &tg, qf, 64, qs * kBMb, h, b);
      const int64_t roff = ((int64_t)b * a.Hq + h) * a.Tpad + (int64_t)qs * kBMb;
      bulk_load(sbase + kBwdStat + s * 512, a.lse2 + roff, 256, qf);
      bulk_load(sbase + kBwdStat + s * 512 + 256, a.dpad + roff, 256, qf);
      ++n;
      hh = nh;
      qs = nq;
      cls = ncls;
      have = next;
      nh = mh;
      nq = mq;
      ncls = mcls;
      next = next2;
    }
    for (int r = (n > kQStages ? n - kQStages : 0); r < n; ++r)
      wait_bar(smem_u32(&ctl->q_full[r % kQStages]), (r / kQStages) & 1, abort_flag, nullptr);
    wait_bar(kvf, 0, abort_flag, nullptr);
  } else if (warp == 1) {
    // ---------------- MMA issuer: S^T/dP^T of step n+1 go ahead of the
    // dV, dK, dQ^T products of step n so the tensor core overlaps the
    // compute warpgroup. The whole warp runs the loop (waits, step info,
    // descriptor arithmetic: warp-uniform values) and one elected lane
    // issues the MMAs and commits; issued from a lone thread, the same
    // loop spent about half again the tensor pipe's time issuing each group.
    const bool leader = elect_one();
    constexpr uint32_t idST = idesc16<kH>(128, 64, 0, 0);   // K Q^T, V dO^T
    constexpr uint32_t idACC = idesc16<kH>(128, 128, 0, 1); // P^T dO, dS^T Q  (B MN-major)
    constexpr uint32_t idDQ = idesc16<kH>(128, 64, 1, 1);   // K^T dS^T (A and B MN-major)
    bool ok = __all_sync(0xffffffffu, wait_bar(smem_u32(&ctl->kv_full), 0, abort_flag, a.status));
    // Descriptors formed once; a K step adds its byte offset >> 4.
    const uint64_t dK = smem_desc_sw128(sbase + kBwdK, 16, 1024), dV = smem_desc_sw128(sbase + kBwdV, 16, 1024);
    const uint64_t dKmn = smem_desc_sw128(sbase + kBwdK, kTileBytes / 2, 1024);
    // Stage i of a ring: the stage-0 descriptor plus i * (stage bytes >> 4).
    const uint64_t dQk0 = smem_desc_sw128(sbase + kBwdQ, 16, 1024), dGk0 = smem_desc_sw128(sbase + kBwdG, 16, 1024);
    const uint64_t dQmn0 = smem_desc_sw128(sbase + kBwdQ, kHalfQ, 1024);
    const uint64_t dGmn0 = smem_desc_sw128(sbase + kBwdG, kHalfQ, 1024);
    const uint64_t dDS0 = smem_desc_sw128(sbase + kBwdDS, 16, 1024);
    const uint64_t dDSmn0 = smem_desc_sw128(sbase + kBwdDS, kHalfQ, 1024);
    auto dQk = [&](int i) { return dQk0 + (uint64_t)(i * (kQTile >> 4)); };
    auto dGk = [&](int i) { return dGk0 + (uint64_t)(i * (kQTile >> 4)); };
    auto dQmn = [&](int i) { return dQmn0 + (uint64_t)(i * (kQTile >> 4)); };
    auto dGmn = [&](int i) { return dGmn0 + (uint64_t)(i * (kQTile >> 4)); };
    auto dDS = [&](int i) { return dDS0 + (uint64_t)(i * (kPTile >> 4)); };
    auto dDSmn = [&](int i) { return dDSmn0 + (uint64_t)(i * (kPTile >> 4)); };
    // Issue S^T and dP^T of step m; returns its qinfo word 0 (0 on abort).
    auto issue_st = [&](int m, uint32_t& info) -> bool {
      const int s = m & 1, sq = m % kQStages;
      const uint32_t par = (m >> 1) & 1;
      if (!__all_sync(0xffffffffu, wait_bar(smem_u32(&ctl->q_full[sq]), (m / kQStages) & 1, abort_flag, a.status)))
        return false;
      info = ctl->qinfo[sq][0];
      if (kDQ && !__all_sync(0xffffffffu, wait_bar(smem_u32(&ctl->dq_empty[s]), par ^ 1, abort_flag, a.status)))
        return false;
      tc_fence_after();
      const uint32_t dst = tmem + s * 128;
      if (leader) {
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t koff = ((kk >> 2) * (kTileBytes / 2) + (kk & 3) * 32) >> 4;
          const uint32_t qoff = ((kk >> 2) * kHalfQ + (kk & 3) * 32) >> 4;
          mma_ss(dst, dK + koff, dQk(sq) + qoff, idST, kk > 0);
        }
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t koff = ((kk >> 2) * (kTileBytes / 2) + (kk & 3) * 32) >> 4;
          const uint32_t qoff = ((kk >> 2) * kHalfQ + (kk & 3) * 32) >> 4;
          mma_ss(dst + 64, dV + koff, dGk(sq) + qoff, idST, kk > 0);
        }
        mma_commit(smem_u32(&ctl->st_full[s]));
      }
      __syncwarp();
      return true;
    };
    int hh0 = 0, qs0 = qs_lo - 1, n = 0;
    uint8_t cls0;
    bool have = ok && bwd_next_step(a, b, kvh, kt, group, qs_lo, qs_hi, hh0, qs0, cls0);
    uint32_t info = 0;
    if (have) ok = issue_st(0, info);
    while (ok && have) {
      const bool next = info & (1u << 30);
      uint32_t ninfo = 0;
      if (next && !(ok = issue_st(n + 1, ninfo))) break;
      const int s = n & 1, sq = n % kQStages;
      if (!(ok = __all_sync(0xffffffffu, wait_bar(smem_u32(&ctl->ds_full[s]), (n >> 1) & 1, abort_flag, a.status))))
        break;
      tc_fence_after();
      auto issue_dq = [&]() {
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)  // K = 128 keys
          mma_ss(tmem + s * 128, dKmn + (uint64_t)(kk * (2048 >> 4)), dDSmn(s) + (uint64_t)(kk * (2048 >> 4)), idDQ,
                 kk > 0);
      };
      // dQ^T first: the dQ warps drain it while dV and dK run, so its TMEM
      // columns are free again before S^T of step n + 2 is issued.
      if (leader) {
        if constexpr (kDQ && kBwdDqFirst) {
          issue_dq();
          mma_commit(smem_u32(&ctl->dq_full[s]));
        }
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)  // K = 64 query rows; A = P~^T from TMEM (16 rows = 8 columns)
          mma_ts(tDV, tmem + s * 128 + 64 + (kk >> 1) * 32 + (kk & 1) * 8, dGmn(sq) + (uint64_t)(kk * (2048 >> 4)),
                 idACC, (n > 0 || kk > 0) ? 1u : 0u);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          mma_ss(tDK, dDS(s) + (uint64_t)(kk * (32 >> 4)), dQmn(sq) + (uint64_t)(kk * (2048 >> 4)), idACC,
                 (n > 0 || kk > 0) ? 1u : 0u);
        if constexpr (kDQ && !kBwdDqFirst) issue_dq();
        mma_commit(smem_u32(&ctl->q_empty[sq]));
        if constexpr (kDQ && !kBwdDqFirst) mma_commit(smem_u32(&ctl->dq_full[s]));
      }
      __syncwarp();
      have = next;
      info = ninfo;
      ++n;
    }
    if (leader) mma_commit(smem_u32(&ctl->acc_done));
    __syncwarp();
  } else if (warp >= 4 && warp < 12) {
    // ---------------- compute warpgroups: thread t owns key row k0 + t. Step
    // n lives in S^T | dP^T buffer n & 1. Without dropout the two warpgroups
    // split every step's 64 query columns (warpgroup w: columns 32 w ..
    // 32 w + 31). With dropout (kAlt) each step carries Philox work as well,
    // and the warpgroups take alternate steps instead (warpgroup w: steps w,
    // w + 2, ..., all 64 columns as two passes of 32), so one warpgroup's
    // element math overlaps the other's waits for the tensor core.
    constexpr bool kAlt = kDrop;
    const int w = (warp - 4) >> 2;
    const int t = ((warp & 3) << 5) | lane;
    const int64_t j = (int64_t)k0 + t;
    const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
    bool ok = true;
    bool any, mine;  // the CTA has a step; this warpgroup's next step exists
    {
      int hh0 = 0, qs0 = qs_lo - 1;
      uint8_t cls0;
      any = bwd_next_step(a, b, kvh, kt, group, qs_lo, qs_hi, hh0, qs0, cls0);
      mine = any && (!kAlt || w == 0 || bwd_next_step(a, b, kvh, kt, group, qs_lo, qs_hi, hh0, qs0, cls0));
    }
    for (int n = kAlt ? w : 0; ok && mine; n += kAlt ? 2 : 1) {
      const int s = n & 1, sq = n % kQStages;
      const uint32_t par = (n >> 1) & 1;
      const uint32_t tbuf = tmem + lane_off + s * 128;  // the step's S^T | dP^T buffer
      // The stage's step info arrives with its Q/dO tiles, long before S^T.
      if (!(ok = __all_sync(0xffffffffu,
                            wait_bar(smem_u32(&ctl->q_full[sq]), (n / kQStages) & 1, abort_flag, a.status))))
        break;
      const uint32_t info = ctl->qinfo[sq][0];
      const int h = kvh * group + (int)ctl->qinfo[sq][1];
      const int qs = (int)(info & 0x0fffffffu);
      const uint8_t cls = (uint8_t)((info >> 28) & 3u);
      mine = kAlt ? (info >> 31) : ((info >> 30) & 1u);  // step n + 2 (n + 1) follows
      const int64_t i0 = (int64_t)qs * kBMb;
      const bool general = cls == kPartial;
      const uint64_t allow64 = general ? bwd_col_bits(a, b, h, i0, j) : ~0ull;
      // Keep bits of query columns 0-31 and 32-63, computed while S^T is on its way.
      uint32_t keep_lo = ~0u, keep_hi = ~0u;
      if constexpr (kDrop) {
        keep_lo = bwd_keep_bits(a.m, b, h, i0, j);
        keep_hi = bwd_keep_bits(a.m, b, h, i0 + 32, j);
      }
      if (!(ok = __all_sync(0xffffffffu, wait_bar(smem_u32(&ctl->st_full[s]), par, abort_flag, a.status)))) break;
      tc_fence_after();
      const uint32_t ds_base = sbase + kBwdDS + s * kPTile;
#pragma unroll 1
      for (int c = kAlt ? 0 : w; c < (kAlt ? 2 : w + 1); ++c) {
        const uint32_t allow = (uint32_t)(allow64 >> (32 * c));
        const uint32_t keep = c ? keep_hi : keep_lo;
        uint32_t rs[32], rp[32];
        tmem_ld32(tbuf + 32 * c, rs);
        tmem_ld32(tbuf + 64 + 32 * c, rp);
        const float* nl = stat + sq * 128 + 32 * c;       // -LSE (base 2) of the 32 columns
        const float* nd = stat + sq * 128 + 64 + 32 * c;  // -delta
        tmem_wait_ld();
        uint32_t ppk[16], dpk[16];
        bwd_chunk_math<kH, kDrop>(rs, rp, nl, nd, general, allow, keep, a.scale_log2, a.m.inv_keep, a.m.dropout, ppk,
                                  dpk);
        // P~^T as bf16 pairs over this pass's own dP^T columns (already read).
        tmem_st16(tbuf + 64 + 32 * c, ppk);
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) {
          const uint32_t off = sw128_offset(t, (c * 4 + cc) * 16);
          st_shared_v4(ds_base + off, dpk[cc * 4], dpk[cc * 4 + 1], dpk[cc * 4 + 2], dpk[cc * 4 + 3]);
        }
      }
      tmem_wait_st();
      tc_fence_before();
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&ctl->ds_full[s]));
    }
    // ---------------- epilogue: warpgroup 0 writes dK = c * sum gamma^T Q,
    // warpgroup 1 writes dV = sum P~^T dO (zeros when the CTA had no step).
    bool have = false;
    if (ok && any) {
      ok = __all_sync(0xffffffffu, wait_bar(smem_u32(&ctl->acc_done), 0, abort_flag, a.status));
      if (ok) tc_fence_after();
      have = ok;
    }
    const float osc = w == 0 ? a.scale : (a.m.dropout ? a.m.inv_keep : 1.f);
    if (ok) {
      uint16_t* orow = w == 0 ? a.dk + b * a.sdk[0] + kvh * a.sdk[1] + j * a.sdk[2]
                              : a.dv + b * a.sdv[0] + kvh * a.sdv[1] + j * a.sdv[2];
      const uint32_t tacc = (w == 0 ? tDK : tDV) + lane_off;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t r[32];
        if (have) {
          tmem_ld32(tacc + c * 32, r);
          tmem_wait_ld();
        }
        if (j < a.Tk) {
#pragma unroll
          for (int c8 = 0; c8 < 4; ++c8) {
            uint32_t pk[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int idx = c8 * 8 + e * 2;
              pk[e] = have ? pack16<kH>(__uint_as_float(r[idx]) * osc, __uint_as_float(r[idx + 1]) * osc) : 0u;
            }
            *reinterpret_cast<uint4*>(orow + c * 32 + c8 * 8) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
          }
        }
      }
    }
  } else if (kDQ && warp >= 12) {
    // ---------------- dQ warpgroup: warp wq reads head-dimension indices
    // 32 wq .. 32 wq + 31 of the dQ^T tile (its TMEM lanes), stages them as a
    // [64 rows][32] fp32 box and adds the box into the fp32 accumulator with
    // a TMA reduce; rows past T are clipped by the tensor map.
    const int wq = warp & 3;
    const uint32_t lane_off = (uint32_t)(wq * 32) << 16;
    const uint32_t stage_s = sbase + kBwdDQ + wq * (kBMb * 32 * 4);
    float* stage = reinterpret_cast<float*>(smem + kBwdDQ + wq * (kBMb * 32 * 4));
    if (lane == 0) tma_prefetch_desc(&tdq);
    int n = 0, hh = 0, qs = qs_lo - 1;
    uint8_t cls;
    bool ok = true;
    while (ok && bwd_next_step(a, b, kvh, kt, group, qs_lo, qs_hi, hh, qs, cls)) {
      const int h = kvh * group + hh;
      const int s = n & 1;
      if (!(ok = __all_sync(0xffffffffu, wait_bar(smem_u32(&ctl->dq_full[s]), (n >> 1) & 1, abort_flag, a.status))))
        break;
      tc_fence_after();
      uint32_t r0[32], r1[32];
      tmem_ld32(tmem + lane_off + s * 128, r0);
      tmem_ld32(tmem + lane_off + s * 128 + 32, r1);
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(smem_u32(&ctl->dq_empty[s]));
        bulk_wait_read0();  // the previous reduce has read this warp's box
      }
      __syncwarp();
#pragma unroll
      for (int e = 0; e < 32; ++e) {
        stage[e * 32 + lane] = __uint_as_float(r0[e]);
        stage[(32 + e) * 32 + lane] = __uint_as_float(r1[e]);
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        tma_reduce_add_3d(&tdq, stage_s, 32 * wq, qs * kBMb, b * a.Hq + h);
        bulk_commit();
      }
      ++n;
    }
    if (lane == 0) bulk_wait0();
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ---------------------------------------------- deterministic dQ (query-centric)
//
// dQ_i = c sum_j gamma_ij K_j evaluated per query tile, key tiles in order,
// with P and gamma recomputed from the saved statistics ("Tiled attention and
// its recomputed reverse pass are exact", proof step 7.1: the reverse rebuilds
// P from the scores and the stored normaliser). Every dQ element is summed by
// one CTA in a fixed order, so the result is bitwise reproducible; the
// key-centric kernel then leaves dQ alone.
//
// One CTA per (128-row query tile, query head, batch row). Warp 0: TMA
// producer (Q and dO once, then K/V stages). Warp 1: MMA issuer. Warps 2-9:
// two warpgroups that split each key tile's columns (warpgroup w: keys
// 64 w .. 64 w + 63); thread t of a warpgroup owns query row t (TMEM lane t).
// TMEM: S double-buffered at columns 0 and 128, dP at 256, dQ at 384. gamma
// (16-bit pairs) is written over the warpgroup's own S columns and read from
// there by the dQ MMA.

struct DqArgs {
  FwdArgs f;             // mask, class table, sizes (o, lse unused)
  const float* lse2;     // [B*Hq, Tpad] minus the base-2 LSE
  const float* dpad;     // [B*Hq, Tpad] minus delta
  uint16_t* dq;          // 16-bit storage
  int64_t sdq[3];
  float scale;
  int Tpad;
};

constexpr uint32_t kDqQ = 0;                              // Q tile
constexpr uint32_t kDqG = kDqQ + kTileBytes;              // dO tile
constexpr uint32_t kDqK = kDqG + kTileBytes;              // K stages
constexpr uint32_t kDqV = kDqK + kStages * kTileBytes;    // V stages
constexpr uint32_t kDqCtl = kDqV + kStages * kTileBytes;
constexpr uint32_t kDqSmem = kDqCtl + 1024 + 1024;
constexpr int kDqThreads = 320;

struct DqCtl {
  uint64_t q_full;
  uint64_t k_full[kStages], v_full[kStages], kv_empty[kStages];
  uint64_t s_full[2], dp_full, g_full;
  uint64_t dq_final;
  uint32_t tmem_base;
  uint32_t abort_flag;
};

// Next key tile after `from` (up to kt_hi) with allowed keys for query tile
// qt; kt_hi + 1 when none. Every role walks the same sequence.
__device__ __forceinline__ int dq_next_tile(const FwdArgs& a, int b, int h, int qt, int kt_hi, int from) {
  for (int kt = from + 1; kt <= kt_hi; ++kt)
    if (wg_class(a, b, h, qt, kt) != kEmpty) return kt;
  return kt_hi + 1;
}

template <bool kH>
__global__ void __launch_bounds__(kDqThreads, 1)
dq_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
          const __grid_constant__ CUtensorMap tv, const __grid_constant__ CUtensorMap tg, const DqArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  DqCtl* ctl = reinterpret_cast<DqCtl*>(smem + kDqCtl);
  volatile uint32_t* abort_flag = &ctl->abort_flag;
  const FwdArgs& f = a.f;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nqt = (f.Tq + kBM - 1) / kBM;
  const int bh = blockIdx.x % (f.B * f.Hq);
  const int qt = nqt - 1 - (int)(blockIdx.x / (f.B * f.Hq));  // longest rows first
  const int h = bh % f.Hq, b = bh / f.Hq;
  const int kvh = h / (f.Hq / f.Hkv);
  const int q0 = qt * kBM;
  int kt_lo, kt_hi;
  fwd_key_tiles(f.m, b, f.Tq, f.Tk, q0, kBM, kt_lo, kt_hi);

  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&ctl->q_full), 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(smem_u32(&ctl->k_full[s]), 1);
      mbar_init(smem_u32(&ctl->v_full[s]), 1);
      mbar_init(smem_u32(&ctl->kv_empty[s]), 1);
    }
    mbar_init(smem_u32(&ctl->s_full[0]), 1);
    mbar_init(smem_u32(&ctl->s_full[1]), 1);
    mbar_init(smem_u32(&ctl->dp_full), 1);
    mbar_init(smem_u32(&ctl->g_full), 8);  // one arrival per compute warp
    mbar_init(smem_u32(&ctl->dq_final), 1);
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
  const int first = dq_next_tile(f, b, h, qt, kt_hi, kt_lo - 1);

  if (warp == 0 && lane == 0) {
    // ---------------- TMA producer
    tma_prefetch_desc(&tq);
    tma_prefetch_desc(&tk);
    tma_prefetch_desc(&tv);
    tma_prefetch_desc(&tg);
    const uint32_t qf = smem_u32(&ctl->q_full);
    mbar_expect_tx(qf, 2 * kTileBytes);
    tma_load_4d(sbase + kDqQ, &tq, qf, 0, q0, h, b);
    tma_load_4d(sbase + kDqQ + kTileBytes / 2, &tq, qf, 64, q0, h, b);
    tma_load_4d(sbase + kDqG, &tg, qf, 0, q0, h, b);
    tma_load_4d(sbase + kDqG + kTileBytes / 2, &tg, qf, 64, q0, h, b);
    int n = 0;
    for (int kt = first; kt <= kt_hi; kt = dq_next_tile(f, b, h, qt, kt_hi, kt), ++n) {
      const int s = n % kStages;
      if (!wait_bar(smem_u32(&ctl->kv_empty[s]), ((n / kStages) & 1) ^ 1, abort_flag, f.status)) break;
      const uint32_t kf = smem_u32(&ctl->k_full[s]), vf = smem_u32(&ctl->v_full[s]);
      const uint32_t kd = sbase + kDqK + s * kTileBytes, vd = sbase + kDqV + s * kTileBytes;
      mbar_expect_tx(kf, kTileBytes);
      tma_load_4d(kd, &tk, kf, 0, kt * kBN, kvh, b);
      tma_load_4d(kd + kTileBytes / 2, &tk, kf, 64, kt * kBN, kvh, b);
      mbar_expect_tx(vf, kTileBytes);
      tma_load_4d(vd, &tv, vf, 0, kt * kBN, kvh, b);
      tma_load_4d(vd + kTileBytes / 2, &tv, vf, 64, kt * kBN, kvh, b);
    }
    for (int r = (n > kStages ? n - kStages : 0); r < n; ++r) {
      const int s = r % kStages;
      wait_bar(smem_u32(&ctl->k_full[s]), (r / kStages) & 1, abort_flag, nullptr);
      wait_bar(smem_u32(&ctl->v_full[s]), (r / kStages) & 1, abort_flag, nullptr);
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer (whole warp; one elected lane issues)
    const bool leader = elect_one();
    auto wait_all = [&](uint32_t bar, uint32_t par) {
      return __all_sync(0xffffffffu, wait_bar(bar, par, abort_flag, f.status));
    };
    constexpr uint32_t idS = idesc16<kH>(128, 128, 0, 0);   // Q K^T and dO V^T
    constexpr uint32_t idDQ = idesc16<kH>(128, 128, 0, 1);  // gamma K (B = K, d contiguous)
    const uint64_t dQ0 = smem_desc_sw128(sbase + kDqQ, 16, 1024), dG0 = smem_desc_sw128(sbase + kDqG, 16, 1024);
    const uint64_t dK0 = smem_desc_sw128(sbase + kDqK, 16, 1024), dV0 = smem_desc_sw128(sbase + kDqV, 16, 1024);
    const uint64_t dKmn0 = smem_desc_sw128(sbase + kDqK, kTileBytes / 2, 1024);
    constexpr uint64_t kTileStep = kTileBytes >> 4;
    auto kstep = [](int kk) { return (uint64_t)(((kk >> 2) * (kTileBytes / 2) + (kk & 3) * 32) >> 4); };
    auto issue_s = [&](int stage, int buf) {
      if (leader) {
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_ss(tmem + buf * 128, dQ0 + kstep(kk), dK0 + (uint64_t)stage * kTileStep + kstep(kk), idS, kk > 0);
        mma_commit(smem_u32(&ctl->s_full[buf]));
      }
      __syncwarp();
    };
    auto issue_dp = [&](int stage) {
      if (leader) {
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_ss(tmem + 256, dG0 + kstep(kk), dV0 + (uint64_t)stage * kTileStep + kstep(kk), idS, kk > 0);
        mma_commit(smem_u32(&ctl->dp_full));
      }
      __syncwarp();
    };
    bool ok = wait_all(smem_u32(&ctl->q_full), 0);
    int n = 0;
    if (ok && first <= kt_hi) {
      ok = wait_all(smem_u32(&ctl->k_full[0]), 0);
      if (ok) {
        tc_fence_after();
        issue_s(0, 0);
        ok = wait_all(smem_u32(&ctl->v_full[0]), 0);
        if (ok) {
          tc_fence_after();
          issue_dp(0);
        }
      }
    }
    for (int kt = first; ok && kt <= kt_hi; ++n) {
      const int nk = dq_next_tile(f, b, h, qt, kt_hi, kt);
      const int s = n % kStages, s1 = (n + 1) % kStages;
      const bool more = nk <= kt_hi;
      if (more) {  // S of the next tile into the other buffer while the warps work on this one
        if (!(ok = wait_all(smem_u32(&ctl->k_full[s1]), ((n + 1) / kStages) & 1))) break;
        tc_fence_after();
        issue_s(s1, (n + 1) & 1);
      }
      if (!(ok = wait_all(smem_u32(&ctl->g_full), n & 1))) break;
      tc_fence_after();
      // dQ += gamma K: keys 16 kk .. 16 kk + 15 of warpgroup kk >> 2, 8 packed columns per step.
      if (leader) {
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_ts(tmem + 384, tmem + (n & 1) * 128 + 64 * (kk >> 2) + 8 * (kk & 3),
                 dKmn0 + (uint64_t)s * kTileStep + (uint64_t)(kk * (2048 >> 4)), idDQ, (n > 0 || kk > 0) ? 1u : 0u);
        mma_commit(smem_u32(&ctl->kv_empty[s]));
      }
      __syncwarp();
      if (more) {
        if (!(ok = wait_all(smem_u32(&ctl->v_full[s1]), ((n + 1) / kStages) & 1))) break;
        tc_fence_after();
        issue_dp(s1);
      }
      kt = nk;
    }
    if (leader) mma_commit(smem_u32(&ctl->dq_final));
    __syncwarp();
  } else if (warp >= 2) {
    // ---------------- compute warpgroups
    const int w = (warp - 2) >> 2;               // key columns 64 w .. 64 w + 63
    const int t = ((warp & 3) << 5) | lane;      // query row within the tile = TMEM lane
    const int64_t row = (int64_t)q0 + t;
    const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
    const int64_t srow = ((int64_t)b * f.Hq + h) * a.Tpad + row;  // row < Tpad = 128 * nqt
    const float nlse2 = row < f.Tq ? a.lse2[srow] : -INFINITY;  // -log2 Z (-inf: no keys)
    const float ndelta = row < f.Tq ? a.dpad[srow] : 0.f;       // -delta
    const float dscale = f.m.dropout ? f.m.inv_keep : 1.f;
    const int slice = 2 * qt + ((warp & 3) >> 1);               // this warp's 64-row slice
    const uint64_t sc2 = f2_pack(f.scale_log2, f.scale_log2), nl2 = f2_pack(nlse2, nlse2);
    const uint64_t nd2 = f2_pack(ndelta, ndelta);
    int n = 0;
    bool ok = true;
    // Tile classes, 32 key tiles per round: lane l holds tile cbase + l
    // (bits 0-1: the query tile's class, bits 2-3: this warp's slice).
    int cbase = kt_lo - 32;
    uint32_t cword = 0;
    for (int kt = kt_lo; ok && kt <= kt_hi; ++kt) {
      if (kt - cbase >= 32) {
        cbase = kt;
        const int mk = kt + lane;
        cword = 0;
        if (mk <= kt_hi) {
          cword = wg_class(f, b, h, qt, mk);
          if (cword == kPartial) cword |= ((uint32_t)lookup_class(f.ct, f.m, f.Tq, f.Tk, b, h, slice, mk) & 3u) << 2;
        }
      }
      const uint32_t cv = __shfl_sync(0xffffffffu, cword, kt - cbase);
      const uint8_t cls = cv & 3u;
      if (cls == kEmpty) continue;
      const bool plain = cls == kFull && !f.m.dropout;
      uint64_t mw = ~0ull, kw = ~0ull;
      if (cls == kPartial) {
        uint64_t w0 = 0ull, w1 = 0ull;
        if (row < f.Tq) fwd_row_bits(f, b, h, row, (int64_t)kt * kBN, (uint8_t)(cv >> 2), w0, w1);
        mw = w ? w1 : w0;
      }
      if (f.m.dropout) {
        uint64_t k0, k1;
        fwd_keep_bits(f.m, b, h, row, (int64_t)kt * kBN, k0, k1);
        kw = w ? k1 : k0;
      }
      const uint32_t tS = tmem + lane_off + (n & 1) * 128 + 64 * w;
      ok = __all_sync(0xffffffffu, wait_bar(smem_u32(&ctl->s_full[n & 1]), (n >> 1) & 1, abort_flag, f.status));
      if (!ok) break;
      tc_fence_after();
      float p[64];
      {
        uint32_t r0[32], r1[32];
        tmem_ld32(tS, r0);
        tmem_ld32(tS + 32, r1);
        tmem_wait_ld();
        if (plain) {  // P = 2^(s c log2(e) - log2 Z) on packed pairs
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            float x0, x1, y0, y1;
            f2_unpack(f2_fma(f2_pack(__uint_as_float(r0[2 * e]), __uint_as_float(r0[2 * e + 1])), sc2, nl2), x0, x1);
            f2_unpack(f2_fma(f2_pack(__uint_as_float(r1[2 * e]), __uint_as_float(r1[2 * e + 1])), sc2, nl2), y0, y1);
            p[2 * e] = ex2(x0);
            p[2 * e + 1] = ex2(x1);
            p[32 + 2 * e] = ex2(y0);
            p[32 + 2 * e + 1] = ex2(y1);
          }
        } else {
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            p[e] = ((mw >> e) & 1ull) ? ex2(fmaf(__uint_as_float(r0[e]), f.scale_log2, nlse2)) : 0.f;
            p[32 + e] = ((mw >> (32 + e)) & 1ull) ? ex2(fmaf(__uint_as_float(r1[e]), f.scale_log2, nlse2)) : 0.f;
          }
        }
      }
      ok = __all_sync(0xffffffffu, wait_bar(smem_u32(&ctl->dp_full), n & 1, abort_flag, f.status));
      if (!ok) break;
      tc_fence_after();
      const uint32_t tP = tmem + lane_off + 256 + 64 * w;
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        uint32_t r[32];
        tmem_ld32(tP + 32 * hh, r);
        tmem_wait_ld();
        uint32_t pk[16];
        if (!f.m.dropout) {  // gamma = P (dP - delta) on packed pairs
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const int c0 = 32 * hh + 2 * e;
            const uint64_t g2 = f2_mul(f2_pack(p[c0], p[c0 + 1]),
                                       f2_add(f2_pack(__uint_as_float(r[2 * e]), __uint_as_float(r[2 * e + 1])), nd2));
            float g0, g1;
            f2_unpack(g2, g0, g1);
            pk[e] = pack16<kH>(g0, g1);
          }
        } else {
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const int c0 = 32 * hh + 2 * e, c1 = c0 + 1;
            const float d0 = ((kw >> c0) & 1ull) ? __uint_as_float(r[2 * e]) * dscale : 0.f;
            const float d1 = ((kw >> c1) & 1ull) ? __uint_as_float(r[2 * e + 1]) * dscale : 0.f;
            pk[e] = pack16<kH>(p[c0] * (d0 + ndelta), p[c1] * (d1 + ndelta));
          }
        }
        // gamma over this warpgroup's own S columns (already read above).
        tmem_st16(tS + 16 * hh, pk);
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&ctl->g_full));
      ++n;
    }
    // ---------------- epilogue: dQ = c * accumulator; warpgroup w writes d columns 64 w .. 64 w + 63
    bool have = false;
    if (ok && n > 0) {
      have = __all_sync(0xffffffffu, wait_bar(smem_u32(&ctl->dq_final), 0, abort_flag, f.status));
      if (have) tc_fence_after();
    }
    if (ok || n == 0) {
      uint16_t* drow = a.dq + b * a.sdq[0] + h * a.sdq[1] + row * a.sdq[2] + 64 * w;
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        uint32_t r[32];
        if (have) {
          tmem_ld32(tmem + lane_off + 384 + 64 * w + 32 * c, r);
          tmem_wait_ld();
        }
        if (row < f.Tq) {
#pragma unroll
          for (int c8 = 0; c8 < 4; ++c8) {
            uint32_t pk[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int idx = c8 * 8 + 2 * e;
              pk[e] = have ? pack16<kH>(__uint_as_float(r[idx]) * a.scale, __uint_as_float(r[idx + 1]) * a.scale)
                           : 0u;
            }
            *reinterpret_cast<uint4*>(drow + 32 * c + 8 * c8) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
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

// Reverse-pass preparation: delta from the stored O and dO (kept, and negated
// in the padded array) and the negated base-2 LSE; with dq_acc set, the row's
// 128 fp32 dQ accumulator entries are zeroed too (the key-centric kernel adds
// into them). A half-warp reads one row with 16-byte loads; a warp takes eight
// rows (B*Hq*Tpad is a multiple of 128, so a warp's rows are all in range or
// all out).
template <bool kH>
__global__ void __launch_bounds__(256)
bwd_prepare_kernel(const uint16_t* o, int64_t so0, int64_t so1, int64_t so2, const uint16_t* g,
                   int64_t sg0, int64_t sg1, int64_t sg2, const float* lse, int64_t sl0, int64_t sl1, int64_t sl2,
                   int B, int Hq, int T, int Tpad, float* lse2, float* dpad, float* delta, float* dq_acc) {
  const int64_t wid = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31, hl = lane & 15;
  const int64_t nrows = (int64_t)B * Hq * Tpad;
#pragma unroll
  for (int it = 0; it < 4; ++it) {
    const int64_t w = wid * 8 + 2 * it + (lane >> 4);
    const bool valid = w < nrows;
    const int i = valid ? (int)(w % Tpad) : 0;
    const int64_t bh = valid ? w / Tpad : 0;
    const int h = (int)(bh % Hq), b = (int)(bh / Hq);
    const bool live = valid && i < T;
    float s = 0.f;
    if (live && dq_acc) {
      float4* z = reinterpret_cast<float4*>(dq_acc + (bh * T + i) * kD + hl * 8);
      z[0] = make_float4(0.f, 0.f, 0.f, 0.f);
      z[1] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
    if (live) {
      const uint4 ov = *reinterpret_cast<const uint4*>(o + b * so0 + h * so1 + (int64_t)i * so2 + hl * 8);
      const uint4 gv = *reinterpret_cast<const uint4*>(g + b * sg0 + h * sg1 + (int64_t)i * sg2 + hl * 8);
      const uint32_t ow[4] = {ov.x, ov.y, ov.z, ov.w}, gw[4] = {gv.x, gv.y, gv.z, gv.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 a2 = unpack16<kH>(ow[e]), b2 = unpack16<kH>(gw[e]);
        s = fmaf(a2.x, b2.x, s);
        s = fmaf(a2.y, b2.y, s);
      }
    }
#pragma unroll
    for (int off = 8; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);  // within the half-warp
    if (valid && hl == 0) {
      if (!live) {
        lse2[w] = -INFINITY;
        dpad[w] = 0.f;
      } else {
        const float L = lse[b * sl0 + h * sl1 + (int64_t)i * sl2];
        lse2[w] = L == -INFINITY ? -INFINITY : -L * kLog2e;  // negated: the reverse adds them
        dpad[w] = -s;
        delta[bh * T + i] = s;
      }
    }
  }
}

// dQ = c * accumulator in the storage type, eight elements per thread.
template <bool kH>
__global__ void __launch_bounds__(256)
dq_finish_kernel(const float* dq_acc, int B, int Hq, int T, float scale, uint16_t* dq, int64_t s0, int64_t s1,
                 int64_t s2) {
  const int64_t e = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) * 8;
  if (e >= (int64_t)B * Hq * T * kD) return;
  const int c = (int)(e % kD);
  const int64_t r = e / kD;
  const int i = (int)(r % T);
  const int h = (int)((r / T) % Hq);
  const int b = (int)(r / ((int64_t)T * Hq));
  const float4 v = *reinterpret_cast<const float4*>(dq_acc + e);
  const float4 u = *reinterpret_cast<const float4*>(dq_acc + e + 4);
  uint4 out;
  out.x = pack16<kH>(v.x * scale, v.y * scale);
  out.y = pack16<kH>(v.z * scale, v.w * scale);
  out.z = pack16<kH>(u.x * scale, u.y * scale);
  out.w = pack16<kH>(u.z * scale, u.w * scale);
  *reinterpret_cast<uint4*>(dq + b * s0 + h * s1 + (int64_t)i * s2 + c) = out;
}

// ----------------------------------------------------------- host helpers

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
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

// 4-D 16-bit (bf16 or fp16) map over (d, T, H, B) with a (64, rows, 1, 1) box
// and 128-byte swizzle.
bool make_map(CUtensorMap* map, const void* base, int T, int H, int B, int64_t st, int64_t sh, int64_t sb,
              int box_rows, bool f16) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[4] = {(cuuint64_t)kD, (cuuint64_t)T, (cuuint64_t)H, (cuuint64_t)B};
  cuuint64_t strides[3] = {(cuuint64_t)st * 2, (cuuint64_t)sh * 2, (cuuint64_t)sb * 2};
  cuuint32_t box[4] = {64, (cuuint32_t)box_rows, 1, 1};
  cuuint32_t es[4] = {1, 1, 1, 1};
  return fn(map, f16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4,
            const_cast<void*>(base), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// A block mask is constant over every (64-row slice, 128-key tile) when its
// block sizes are multiples of those; then the tile class already says all.
int block_aligned(const MaskP& m) {
  if (!(m.flags & ATTN_MASK_BLOCK)) return 1;
  return (m.bq % kBMb == 0 && m.bk % kBN == 0) ? 1 : 0;
}

// 3-D fp32 map over the dQ accumulator [B*Hq][T][128] with a (32, 64, 1) box,
// no swizzle: the reduce-add target of the reverse kernel.
bool make_dq_map(CUtensorMap* map, float* base, int T, int BH) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {(cuuint64_t)kD, (cuuint64_t)T, (cuuint64_t)BH};
  cuuint64_t strides[2] = {(cuuint64_t)kD * 4, (cuuint64_t)T * kD * 4};
  cuuint32_t box[3] = {32, (cuuint32_t)kBMb, 1};
  cuuint32_t es[3] = {1, 1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, base, dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool tma_ok(const attn_tensor* t) {
  if (!t || (t->dtype != ATTN_BF16 && t->dtype != ATTN_F16) || t->ndim != 4 || t->stride[3] != 1) return false;
  if (reinterpret_cast<uintptr_t>(t->data) % 16) return false;
  for (int i = 0; i < 3; ++i) {
    if ((t->stride[i] * 2) % 16) return false;
    if (t->stride[i] <= 0 && t->shape[i] > 1) return false;
  }
  return true;
}

// Raise a kernel's dynamic shared-memory limit once per device. which names
// the kernel instantiation, one slot each: forward 0-3, query-centric dQ 4-5,
// reverse 8-15.
cudaError_t set_smem_attr(const void* fn, uint32_t bytes, int which) {
  static bool done[16][64] = {};
  if (which < 0 || which >= 16) return cudaErrorInvalidValue;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 64 && done[which][dev]) return cudaSuccess;
  e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
  if (e == cudaSuccess && dev < 64) done[which][dev] = true;
  return e;
}

constexpr uint32_t kTableFlags = ATTN_MASK_BLOCK | ATTN_MASK_LENGTHS | ATTN_MASK_STARTS;

// A class table is kept per batch row when the block mask, the lengths or the
// starts differ between batch rows, per head when the block mask does.
int table_batches(uint32_t flags, int B, int64_t bm_sb, int64_t st_sb) {
  const bool per_b = ((flags & ATTN_MASK_BLOCK) && bm_sb) || (flags & ATTN_MASK_LENGTHS) ||
                     ((flags & ATTN_MASK_STARTS) && st_sb);
  return per_b ? B : 1;
}

size_t class_bytes(int B, int Hq, int Tq, int Tk, const attn_mask* m) {
  if (!m || !(m->flags & kTableFlags)) return 0;
  const int nb = table_batches(m->flags, B, m->bm_stride_b, m->starts_stride_b);
  const int nh = (m->flags & ATTN_MASK_BLOCK) && m->bm_stride_h ? Hq : 1;
  const size_t nqs = (Tq + kBMb - 1) / kBMb, nkt = (Tk + kBN - 1) / kBN;
  return align_up((size_t)nb * nh * nqs * nkt, 256);
}

ClassTable build_class_table(const DenseP& p, void* ws, cudaStream_t st, cudaError_t& err) {
  ClassTable ct;
  ct.cls = nullptr;
  ct.nb = table_batches(p.m.flags, p.B, p.m.bm_sb, p.m.st_sb);
  ct.nh = (p.m.flags & ATTN_MASK_BLOCK) && p.m.bm_sh ? p.Hq : 1;
  ct.nqs = (p.Tq + kBMb - 1) / kBMb;
  ct.nkt = (p.Tk + kBN - 1) / kBN;
  err = cudaSuccess;
  if (!(p.m.flags & kTableFlags)) return ct;
  uint8_t* out = static_cast<uint8_t*>(ws);
  const int64_t n = (int64_t)ct.nb * ct.nh * ct.nqs * ct.nkt;
  const int blocks = (int)((n + 255) / 256 < 4096 ? (n + 255) / 256 : 4096);
  classify_kernel<<<blocks, 256, 0, st>>>(p.m, p.Tq, p.Tk, p.B, p.Hq, ct, out);
  err = cudaGetLastError();
  ct.cls = out;
  return ct;
}

}  // namespace

size_t sm100_fwd_workspace_bytes(int B, int Hq, int Tq, int Tk, const attn_mask* m) {
  return class_bytes(B, Hq, Tq, Tk, m);
}

size_t sm100_bwd_extra_workspace_bytes(int B, int Hq, int Hkv, int Tq, int Tk, const attn_mask* m) {
  (void)Hkv;
  const size_t Tpad = (size_t)((Tq + kBN - 1) / kBN) * kBN;
  return 2 * align_up((size_t)B * Hq * Tpad * sizeof(float), 256) + class_bytes(B, Hq, Tq, Tk, m);
}

bool sm100_dense_supported(const DenseP& p, const attn_tensor* q, const attn_tensor* k, const attn_tensor* v,
                           const attn_tensor* o) {
  if (p.d != kD || p.dv != kD || p.Tq < 1 || p.Tk < 1) return false;
  if (!tma_ok(q) || !tma_ok(k) || !tma_ok(v) || !tma_ok(o)) return false;
  if (!encode_fn()) return false;
  int dev = 0, major = 0, minor = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return false;
  cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
  cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
  return major == 10 && minor == 0;
}

bool sm100_dense_bwd_supported(const DenseP&, const attn_tensor* do_, const attn_tensor* dq, const attn_tensor* dk,
                               const attn_tensor* dv) {
  return tma_ok(do_) && tma_ok(dq) && tma_ok(dk) && tma_ok(dv);
}

cudaError_t sm100_dense_fwd(const DenseP& p, void* o, const int64_t so[3], float* lse, const int64_t sl[3], void* ws,
                            uint32_t* status, cudaStream_t st) {
  cudaError_t err;
  ClassTable ct = build_class_table(p, ws, st, err);
  if (err != cudaSuccess) return err;
  const bool f16 = p.dtype == ATTN_F16;
  CUtensorMap mq, mk, mv;
  if (!make_map(&mq, p.q, p.Tq, p.Hq, p.B, p.sq[2], p.sq[1], p.sq[0], kBM, f16) ||
      !make_map(&mk, p.k, p.Tk, p.Hkv, p.B, p.sk[2], p.sk[1], p.sk[0], kBN, f16) ||
      !make_map(&mv, p.v, p.Tk, p.Hkv, p.B, p.sv[2], p.sv[1], p.sv[0], kBN, f16))
    return cudaErrorInvalidValue;
  FwdArgs a;
  a.m = p.m;
  a.ct = ct;
  a.block_aligned = block_aligned(p.m);
  a.B = p.B;
  a.Hq = p.Hq;
  a.Hkv = p.Hkv;
  a.Tq = p.Tq;
  a.Tk = p.Tk;
  a.scale_log2 = p.scale * kLog2e;
  a.o = static_cast<uint16_t*>(o);
  for (int i = 0; i < 3; ++i) {
    a.so[i] = so[i];
    a.sl[i] = sl[i];
  }
  a.lse = lse;
  a.status = status;
  const bool drop = p.m.dropout != 0;
  auto kern = f16 ? (drop ? fwd_kernel<true, true> : fwd_kernel<true, false>)
                  : (drop ? fwd_kernel<false, true> : fwd_kernel<false, false>);
  if ((err = set_smem_attr(reinterpret_cast<const void*>(kern), kFwdSmem, (f16 ? 1 : 0) + (drop ? 2 : 0))) !=
      cudaSuccess)
    return err;
  const int nct = (p.Tq + kFwdRows - 1) / kFwdRows;
  main_kernel_begin(st);
  kern<<<nct * p.B * p.Hq, kFwdThreads, kFwdSmem, st>>>(mq, mk, mv, a);
  main_kernel_end(st);
  return cudaGetLastError();
}

cudaError_t sm100_dense_bwd(const DenseP& p, const void* o, const int64_t so[3], const void* g, const int64_t sg[3],
                            const float* lse, const int64_t sl[3], float* delta, float* dq_acc, void* dq,
                            const int64_t sdq[3], void* dk, const int64_t sdk[3], void* dv, const int64_t sdv[3],
                            void* ws_extra, uint32_t* status, cudaStream_t st) {
  const int Tpad = ((p.Tq + kBN - 1) / kBN) * kBN;
  const size_t padb = align_up((size_t)p.B * p.Hq * Tpad * sizeof(float), 256);
  float* lse2 = static_cast<float*>(ws_extra);
  float* dpad = reinterpret_cast<float*>(static_cast<char*>(ws_extra) + padb);
  cudaError_t err;
  ClassTable ct = build_class_table(p, static_cast<char*>(ws_extra) + 2 * padb, st, err);
  if (err != cudaSuccess) return err;
  const bool f16 = p.dtype == ATTN_F16;
  const bool det = p.bwd_flags & ATTN_BWD_DETERMINISTIC;
  const int64_t rows = (int64_t)p.B * p.Hq * Tpad;  // a multiple of 128: eight rows per warp
  (f16 ? bwd_prepare_kernel<true> : bwd_prepare_kernel<false>)<<<(unsigned)((rows * 4 + 255) / 256), 256, 0, st>>>(
      static_cast<const uint16_t*>(o), so[0], so[1], so[2], static_cast<const uint16_t*>(g), sg[0], sg[1], sg[2], lse,
      sl[0], sl[1], sl[2], p.B, p.Hq, p.Tq, Tpad, lse2, dpad, delta, det ? nullptr : dq_acc);
  if ((err = cudaGetLastError()) != cudaSuccess) return err;
  CUtensorMap mq, mk, mv, mg, mdq;
  if (!make_dq_map(&mdq, dq_acc, p.Tq, p.B * p.Hq) ||
      !make_map(&mq, p.q, p.Tq, p.Hq, p.B, p.sq[2], p.sq[1], p.sq[0], kBMb, f16) ||
      !make_map(&mk, p.k, p.Tk, p.Hkv, p.B, p.sk[2], p.sk[1], p.sk[0], kBN, f16) ||
      !make_map(&mv, p.v, p.Tk, p.Hkv, p.B, p.sv[2], p.sv[1], p.sv[0], kBN, f16) ||
      !make_map(&mg, g, p.Tq, p.Hq, p.B, sg[2], sg[1], sg[0], kBMb, f16))
    return cudaErrorInvalidValue;
  BwdArgs a;
  a.m = p.m;
  a.ct = ct;
  a.block_aligned = block_aligned(p.m);
  a.B = p.B;
  a.Hq = p.Hq;
  a.Hkv = p.Hkv;
  a.Tq = p.Tq;
  a.Tk = p.Tk;
  a.Tpad = Tpad;
  a.scale_log2 = p.scale * kLog2e;
  a.lse2 = lse2;
  a.dpad = dpad;
  a.dq_acc = dq_acc;
  a.dk = static_cast<uint16_t*>(dk);
  a.dv = static_cast<uint16_t*>(dv);
  for (int i = 0; i < 3; ++i) {
    a.sdk[i] = sdk[i];
    a.sdv[i] = sdv[i];
  }
  a.scale = p.scale;
  a.status = status;
  const bool drop = p.m.dropout != 0;
  using BwdFn = void (*)(const CUtensorMap, const CUtensorMap, const CUtensorMap, const CUtensorMap,
                         const CUtensorMap, const BwdArgs);
  // [fp16][no dQ][dropout]
  const BwdFn table[2][2][2] = {{{bwd_kernel<false, true, false>, bwd_kernel<false, true, true>},
                                 {bwd_kernel<false, false, false>, bwd_kernel<false, false, true>}},
                                {{bwd_kernel<true, true, false>, bwd_kernel<true, true, true>},
                                 {bwd_kernel<true, false, false>, bwd_kernel<true, false, true>}}};
  auto kern = table[f16][det][drop];
  const int which = 8 + (f16 ? 4 : 0) + (det ? 2 : 0) + (drop ? 1 : 0);  // 8 .. 15
  if ((err = set_smem_attr(reinterpret_cast<const void*>(kern), kBwdSmem, which)) != cudaSuccess) return err;
  const int nkt = (p.Tk + kBN - 1) / kBN;
  main_kernel_begin(st);
  kern<<<nkt * p.B * p.Hkv, kBwdThreads, kBwdSmem, st>>>(mq, mk, mv, mg, mdq, a);
  main_kernel_end(st);
  if ((err = cudaGetLastError()) != cudaSuccess) return err;
  if (p.bwd_flags & ATTN_BWD_DETERMINISTIC) {
    // dQ from the query-centric pass: one CTA sums each element in key order.
    CUtensorMap dq_mq, dq_mg;
    if (!make_map(&dq_mq, p.q, p.Tq, p.Hq, p.B, p.sq[2], p.sq[1], p.sq[0], kBM, f16) ||
        !make_map(&dq_mg, g, p.Tq, p.Hq, p.B, sg[2], sg[1], sg[0], kBM, f16))
      return cudaErrorInvalidValue;
    DqArgs d;
    d.f.m = p.m;
    d.f.ct = ct;
    d.f.block_aligned = block_aligned(p.m);
    d.f.B = p.B;
    d.f.Hq = p.Hq;
    d.f.Hkv = p.Hkv;
    d.f.Tq = p.Tq;
    d.f.Tk = p.Tk;
    d.f.scale_log2 = p.scale * kLog2e;
    d.f.o = nullptr;
    d.f.lse = nullptr;
    for (int i = 0; i < 3; ++i) d.f.so[i] = d.f.sl[i] = 0;
    d.f.status = status;
    d.lse2 = lse2;
    d.dpad = dpad;
    d.dq = static_cast<uint16_t*>(dq);
    for (int i = 0; i < 3; ++i) d.sdq[i] = sdq[i];
    d.scale = p.scale;
    d.Tpad = Tpad;
    auto kdq = f16 ? dq_kernel<true> : dq_kernel<false>;
    if ((err = set_smem_attr(reinterpret_cast<const void*>(kdq), kDqSmem, f16 ? 5 : 4)) != cudaSuccess) return err;
    const int nqt = (p.Tq + kBM - 1) / kBM;
    kdq<<<nqt * p.B * p.Hq, kDqThreads, kDqSmem, st>>>(dq_mq, mk, mv, dq_mg, d);
    return cudaGetLastError();
  }
  const int64_t n8 = (int64_t)p.B * p.Hq * p.Tq * kD / 8;
  (f16 ? dq_finish_kernel<true> : dq_finish_kernel<false>)<<<(unsigned)((n8 + 255) / 256), 256, 0, st>>>(
      dq_acc, p.B, p.Hq, p.Tq, p.scale, static_cast<uint16_t*>(dq), sdq[0], sdq[1], sdq[2]);
  return cudaGetLastError();
}

}  // namespace attn
