// Exact top-k of one row of float scores in shared memory, by one warp:
// larger score first, lower index on equal scores, result in ascending index
// order.  Used by the pooled selection and its fallback, and by the
// restoration-based selection.
#pragma once

#include "ress_common.cuh"

namespace ress {
namespace {

// Order-preserving map from float to uint32 (larger float -> larger key);
// -0 maps like +0 and NaN maps to 0 (below -inf).
__device__ __forceinline__ uint32_t order_key(float f) {
  if (f != f) return 0u;
  uint32_t b = __float_as_uint(f);
  if ((b << 1) == 0u) b = 0u;
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

// Exact selection of `budget` largest keys of a shared-memory row (one warp):
// four 8-bit radix passes find the key T of the budget-th largest element and
// how many elements equal to T are kept; a final ascending pass writes every
// index with key > T plus the lowest-index elements with key == T.
__device__ __forceinline__ void warp_topk_row(const float* row, int nb, int budget,
                                              uint32_t* hist, int32_t* out, int lane) {
  uint32_t prefix = 0u, pmask = 0u;
  int rem = budget;
#pragma unroll 1
  for (int shift = 24; shift >= 0; shift -= 8) {
    for (int b = lane; b < 256; b += 32) hist[b] = 0u;
    __syncwarp();
    for (int j = lane; j < nb; j += 32) {
      const uint32_t key = order_key(row[j]);
      if ((key & pmask) == prefix) atomicAdd(&hist[(key >> shift) & 255u], 1u);
    }
    __syncwarp();
    int cnt[8];
    int tot = 0;
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      cnt[u] = (int)hist[255 - 8 * lane - u];
      tot += cnt[u];
    }
    int incl = tot;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    const int excl = incl - tot;
    const unsigned ball = __ballot_sync(0xffffffffu, excl < rem && rem <= incl);
    const int src = ball ? __ffs(ball) - 1 : 0;
    int bin = 0, above = 0;
    if (lane == src) {
      int acc = excl;
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        if (acc + cnt[u] >= rem) {
          bin = 255 - 8 * lane - u;
          above = acc;
          break;
        }
        acc += cnt[u];
      }
    }
    bin = __shfl_sync(0xffffffffu, bin, src);
    above = __shfl_sync(0xffffffffu, above, src);
    rem -= above;
    prefix |= (uint32_t)bin << shift;
    pmask |= 255u << shift;
    __syncwarp();
  }
  const uint32_t lt_mask = (1u << lane) - 1u;
  int pos = 0, eq_seen = 0;
  for (int j0 = 0; j0 < nb; j0 += 32) {
    const int j = j0 + lane;
    const uint32_t key = (j < nb) ? order_key(row[j]) : 0u;
    const bool gt = (j < nb) && key > prefix;
    const bool eq = (j < nb) && key == prefix;
    const unsigned eqb = __ballot_sync(0xffffffffu, eq);
    const bool take = gt || (eq && (eq_seen + __popc(eqb & lt_mask)) < rem);
    const unsigned tb = __ballot_sync(0xffffffffu, take);
    if (take) out[pos + __popc(tb & lt_mask)] = j;
    pos += __popc(tb);
    eq_seen += __popc(eqb);
  }
}

constexpr int kBins = 512;        // histogram bins, linear in the value over [row min, row max]
constexpr int kMaxCand = 64;      // values of the threshold bin that are ranked exactly
constexpr int kBitmapWords = 128; // kept-block bitmap: nb <= 4096
constexpr int kWarpScratchWords = kBins + kBitmapWords + 2 * kMaxCand;
constexpr int kCdfBins = 256;     // histogram bins of the CDF count
// Per-row-warp scratch: the top-k (kWarpScratchWords) or the CDF count
// (counts, 64-bit masses and candidates of kCdfBins bins).
constexpr int kWarpScratchStride = 1024;
static_assert(kWarpScratchWords <= kWarpScratchStride &&
              kCdfBins + 2 * kCdfBins + 4 * kMaxCand <= kWarpScratchStride, "row-warp scratch");

// Shared-memory histogram increment; the result is not returned.
__device__ __forceinline__ void red_add_shared(uint32_t addr, uint32_t v) {
  asm volatile("red.shared.add.u32 [%0], %1;" ::"r"(addr), "r"(v));
}

// Bin of v: round((v - lo) * scale) clamped to [0, kBins - 1], through the
// round-to-nearest of adding 1.5 * 2^23.  Monotone non-decreasing in v (NaN
// -> 0, below every number, as in order_key); always a valid index.
__device__ __forceinline__ uint32_t value_bin(float v, float lo, float scale) {
  const float d = fmaxf(v - lo, 0.f);
  const uint32_t b = __float_as_uint(fmaf(d, scale, 12582912.0f)) - 0x4B400000u;
  return min(b, (uint32_t)(kBins - 1));
}

// The same with `bins` bins (scale = (bins - 1) / range).
__device__ __forceinline__ uint32_t value_bin_n(float v, float lo, float scale, uint32_t bins) {
  const float d = fmaxf(v - lo, 0.f);
  const uint32_t b = __float_as_uint(fmaf(d, scale, 12582912.0f)) - 0x4B400000u;
  return min(b, bins - 1u);
}

// Exact top-`budget` of a shared-memory row (one warp), lowest index on ties.
//  1. row min and max, and
//  2. a histogram over kBins bins linear in the value, both with lane l
//     reading the contiguous run [l * run, (l + 1) * run) as float4 (run =
//     4 x an odd number: the eight lanes of one 128-bit access phase hit
//     disjoint banks, and neighbouring lanes hold distant, differently valued
//     blocks, so their histogram increments rarely collide); the bin b*
//     holding the budget-th largest value and the count above it follow from
//     a scan over the bins;
//  3. the values of b* are gathered in ascending index order (32 consecutive
//     blocks per lane step, ballot compaction) and ranked exactly by (order
//     key desc, index asc);
//  4. a last pass over 32 consecutive blocks per step writes every block
//     above b* and the winners of b*, compacted by ballot, in ascending order.
// Every pass issues four independent loads before using any of them, so that
// one warp keeps several shared-memory accesses in flight.
// A threshold bin with more than kMaxCand values falls back to the radix
// select (same result, slower).
__device__ __forceinline__ void warp_topk_row_binned(const float* row, int nb, int budget,
                                                     uint32_t* scratch, int32_t* out, int lane) {
  uint32_t* hist = scratch;                          // [kBins]
  uint32_t* wins = hist + kBins;                     // [kBitmapWords] kept-block bitmap
  uint32_t* cand_key = wins + kBitmapWords;          // [kMaxCand]
  uint32_t* cand_j = cand_key + kMaxCand;            // [kMaxCand]
  const uint32_t hist_s = smem_addr(hist);
  const uint32_t lt_mask = (1u << lane) - 1u;
  const int run = 4 * ((((nb + 31) >> 5) + 3) >> 2 | 1);
  const int j0 = min(lane * run, nb);
  const int j1 = min(j0 + run, nb);
  const int n4 = (j1 - j0) >> 2;          // float4s of the run; [j0 + 4 n4, j1) one by one
  const float4* run4 = reinterpret_cast<const float4*>(row + j0);
  float lo = INFINITY, hi = -INFINITY;
  for (int g = 0; g < n4; g += 4) {
    float4 v[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) v[u] = run4[min(g + u, n4 - 1)];   // repeats are harmless
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      lo = fminf(lo, fminf(fminf(v[u].x, v[u].y), fminf(v[u].z, v[u].w)));
      hi = fmax3(hi, fmaxf(v[u].x, v[u].y), fmaxf(v[u].z, v[u].w));
    }
  }
  for (int j = j0 + 4 * n4; j < j1; ++j) {
    lo = fminf(lo, row[j]);
    hi = fmaxf(hi, row[j]);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    lo = fminf(lo, __shfl_xor_sync(0xffffffffu, lo, o));
    hi = fmaxf(hi, __shfl_xor_sync(0xffffffffu, hi, o));
  }
  float scale = (float)(kBins - 1) / (hi - lo);
  if (!(scale < INFINITY)) scale = 0.f;   // constant row (or non-finite range): one bin
  for (int b = 4 * lane; b < kBins; b += 128)
    *reinterpret_cast<uint4*>(hist + b) = make_uint4(0u, 0u, 0u, 0u);
  for (int w = 4 * lane; w < kBitmapWords; w += 128)
    *reinterpret_cast<uint4*>(wins + w) = make_uint4(0u, 0u, 0u, 0u);
  __syncwarp();
  for (int g = 0; g < n4; g += 4) {
    float4 v[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) v[u] = run4[min(g + u, n4 - 1)];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      if (g + u < n4) {
        red_add_shared(hist_s + 4u * value_bin(v[u].x, lo, scale), 1u);
        red_add_shared(hist_s + 4u * value_bin(v[u].y, lo, scale), 1u);
        red_add_shared(hist_s + 4u * value_bin(v[u].z, lo, scale), 1u);
        red_add_shared(hist_s + 4u * value_bin(v[u].w, lo, scale), 1u);
      }
    }
  }
  for (int j = j0 + 4 * n4; j < j1; ++j) red_add_shared(hist_s + 4u * value_bin(row[j], lo, scale), 1u);
  __syncwarp();
  // Lane l owns bins kBins-1-16l .. kBins-16-16l (descending).
  constexpr int kPer = kBins / 32;
  int cnt[kPer];
  int tot = 0;
#pragma unroll
  for (int u = 0; u < kPer; ++u) {
    cnt[u] = (int)hist[kBins - 1 - kPer * lane - u];
    tot += cnt[u];
  }
  int incl = tot;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  const int excl = incl - tot;
  const unsigned ball = __ballot_sync(0xffffffffu, excl < budget && budget <= incl);
  const int src = ball ? __ffs(ball) - 1 : 0;
  int bstar_i = 0, above = 0;
  if (lane == src) {
    int acc = excl;
#pragma unroll
    for (int u = 0; u < kPer; ++u) {
      if (acc + cnt[u] >= budget) {
        bstar_i = kBins - 1 - kPer * lane - u;
        above = acc;
        break;
      }
      acc += cnt[u];
    }
  }
  const uint32_t bstar = (uint32_t)__shfl_sync(0xffffffffu, bstar_i, src);
  above = __shfl_sync(0xffffffffu, above, src);
  const int need = budget - above;
  const int in_bin = (int)hist[bstar];
  if (in_bin > kMaxCand) {                     // crowded threshold bin: exact radix select
    __syncwarp();
    warp_topk_row(row, nb, budget, hist, out, lane);
    return;
  }
  // One pass, 4 x 32 consecutive blocks a step: the blocks above b* go into
  // the bitmap (one ballot word per 32 blocks); the values of b* are gathered
  // in ascending index order.
  int ncand = 0;
  for (int c0 = 0; c0 < nb; c0 += 128) {
    float v[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) v[u] = row[min(c0 + 32 * u + lane, nb - 1)];
    unsigned ma[4], mc[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const uint32_t b = value_bin(v[u], lo, scale);
      const bool valid = c0 + 32 * u + lane < nb;
      ma[u] = __ballot_sync(0xffffffffu, valid && b > bstar);
      mc[u] = __ballot_sync(0xffffffffu, valid && b == bstar);
    }
    if (lane < 4 && c0 + 32 * lane < nb)
      wins[(c0 >> 5) + lane] = lane == 0 ? ma[0] : lane == 1 ? ma[1] : lane == 2 ? ma[2] : ma[3];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      if (mc[u] != 0u) {                       // warp-uniform; rare
        if ((mc[u] >> lane) & 1u) {
          const int slot = ncand + __popc(mc[u] & lt_mask);
          cand_key[slot] = order_key(v[u]);
          cand_j[slot] = (uint32_t)(c0 + 32 * u + lane);
        }
        ncand += __popc(mc[u]);
      }
    }
  }
  __syncwarp();
  // Rank the candidates: larger key first, lower index first on equal keys;
  // the winners join the bitmap.
  for (int c = lane; c < in_bin; c += 32) {
    const uint32_t kc = cand_key[c], jc = cand_j[c];
    int rank = 0;
    for (int o = 0; o < in_bin; ++o) {
      const uint32_t ko = cand_key[o], jo = cand_j[o];
      rank += (ko > kc || (ko == kc && jo < jc)) ? 1 : 0;
    }
    if (rank < need) atomicOr(&wins[jc >> 5], 1u << (jc & 31));
  }
  __syncwarp();
  // Emit the bitmap in ascending order, four words a step.
  const int words = (nb + 31) >> 5;
  int base = 0;
  for (int w0 = 0; w0 < words; w0 += 4) {
    const uint4 m4 = *reinterpret_cast<const uint4*>(wins + w0);   // words >= `words` are 0
    const uint32_t m[4] = {m4.x, m4.y, m4.z, m4.w};
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      if ((m[u] >> lane) & 1u) out[base + __popc(m[u] & lt_mask)] = 32 * (w0 + u) + lane;
      base += __popc(m[u]);
    }
  }
}

}  // namespace
}  // namespace ress
