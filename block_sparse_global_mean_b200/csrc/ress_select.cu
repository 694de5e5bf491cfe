// Stage 1: pooled block selection.
//
//   pool_kernel        one streaming pass over Q and K (and V when lambda > 0):
//                      per-block means with 16-byte loads and fp32 sums.
//   contrast_kernel    c[h][j] = ||Vbar_j - Vbar_{j-1}||_2, c[h][0] = 0.
//   score_topk_kernel  per (head, R query blocks): pooled logits for every key
//                      block into shared memory (fp32 FMA), optional softmax +
//                      contrast, then an exact selection per row (one warp per
//                      row: a value-linear histogram finds the threshold bin,
//                      whose few values are ranked exactly) that keeps
//                      `budget` blocks, ties to the lower index, written in
//                      ascending order.
//                      In its CDF mode each row keeps instead the fewest top
//                      blocks whose probabilities reach tau (warp_cdf_count),
//                      padded to a fixed capacity.
//
// Sources: ReSS (thelatestinai.com) Table S5, SpargeAttn row - selection by
// pooled query/key inner products, which reduces to SparseVGGT's cumulative
// threshold (Table 2, "+ CDF threshold"); VASC (paperlayer.ai) 4.1 - pooled
// relevance plus neighbouring value contrast; VASC A.2 - an exact-capacity
// binary Top-K.
#include "ress_common.cuh"
#include "ress_internal.h"
#include "ress_topk.cuh"

namespace ress {

namespace {

constexpr int kPoolMaxTensors = 3;

struct PoolArgs {
  const void* src[kPoolMaxTensors];
  float* dst[kPoolMaxTensors];
  int layout[kPoolMaxTensors];  // 0: [H][nb][64]; 1: [H][64][nb_pad] (transposed)
  int nb, nb_pad, block, heads, vpr;
  // Extra outputs for the keys (tensor 1), written when khi != null: the
  // pooled keys split into a tf32 high part and a tf32 low part, both
  // [H][nb_pad][64] (key-major), the high parts of 128 evenly spaced sample
  // keys [H][128][64] (sample t is key (t * nb) / 128), and the key norms
  // [H][nb].
  float* khi;
  float* klo;
  float* ksample;
  float* knorm;
  int lay_t, lay_r;   // per-view layout (lay_t == 0: none): only valid tokens are pooled
};

// float32 -> nearest tf32 (10 explicit mantissa bits), kept in a float.
__device__ __forceinline__ float round_tf32(float x) {
  return __uint_as_float((__float_as_uint(x) + 0x1000u) & 0xFFFFE000u);
}

__device__ __forceinline__ void accum_vec(float* acc, const uint4& v, const __nv_bfloat16*) {
  const __nv_bfloat162* p = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const float2 f = __bfloat1622float2(p[u]);
    acc[2 * u] += f.x;
    acc[2 * u + 1] += f.y;
  }
}

__device__ __forceinline__ void accum_vec(float* acc, const uint4& v, const float*) {
  acc[0] += __uint_as_float(v.x);
  acc[1] += __uint_as_float(v.y);
  acc[2] += __uint_as_float(v.z);
  acc[3] += __uint_as_float(v.w);
}

// grid (nb, tensors); block = vpr * phases threads; thread (col, phase) sums
// the 16-byte column `col` of tokens phase, phase + phases, ... of its block.
template <typename T>
__global__ void __launch_bounds__(1024, 1) pool_kernel(const PoolArgs a) {
  constexpr int EPV = 16 / sizeof(T);
  extern __shared__ float red[];
  const int i = blockIdx.x;
  const int t = blockIdx.y;
  const int vpr = a.vpr;
  const int phases = blockDim.x / vpr;
  const int col = threadIdx.x % vpr;
  const int ph = threadIdx.x / vpr;
  // Picked by value: indexing the parameter arrays with t would copy them to
  // local memory.
  const void* src = t == 0 ? a.src[0] : (t == 1 ? a.src[1] : a.src[2]);
  float* dst = t == 0 ? a.dst[0] : (t == 1 ? a.dst[1] : a.dst[2]);
  const int layout = t == 0 ? a.layout[0] : (t == 1 ? a.layout[1] : a.layout[2]);
  const uint4* base = reinterpret_cast<const uint4*>(src) + (size_t)i * a.block * vpr + col;
  // Tokens pooled: the block's valid prefix (all of it without a layout).
  const int cnt = layout_valid(a.lay_t, a.lay_r, (long long)i * a.block, a.block);
  float acc[EPV];
#pragma unroll
  for (int u = 0; u < EPV; ++u) acc[u] = 0.f;
  int tok = ph;
#pragma unroll 1
  for (; tok + 7 * phases < cnt; tok += 8 * phases) {
    uint4 v[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) v[u] = __ldg(base + (size_t)(tok + u * phases) * vpr);
#pragma unroll
    for (int u = 0; u < 8; ++u) accum_vec(acc, v[u], (const T*)nullptr);
  }
  for (; tok < cnt; tok += phases) {
    const uint4 v = __ldg(base + (size_t)tok * vpr);
    accum_vec(acc, v, (const T*)nullptr);
  }
  if (phases > 1) {
#pragma unroll
    for (int u = 0; u < EPV; ++u) red[(ph * vpr + col) * EPV + u] = acc[u];
    __syncthreads();
    if (ph != 0) return;
    for (int q = 1; q < phases; ++q) {
#pragma unroll
      for (int u = 0; u < EPV; ++u) acc[u] += red[(q * vpr + col) * EPV + u];
    }
  }
  // An empty block (no valid token) pools to zero.
  const float inv = cnt > 0 ? 1.0f / (float)cnt : 0.f;
  const int e0 = col * EPV;           // element within the token row (H * 64)
  const int hh = e0 / kHeadDim;
  const int dd = e0 % kHeadDim;
  if (t == 1 && a.khi != nullptr) {
    // Lanes holding one head's 64 values: 64 / EPV consecutive lanes, all in
    // phase 0 (the lanes of other phases have returned above).
    constexpr int G = kHeadDim / EPV;
    const int lane = threadIdx.x & 31;
    const unsigned gmask = (G == 32 ? 0xffffffffu : ((1u << G) - 1u)) << (lane & ~(G - 1));
    float v[EPV], hi[EPV], lo[EPV];
    float ss = 0.f;
#pragma unroll
    for (int u = 0; u < EPV; ++u) {
      v[u] = acc[u] * inv;
      hi[u] = round_tf32(v[u]);
      lo[u] = round_tf32(v[u] - hi[u]);
      ss = fmaf(v[u], v[u], ss);
    }
#pragma unroll
    for (int o = G / 2; o > 0; o >>= 1) ss += __shfl_xor_sync(gmask, ss, o);
    const size_t krow = ((size_t)hh * a.nb_pad + i) * kHeadDim + dd;
#pragma unroll
    for (int u = 0; u < EPV; u += 4) {
      *reinterpret_cast<float4*>(a.khi + krow + u) = make_float4(hi[u], hi[u + 1], hi[u + 2], hi[u + 3]);
      *reinterpret_cast<float4*>(a.klo + krow + u) = make_float4(lo[u], lo[u + 1], lo[u + 2], lo[u + 3]);
    }
    if ((lane & (G - 1)) == 0) a.knorm[(size_t)hh * a.nb + i] = sqrtf(ss);
    // Sample slots whose key is this block: t_s with (t_s * nb) / 128 == i.
    for (int ts = (i * 128 + a.nb - 1) / a.nb; ts < 128 && (ts * a.nb) / 128 == i; ++ts) {
      float* srow = a.ksample + ((size_t)hh * 128 + ts) * kHeadDim + dd;
#pragma unroll
      for (int u = 0; u < EPV; u += 4)
        *reinterpret_cast<float4*>(srow + u) = make_float4(hi[u], hi[u + 1], hi[u + 2], hi[u + 3]);
    }
  }
  if (dst == nullptr) return;
  if (layout == 0) {
    float4* o = reinterpret_cast<float4*>(dst + ((size_t)hh * a.nb + i) * kHeadDim + dd);
#pragma unroll
    for (int u = 0; u < EPV / 4; ++u)
      o[u] = make_float4(acc[4 * u] * inv, acc[4 * u + 1] * inv, acc[4 * u + 2] * inv,
                         acc[4 * u + 3] * inv);
  } else {
#pragma unroll
    for (int u = 0; u < EPV; ++u)
      dst[((size_t)hh * kHeadDim + dd + u) * a.nb_pad + i] = acc[u] * inv;
  }
}

// One warp per (h, j): c[h][j] = ||Vbar[h][j] - Vbar[h][j-1]||_2, c[h][0] = 0.
__global__ void __launch_bounds__(256) contrast_kernel(const float* __restrict__ vbar,
                                                       float* __restrict__ c, int heads, int nb) {
  const int w = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (w >= heads * nb) return;
  const int j = w % nb;
  float s = 0.f;
  if (j > 0) {
    const float* cur = vbar + (size_t)w * kHeadDim;
    const float* prv = cur - kHeadDim;
    const float d0 = cur[lane] - prv[lane];
    const float d1 = cur[lane + 32] - prv[lane + 32];
    s = d0 * d0 + d1 * d1;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  }
  if (lane == 0) c[w] = sqrtf(s);
}

struct ScoreArgs {
  DeviceError* err;
  const float* qbar;     // [H][nb][64]
  const float* kbar_t;   // [H][64][nb_pad]
  const float* contrast; // [H][nb] or null
  int32_t* idx;          // [H][nb][budget]
  int heads, nb, nb_pad, budget, tiles_per_head;
  int row_stride;         // floats between score rows in shared memory
  int stages;             // ring stages
  float lambda;
  float tau;              // CDF threshold (cdf_counts != null)
  int32_t* cdf_counts;    // [H][nb] CDF counts, or null for the fixed budget
  int block, lay_t, lay_r, lay_s;   // per-view layout (lay_t == 0: none)
  // VASC mode: the pair contrast and the memory's ranking copy [H][n_pairs],
  // the demand (units of 2^-32) and service sums they add to, and c_h.
  const float* vasc_rho;
  const float* vasc_mhat;
  unsigned long long* vasc_dsum;
  uint32_t* vasc_ssum;
  int n_pairs;
  int vasc_budget[kMaxHeads];
};

// Modes of score_topk_kernel.
constexpr int kModeBudget = 0;   // fixed budget: logits, or p + lambda c, or the layout ranks
constexpr int kModeCdf = 1;      // CDF threshold
constexpr int kModeVasc = 2;     // VASC demand plus memory, per-head budgets

// Probability of logit s in units of 2^-40: p = exp(s - hi) / z in float32,
// rounded to the nearest unit.  Sums of up to 4,096 of them are exact in 64
// bits, so every mass below is independent of the summation order.
__device__ __forceinline__ unsigned long long mass_fixed(float s, float hi, float inv_z) {
  return __float2ull_rn(expf(s - hi) * inv_z * 1099511627776.0f);
}

__device__ __forceinline__ unsigned long long shfl_up_u64(unsigned long long v, int o) {
  return __shfl_up_sync(0xffffffffu, v, o);
}

// CDF count of one shared-memory row of pooled logits (one warp): the
// smallest m >= 1 such that the m largest probabilities (equal logits in
// index order) sum to at least tau_f (units of 2^-40); nb if the total does
// not reach it.  Probabilities follow the logits, so logits are ranked.
//  1. row max hi, z = sum exp(s - hi), and the total mass;
//  2. over the current logit interval [a, b] (first the whole row): counts
//     and masses in kCdfBins value-linear bins; the bin b* where the mass
//     from the top reaches tau_f; the blocks above b* are kept;
//  3. if b* holds at most kMaxCand blocks, they are ranked exactly by (logit
//     desc, index asc) and taken in that order until the mass reaches tau_f;
//     if its blocks all have one logit, the count follows by division;
//     otherwise [a, b] becomes the logit range of b* and step 2 repeats.
// Each level separates the distinct logits of b* by a factor of about
// kCdfBins, so four levels suffice for float32; after six the remaining
// blocks are taken one at a time in rank order (never reached in practice).
__device__ __noinline__ int warp_cdf_count(const float* row, int nb, unsigned long long tau_f,
                                           uint32_t* scratch, int lane) {
  uint32_t* cnt = scratch;                                                      // [kCdfBins]
  unsigned long long* mass = reinterpret_cast<unsigned long long*>(scratch + kCdfBins);  // [kCdfBins]
  uint32_t* ckey = scratch + 3 * kCdfBins;                                      // [kMaxCand]
  uint32_t* cj = ckey + kMaxCand;                                               // [kMaxCand]
  unsigned long long* cm = reinterpret_cast<unsigned long long*>(cj + kMaxCand);  // [kMaxCand]
  const uint32_t lt_mask = (1u << lane) - 1u;
  const int run = 4 * ((((nb + 31) >> 5) + 3) >> 2 | 1);
  const int j0 = min(lane * run, nb);
  const int j1 = min(j0 + run, nb);

  float lo = INFINITY, hi = -INFINITY;
  for (int j = j0; j < j1; ++j) {
    lo = fminf(lo, row[j]);
    hi = fmaxf(hi, row[j]);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    lo = fminf(lo, __shfl_xor_sync(0xffffffffu, lo, o));
    hi = fmaxf(hi, __shfl_xor_sync(0xffffffffu, hi, o));
  }
  float z = 0.f;
  for (int j = j0; j < j1; ++j) z += expf(row[j] - hi);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) z += __shfl_xor_sync(0xffffffffu, z, o);
  const float inv_z = 1.0f / z;
  unsigned long long tot = 0ull;
  for (int j = j0; j < j1; ++j) tot += mass_fixed(row[j], hi, inv_z);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) tot += __shfl_xor_sync(0xffffffffu, tot, o);
  if (!(hi >= lo) || tot < tau_f) return nb;   // never reached (or no finite logit)

  float a = lo, b = hi;
  int cnt_above = 0;                // blocks above the interval, all kept
  unsigned long long cum_above = 0; // and their mass
  for (int level = 0; level < 6; ++level) {
    float scale = (float)(kCdfBins - 1) / (b - a);
    if (!(scale < INFINITY)) scale = 0.f;
    for (int t = lane; t < kCdfBins; t += 32) {
      cnt[t] = 0u;
      mass[t] = 0ull;
    }
    __syncwarp();
    for (int j = j0; j < j1; ++j) {
      const float sv = row[j];
      if (sv >= a && sv <= b) {
        const uint32_t bin = value_bin_n(sv, a, scale, kCdfBins);
        atomicAdd(&cnt[bin], 1u);
        atomicAdd(&mass[bin], mass_fixed(sv, hi, inv_z));
      }
    }
    __syncwarp();
    // Lane l owns bins kCdfBins-1-8l .. kCdfBins-8-8l (descending).
    constexpr int kPer = kCdfBins / 32;
    unsigned long long lm[kPer];
    int lc[kPer];
    unsigned long long tm = 0ull;
    int tc = 0;
#pragma unroll
    for (int u = 0; u < kPer; ++u) {
      lm[u] = mass[kCdfBins - 1 - kPer * lane - u];
      lc[u] = (int)cnt[kCdfBins - 1 - kPer * lane - u];
      tm += lm[u];
      tc += lc[u];
    }
    unsigned long long im = tm;
    int ic = tc;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const unsigned long long ym = shfl_up_u64(im, o);
      const int yc = __shfl_up_sync(0xffffffffu, ic, o);
      if (lane >= o) {
        im += ym;
        ic += yc;
      }
    }
    const unsigned long long em = im - tm;
    const int ec = ic - tc;
    const unsigned ball =
        __ballot_sync(0xffffffffu, cum_above + em < tau_f && cum_above + im >= tau_f);
    if (ball == 0u) return nb;      // unreachable: the interval's mass reaches tau_f
    const int src = __ffs(ball) - 1;
    int bstar_i = 0, above_c = 0;
    unsigned long long above_m = 0ull;
    if (lane == src) {
      unsigned long long accm = cum_above + em;
      int accc = ec;
#pragma unroll
      for (int u = 0; u < kPer; ++u) {
        if (accm + lm[u] >= tau_f) {
          bstar_i = kCdfBins - 1 - kPer * lane - u;
          above_m = accm;
          above_c = accc;
          break;
        }
        accm += lm[u];
        accc += lc[u];
      }
    }
    const uint32_t bstar = (uint32_t)__shfl_sync(0xffffffffu, bstar_i, src);
    above_c = __shfl_sync(0xffffffffu, above_c, src);
    above_m = __shfl_sync(0xffffffffu, above_m, src);
    cnt_above += above_c;
    cum_above = above_m;
    const int in_bin = (int)cnt[bstar];
    if (in_bin <= kMaxCand) {
      // Gather b* in ascending index order, rank exactly, take in rank order.
      int n = 0;
      for (int c0 = 0; c0 < nb; c0 += 32) {
        const int j = c0 + lane;
        const float sv = row[min(j, nb - 1)];
        const bool c = j < nb && sv >= a && sv <= b && value_bin_n(sv, a, scale, kCdfBins) == bstar;
        const unsigned m = __ballot_sync(0xffffffffu, c);
        if (c) {
          const int slot = n + __popc(m & lt_mask);
          ckey[slot] = order_key(sv);
          cj[slot] = (uint32_t)j;
          cm[slot] = mass_fixed(sv, hi, inv_z);
        }
        n += __popc(m);
      }
      __syncwarp();
      int best = in_bin;
      for (int c = lane; c < in_bin; c += 32) {
        const uint32_t kc = ckey[c], jc = cj[c];
        int rank = 0;
        unsigned long long upto = cm[c];
        for (int o = 0; o < in_bin; ++o) {
          const bool before = ckey[o] > kc || (ckey[o] == kc && cj[o] < jc);
          rank += before ? 1 : 0;
          upto += before ? cm[o] : 0ull;
        }
        if (cum_above + upto >= tau_f) best = min(best, rank);
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) best = min(best, __shfl_xor_sync(0xffffffffu, best, o));
      return cnt_above + min(best + 1, in_bin);
    }
    // Crowded b*: its logit range becomes the next interval.
    float na = INFINITY, nbv = -INFINITY;
    for (int j = j0; j < j1; ++j) {
      const float sv = row[j];
      if (sv >= a && sv <= b && value_bin_n(sv, a, scale, kCdfBins) == bstar) {
        na = fminf(na, sv);
        nbv = fmaxf(nbv, sv);
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      na = fminf(na, __shfl_xor_sync(0xffffffffu, na, o));
      nbv = fmaxf(nbv, __shfl_xor_sync(0xffffffffu, nbv, o));
    }
    if (na == nbv) {
      // One logit: every block of b* carries the same mass.
      const unsigned long long pm = mass_fixed(na, hi, inv_z);
      const unsigned long long need = tau_f - cum_above;
      const unsigned long long take = pm ? (need + pm - 1ull) / pm : (unsigned long long)in_bin;
      return cnt_above + (int)min(take, (unsigned long long)in_bin);
    }
    a = na;
    b = nbv;
    __syncwarp();
  }
  // Last resort: take the blocks of [a, b] one at a time in rank order.
  uint32_t prev_key = 0xffffffffu;
  int prev_j = -1;
  bool first = true;
  unsigned long long cum = cum_above;
  int taken = 0;
  for (int guard = 0; guard < nb; ++guard) {
    uint32_t bk = 0u;
    int bj = nb;
    for (int j = j0; j < j1; ++j) {
      const float sv = row[j];
      if (!(sv >= a && sv <= b)) continue;
      const uint32_t kk = order_key(sv);
      const bool after = first || kk < prev_key || (kk == prev_key && j > prev_j);
      if (after && (kk > bk || (kk == bk && j < bj) || bj == nb)) {
        bk = kk;
        bj = j;
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const uint32_t ok2 = __shfl_xor_sync(0xffffffffu, bk, o);
      const int oj = __shfl_xor_sync(0xffffffffu, bj, o);
      if (oj != nb && (bj == nb || ok2 > bk || (ok2 == bk && oj < bj))) {
        bk = ok2;
        bj = oj;
      }
    }
    if (bj == nb) break;
    ++taken;
    cum += mass_fixed(row[bj], hi, inv_z);
    if (cum >= tau_f) break;
    prev_key = bk;
    prev_j = bj;
    first = false;
  }
  return cnt_above + max(taken, 1);
}

// VASC row (one warp; row holds the pooled logits s_j of query block i).
// With e_j = exp(s_j - max s) and rho the contrast of j's pair, the demand is
//   a_j = min(1, e_j rho_j * c_h / sum_j e_j rho_j)
// (the relevance p_j = e_j / sum e, times the contrast, rescaled so the row
// totals c_h, clipped at one: VASC 4.1 and A.2); the ranking score is
// a_j + mhat[pair(j)] (VASC 4.2), of which the c_h largest are kept (ties to
// the lower index), listed ascending and padded with the last kept block to
// the row length.  The demand (units of 2^-32, exact in 64 bits) and the
// executed children are summed per pair into the CTA's counters.
__device__ __forceinline__ void vasc_row(const ScoreArgs& a, float* row, uint32_t* whist, int h,
                                      int i, unsigned long long* dacc, uint32_t* sacc,
                                      int lane) {
  const int nb = a.nb;
  const int c = a.vasc_budget[h];
  const float* rho = a.vasc_rho + (size_t)h * a.n_pairs;
  const float* mhat = a.vasc_mhat + (size_t)h * a.n_pairs;
  float m = -INFINITY;
  for (int j = lane; j < nb; j += 32) m = fmaxf(m, row[j]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  // e_j rho_j replaces the logit (one exponential per entry).
  float z = 0.f;
  for (int j = lane; j < nb; j += 32) {
    const float w = expf(row[j] - m) * rho[j >> 1];
    row[j] = w;
    z += w;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) z += __shfl_xor_sync(0xffffffffu, z, o);
  const float scale = z > 0.f ? (float)c / z : 0.f;
  // Lanes 2l and 2l + 1 hold the two children of one pair (32 is even), so
  // the even lane adds both demands to the pair's counter.
  for (int j0 = 0; j0 < nb; j0 += 32) {
    const int j = j0 + lane;
    unsigned long long fx = 0ull;
    if (j < nb) {
      const float dem = fminf(1.f, row[j] * scale);
      fx = __float2ull_rn(dem * 4294967296.0f);
      row[j] = dem + mhat[j >> 1];
    }
    fx += __shfl_xor_sync(0xffffffffu, fx, 1);
    if ((lane & 1) == 0 && j < nb) atomicAdd(&dacc[j >> 1], fx);
  }
  __syncwarp();
  int32_t* out = a.idx + ((size_t)h * nb + i) * a.budget;
  warp_topk_row_binned(row, nb, c, whist, out, lane);
  __syncwarp();
  const int32_t last = out[c - 1];
  for (int r = c + lane; r < a.budget; r += 32) out[r] = last;
  for (int r = lane; r < c; r += 32) atomicAdd(&sacc[out[r] >> 1], 1u);
}

// CTA = one head and R consecutive query blocks.  The pooled keys stream
// through a ring of 16 KB shared-memory stages, each [4 d][1024 keys] fp32,
// filled by bulk copies that the producer (the last warp) issues as soon as
// the eight score warps have released the stage.  Lane l of score warp w
// accumulates all R rows against keys 128 w + 4 l .. + 3 of the tile, two
// rows per packed fp32 FMA, d in ascending order; the R score rows (all nb
// key blocks) stay in shared memory.  Then every warp 0 .. R-1 (the producer
// included when R = 16) selects the top `budget` of one row.
constexpr uint32_t kStageBytes = 16384;
constexpr int kScoreTK = 1024;                          // keys per tile
constexpr int kScoreTD = kStageBytes / (4 * kScoreTK);  // d per stage (4)
constexpr int kStagesPerTile = kHeadDim / kScoreTD;
constexpr int kScoreWarps = 8;                          // warps that compute scores
static_assert(kScoreWarps * 32 * 4 == kScoreTK, "four keys per score lane");

template <int R>
struct ScoreCfg {
  static constexpr int kWarps = R > kScoreWarps ? R : kScoreWarps + 1;
  static constexpr int kThreads = 32 * kWarps;
  static constexpr int kProducer = kWarps - 1;
  // The top-k scratch of the R row warps reuses the stage ring, which has at
  // least 4 stages for R = 16 and 2 for R = 8.
  static_assert(R * kWarpScratchStride * 4 <= (R == 16 ? 4 : 2) * (int)kStageBytes,
                "row-warp scratch fits the stage ring");
};

// Registers are capped at 128 so that four warps of one SM sub-partition fit
// its register file (4 x 32 x 128 = 16,384).
template <int R, int kMode>
__global__ void __maxnreg__(128) score_topk_kernel(const ScoreArgs a) {
  using C = ScoreCfg<R>;
  constexpr int TK = kScoreTK, TD = kScoreTD;
  extern __shared__ __align__(16) float sm[];
  const int S = a.stages;
  float* stages = sm;                                    // [S][TD][TK]; top-k scratch later
  float* qs = stages + (size_t)S * TD * TK;              // [64][R]
  float* scores = qs + kHeadDim * R;                     // [R][row_stride]
  const int nb = a.nb, nb_pad = a.nb_pad, rs = a.row_stride;
  uint64_t* bars = reinterpret_cast<uint64_t*>(scores + (size_t)R * rs);   // full[S], empty[S]
  int* abortf = reinterpret_cast<int*>(bars + 2 * S);
  // VASC mode: this CTA's demand sums [n_pairs] and service counts [n_pairs].
  unsigned long long* dacc = reinterpret_cast<unsigned long long*>(bars + 2 * S + 2);
  uint32_t* sacc = reinterpret_cast<uint32_t*>(dacc + a.n_pairs);

  const int h = blockIdx.x / a.tiles_per_head;
  const int i0 = (blockIdx.x % a.tiles_per_head) * R;
  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const int n_tiles = (nb_pad + TK - 1) / TK;
  const int n_seq = n_tiles * kStagesPerTile;
  const float* kbt = a.kbar_t + (size_t)h * kHeadDim * nb_pad;
  const uint32_t full0 = smem_addr(&bars[0]);
  const uint32_t empty0 = smem_addr(&bars[S]);

  if (tid == 0) {
    for (int st = 0; st < S; ++st) {
      mbar_init(full0 + 8u * st, 1);
      mbar_init(empty0 + 8u * st, kScoreWarps);
    }
    *abortf = 0;
    fence_mbarrier_init();
  }
  for (int e = tid; e < R * kHeadDim; e += C::kThreads) {
    const int r = e / kHeadDim, d = e % kHeadDim;
    qs[d * R + r] = (i0 + r < nb) ? a.qbar[((size_t)h * nb + i0 + r) * kHeadDim + d] : 0.f;
  }
  if constexpr (kMode == kModeVasc) {
    for (int p = tid; p < a.n_pairs; p += C::kThreads) {
      dacc[p] = 0ull;
      sacc[p] = 0u;
    }
  }
  __syncthreads();

  if (warp == C::kProducer) {
    // Stage seq holds d rows TD*(seq % kStagesPerTile) .. +TD-1 of tile
    // seq / kStagesPerTile (its keys below nb_pad).
    int issued = 0;
    for (int seq = 0; seq < n_seq; ++seq) {
      const int st = seq % S;
      const uint32_t k = (uint32_t)(seq / S);
      bool ok = true;
      if (seq >= S) ok = mbar_wait(empty0 + 8u * st, (k - 1u) & 1u, abortf, a.err, 72);
      if (!__all_sync(0xffffffffu, ok)) break;
      const int t = seq / kStagesPerTile, dq = seq % kStagesPerTile;
      const int keys = min(TK, nb_pad - t * TK);        // a multiple of 256
      const uint32_t full = full0 + 8u * st;
      if (lane == 0) mbar_arrive_expect_tx(full, (uint32_t)(TD * keys * 4));
      __syncwarp();
      if (lane < TD)
        bulk_load(smem_addr(stages + ((size_t)st * TD + lane) * TK),
                  kbt + (size_t)(TD * dq + lane) * nb_pad + (size_t)t * TK, (uint32_t)keys * 4u,
                  full);
      issued = seq + 1;
    }
    // Copies still in flight (only after a timeout) land before the buffers
    // are reused or released.
    if (lane == 0)
      for (int seq = issued > S ? issued - S : 0; seq < issued; ++seq)
        mbar_wait_drain(full0 + 8u * (seq % S), (uint32_t)(seq / S) & 1u, a.err, 73);
  } else if (warp < kScoreWarps) {
    const int kw = 128 * warp + 4 * lane;           // first of this lane's four keys in a tile
    bool ok = true;
#pragma unroll 1
    for (int t = 0; t < n_tiles && ok; ++t) {
      // Warps whose 128 keys all lie beyond nb only keep the stage protocol.
      const bool active = t * TK + 128 * warp < nb;
      float2 acc[R / 2][4];   // acc[p][u] = rows (2p, 2p + 1) x key u
#pragma unroll
      for (int p = 0; p < R / 2; ++p)
#pragma unroll
        for (int u = 0; u < 4; ++u) acc[p][u] = make_float2(0.f, 0.f);
#pragma unroll 1
      for (int dq = 0; dq < kStagesPerTile; ++dq) {
        const int seq = t * kStagesPerTile + dq;
        const int st = seq % S;
        ok = mbar_wait(full0 + 8u * st, (uint32_t)(seq / S) & 1u, abortf, a.err, 70);
        if (!__all_sync(0xffffffffu, ok)) {
          ok = false;
          break;
        }
        if (active) {
          const float* kb = stages + (size_t)st * TD * TK + kw;
          const float* qb = qs + TD * dq * R;
#pragma unroll 2   // full unrolling spills at 128 registers
          for (int dd = 0; dd < TD; ++dd) {
            const float4 kv = *reinterpret_cast<const float4*>(kb + dd * TK);
            const float kk[4] = {kv.x, kv.y, kv.z, kv.w};
#pragma unroll
            for (int m = 0; m < R / 4; ++m) {
              const float4 qv = *reinterpret_cast<const float4*>(qb + dd * R + 4 * m);
              const float2 qa = make_float2(qv.x, qv.y), qc = make_float2(qv.z, qv.w);
#pragma unroll
              for (int u = 0; u < 4; ++u) {
                const float2 ku = make_float2(kk[u], kk[u]);
                acc[2 * m][u] = ffma2(qa, ku, acc[2 * m][u]);
                acc[2 * m + 1][u] = ffma2(qc, ku, acc[2 * m + 1][u]);
              }
            }
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(empty0 + 8u * st);
      }
      if (!ok || !active) continue;
      const int j = t * TK + kw;
      // 1 / sqrt(64) = 0.125 is exact.
#pragma unroll
      for (int p = 0; p < R / 2; ++p) {
        float* r0 = scores + (size_t)(2 * p) * rs;
        float* r1 = r0 + rs;
        if (j + 3 < nb) {
          *reinterpret_cast<float4*>(r0 + j) = make_float4(acc[p][0].x * 0.125f, acc[p][1].x * 0.125f,
                                                           acc[p][2].x * 0.125f, acc[p][3].x * 0.125f);
          *reinterpret_cast<float4*>(r1 + j) = make_float4(acc[p][0].y * 0.125f, acc[p][1].y * 0.125f,
                                                           acc[p][2].y * 0.125f, acc[p][3].y * 0.125f);
        } else {
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            if (j + u < nb) {
              r0[j + u] = acc[p][u].x * 0.125f;
              r1[j + u] = acc[p][u].y * 0.125f;
            }
          }
        }
      }
    }
  }
  __syncthreads();
  if constexpr (kMode == kModeVasc) {
    if (*abortf != 0) return;   // read after the barrier: the same for every thread
    if (warp < R && i0 + warp < nb)
      vasc_row(a, scores + (size_t)warp * rs,
               reinterpret_cast<uint32_t*>(stages) + warp * kWarpScratchStride, h, i0 + warp,
               dacc, sacc, lane);
    __syncthreads();
    // This CTA's sums join the head's totals (integer adds: the totals do not
    // depend on the order of the CTAs).
    for (int p = tid; p < a.n_pairs; p += C::kThreads) {
      const size_t at = (size_t)h * a.n_pairs + p;
      if (dacc[p] != 0ull) atomicAdd(&a.vasc_dsum[at], dacc[p]);
      if (sacc[p] != 0u) atomicAdd(&a.vasc_ssum[at], sacc[p]);
    }
    return;
  }
  if (*abortf != 0 || warp >= R) return;
  // One warp per row; the stage buffers now hold each row warp's scratch.
  const int i = i0 + warp;
  if (i >= nb) return;
  uint32_t* whist = reinterpret_cast<uint32_t*>(stages) + warp * kWarpScratchStride;
  float* row = scores + (size_t)warp * rs;
  int32_t* out = a.idx + ((size_t)h * nb + i) * a.budget;
  if constexpr (kMode == kModeCdf) {
    // CDF threshold: the count, then the exact top min(count, capacity) of the
    // logits (the probabilities' order), padded with the last kept block.
    // At least one unit: every row keeps at least its top block.
    const unsigned long long tau_f = max(__double2ull_rn((double)a.tau * 1099511627776.0), 1ull);
    const int k = warp_cdf_count(row, nb, tau_f, whist, lane);
    const int keep = min(k, a.budget);
    __syncwarp();
    warp_topk_row_binned(row, nb, keep, whist, out, lane);
    __syncwarp();
    const int32_t last = out[keep - 1];
    for (int r = keep + lane; r < a.budget; r += 32) out[r] = last;
    if (lane == 0) a.cdf_counts[(size_t)h * nb + i] = k;
    return;
  }
  if (a.lay_t != 0) {
    // Layout: an empty key block (no valid token) ranks below every other
    // block, a key block whose valid tokens are all special ranks above
    // (kept first, lowest index first when there are more than the budget).
    for (int j = lane; j < nb; j += 32) {
      const long long t0 = (long long)j * a.block;
      const int cnt = layout_valid(a.lay_t, a.lay_r, t0, a.block);
      const int sp = layout_valid(a.lay_t, a.lay_s, t0, a.block);
      if (cnt == 0) row[j] = -INFINITY;
      else if (sp == cnt) row[j] = INFINITY;
    }
    __syncwarp();
  }
  if (a.lambda != 0.f) {
    float m = -INFINITY;
    for (int j = lane; j < nb; j += 32) m = fmaxf(m, row[j]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    float z = 0.f;
    for (int j = lane; j < nb; j += 32) z += expf(row[j] - m);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) z += __shfl_xor_sync(0xffffffffu, z, o);
    const float* ch = a.contrast + (size_t)h * nb;
    for (int j = lane; j < nb; j += 32) row[j] = expf(row[j] - m) / z + a.lambda * ch[j];
    __syncwarp();
  }
  warp_topk_row_binned(row, nb, a.budget, whist, out, lane);
}

// Shared memory of score_topk_kernel<R> with `stages` ring stages and score
// rows of `row_stride` floats.
template <int R>
size_t score_smem_bytes(int stages, int row_stride, int n_pairs = 0) {
  return (size_t)stages * kStageBytes +
         sizeof(float) * ((size_t)kHeadDim * R + (size_t)R * row_stride) +
         2 * sizeof(uint64_t) * (size_t)stages + 16 +
         (sizeof(unsigned long long) + sizeof(uint32_t)) * (size_t)n_pairs;
}

constexpr size_t kMaxSmem = 227 * 1024;
constexpr int kMaxStages = 6;

// Deepest ring (up to kMaxStages) that fits; 0 if fewer than `min_stages` fit.
template <int R>
int score_stages(int row_stride, int min_stages, int n_pairs = 0) {
  for (int s = kMaxStages; s >= min_stages; --s)
    if (score_smem_bytes<R>(s, row_stride, n_pairs) <= kMaxSmem) return s;
  return 0;
}

template <int R, int kMode>
ress_status launch_score_mode(const ScoreArgs& a0, int stages, cudaStream_t st) {
  ScoreArgs a = a0;
  a.tiles_per_head = (a.nb + R - 1) / R;
  a.stages = stages;
  const size_t smem =
      score_smem_bytes<R>(stages, a.row_stride, kMode == kModeVasc ? a.n_pairs : 0);
  if (ress_status st_ = record_cuda(cudaFuncSetAttribute(
          score_topk_kernel<R, kMode>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem)))
    return st_;
  score_topk_kernel<R, kMode><<<a.heads * a.tiles_per_head, ScoreCfg<R>::kThreads, smem, st>>>(a);
  return record_cuda(cudaGetLastError());
}

// The CDF and VASC modes are separate instantiations, so that their code does
// not weigh on the register allocation and code layout of the fixed-budget
// kernel.
template <int R>
ress_status launch_score(const ScoreArgs& a, int stages, cudaStream_t st) {
  if (a.vasc_rho != nullptr) return launch_score_mode<R, kModeVasc>(a, stages, st);
  return a.cdf_counts != nullptr ? launch_score_mode<R, kModeCdf>(a, stages, st)
                                 : launch_score_mode<R, kModeBudget>(a, stages, st);
}

// Exact top-k of the rows that the tensor-core kernel handed over (its check
// failed: a crowded threshold band, or a band that missed the budget-th
// score).  A persistent grid walks the list; per row the pooled scores are
// float32 FMA dot products over d in ascending order, scaled by the exact
// 1/8 (the shared-memory kernel's arithmetic), with the keys read back as
// their tf32 high + low parts, and warp 0 selects the top `budget`.
struct FallbackArgs {
  const float* qbar;          // [H][nb][64]
  const float* khi;           // [H][nb_pad][64]
  const float* klo;           // [H][nb_pad][64]
  const int32_t* fb_count;
  const int32_t* fb_list;
  int32_t* idx;
  int nb, nb_pad, budget, row_stride;
};

__global__ void __launch_bounds__(512) topk_fallback_kernel(const FallbackArgs a) {
  extern __shared__ __align__(16) float fsm[];
  float* row = fsm;                                  // [row_stride]
  float* qs = row + a.row_stride;                    // [64]
  uint32_t* scratch = reinterpret_cast<uint32_t*>(qs + kHeadDim);   // [kWarpScratchStride]
  const int count = *a.fb_count;
  for (int t = blockIdx.x; t < count; t += gridDim.x) {
    const int code = a.fb_list[t];
    const int h = code / a.nb, i = code - h * a.nb;
    if (threadIdx.x < kHeadDim) qs[threadIdx.x] = a.qbar[((size_t)h * a.nb + i) * kHeadDim + threadIdx.x];
    __syncthreads();
    for (int j = threadIdx.x; j < a.nb; j += blockDim.x) {
      const float* kh = a.khi + ((size_t)h * a.nb_pad + j) * kHeadDim;
      const float* kl = a.klo + ((size_t)h * a.nb_pad + j) * kHeadDim;
      float acc = 0.f;
#pragma unroll 16
      for (int d = 0; d < kHeadDim; ++d) acc = fmaf(qs[d], kh[d] + kl[d], acc);
      row[j] = acc * 0.125f;
    }
    __syncthreads();
    if (threadIdx.x < 32)
      warp_topk_row_binned(row, a.nb, a.budget, scratch,
                           a.idx + ((size_t)h * a.nb + i) * a.budget, threadIdx.x);
    __syncthreads();
  }
}

}  // namespace

ress_status launch_pool(const Geometry& g, const void* q, const void* k, const void* v,
                        float* qbar, float* kbar_t, float* vbar_t, cudaStream_t st) {
  PoolArgs pa{};
  pa.src[0] = q;  pa.dst[0] = qbar;   pa.layout[0] = 0;
  pa.src[1] = k;  pa.dst[1] = kbar_t; pa.layout[1] = 1;
  pa.src[2] = v;  pa.dst[2] = vbar_t; pa.layout[2] = 1;
  pa.nb = g.nb;
  pa.nb_pad = g.nb_pad;
  pa.block = g.block;
  pa.heads = g.heads;
  const int epv = g.f32 ? 4 : 8;
  pa.vpr = g.heads * kHeadDim / epv;
  const int phases = pa.vpr >= 256 ? 1 : 256 / pa.vpr;
  const dim3 grid(g.nb, v != nullptr ? 3 : 2);
  const int threads = pa.vpr * phases;
  const size_t red = phases > 1 ? sizeof(float) * (size_t)phases * pa.vpr * epv : 0;
  if (g.f32)
    pool_kernel<float><<<grid, threads, red, st>>>(pa);
  else
    pool_kernel<__nv_bfloat16><<<grid, threads, red, st>>>(pa);
  return record_cuda(cudaGetLastError());
}

ress_status launch_score_vasc(const Geometry& g, const float* qbar, const float* kbar_t,
                              int capacity, int32_t* idx, const VascSelect& vs,
                              cudaStream_t st) {
  ScoreArgs sa{};
  sa.err = device_error_ptr();
  if (sa.err == nullptr) return RESS_ERR_CUDA;
  sa.qbar = qbar;
  sa.kbar_t = kbar_t;
  sa.idx = idx;
  sa.heads = g.heads;
  sa.nb = g.nb;
  sa.nb_pad = g.nb_pad;
  sa.budget = capacity;
  sa.block = g.block;
  sa.row_stride = (g.nb + 3) & ~3;
  sa.vasc_rho = vs.rho;
  sa.vasc_mhat = vs.mhat;
  sa.vasc_dsum = vs.dsum;
  sa.vasc_ssum = vs.ssum;
  sa.n_pairs = vasc_pairs(g.nb);
  for (int h = 0; h < g.heads; ++h) sa.vasc_budget[h] = vs.budgets[h];
  // As for the fixed budget, with the CTA's pair counters next to the rows.
  const int s16 = score_stages<16>(sa.row_stride, 4, sa.n_pairs);
  if (s16 != 0) return launch_score<16>(sa, s16, st);
  const int s8 = score_stages<8>(sa.row_stride, 2, sa.n_pairs);
  if (s8 == 0) return RESS_ERR_UNSUPPORTED;
  return launch_score<8>(sa, s8, st);
}

ress_status launch_topk_fallback(const Geometry& g, int budget, int32_t* idx, uint8_t* ws,
                                 const SelectLayout& lay, cudaStream_t st) {
  FallbackArgs a{};
  a.qbar = reinterpret_cast<const float*>(ws + lay.qbar);
  a.khi = reinterpret_cast<const float*>(ws + lay.tc_khi);
  a.klo = reinterpret_cast<const float*>(ws + lay.tc_klo);
  a.fb_count = reinterpret_cast<const int32_t*>(ws + lay.tc_fb_count);
  a.fb_list = reinterpret_cast<const int32_t*>(ws + lay.tc_fb_list);
  a.idx = idx;
  a.nb = g.nb;
  a.nb_pad = g.nb_pad;
  a.budget = budget;
  a.row_stride = (g.nb + 3) & ~3;
  const size_t smem = sizeof(float) * ((size_t)a.row_stride + kHeadDim) +
                      sizeof(uint32_t) * kWarpScratchStride;
  if (ress_status st_ = record_cuda(cudaFuncSetAttribute(
          topk_fallback_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem)))
    return st_;
  topk_fallback_kernel<<<148, 512, smem, st>>>(a);
  return record_cuda(cudaGetLastError());
}

SelectLayout select_layout(const Geometry& g, bool with_v) {
  SelectLayout l{};
  size_t off = 0;
  l.qbar = off;
  off += align256(sizeof(float) * (size_t)g.heads * g.nb * kHeadDim);
  const size_t after_qbar = off;
  l.kbar_t = off;
  off += align256(sizeof(float) * (size_t)g.heads * kHeadDim * g.nb_pad);
  if (with_v) {
    l.vbar = off;
    off += align256(sizeof(float) * (size_t)g.heads * g.nb * kHeadDim);
    l.contrast = off;
    off += align256(sizeof(float) * (size_t)g.heads * g.nb);
    l.total = off;
    return l;
  }
  l.vbar = l.contrast = 0;
  // Tensor-core path (lambda == 0): the key planes overlay kbar_t and beyond.
  size_t t = after_qbar;
  const size_t plane = align256(sizeof(float) * (size_t)g.heads * g.nb_pad * kHeadDim);
  l.tc_khi = t;
  t += plane;
  l.tc_klo = t;
  t += plane;
  l.tc_ksample = t;
  t += align256(sizeof(float) * (size_t)g.heads * 128 * kHeadDim);
  l.tc_knorm = t;
  t += align256(sizeof(float) * (size_t)g.heads * g.nb);
  l.tc_fb_count = t;
  t += 256;
  l.tc_fb_list = t;
  t += align256(sizeof(int32_t) * (size_t)g.heads * g.nb);
  l.total = off > t ? off : t;
  return l;
}

bool select_uses_tc(const Geometry& g, int budget, bool with_v, bool cdf) {
  return !with_v && !cdf && g.lay_t == 0 && budget < g.nb && g.nb <= kMaxBlocksTc;
}

ress_status launch_select(const Geometry& g, const void* q, const void* k, const void* v,
                          int budget, float lambda, int32_t* idx, void* ws, cudaStream_t st,
                          const CdfSelect* cdf) {
  const bool with_v = lambda != 0.f;
  const SelectLayout lay = select_layout(g, with_v);
  uint8_t* w = static_cast<uint8_t*>(ws);
  float* qbar = reinterpret_cast<float*>(w + lay.qbar);
  float* kbar_t = reinterpret_cast<float*>(w + lay.kbar_t);
  float* vbar = with_v ? reinterpret_cast<float*>(w + lay.vbar) : nullptr;
  float* contrast = with_v ? reinterpret_cast<float*>(w + lay.contrast) : nullptr;

  const bool tc = select_uses_tc(g, budget, with_v, cdf != nullptr);
  PoolArgs pa{};
  pa.src[0] = q;  pa.dst[0] = qbar;   pa.layout[0] = 0;
  pa.src[1] = k;  pa.dst[1] = tc ? nullptr : kbar_t; pa.layout[1] = 1;
  pa.src[2] = v;  pa.dst[2] = vbar;   pa.layout[2] = 0;
  if (tc) {
    pa.khi = reinterpret_cast<float*>(w + lay.tc_khi);
    pa.klo = reinterpret_cast<float*>(w + lay.tc_klo);
    pa.ksample = reinterpret_cast<float*>(w + lay.tc_ksample);
    pa.knorm = reinterpret_cast<float*>(w + lay.tc_knorm);
  }
  pa.nb = g.nb;
  pa.nb_pad = g.nb_pad;
  pa.block = g.block;
  pa.heads = g.heads;
  pa.lay_t = g.lay_t;
  pa.lay_r = g.lay_r;
  const int epv = g.f32 ? 4 : 8;
  pa.vpr = g.heads * kHeadDim / epv;
  const int phases = pa.vpr >= 256 ? 1 : 256 / pa.vpr;
  const dim3 grid(g.nb, with_v ? 3 : 2);
  const int threads = pa.vpr * phases;
  const size_t red = phases > 1 ? sizeof(float) * (size_t)phases * pa.vpr * epv : 0;
  if (g.f32)
    pool_kernel<float><<<grid, threads, red, st>>>(pa);
  else
    pool_kernel<__nv_bfloat16><<<grid, threads, red, st>>>(pa);
  if (ress_status st_ = record_cuda(cudaGetLastError())) return st_;
  if (with_v) {
    const int warps = g.heads * g.nb;
    contrast_kernel<<<(warps + 7) / 8, 256, 0, st>>>(vbar, contrast, g.heads, g.nb);
    if (ress_status st_ = record_cuda(cudaGetLastError())) return st_;
  }
  if (tc) {
    if (ress_status st_ = launch_topk_tc(g, budget, idx, w, lay, st)) return st_;
    return launch_topk_fallback(g, budget, idx, w, lay, st);
  }
  ScoreArgs sa{};
  sa.err = device_error_ptr();
  if (sa.err == nullptr) return RESS_ERR_CUDA;
  sa.qbar = qbar;
  sa.kbar_t = kbar_t;
  sa.contrast = contrast;
  sa.idx = idx;
  sa.heads = g.heads;
  sa.nb = g.nb;
  sa.nb_pad = g.nb_pad;
  sa.budget = budget;
  sa.lambda = lambda;
  sa.tau = cdf ? cdf->tau : 0.f;
  sa.cdf_counts = cdf ? cdf->counts : nullptr;
  sa.block = g.block;
  sa.lay_t = g.lay_t;
  sa.lay_r = g.lay_r;
  sa.lay_s = g.lay_s;
  sa.row_stride = (g.nb + 3) & ~3;
  // Sixteen rows per CTA while at least four stages fit next to the score rows
  // (nb <= 2,304), else eight.  The stage ring also holds the top-k scratch of
  // every consumer warp afterwards.
  const int s16 = score_stages<16>(sa.row_stride, 4);
  if (s16 != 0) return launch_score<16>(sa, s16, st);
  const int s8 = score_stages<8>(sa.row_stride, 2);
  if (s8 == 0) return RESS_ERR_UNSUPPORTED;
  return launch_score<8>(sa, s8, st);
}

}  // namespace ress
