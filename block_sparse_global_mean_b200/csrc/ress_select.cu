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
//
// Sources: ReSS (thelatestinai.com) Table S5, SpargeAttn row - selection by
// pooled query/key inner products; VASC (paperlayer.ai) 4.1 - pooled relevance
// plus neighbouring value contrast; VASC A.2 - an exact-capacity binary Top-K.
#include "ress_common.cuh"
#include "ress_internal.h"

namespace ress {

namespace {

constexpr int kPoolMaxTensors = 3;

struct PoolArgs {
  const void* src[kPoolMaxTensors];
  float* dst[kPoolMaxTensors];
  int layout[kPoolMaxTensors];  // 0: [H][nb][64]; 1: [H][64][nb_pad] (transposed)
  int nb, nb_pad, block, heads, vpr;
};

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
__global__ void __launch_bounds__(1024) pool_kernel(const PoolArgs a) {
  constexpr int EPV = 16 / sizeof(T);
  extern __shared__ float red[];
  const int i = blockIdx.x;
  const int t = blockIdx.y;
  const int vpr = a.vpr;
  const int phases = blockDim.x / vpr;
  const int col = threadIdx.x % vpr;
  const int ph = threadIdx.x / vpr;
  const uint4* base =
      reinterpret_cast<const uint4*>(a.src[t]) + (size_t)i * a.block * vpr + col;
  float acc[EPV];
#pragma unroll
  for (int u = 0; u < EPV; ++u) acc[u] = 0.f;
  int tok = ph;
#pragma unroll 1
  for (; tok + 7 * phases < a.block; tok += 8 * phases) {
    uint4 v[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) v[u] = __ldg(base + (size_t)(tok + u * phases) * vpr);
#pragma unroll
    for (int u = 0; u < 8; ++u) accum_vec(acc, v[u], (const T*)nullptr);
  }
  for (; tok < a.block; tok += phases) {
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
  const float inv = 1.0f / (float)a.block;
  const int e0 = col * EPV;           // element within the token row (H * 64)
  const int hh = e0 / kHeadDim;
  const int dd = e0 % kHeadDim;
  float* dst = a.dst[t];
  if (a.layout[t] == 0) {
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

// Order-preserving map from float to uint32 (larger float -> larger key);
// -0 maps like +0 and NaN maps to 0 (below -inf).
__device__ __forceinline__ uint32_t order_key(float f) {
  if (f != f) return 0u;
  uint32_t b = __float_as_uint(f);
  if ((b << 1) == 0u) b = 0u;
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

struct ScoreArgs {
  const float* qbar;     // [H][nb][64]
  const float* kbar_t;   // [H][64][nb_pad]
  const float* contrast; // [H][nb] or null
  int32_t* idx;          // [H][nb][budget]
  int heads, nb, nb_pad, budget, tiles_per_head;
  float lambda;
};

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

constexpr int kBins = 512;        // linear histogram bins over [row min, row max]
constexpr int kMaxCand = 64;      // candidates resolved exactly in the threshold bin
constexpr int kBitmapWords = 128; // selection bitmap: nb <= 4096
constexpr int kWarpScratchWords = kBins + kBitmapWords + 2 * kMaxCand + 4;

// Exact top-`budget` of a shared-memory row (one warp), lowest index on ties:
//  1. row min and max;
//  2. histogram over kBins bins linear in the value (a monotone map, equal
//     values share a bin); lanes walk the row with a stride of ceil(nb/32) so
//     that neighbouring lanes touch distant (differently valued) blocks;
//  3. the bin b* holding the budget-th largest value and the count above it;
//  4. everything above b* goes into a bitmap; the values of b* are gathered
//     and ranked exactly by (order key desc, index asc) to fill the rest;
//  5. the bitmap is written out in ascending block order.
// A threshold bin with more than kMaxCand values falls back to the radix
// select (same result, slower).
__device__ __forceinline__ void warp_topk_row_binned(const float* row, int nb, int budget,
                                                     uint32_t* scratch, int32_t* out, int lane) {
  uint32_t* hist = scratch;                          // [kBins]
  uint32_t* bits = hist + kBins;                     // [kBitmapWords]
  uint32_t* cand_key = bits + kBitmapWords;          // [kMaxCand]
  uint32_t* cand_j = cand_key + kMaxCand;            // [kMaxCand]
  uint32_t* cand_n = cand_j + kMaxCand;              // [1]
  float lo = INFINITY, hi = -INFINITY;
  for (int j = lane; j < nb; j += 32) {
    const float v = row[j];
    lo = fminf(lo, v);
    hi = fmaxf(hi, v);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    lo = fminf(lo, __shfl_xor_sync(0xffffffffu, lo, o));
    hi = fmaxf(hi, __shfl_xor_sync(0xffffffffu, hi, o));
  }
  const float scale = (float)kBins / (hi - lo);
  for (int b = lane; b < kBins; b += 32) hist[b] = 0u;
  for (int w = lane; w < kBitmapWords; w += 32) bits[w] = 0u;
  if (lane == 0) *cand_n = 0u;
  __syncwarp();
  const int stride = (nb + 31) >> 5;
  auto bin_of = [&](float v) -> int {
    const float t = (v - lo) * scale;           // monotone in v; NaN -> bin 0
    int b = (t >= 0.f) ? (int)fminf(t, (float)(kBins - 1)) : 0;
    return b;
  };
  for (int it = 0; it < stride; ++it) {
    const int j = lane * stride + it;
    if (j < nb) atomicAdd(&hist[bin_of(row[j])], 1u);
  }
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
  int bstar = 0, above = 0;
  if (lane == src) {
    int acc = excl;
#pragma unroll
    for (int u = 0; u < kPer; ++u) {
      if (acc + cnt[u] >= budget) {
        bstar = kBins - 1 - kPer * lane - u;
        above = acc;
        break;
      }
      acc += cnt[u];
    }
  }
  bstar = __shfl_sync(0xffffffffu, bstar, src);
  above = __shfl_sync(0xffffffffu, above, src);
  const int need = budget - above;
  const int in_bin = (int)hist[bstar];
  if (in_bin > kMaxCand) {                     // crowded threshold bin: exact radix select
    __syncwarp();
    warp_topk_row(row, nb, budget, hist, out, lane);
    return;
  }
  for (int it = 0; it < stride; ++it) {
    const int j = lane * stride + it;
    if (j < nb) {
      const float v = row[j];
      const int b = bin_of(v);
      if (b > bstar) {
        atomicOr(&bits[j >> 5], 1u << (j & 31));
      } else if (b == bstar) {
        const uint32_t slot = atomicAdd(cand_n, 1u);
        cand_key[slot] = order_key(v);
        cand_j[slot] = (uint32_t)j;
      }
    }
  }
  __syncwarp();
  // Rank the candidates: larger key first, lower index first on equal keys.
  for (int c = lane; c < in_bin; c += 32) {
    const uint32_t kc = cand_key[c], jc = cand_j[c];
    int rank = 0;
    for (int o = 0; o < in_bin; ++o) {
      const uint32_t ko = cand_key[o], jo = cand_j[o];
      rank += (ko > kc || (ko == kc && jo < jc)) ? 1 : 0;
    }
    if (rank < need) atomicOr(&bits[jc >> 5], 1u << (jc & 31));
  }
  __syncwarp();
  // Bitmap -> ascending list.
  const int words = (nb + 31) >> 5;
  int base = 0;
  for (int w0 = 0; w0 < words; w0 += 32) {
    const int w = w0 + lane;
    uint32_t m = (w < words) ? bits[w] : 0u;
    const int c = __popc(m);
    int inc = c;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, inc, o);
      if (lane >= o) inc += y;
    }
    int pos = base + inc - c;
    while (m) {
      const int bit = __ffs(m) - 1;
      m &= m - 1u;
      out[pos++] = w * 32 + bit;
    }
    base += __shfl_sync(0xffffffffu, inc, 31);
  }
}

// CTA = one head and R consecutive query blocks; 256 threads.  Scores of the
// R rows over all nb key blocks stay in shared memory.
template <int R>
__global__ void __launch_bounds__(256, 1) score_topk_kernel(const ScoreArgs a) {
  constexpr int TK = 2048 / R;   // key blocks per shared-memory tile
  constexpr int KP = TK / 2;     // key pairs per row group
  extern __shared__ __align__(16) float sm[];
  float* kt = sm;                          // [64][TK]
  float* qs = kt + kHeadDim * TK;          // [64][R]
  uint32_t* hist = reinterpret_cast<uint32_t*>(qs + kHeadDim * R);  // [8][kWarpScratchWords]
  float* scores = reinterpret_cast<float*>(hist + 8 * kWarpScratchWords);  // [R][nb_pad]

  const int h = blockIdx.x / a.tiles_per_head;
  const int i0 = (blockIdx.x % a.tiles_per_head) * R;
  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const int nb = a.nb, nb_pad = a.nb_pad;

  for (int e = tid; e < R * kHeadDim; e += 256) {
    const int r = e / kHeadDim, d = e % kHeadDim;
    qs[d * R + r] = (i0 + r < nb) ? a.qbar[((size_t)h * nb + i0 + r) * kHeadDim + d] : 0.f;
  }
  const int rg = tid / KP;   // rows 4*rg .. 4*rg+3
  const int kp = tid % KP;   // key blocks 2*kp, 2*kp+1 of the tile
  const float* kbt = a.kbar_t + (size_t)h * kHeadDim * nb_pad;
#pragma unroll 1
  for (int j0 = 0; j0 < nb; j0 += TK) {
    __syncthreads();
    for (int e = tid; e < kHeadDim * (TK / 4); e += 256) {
      const int d = e / (TK / 4), c4 = e % (TK / 4);
      reinterpret_cast<float4*>(kt + d * TK)[c4] =
          reinterpret_cast<const float4*>(kbt + (size_t)d * nb_pad + j0)[c4];
    }
    __syncthreads();
    float acc[4][2];
#pragma unroll
    for (int r = 0; r < 4; ++r) acc[r][0] = acc[r][1] = 0.f;
#pragma unroll 16
    for (int d = 0; d < kHeadDim; ++d) {
      const float4 qv = *reinterpret_cast<const float4*>(qs + d * R + 4 * rg);
      const float2 kv = *reinterpret_cast<const float2*>(kt + d * TK + 2 * kp);
      acc[0][0] = fmaf(qv.x, kv.x, acc[0][0]);
      acc[0][1] = fmaf(qv.x, kv.y, acc[0][1]);
      acc[1][0] = fmaf(qv.y, kv.x, acc[1][0]);
      acc[1][1] = fmaf(qv.y, kv.y, acc[1][1]);
      acc[2][0] = fmaf(qv.z, kv.x, acc[2][0]);
      acc[2][1] = fmaf(qv.z, kv.y, acc[2][1]);
      acc[3][0] = fmaf(qv.w, kv.x, acc[3][0]);
      acc[3][1] = fmaf(qv.w, kv.y, acc[3][1]);
    }
    const int j = j0 + 2 * kp;
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      float* srow = scores + (size_t)(4 * rg + r) * nb_pad;
      if (j < nb) srow[j] = acc[r][0] * 0.125f;       // 1 / sqrt(64), exact
      if (j + 1 < nb) srow[j + 1] = acc[r][1] * 0.125f;
    }
  }
  __syncthreads();

  // One warp per row.
  uint32_t* whist = hist + warp * kWarpScratchWords;
#pragma unroll 1
  for (int r = warp; r < R; r += 8) {
    const int i = i0 + r;
    if (i >= nb) break;
    float* row = scores + (size_t)r * nb_pad;
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
    warp_topk_row_binned(row, nb, a.budget, whist, a.idx + ((size_t)h * nb + i) * a.budget, lane);
  }
}

template <int R>
size_t score_smem_bytes(int nb_pad) {
  return sizeof(float) * ((size_t)kHeadDim * (2048 / R) + (size_t)kHeadDim * R +
                          8 * (size_t)kWarpScratchWords + (size_t)R * nb_pad);
}

template <int R>
ress_status launch_score(const ScoreArgs& a0, cudaStream_t st) {
  ScoreArgs a = a0;
  a.tiles_per_head = (a.nb + R - 1) / R;
  const size_t smem = score_smem_bytes<R>(a.nb_pad);
  if (ress_status st_ = record_cuda(cudaFuncSetAttribute(score_topk_kernel<R>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)smem)))
    return st_;
  score_topk_kernel<R><<<a.heads * a.tiles_per_head, 256, smem, st>>>(a);
  return record_cuda(cudaGetLastError());
}

}  // namespace

SelectLayout select_layout(const Geometry& g, bool with_v) {
  SelectLayout l{};
  size_t off = 0;
  l.qbar = off;
  off += align256(sizeof(float) * (size_t)g.heads * g.nb * kHeadDim);
  l.kbar_t = off;
  off += align256(sizeof(float) * (size_t)g.heads * kHeadDim * g.nb_pad);
  if (with_v) {
    l.vbar = off;
    off += align256(sizeof(float) * (size_t)g.heads * g.nb * kHeadDim);
    l.contrast = off;
    off += align256(sizeof(float) * (size_t)g.heads * g.nb);
  } else {
    l.vbar = l.contrast = 0;
  }
  l.total = off;
  return l;
}

ress_status launch_select(const Geometry& g, const void* q, const void* k, const void* v,
                          int budget, float lambda, int32_t* idx, void* ws, cudaStream_t st) {
  const bool with_v = lambda != 0.f;
  const SelectLayout lay = select_layout(g, with_v);
  uint8_t* w = static_cast<uint8_t*>(ws);
  float* qbar = reinterpret_cast<float*>(w + lay.qbar);
  float* kbar_t = reinterpret_cast<float*>(w + lay.kbar_t);
  float* vbar = with_v ? reinterpret_cast<float*>(w + lay.vbar) : nullptr;
  float* contrast = with_v ? reinterpret_cast<float*>(w + lay.contrast) : nullptr;

  PoolArgs pa{};
  pa.src[0] = q;  pa.dst[0] = qbar;   pa.layout[0] = 0;
  pa.src[1] = k;  pa.dst[1] = kbar_t; pa.layout[1] = 1;
  pa.src[2] = v;  pa.dst[2] = vbar;   pa.layout[2] = 0;
  pa.nb = g.nb;
  pa.nb_pad = g.nb_pad;
  pa.block = g.block;
  pa.heads = g.heads;
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
  ScoreArgs sa{};
  sa.qbar = qbar;
  sa.kbar_t = kbar_t;
  sa.contrast = contrast;
  sa.idx = idx;
  sa.heads = g.heads;
  sa.nb = g.nb;
  sa.nb_pad = g.nb_pad;
  sa.budget = budget;
  sa.lambda = lambda;
  if (g.nb <= 2304) return launch_score<16>(sa, st);
  return launch_score<8>(sa, st);
}

}  // namespace ress
