// ReSS-style drift-based selection with iterative restoration, on pooled
// contributions (one warp per (head, query block) row).
//
// For query block i of head h, with p_ij the pooled probabilities of stage 1
// (softmax over all key blocks of Qbar_i . Kbar_j / sqrt(d)) and Vbar_j the
// pooled values, key block j contributes c_j = p_ij Vbar_j to the pooled
// output.  The drift score of block j is |c_j|; the initial kept set is the
// `budget` blocks of largest score (ties to the lower index).  Each
// restoration round then looks at the drop set D (the complement) and its
// sum T = sum_{j in D} c_j: the `cand` dropped blocks of largest gain
// 2 <T, c_b> - |c_b|^2 and the `cand` kept blocks of smallest cost
// 2 <T, c_a> + |c_a|^2 (ties to the lower index) form the candidate pairs, and
// the pair of smallest |T - c_b + c_a| (ties: lower b, then lower a) is
// swapped if that is below |T|; otherwise restoration stops.  The result is
// the last accepted set, which has the smallest drift of all rounds.
//
// One warp per row; the row's probabilities, drift scores, value norms and
// candidate contributions live in shared memory, the pooled keys and values
// (transposed, [64][nb_pad] per head) are read from the workspace.
//
// Sources: ReSS (thelatestinai.com) Abstract and Fig. 1 (drift: the shift a
// masked block leaves in the residual stream; the drift of a drop set depends
// on the directions of the contributions), Fig. 3(b) (the blocks of highest
// drift score form the initial set), Fig. 3(c) and Fig. 7 (restoration swaps
// blocks while preserving the budget; three to four rounds saturate), Table
// S3 (track-best).  The swap rule and the pooled contributions are this
// library's reading; the pages give neither.
#include "ress_common.cuh"
#include "ress_internal.h"
#include "ress_topk.cuh"

namespace ress {

namespace {

constexpr int kRsMaxWarps = 4;       // rows per CTA, at most
constexpr int kRsMaxCand = 16;

struct RestoreArgs {
  const float* qbar;     // [H][nb][64]
  const float* kbar_t;   // [H][64][nb_pad]
  const float* vbar_t;   // [H][64][nb_pad]
  int32_t* idx;          // [H][nb][budget]
  float* j_init;         // [H][nb] or null
  float* j_final;        // [H][nb] or null
  int heads, nb, nb_pad, budget, rounds, cand;
  int row_stride;        // floats of one shared-memory row (nb rounded up to 4)
  int warp_floats;       // floats of one warp's shared memory
};

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ float warp_add(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Warp-wide best (value, index): the largest (kLargest) or smallest value,
// ties to the lower index; entries with index INT_MAX do not count.
template <bool kLargest>
__device__ __forceinline__ void warp_best(float& v, int& j) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const float ov = __shfl_xor_sync(0xffffffffu, v, o);
    const int oj = __shfl_xor_sync(0xffffffffu, j, o);
    const bool take = (oj != INT_MAX) &&
                      (j == INT_MAX || (kLargest ? ov > v : ov < v) || (ov == v && oj < j));
    if (take) {
      v = ov;
      j = oj;
    }
  }
}

// out[j] = sum_d x[d] * mt[d][j] for every j < nb (d ascending, float32
// FMA): lane l takes blocks l, l + 32, l + 64, l + 96 of each group of 128 at
// once, four independent chains with their loads in flight together.  Loads
// past nb stay inside the padded row (index clamped to nb_pad - 1) and are
// not stored.
__device__ __forceinline__ void dots4(const float* x, const float* __restrict__ mt, int nb_pad,
                                      int nb, float* out, int lane) {
  for (int j0 = lane; j0 < nb; j0 += 128) {
    int jj[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) jj[u] = min(j0 + 32 * u, nb_pad - 1);
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 4
    for (int d = 0; d < kHeadDim; ++d) {
      const float xd = x[d];
      const float* row = mt + (size_t)d * nb_pad;
#pragma unroll
      for (int u = 0; u < 4; ++u) acc[u] = fmaf(xd, row[jj[u]], acc[u]);
    }
#pragma unroll
    for (int u = 0; u < 4; ++u)
      if (j0 + 32 * u < nb) out[j0 + 32 * u] = acc[u];
  }
}

__global__ void __launch_bounds__(32 * kRsMaxWarps) restore_kernel(const RestoreArgs a) {
  extern __shared__ __align__(16) float rsm[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int row = blockIdx.x * (blockDim.x >> 5) + warp;
  if (row >= a.heads * a.nb) return;
  const int nb = a.nb, rs = a.row_stride;
  const int words = (nb + 31) >> 5;
  // This warp's shared memory: p, the drift score / <T, Vbar_j>, |Vbar_j|^2
  // (one row each), T, the candidates' contributions, their indices, the
  // kept bitmap, the top-k scratch and the initial kept list.
  float* p = rsm + (size_t)warp * a.warp_floats;
  float* dot = p + rs;
  float* vn2 = dot + rs;
  float* T = vn2 + rs;                                         // [64]
  float* cbv = T + 64;                                         // [kRsMaxCand][64]
  float* cav = cbv + kRsMaxCand * 64;                          // [kRsMaxCand][64]
  int* cb = reinterpret_cast<int*>(cav + kRsMaxCand * 64);     // [kRsMaxCand]
  int* ca = cb + kRsMaxCand;                                   // [kRsMaxCand]
  uint32_t* kept = reinterpret_cast<uint32_t*>(ca + kRsMaxCand);   // [128]
  uint32_t* scratch = kept + 128;                              // [kWarpScratchStride]
  int32_t* list = reinterpret_cast<int32_t*>(scratch + kWarpScratchStride);   // [rs]

  const int h = row / nb, i = row - h * nb;
  const float* kt = a.kbar_t + (size_t)h * kHeadDim * a.nb_pad;
  const float* vt = a.vbar_t + (size_t)h * kHeadDim * a.nb_pad;
  const float* qrow = a.qbar + ((size_t)h * nb + i) * kHeadDim;
  if (lane < 16) reinterpret_cast<float4*>(T)[lane] = reinterpret_cast<const float4*>(qrow)[lane];
  __syncwarp();

  // Pooled logits (d ascending, float32 FMA, exact 1/8) and probabilities.
  dots4(T, kt, a.nb_pad, nb, p, lane);
  float m = -INFINITY;
  for (int j = lane; j < nb; j += 32) {
    const float s = p[j] * 0.125f;
    p[j] = s;
    m = fmaxf(m, s);
  }
  m = warp_max(m);
  float z = 0.f;
  for (int j = lane; j < nb; j += 32) z += expf(p[j] - m);
  z = warp_add(z);
  const float inv_z = 1.0f / z;
  // p_j, |Vbar_j|^2, the drift score p_j |Vbar_j| and the pooled output
  // O = sum_j c_j, accumulated per lane over its blocks and reduced (d by d).
  float o[kHeadDim];
#pragma unroll
  for (int d = 0; d < kHeadDim; ++d) o[d] = 0.f;
  for (int j = lane; j < nb; j += 32) {
    const float pj = expf(p[j] - m) * inv_z;
    float vv = 0.f;
#pragma unroll
    for (int d = 0; d < kHeadDim; ++d) {
      const float x = vt[(size_t)d * a.nb_pad + j];
      o[d] = fmaf(pj, x, o[d]);
      vv = fmaf(x, x, vv);
    }
    p[j] = pj;
    vn2[j] = vv;
    dot[j] = pj * sqrtf(vv);
  }
#pragma unroll
  for (int d = 0; d < kHeadDim; ++d) o[d] = warp_add(o[d]);
  __syncwarp();
  // Initial kept set: the budget largest drift scores, ties to the lower index.
  warp_topk_row_binned(dot, nb, a.budget, scratch, list, lane);
  __syncwarp();
  for (int w = lane; w < 128; w += 32) kept[w] = 0u;
  __syncwarp();
  for (int r = lane; r < a.budget; r += 32) atomicOr(&kept[list[r] >> 5], 1u << (list[r] & 31));
  __syncwarp();
  // T = O - sum over the kept blocks of c_j (lane l holds d = l and l + 32).
  float t0 = 0.f, t1 = 0.f;
#pragma unroll
  for (int d = 0; d < kHeadDim; ++d) {
    if (d == lane) t0 = o[d];
    if (d == lane + 32) t1 = o[d];
  }
  for (int r = 0; r < a.budget; ++r) {
    const int j = list[r];
    t0 = fmaf(-p[j], vt[(size_t)lane * a.nb_pad + j], t0);
    t1 = fmaf(-p[j], vt[(size_t)(lane + 32) * a.nb_pad + j], t1);
  }
  float jcur2 = warp_add(t0 * t0 + t1 * t1);
  const float j_init = sqrtf(jcur2);

  for (int round = 0; round < a.rounds; ++round) {
    __syncwarp();
    T[lane] = t0;
    T[lane + 32] = t1;
    __syncwarp();
    dots4(T, vt, a.nb_pad, nb, dot, lane);
    __syncwarp();
    // Candidates: the dropped blocks of largest gain 2 <T, c_b> - |c_b|^2 and
    // the kept blocks of smallest cost 2 <T, c_a> + |c_a|^2.
    int nbc = 0, nac = 0;
#pragma unroll 1
    for (int side = 0; side < 2; ++side) {
#pragma unroll 1
      for (int t = 0; t < a.cand; ++t) {
        float bv = 0.f;
        int bj = INT_MAX;
        for (int j = lane; j < nb; j += 32) {
          const bool in_k = (kept[j >> 5] >> (j & 31)) & 1u;
          if (side == 0 ? in_k : !in_k) continue;
          bool taken = false;
          for (int u = 0; u < t; ++u) taken |= (side == 0 ? cb[u] : ca[u]) == j;
          if (taken) continue;
          const float pj = p[j];
          const float c2 = pj * pj * vn2[j];
          const float lin = 2.0f * pj * dot[j];
          const float val = side == 0 ? lin - c2 : lin + c2;
          if (bj == INT_MAX || (side == 0 ? val > bv : val < bv)) {
            bv = val;
            bj = j;
          }
        }
        if (side == 0) warp_best<true>(bv, bj); else warp_best<false>(bv, bj);
        if (bj == INT_MAX) break;
        if (lane == 0) {
          if (side == 0) cb[t] = bj; else ca[t] = bj;
        }
        __syncwarp();
        if (side == 0) nbc = t + 1; else nac = t + 1;
      }
    }
    if (nbc == 0 || nac == 0) break;
    for (int u = 0; u < nbc; ++u) {
      const int j = cb[u];
      cbv[u * 64 + lane] = p[j] * vt[(size_t)lane * a.nb_pad + j];
      cbv[u * 64 + lane + 32] = p[j] * vt[(size_t)(lane + 32) * a.nb_pad + j];
    }
    for (int u = 0; u < nac; ++u) {
      const int j = ca[u];
      cav[u * 64 + lane] = p[j] * vt[(size_t)lane * a.nb_pad + j];
      cav[u * 64 + lane + 32] = p[j] * vt[(size_t)(lane + 32) * a.nb_pad + j];
    }
    __syncwarp();
    // The pair of smallest |T - c_b + c_a|^2 (ties: lower b, then lower a).
    float best = 0.f;
    int best_code = INT_MAX;
    for (int e = lane; e < nbc * nac; e += 32) {
      const int ub = e / nac, ua = e - ub * nac;
      float s = 0.f;
#pragma unroll 8
      for (int d = 0; d < kHeadDim; ++d) {
        const float x = T[d] - cbv[ub * 64 + d] + cav[ua * 64 + d];
        s = fmaf(x, x, s);
      }
      const int code = cb[ub] * nb + ca[ua];
      if (best_code == INT_MAX || s < best || (s == best && code < best_code)) {
        best = s;
        best_code = code;
      }
    }
    warp_best<false>(best, best_code);
    if (!(best < jcur2)) break;
    const int b = best_code / nb, aa = best_code - b * nb;
    __syncwarp();
    if (lane == 0) {
      kept[aa >> 5] &= ~(1u << (aa & 31));
      kept[b >> 5] |= 1u << (b & 31);
    }
    __syncwarp();
    t0 = t0 - p[b] * vt[(size_t)lane * a.nb_pad + b] + p[aa] * vt[(size_t)lane * a.nb_pad + aa];
    t1 = t1 - p[b] * vt[(size_t)(lane + 32) * a.nb_pad + b] +
         p[aa] * vt[(size_t)(lane + 32) * a.nb_pad + aa];
    jcur2 = best;
  }
  // The kept blocks in ascending order.
  int32_t* out = a.idx + ((size_t)h * nb + i) * a.budget;
  int pos = 0;
  for (int w0 = 0; w0 < words; w0 += 32) {
    const int w = w0 + lane;
    const uint32_t m32 = w < words ? kept[w] : 0u;
    const int cnt = __popc(m32);
    int incl = cnt;
#pragma unroll
    for (int o2 = 1; o2 < 32; o2 <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o2);
      if (lane >= o2) incl += y;
    }
    int at = pos + incl - cnt;
    uint32_t mm = m32;
    while (mm) {
      const int bit = __ffs(mm) - 1;
      mm &= mm - 1u;
      if (at < a.budget) out[at] = 32 * w + bit;
      ++at;
    }
    pos += __shfl_sync(0xffffffffu, incl, 31);
  }
  if (lane == 0) {
    if (a.j_init) a.j_init[(size_t)h * nb + i] = j_init;
    if (a.j_final) a.j_final[(size_t)h * nb + i] = sqrtf(jcur2);
  }
}

}  // namespace

RestoreLayout restore_layout(const Geometry& g) {
  RestoreLayout l{};
  size_t off = 0;
  l.qbar = off;
  off += align256(sizeof(float) * (size_t)g.heads * g.nb * kHeadDim);
  l.kbar_t = off;
  off += align256(sizeof(float) * (size_t)g.heads * kHeadDim * g.nb_pad);
  l.vbar_t = off;
  off += align256(sizeof(float) * (size_t)g.heads * kHeadDim * g.nb_pad);
  l.total = off;
  return l;
}

ress_status launch_restore(const Geometry& g, const void* q, const void* k, const void* v,
                           int budget, int rounds, int cand, int32_t* idx, float* j_init,
                           float* j_final, uint8_t* ws, cudaStream_t st) {
  const RestoreLayout lay = restore_layout(g);
  float* qbar = reinterpret_cast<float*>(ws + lay.qbar);
  float* kbar_t = reinterpret_cast<float*>(ws + lay.kbar_t);
  float* vbar_t = reinterpret_cast<float*>(ws + lay.vbar_t);
  if (ress_status s = launch_pool(g, q, k, v, qbar, kbar_t, vbar_t, st)) return s;
  RestoreArgs a{};
  a.qbar = qbar;
  a.kbar_t = kbar_t;
  a.vbar_t = vbar_t;
  a.idx = idx;
  a.j_init = j_init;
  a.j_final = j_final;
  a.heads = g.heads;
  a.nb = g.nb;
  a.nb_pad = g.nb_pad;
  a.budget = budget;
  a.rounds = rounds;
  a.cand = cand;
  a.row_stride = (g.nb + 3) & ~3;
  a.warp_floats = 4 * a.row_stride + 64 + 2 * kRsMaxCand * 64 + 2 * kRsMaxCand + 128 +
                  kWarpScratchStride;
  a.warp_floats = (a.warp_floats + 3) & ~3;
  // As many rows per CTA as fit (nb = 4,096 leaves room for two).
  const size_t per_warp = sizeof(float) * (size_t)a.warp_floats;
  int warps = (int)((227 * 1024) / per_warp);
  if (warps > kRsMaxWarps) warps = kRsMaxWarps;
  if (warps < 1) return RESS_ERR_UNSUPPORTED;
  const size_t smem = per_warp * warps;
  if (ress_status s = record_cuda(cudaFuncSetAttribute(
          restore_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem)))
    return s;
  const int rows = g.heads * g.nb;
  restore_kernel<<<(rows + warps - 1) / warps, 32 * warps, smem, st>>>(a);
  return record_cuda(cudaGetLastError());
}

}  // namespace ress
