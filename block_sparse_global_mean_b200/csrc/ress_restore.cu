// ReSS-style drift-based selection with iterative restoration, on pooled
// contributions (one CTA per (head, query block) row).
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
// One CTA of four warps per row: the passes over the row's key blocks (logits,
// values, the per-round products with T) are split over all 128 threads, the
// row's probabilities, drift scores, value norms and candidate contributions
// live in shared memory, and the pooled keys and values (transposed,
// [64][nb_pad] per head) are read from the workspace.  Each thread keeps its
// best candidates of a side in registers and the CTA merges them.  Sums
// across threads follow a fixed order, so the result is deterministic.
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

constexpr int kRsThreads = 128;      // one row per CTA
constexpr int kRsWarps = kRsThreads / 32;
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

// (value, index) v beats (ov, oj): the larger (kLargest) or smaller value,
// ties to the lower index; index INT_MAX is no entry.
template <bool kLargest>
__device__ __forceinline__ bool beats(float v, int j, float ov, int oj) {
  if (j == INT_MAX) return false;
  if (oj == INT_MAX) return true;
  return (kLargest ? v > ov : v < ov) || (v == ov && j < oj);
}

template <bool kLargest>
__device__ __forceinline__ void warp_best(float& v, int& j) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const float ov = __shfl_xor_sync(0xffffffffu, v, o);
    const int oj = __shfl_xor_sync(0xffffffffu, j, o);
    if (beats<kLargest>(ov, oj, v, j)) {
      v = ov;
      j = oj;
    }
  }
}

// CTA-wide best (value, index) of every thread's candidate; the same result
// in every thread.  Uses red_v / red_j [kRsWarps] and two barriers.
template <bool kLargest>
__device__ __forceinline__ void cta_best(float& v, int& j, float* red_v, int* red_j, int warp,
                                         int lane) {
  warp_best<kLargest>(v, j);
  if (lane == 0) {
    red_v[warp] = v;
    red_j[warp] = j;
  }
  __syncthreads();
  v = red_v[0];
  j = red_j[0];
#pragma unroll
  for (int w = 1; w < kRsWarps; ++w)
    if (beats<kLargest>(red_v[w], red_j[w], v, j)) {
      v = red_v[w];
      j = red_j[w];
    }
  __syncthreads();
}

// CTA-wide sum (fixed order: lanes by a shuffle tree, then warps 0..3).
__device__ __forceinline__ float cta_add(float v, float* red, int warp, int lane) {
  v = warp_add(v);
  if (lane == 0) red[warp] = v;
  __syncthreads();
  float s = red[0];
#pragma unroll
  for (int w = 1; w < kRsWarps; ++w) s += red[w];
  __syncthreads();
  return s;
}

// out[j] = sum_d x[d] * mt[d][j] for every j < nb (d ascending, float32
// FMA, one chain per j): thread t takes the four consecutive blocks 4t .. 4t+3
// of each group of 512 with one 16-byte load per d and two packed FMAs.  The
// rows of mt are nb_pad (a multiple of 256) floats, so the loads past nb stay
// inside the row; those results are not stored.
__device__ __forceinline__ void dots4(const float* x, const float* __restrict__ mt, int nb_pad,
                                      int nb, float* out, int tid) {
  for (int j0 = 4 * tid; j0 < nb; j0 += 4 * kRsThreads) {
    float2 a01 = make_float2(0.f, 0.f), a23 = make_float2(0.f, 0.f);
#pragma unroll 4
    for (int d4 = 0; d4 < kHeadDim; d4 += 4) {
      const float4 xv = *reinterpret_cast<const float4*>(x + d4);
      const float xs[4] = {xv.x, xv.y, xv.z, xv.w};
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const float4 m = *reinterpret_cast<const float4*>(mt + (size_t)(d4 + u) * nb_pad + j0);
        const float2 xx = make_float2(xs[u], xs[u]);
        a01 = ffma2(xx, make_float2(m.x, m.y), a01);
        a23 = ffma2(xx, make_float2(m.z, m.w), a23);
      }
    }
    if (j0 + 3 < nb) {
      *reinterpret_cast<float4*>(out + j0) = make_float4(a01.x, a01.y, a23.x, a23.y);
    } else {
      const float r[4] = {a01.x, a01.y, a23.x, a23.y};
#pragma unroll
      for (int u = 0; u < 4; ++u)
        if (j0 + u < nb) out[j0 + u] = r[u];
    }
  }
}

// The `a.cand` best blocks of one side into out[] (kLargest: the dropped
// blocks of largest gain; else the kept blocks of smallest cost), ties to the
// lower index; their number goes to n.  Returns whether any was found.
template <bool kLargest>
__device__ __forceinline__ bool side_candidates(const RestoreArgs& a, const uint32_t* kept,
                                                const float* p, const float* vn2,
                                                const float* dot, int* out, float* red_v,
                                                int* red_j, int tid, int warp, int lane, int nb,
                                                int& n) {
  float v[kRsMaxCand];
  int jx[kRsMaxCand];
#pragma unroll
  for (int u = 0; u < kRsMaxCand; ++u) {
    v[u] = 0.f;
    jx[u] = INT_MAX;
  }
  for (int j = tid; j < nb; j += kRsThreads) {
    const bool in_k = (kept[j >> 5] >> (j & 31)) & 1u;
    if (kLargest ? in_k : !in_k) continue;
    const float pj = p[j];
    const float c2 = pj * pj * vn2[j];
    const float lin = 2.0f * pj * dot[j];
    float cv = kLargest ? lin - c2 : lin + c2;
    int cj = j;
    if (!beats<kLargest>(cv, cj, v[kRsMaxCand - 1], jx[kRsMaxCand - 1])) continue;
    // Insert: the carried entry swaps with every slot it beats.
#pragma unroll
    for (int u = 0; u < kRsMaxCand; ++u) {
      if (beats<kLargest>(cv, cj, v[u], jx[u])) {
        const float tv = v[u];
        const int tj = jx[u];
        v[u] = cv;
        jx[u] = cj;
        cv = tv;
        cj = tj;
      }
    }
  }
  n = 0;
#pragma unroll 1
  for (int t = 0; t < a.cand; ++t) {
    float bv = v[0];
    int bj = jx[0];
    cta_best<kLargest>(bv, bj, red_v, red_j, warp, lane);
    if (bj == INT_MAX) break;
    if (jx[0] == bj) {   // this thread's head won: pop it
#pragma unroll
      for (int u = 0; u + 1 < kRsMaxCand; ++u) {
        v[u] = v[u + 1];
        jx[u] = jx[u + 1];
      }
      v[kRsMaxCand - 1] = 0.f;
      jx[kRsMaxCand - 1] = INT_MAX;
    }
    if (tid == 0) out[t] = bj;
    n = t + 1;
  }
  __syncthreads();
  return n > 0;
}

__global__ void __launch_bounds__(kRsThreads) restore_kernel(const RestoreArgs a) {
  extern __shared__ __align__(16) float rsm[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int row = blockIdx.x;
  const int nb = a.nb, rs = a.row_stride;
  const int words = (nb + 31) >> 5;
  // Shared memory: p, the drift score / <T, Vbar_j>, |Vbar_j|^2, the initial
  // kept list (one row each), T, the candidates' contributions, their
  // indices, the kept bitmap, the top-k scratch and reduction slots.
  float* p = rsm;
  float* dot = p + rs;
  float* vn2 = dot + rs;
  int32_t* list = reinterpret_cast<int32_t*>(vn2 + rs);                 // [rs]
  float* T = reinterpret_cast<float*>(list + rs);                      // [64]
  float* cbv = T + 64;                                                 // [kRsMaxCand][64]
  float* cav = cbv + kRsMaxCand * 64;                                  // [kRsMaxCand][64]
  int* cb = reinterpret_cast<int*>(cav + kRsMaxCand * 64);             // [kRsMaxCand]
  int* ca = cb + kRsMaxCand;                                           // [kRsMaxCand]
  uint32_t* kept = reinterpret_cast<uint32_t*>(ca + kRsMaxCand);       // [128]
  float* ored = reinterpret_cast<float*>(kept + 128);                  // [kRsWarps][64]
  float* red_v = ored + kRsWarps * 64;                                 // [kRsWarps]
  int* red_j = reinterpret_cast<int*>(red_v + kRsWarps);               // [kRsWarps]
  uint32_t* scratch = reinterpret_cast<uint32_t*>(red_j + kRsWarps);   // [kWarpScratchStride]

  const int h = row / nb, i = row - h * nb;
  const float* kt = a.kbar_t + (size_t)h * kHeadDim * a.nb_pad;
  const float* vt = a.vbar_t + (size_t)h * kHeadDim * a.nb_pad;
  const float* qrow = a.qbar + ((size_t)h * nb + i) * kHeadDim;
  if (tid < 16) reinterpret_cast<float4*>(T)[tid] = reinterpret_cast<const float4*>(qrow)[tid];
  for (int w = tid; w < 128; w += kRsThreads) kept[w] = 0u;
  __syncthreads();

  // Pooled logits (d ascending, float32 FMA, exact 1/8) and probabilities.
  dots4(T, kt, a.nb_pad, nb, p, tid);
  __syncthreads();   // the logits were written by other threads than read them below
  float m = -INFINITY;
  for (int j = tid; j < nb; j += kRsThreads) {
    const float s = p[j] * 0.125f;
    p[j] = s;
    m = fmaxf(m, s);
  }
  m = warp_max(m);
  if (lane == 0) red_v[warp] = m;
  __syncthreads();
  m = fmaxf(fmaxf(red_v[0], red_v[1]), fmaxf(red_v[2], red_v[3]));
  __syncthreads();
  float z = 0.f;
  for (int j = tid; j < nb; j += kRsThreads) z += expf(p[j] - m);
  z = cta_add(z, red_v, warp, lane);
  const float inv_z = 1.0f / z;
  // p_j, |Vbar_j|^2, the drift score p_j |Vbar_j| and the pooled output
  // O = sum_j c_j, accumulated per thread over its blocks and reduced.
  float o[kHeadDim];
#pragma unroll
  for (int d = 0; d < kHeadDim; ++d) o[d] = 0.f;
  for (int j = tid; j < nb; j += kRsThreads) {
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
  for (int d = 0; d < kHeadDim; ++d) {
    const float od = warp_add(o[d]);
    if (lane == 0) ored[warp * 64 + d] = od;
  }
  __syncthreads();
  // Initial kept set: the budget largest drift scores, ties to the lower index.
  if (warp == 0) warp_topk_row_binned(dot, nb, a.budget, scratch, list, lane);
  __syncthreads();
  for (int r = tid; r < a.budget; r += kRsThreads)
    atomicOr(&kept[list[r] >> 5], 1u << (list[r] & 31));
  // T = O - sum over the kept blocks of c_j: thread (d, half) sums half of the
  // kept list for dimension d.
  {
    const int d = tid & 63, half = tid >> 6;
    float acc = 0.f;
    for (int r = half; r < a.budget; r += 2) {
      const int j = list[r];
      acc = fmaf(p[j], vt[(size_t)d * a.nb_pad + j], acc);
    }
    cbv[half * 64 + d] = acc;   // scratch use of the candidate area
  }
  __syncthreads();
  if (tid < 64)
    T[tid] = ((ored[tid] + ored[64 + tid]) + (ored[128 + tid] + ored[192 + tid])) -
             (cbv[tid] + cbv[64 + tid]);
  __syncthreads();
  float jcur2 = 0.f;
  {
    const float t = tid < 64 ? T[tid] : 0.f;
    jcur2 = cta_add(t * t, red_v, warp, lane);
  }
  const float j_init = sqrtf(jcur2);

  for (int round = 0; round < a.rounds; ++round) {
    dots4(T, vt, a.nb_pad, nb, dot, tid);
    __syncthreads();
    // Candidates: the dropped blocks of largest gain 2 <T, c_b> - |c_b|^2 and
    // the kept blocks of smallest cost 2 <T, c_a> + |c_a|^2 (ties to the
    // lower index).  Each thread keeps its best kRsMaxCand of a side in
    // registers in one pass over its blocks, then the CTA takes the best
    // `cand` by repeatedly choosing among the threads' heads.
    int nbc = 0, nac = 0;   // the same in every thread: every branch below is uniform
    if (side_candidates<true>(a, kept, p, vn2, dot, cb, red_v, red_j, tid, warp, lane, nb, nbc))
      side_candidates<false>(a, kept, p, vn2, dot, ca, red_v, red_j, tid, warp, lane, nb, nac);
    if (nbc == 0 || nac == 0) break;
    for (int e = tid; e < nbc * 64; e += kRsThreads) {
      const int u = e >> 6, d = e & 63;
      cbv[e] = p[cb[u]] * vt[(size_t)d * a.nb_pad + cb[u]];
    }
    for (int e = tid; e < nac * 64; e += kRsThreads) {
      const int u = e >> 6, d = e & 63;
      cav[e] = p[ca[u]] * vt[(size_t)d * a.nb_pad + ca[u]];
    }
    __syncthreads();
    // The pair of smallest |T - c_b + c_a|^2 (ties: lower b, then lower a).
    float best = 0.f;
    int best_code = INT_MAX;
    for (int e = tid; e < nbc * nac; e += kRsThreads) {
      const int ub = e / nac, ua = e - ub * nac;
      float s = 0.f;
#pragma unroll 8
      for (int d = 0; d < kHeadDim; ++d) {
        const float x = T[d] - cbv[ub * 64 + d] + cav[ua * 64 + d];
        s = fmaf(x, x, s);
      }
      const int code = cb[ub] * nb + ca[ua];
      if (beats<false>(s, code, best, best_code)) {
        best = s;
        best_code = code;
      }
    }
    cta_best<false>(best, best_code, red_v, red_j, warp, lane);
    if (!(best < jcur2)) break;
    const int b = best_code / nb, aa = best_code - b * nb;
    if (tid == 0) {
      kept[aa >> 5] &= ~(1u << (aa & 31));
      kept[b >> 5] |= 1u << (b & 31);
    }
    if (tid < 64)
      T[tid] = T[tid] - p[b] * vt[(size_t)tid * a.nb_pad + b] +
               p[aa] * vt[(size_t)tid * a.nb_pad + aa];
    __syncthreads();
    jcur2 = best;
  }
  // The kept blocks in ascending order (warp 0).
  if (warp == 0) {
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
  const size_t floats = 4 * (size_t)a.row_stride + 64 + 2 * kRsMaxCand * 64 + 2 * kRsMaxCand +
                        128 + kRsWarps * 64 + 2 * kRsWarps + kWarpScratchStride;
  const size_t smem = sizeof(float) * floats;
  if (smem > 227 * 1024) return RESS_ERR_UNSUPPORTED;
  if (ress_status s = record_cuda(cudaFuncSetAttribute(
          restore_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem)))
    return s;
  restore_kernel<<<g.heads * g.nb, kRsThreads, smem, st>>>(a);
  return record_cuda(cudaGetLastError());
}

}  // namespace ress
