// VASC selection: value-aware demand, budgeted binary execution and
// cross-layer memory, one global layer per call.
//
// Per head h, key blocks form fixed pairs of native neighbours (2p, 2p+1);
// an odd final block is a singleton (VASC A.1).  A call
//   1. pools Q, K, V per block (the pooling pass of the other selections);
//   2. vasc_prep_kernel: the RMS contrast of every pair,
//        rho_p = sqrt(mean_d (Vbar_2p - Vbar_2p+1)^2), 0 for a singleton
//      (VASC 4.1, A.3; 1 everywhere when the contrast is switched off, the
//      ablation of VASC Appendix D), and the ranking copy of the memory, each
//      head's balances divided by its largest one (VASC A.4);
//   3. the score kernel in its VASC mode: per (h, i) the demand
//        a_ij = min(1, c_h p_ij rho_pair(j) / sum_j p_ij rho_pair(j))
//      (VASC 4.1, A.2), the ranking score a_ij + mhat_pair(j) (VASC 4.2) and
//      its exact top c_h, ties to the lower index; demand and executed
//      children summed per pair in fixed point;
//   4. vasc_settle_kernel: with D and S the demand and service averaged over
//      query blocks and paired children,
//        memory <- max(0, memory + D - S)
//      (VASC 4.3, A.5: deficits accumulate, clipped at zero).
// The memory is the caller's [H][pairs] float32 array; `reset` treats it as
// zero on entry (a new inference, or a new layout).
//
// Sources: VASC: Value-Aware Sparse Attention with Cross-Layer Memory
// (paperlayer.ai), sections 4.1, 4.2, 4.3, A.1 - A.5 and Appendix D; ReSS
// (thelatestinai.com) Fig. 3 and Table 2 (a budget c_h per head).
#include "ress_common.cuh"
#include "ress_internal.h"

namespace ress {

namespace {

constexpr int kPrepThreads = 1024;   // one or two pairs per thread at nb = 2,200

struct VascPrepArgs {
  const float* vbar_t;   // [H][64][nb_pad] (null when the contrast is off)
  const float* memory;   // [H][pairs]
  float* rho;            // [H][pairs]
  float* mhat;           // [H][pairs]
  unsigned long long* dsum;
  uint32_t* ssum;
  int nb, nb_pad, pairs, value_aware, reset;
};

// One CTA per head.
__global__ void __launch_bounds__(kPrepThreads) vasc_prep_kernel(const VascPrepArgs a) {
  __shared__ float red[kPrepThreads / 32];
  const int h = blockIdx.x;
  const size_t base = (size_t)h * a.pairs;
  const float* mem = a.memory + base;
  float top = 0.f;
  for (int p = threadIdx.x; p < a.pairs; p += kPrepThreads) {
    float r = 1.f;
    if (a.value_aware) {
      r = 0.f;
      if (2 * p + 1 < a.nb) {
        const float* vt = a.vbar_t + (size_t)h * kHeadDim * a.nb_pad + 2 * p;
        // Four partial sums over d (independent loads in flight), added in a
        // fixed order.
        float s4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 4
        for (int d = 0; d < kHeadDim; d += 4) {
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const float x = vt[(size_t)(d + u) * a.nb_pad] - vt[(size_t)(d + u) * a.nb_pad + 1];
            s4[u] = fmaf(x, x, s4[u]);
          }
        }
        const float s = (s4[0] + s4[1]) + (s4[2] + s4[3]);
        r = sqrtf(s * (1.0f / kHeadDim));   // 1/64 is exact
      }
    }
    a.rho[base + p] = r;
    a.dsum[base + p] = 0ull;
    a.ssum[base + p] = 0u;
    if (!a.reset) top = fmaxf(top, mem[p]);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) top = fmaxf(top, __shfl_xor_sync(0xffffffffu, top, o));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = top;
  __syncthreads();
  top = red[0];
#pragma unroll
  for (int w = 1; w < kPrepThreads / 32; ++w) top = fmaxf(top, red[w]);
  for (int p = threadIdx.x; p < a.pairs; p += kPrepThreads)
    a.mhat[base + p] = (a.reset || !(top > 0.f)) ? 0.f : mem[p] / top;
}

struct VascSettleArgs {
  const unsigned long long* dsum;
  const uint32_t* ssum;
  float* memory;
  float* demand;    // [H][pairs] or null
  float* service;   // [H][pairs] or null
  int nb, pairs, total, reset;
};

__global__ void __launch_bounds__(256) vasc_settle_kernel(const VascSettleArgs a) {
  for (int e = blockIdx.x * blockDim.x + threadIdx.x; e < a.total; e += gridDim.x * blockDim.x) {
    const int p = e % a.pairs;
    const int children = (2 * p + 1 < a.nb) ? 2 : 1;
    const double n = (double)a.nb * (double)children;   // query blocks x children
    const double dm = (double)a.dsum[e] * (1.0 / 4294967296.0) / n;
    const double sv = (double)a.ssum[e] / n;
    const double in = a.reset ? 0.0 : (double)a.memory[e];
    a.memory[e] = (float)fmax(0.0, in + dm - sv);
    if (a.demand) a.demand[e] = (float)dm;
    if (a.service) a.service[e] = (float)sv;
  }
}

}  // namespace

VascLayout vasc_layout(const Geometry& g) {
  VascLayout l{};
  const size_t pairs = (size_t)g.heads * vasc_pairs(g.nb);
  size_t off = 0;
  l.qbar = off;
  off += align256(sizeof(float) * (size_t)g.heads * g.nb * kHeadDim);
  l.kbar_t = off;
  off += align256(sizeof(float) * (size_t)g.heads * kHeadDim * g.nb_pad);
  l.vbar_t = off;
  off += align256(sizeof(float) * (size_t)g.heads * kHeadDim * g.nb_pad);
  l.rho = off;
  off += align256(sizeof(float) * pairs);
  l.mhat = off;
  off += align256(sizeof(float) * pairs);
  l.dsum = off;
  off += align256(sizeof(unsigned long long) * pairs);
  l.ssum = off;
  off += align256(sizeof(uint32_t) * pairs);
  l.total = off;
  return l;
}

ress_status launch_vasc(const Geometry& g, const void* q, const void* k, const void* v,
                        const int32_t* budgets, int capacity, bool value_aware, bool reset,
                        float* memory, int32_t* idx, float* demand, float* service, uint8_t* ws,
                        cudaStream_t st) {
  const VascLayout lay = vasc_layout(g);
  float* qbar = reinterpret_cast<float*>(ws + lay.qbar);
  float* kbar_t = reinterpret_cast<float*>(ws + lay.kbar_t);
  float* vbar_t = value_aware ? reinterpret_cast<float*>(ws + lay.vbar_t) : nullptr;
  float* rho = reinterpret_cast<float*>(ws + lay.rho);
  float* mhat = reinterpret_cast<float*>(ws + lay.mhat);
  auto* dsum = reinterpret_cast<unsigned long long*>(ws + lay.dsum);
  auto* ssum = reinterpret_cast<uint32_t*>(ws + lay.ssum);
  const int pairs = vasc_pairs(g.nb);
  if (ress_status s = launch_pool(g, q, k, value_aware ? v : nullptr, qbar, kbar_t, vbar_t, st))
    return s;
  VascPrepArgs pa{};
  pa.vbar_t = vbar_t;
  pa.memory = memory;
  pa.rho = rho;
  pa.mhat = mhat;
  pa.dsum = dsum;
  pa.ssum = ssum;
  pa.nb = g.nb;
  pa.nb_pad = g.nb_pad;
  pa.pairs = pairs;
  pa.value_aware = value_aware ? 1 : 0;
  pa.reset = reset ? 1 : 0;
  vasc_prep_kernel<<<g.heads, kPrepThreads, 0, st>>>(pa);
  if (ress_status s = record_cuda(cudaGetLastError())) return s;
  const VascSelect vs{budgets, rho, mhat, dsum, ssum};
  if (ress_status s = launch_score_vasc(g, qbar, kbar_t, capacity, idx, vs, st)) return s;
  VascSettleArgs sa{};
  sa.dsum = dsum;
  sa.ssum = ssum;
  sa.memory = memory;
  sa.demand = demand;
  sa.service = service;
  sa.nb = g.nb;
  sa.pairs = pairs;
  sa.total = g.heads * pairs;
  sa.reset = reset ? 1 : 0;
  const int blocks = (sa.total + 255) / 256;
  vasc_settle_kernel<<<blocks, 256, 0, st>>>(sa);
  return record_cuda(cudaGetLastError());
}

}  // namespace ress
