// Stage 2: block-sparse attention forward on tcgen05 tensor cores.
//
// One CTA computes a 128-row query tile of one head: two consecutive 64-token
// query blocks (block 64) or one 128-token query block (block 128).  The key
// blocks it visits are the union of the tile's kept sets, in ascending order,
// two 64-key sub-blocks per 128-key chunk; each row half applies its own kept
// set as a warp-uniform mask, so every row is normalised over its own kept
// tokens only (ReSS Table S6 / VASC 4.2: the selection's binary block mask
// drives one shared sparse kernel; ReSS Table S5: no causal mask).
//
// Warp roles (192 threads, two CTAs per SM):
//   warp 0     TMA producer: Q tile once, then K/V sub-blocks of each chunk
//              into a 2-stage ring (128-byte swizzle).
//   warp 1     TMEM owner and MMA issuer: S = Q K^T (M=128, N=128, K=64) into
//              TMEM, then O += P V (M=128, N=64, K=128) with P read from TMEM.
//   warps 2-5  softmax: one query row per thread; S from TMEM, online softmax
//              in the log2 domain with a lazy rescale of O (only when the
//              running maximum grows by more than 2^8), P written back to TMEM
//              as bf16 over the first 64 columns of S; epilogue O / sum(P) and lse.
//
// Every mbarrier wait is bounded; on timeout the CTA raises the device error,
// drains its copies and MMAs in flight, frees TMEM and exits.
#include "ress_common.cuh"
#include "ress_internal.h"

namespace ress {

namespace {

constexpr int kRows = 128;
constexpr int kStages = 2;
constexpr int kThreads = 192;
constexpr uint32_t kQBytes = 128 * 128;            // 128 rows x 64 bf16
constexpr uint32_t kSubBytes = 64 * 128;           // 64 keys x 64 bf16
constexpr uint32_t kStageBytes = 4 * kSubBytes;    // K sub0, K sub1, V sub0, V sub1
constexpr uint32_t kTmemCols = 256;
constexpr uint32_t kColS = 0;                      // S: 128 fp32 columns; P: bf16 in cols 0..63
constexpr uint32_t kColO = 128;                    // O: 64 fp32 columns

struct AttnParams {
  DeviceError* err;
  int n;
  int heads;
  int nb;
  int block;
  int budget;
  int tiles_per_head;
  const int32_t* idx;
  void* out;
  float* lse;
};

struct __align__(8) Ctl {
  uint64_t q_full;
  uint64_t kv_full[kStages];
  uint64_t kv_empty[kStages];
  uint64_t s_full;
  uint64_t p_full;
  uint64_t o_full;
  uint64_t mma_done;
  uint32_t tmem_base;
  int abort_flag;
  int n_entries;
  int pad;
};

__host__ __device__ inline int words_for(int nb) { return (nb + 31) >> 5; }

size_t attn_smem_bytes(int nb) {
  return 1024 + kQBytes + kStages * kStageBytes + sizeof(Ctl) +
         sizeof(uint32_t) * (2 * (size_t)words_for(nb) + (size_t)nb);
}

// Chunk c of the sorted entry list -> token starts of its two 64-key
// sub-blocks and, per sub-block, which row halves use it (bit 0: rows 0..63,
// bit 1: rows 64..127).
__device__ __forceinline__ void chunk_info(const uint32_t* list, int n_entries, int block, int c,
                                           int& t0, int& t1, uint32_t& m0, uint32_t& m1) {
  if (block == 64) {
    const uint32_t e0 = list[2 * c];
    t0 = (int)(e0 & 0x3FFFFFFFu) * 64;
    m0 = e0 >> 30;
    if (2 * c + 1 < n_entries) {
      const uint32_t e1 = list[2 * c + 1];
      t1 = (int)(e1 & 0x3FFFFFFFu) * 64;
      m1 = e1 >> 30;
    } else {  // odd count: repeat a valid sub-block, masked for every row
      t1 = t0;
      m1 = 0;
    }
  } else {
    const uint32_t e0 = list[c];
    t0 = (int)(e0 & 0x3FFFFFFFu) * 128;
    t1 = t0 + 64;
    m0 = m1 = 3u;
  }
}

__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                          DeviceError* err, int detail) {
  const bool ok = mbar_wait(bar, parity, abort_flag, err, detail);
  return __all_sync(0xffffffffu, ok);
}

template <typename OutT>
__device__ __forceinline__ void store_row(OutT* dst, const float* o, float inv);

template <>
__device__ __forceinline__ void store_row<__nv_bfloat16>(__nv_bfloat16* dst, const float* o,
                                                         float inv) {
  uint4* d4 = reinterpret_cast<uint4*>(dst);
#pragma unroll
  for (int u = 0; u < 8; ++u) {
    uint4 v;
    v.x = pack_bf16x2(o[8 * u + 0] * inv, o[8 * u + 1] * inv);
    v.y = pack_bf16x2(o[8 * u + 2] * inv, o[8 * u + 3] * inv);
    v.z = pack_bf16x2(o[8 * u + 4] * inv, o[8 * u + 5] * inv);
    v.w = pack_bf16x2(o[8 * u + 6] * inv, o[8 * u + 7] * inv);
    d4[u] = v;
  }
}

template <>
__device__ __forceinline__ void store_row<float>(float* dst, const float* o, float inv) {
  float4* d4 = reinterpret_cast<float4*>(dst);
#pragma unroll
  for (int u = 0; u < 16; ++u)
    d4[u] = make_float4(o[4 * u] * inv, o[4 * u + 1] * inv, o[4 * u + 2] * inv,
                        o[4 * u + 3] * inv);
}

template <typename OutT>
__global__ void __launch_bounds__(kThreads, 2)
    block_sparse_attn_kernel(const __grid_constant__ CUtensorMap tm_q,
                             const __grid_constant__ CUtensorMap tm_k,
                             const __grid_constant__ CUtensorMap tm_v, const AttnParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* sQ = smem;
  uint8_t* sKV = smem + kQBytes;
  Ctl* ctl = reinterpret_cast<Ctl*>(sKV + kStages * kStageBytes);
  const int W = words_for(p.nb);
  uint32_t* bmA = reinterpret_cast<uint32_t*>(ctl + 1);
  uint32_t* bmB = bmA + W;
  uint32_t* list = bmB + W;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int h = blockIdx.x / p.tiles_per_head;
  const int tile = blockIdx.x % p.tiles_per_head;
  const int row0 = tile * kRows;
  const int nsets = (p.block == 64) ? 2 : 1;
  const int qb0 = (p.block == 64) ? 2 * tile : tile;

  const uint32_t bar_q = smem_addr(&ctl->q_full);
  const uint32_t bar_s = smem_addr(&ctl->s_full);
  const uint32_t bar_p = smem_addr(&ctl->p_full);
  const uint32_t bar_o = smem_addr(&ctl->o_full);
  const uint32_t bar_done = smem_addr(&ctl->mma_done);
  volatile int* abortf = &ctl->abort_flag;

  if (threadIdx.x == 0) {
    mbar_init(bar_q, 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(smem_addr(&ctl->kv_full[s]), 1);
      mbar_init(smem_addr(&ctl->kv_empty[s]), 1);
    }
    mbar_init(bar_s, 1);
    mbar_init(bar_p, 128);
    mbar_init(bar_o, 1);
    mbar_init(bar_done, 1);
    ctl->abort_flag = 0;
    fence_mbarrier_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_addr(&ctl->tmem_base), kTmemCols);
    tmem_relinquish();
  }
  for (int w = threadIdx.x; w < 2 * W; w += kThreads) bmA[w] = 0u;
  __syncthreads();

  // Kept sets of the tile's query blocks as bitmaps (duplicates collapse,
  // out-of-range entries are skipped and flagged).
  for (int e = threadIdx.x; e < nsets * p.budget; e += kThreads) {
    const int s = e / p.budget;
    const int r = e - s * p.budget;
    const int qb = qb0 + s;
    if (qb >= p.nb) continue;
    const int j = p.idx[((size_t)h * p.nb + qb) * p.budget + r];
    if (j < 0 || j >= p.nb) {
      raise_device_error(p.err, RESS_ERR_BAD_INDEX, 1);
      continue;
    }
    atomicOr(&(s ? bmB : bmA)[j >> 5], 1u << (j & 31));
  }
  __syncthreads();

  // Union list in ascending block order with per-half membership.
  if (warp == 0) {
    int base = 0;
    for (int w0 = 0; w0 < W; w0 += 32) {
      const int w = w0 + lane;
      const uint32_t a = (w < W) ? bmA[w] : 0u;
      const uint32_t b = (w < W) ? (nsets == 2 ? bmB[w] : a) : 0u;
      uint32_t u = a | b;
      const int cnt = __popc(u);
      int incl = cnt;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      int pos = base + incl - cnt;
      while (u) {
        const int bit = __ffs(u) - 1;
        u &= u - 1u;
        const uint32_t mem = ((a >> bit) & 1u) | (((b >> bit) & 1u) << 1);
        list[pos++] = (uint32_t)(w * 32 + bit) | (mem << 30);
      }
      base += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (lane == 0) ctl->n_entries = base;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();

  const uint32_t tmem = ctl->tmem_base;
  const int n_entries = ctl->n_entries;
  const int n_chunks = (p.block == 64) ? (n_entries + 1) / 2 : n_entries;

  if (warp == 0) {
    // ---------------- TMA producer ----------------
    if (lane == 0 && n_chunks > 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      mbar_arrive_expect_tx(bar_q, kQBytes);
      tma_load_3d(smem_addr(sQ), &tm_q, bar_q, 0, h, row0);
      int issued = 0;
      for (int c = 0; c < n_chunks; ++c) {
        const int s = c % kStages;
        if (c >= kStages &&
            !mbar_wait(smem_addr(&ctl->kv_empty[s]), ((c / kStages) - 1) & 1, abortf, p.err, 10))
          break;
        int t0, t1;
        uint32_t m0, m1;
        chunk_info(list, n_entries, p.block, c, t0, t1, m0, m1);
        uint8_t* st = sKV + s * kStageBytes;
        const uint32_t bar = smem_addr(&ctl->kv_full[s]);
        mbar_arrive_expect_tx(bar, kStageBytes);
        tma_load_3d(smem_addr(st), &tm_k, bar, 0, h, t0);
        tma_load_3d(smem_addr(st + kSubBytes), &tm_k, bar, 0, h, t1);
        tma_load_3d(smem_addr(st + 2 * kSubBytes), &tm_v, bar, 0, h, t0);
        tma_load_3d(smem_addr(st + 3 * kSubBytes), &tm_v, bar, 0, h, t1);
        issued = c + 1;
      }
      // Copies still in flight must land before the CTA can exit.
      for (int c = issued > kStages ? issued - kStages : 0; c < issued; ++c)
        mbar_wait_drain(smem_addr(&ctl->kv_full[c % kStages]), (c / kStages) & 1, p.err, 11);
      mbar_wait_drain(bar_q, 0, p.err, 12);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    if (lane == 0 && n_chunks > 0) {
      constexpr uint32_t idS = idesc_bf16_f32(128, 128, false);
      constexpr uint32_t idPV = idesc_bf16_f32(128, 64, true);
      const uint32_t tS = tmem + kColS;
      const uint32_t tO = tmem + kColO;
      const uint64_t dq = smem_desc_sw128(smem_addr(sQ), 16, 1024);
      bool ok = mbar_wait(bar_q, 0, abortf, p.err, 20);
      auto issue_pv = [&](int c) {
        const int sp = c % kStages;
        const uint32_t vaddr = smem_addr(sKV + sp * kStageBytes + 2 * kSubBytes);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint64_t dv = smem_desc_sw128(vaddr + kk * 2048, 16384, 1024);
          mma_ts(tO, tS + kk * 8, dv, idPV, (c > 0 || kk > 0) ? 1u : 0u);
        }
        mma_commit(smem_addr(&ctl->kv_empty[sp]));
      };
      for (int c = 0; ok && c < n_chunks; ++c) {
        if (c > 0) {
          // P(c-1) must be consumed before S(c) overwrites its columns; the
          // tensor core runs this thread's MMAs in issue order.
          if (!mbar_wait(bar_p, (c - 1) & 1, abortf, p.err, 21)) { ok = false; break; }
          tc_fence_after();
          issue_pv(c - 1);
        }
        const int s = c % kStages;
        if (!mbar_wait(smem_addr(&ctl->kv_full[s]), (c / kStages) & 1, abortf, p.err, 22)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint64_t dk = smem_desc_sw128(smem_addr(sKV + s * kStageBytes), 16, 1024);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          mma_ss(tS, dq + (uint64_t)(kk * 2), dk + (uint64_t)(kk * 2), idS, kk > 0 ? 1u : 0u);
        mma_commit(bar_s);
      }
      if (ok && mbar_wait(bar_p, (n_chunks - 1) & 1, abortf, p.err, 23)) {
        tc_fence_after();
        issue_pv(n_chunks - 1);
        mma_commit(bar_o);
      }
      mma_commit(bar_done);
      mbar_wait_drain(bar_done, 0, p.err, 24);
    }
    __syncwarp();
  } else {
    // ---------------- softmax + epilogue (warps 2..5) ----------------
    const int quad = warp & 3;             // TMEM lanes 32*quad .. 32*quad+31
    const int row = quad * 32 + lane;
    const int half = row >> 6;
    const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
    const uint32_t tS = tmem + kColS + lane_off;
    const uint32_t tO = tmem + kColO + lane_off;
    const float kScaleLog2 = 1.4426950408889634f * 0.125f;   // log2(e) / sqrt(64)
    float m_ref = -INFINITY;
    float l = 0.f;    // sum of the float32 probabilities (for lse)
    float lr = 0.f;   // sum of the same probabilities rounded to bf16 (normaliser of P V)
    bool ok = true;
    for (int c = 0; c < n_chunks; ++c) {
      if (!warp_wait(bar_s, c & 1, abortf, p.err, 30)) { ok = false; break; }
      tc_fence_after();
      int t0, t1;
      uint32_t m0, m1;
      chunk_info(list, n_entries, p.block, c, t0, t1, m0, m1);
      const bool use0 = (m0 >> half) & 1u;
      const bool use1 = (m1 >> half) & 1u;
      if (!use0 && !use1) {
        uint32_t z[32];
#pragma unroll
        for (int u = 0; u < 32; ++u) z[u] = 0u;
        tmem_st32(tS, z);
        tmem_st32(tS + 32, z);
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(bar_p);
        continue;
      }
      uint32_t r[4][32];
      tmem_ld32(tS, r[0]);
      tmem_ld32(tS + 32, r[1]);
      tmem_ld32(tS + 64, r[2]);
      tmem_ld32(tS + 96, r[3]);
      tmem_ld_wait();
      float mx = -INFINITY;
      if (use0) {
#pragma unroll
        for (int u = 0; u < 32; ++u) mx = fmaxf(mx, fmaxf(__uint_as_float(r[0][u]), __uint_as_float(r[1][u])));
      }
      if (use1) {
#pragma unroll
        for (int u = 0; u < 32; ++u) mx = fmaxf(mx, fmaxf(__uint_as_float(r[2][u]), __uint_as_float(r[3][u])));
      }
      // Lazy rescale: a row moves its reference maximum only when the chunk's
      // maximum exceeds it by more than 8 (a factor 2^8 in p).  The TMEM
      // accesses below are warp-collective, so the decision is taken per warp;
      // rows that keep their reference use alpha = 1.
      const float m_new = mx * kScaleLog2;
      const bool grow = m_new > m_ref + 8.0f;
      if (__any_sync(0xffffffffu, grow)) {
        const float alpha = grow ? fast_exp2(m_ref - m_new) : 1.0f;
        if (c > 0) {
          // The PV of chunk c-1 completed before S(c) was signalled.
          uint32_t o[32];
#pragma unroll
          for (int g = 0; g < 2; ++g) {
            tmem_ld32(tO + 32 * g, o);
            tmem_ld_wait();
#pragma unroll
            for (int u = 0; u < 32; ++u) o[u] = __float_as_uint(__uint_as_float(o[u]) * alpha);
            tmem_st32(tO + 32 * g, o);
          }
        }
        if (grow) {
          l *= alpha;
          lr *= alpha;
          m_ref = m_new;
        }
      }
      const float neg_m = -m_ref;
#pragma unroll
      for (int g = 0; g < 4; ++g) {
        const bool use = (g < 2) ? use0 : use1;
        uint32_t pk[16];
        if (use) {
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const float p0 = fast_exp2(fmaf(__uint_as_float(r[g][2 * e]), kScaleLog2, neg_m));
            const float p1 = fast_exp2(fmaf(__uint_as_float(r[g][2 * e + 1]), kScaleLog2, neg_m));
            l += p0 + p1;
            pk[e] = pack_bf16x2(p0, p1);
            lr += __uint_as_float(pk[e] << 16) + __uint_as_float(pk[e] & 0xFFFF0000u);
          }
        } else {
#pragma unroll
          for (int e = 0; e < 16; ++e) pk[e] = 0u;
        }
        tmem_st16(tS + 16 * g, pk);
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(bar_p);
    }
    // Epilogue
    const int tok = row0 + row;
    if (n_chunks == 0) {
      if (tok < p.n) {
        float zero[64];
#pragma unroll
        for (int u = 0; u < 64; ++u) zero[u] = 0.f;
        store_row(reinterpret_cast<OutT*>(p.out) + ((size_t)tok * p.heads + h) * kHeadDim, zero,
                  0.f);
        if (p.lse) p.lse[(size_t)h * p.n + tok] = -INFINITY;
      }
    } else if (ok && warp_wait(bar_o, 0, abortf, p.err, 31)) {
      tc_fence_after();
      uint32_t o[2][32];
      tmem_ld32(tO, o[0]);
      tmem_ld32(tO + 32, o[1]);
      tmem_ld_wait();
      if (tok < p.n) {
        float of[64];
#pragma unroll
        for (int u = 0; u < 32; ++u) {
          of[u] = __uint_as_float(o[0][u]);
          of[32 + u] = __uint_as_float(o[1][u]);
        }
        const float inv = 1.0f / lr;
        store_row(reinterpret_cast<OutT*>(p.out) + ((size_t)tok * p.heads + h) * kHeadDim, of,
                  inv);
        if (p.lse) p.lse[(size_t)h * p.n + tok] = (m_ref + __log2f(l)) * 0.6931471805599453f;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace

bool make_token_map(CUtensorMap* map, const void* base, const Geometry& g, int rows);

ress_status launch_attn(const Geometry& g, const void* q, const void* k, const void* v,
                        int budget, const int32_t* idx, void* out, bool out_f32, float* lse,
                        cudaStream_t st) {
  CUtensorMap tq, tk, tv;
  if (!make_token_map(&tq, q, g, 128) || !make_token_map(&tk, k, g, 64) ||
      !make_token_map(&tv, v, g, 64))
    return RESS_ERR_CUDA;
  AttnParams p{};
  p.err = device_error_ptr();
  if (p.err == nullptr) return RESS_ERR_CUDA;
  p.n = (int)g.n;
  p.heads = g.heads;
  p.nb = g.nb;
  p.block = g.block;
  p.budget = budget;
  p.tiles_per_head = (g.block == 64) ? (g.nb + 1) / 2 : g.nb;
  p.idx = idx;
  p.out = out;
  p.lse = lse;
  const size_t smem = attn_smem_bytes(g.nb);
  const dim3 grid((unsigned)(g.heads * p.tiles_per_head));
  if (out_f32) {
    if (cudaFuncSetAttribute(block_sparse_attn_kernel<float>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
      return RESS_ERR_CUDA;
    block_sparse_attn_kernel<float><<<grid, kThreads, smem, st>>>(tq, tk, tv, p);
  } else {
    if (cudaFuncSetAttribute(block_sparse_attn_kernel<__nv_bfloat16>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
      return RESS_ERR_CUDA;
    block_sparse_attn_kernel<__nv_bfloat16><<<grid, kThreads, smem, st>>>(tq, tk, tv, p);
  }
  return cudaGetLastError() == cudaSuccess ? RESS_OK : RESS_ERR_CUDA;
}

}  // namespace ress
