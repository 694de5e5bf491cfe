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
// Warp roles (320 threads, one CTA per SM):
//   warp 0     TMA producer: Q tile once, then K/V sub-blocks of each chunk
//              into a 5-stage ring (128-byte swizzle).
//   warp 1     TMEM owner and MMA issuer: S = Q K^T (M=128, N=128, K=64) into
//              one of three TMEM buffers, so the S of a softmax group's next
//              chunk is ready when it finishes the current one; then
//              O += P V (M=128, N=64, K=128) with P read from TMEM.
//   warps 2-9  softmax, one query row per thread, in two groups: warps 2-5
//              take the even chunks and warps 6-9 the odd ones, each group with
//              its own running maximum, sums and O accumulator in TMEM (a
//              split over chunks, merged in the epilogue), so one group's
//              TMEM and barrier latency overlaps the other's exponentials.
//              S is read from TMEM, the online softmax runs in the log2 domain
//              with a lazy rescale of O (only when the running maximum grows
//              by more than 2^8), and P goes back to TMEM as bf16 over the
//              first 64 columns of S; epilogue O / sum(P) and lse, where
//              sum(P) adds the same bf16-rounded values that enter P V (so
//              that the rounding of a dominant probability cancels in O).
//              Three exponentials in four go to MUFU and one to a
//              polynomial on the FMA pipe.
//
// Every mbarrier wait is bounded; on timeout the CTA raises the device error,
// drains its copies and MMAs in flight, frees TMEM and exits.
#include "ress_common.cuh"
#include "ress_internal.h"

namespace ress {

namespace {

constexpr int kRows = 128;
constexpr int kStages = 5;
constexpr int kSBufs = 3;
constexpr int kThreads = 320;
constexpr uint32_t kQBytes = 128 * 128;            // 128 rows x 64 bf16
constexpr uint32_t kSubBytes = 64 * 128;           // 64 keys x 64 bf16
constexpr uint32_t kStageBytes = 4 * kSubBytes;    // K sub0, K sub1, V sub0, V sub1
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS = 0;                      // S buffers at 0, 128, 256 (128 fp32 columns each;
                                                   // P as bf16 in the first 64 columns of its buffer)
constexpr uint32_t kColO = 384;                    // O of the even / odd chunks: 2 x 64 fp32 columns

struct AttnParams {
  DeviceError* err;
  int n;          // key tokens
  int nq;         // query tokens (rows of Q, out and lse); n except in the dense pass
  int heads;
  int nb;         // key blocks
  int nbq;        // query blocks
  int block;
  int budget;
  int tiles_per_head;
  int dense;      // every key block is kept for every query row (idx unused)
  int lay_t, lay_r, lay_s;   // per-view layout (lay_t == 0: none)
  const int32_t* idx;
  void* out;
  float* lse;
};

// Sets the S columns of one 64-key sub-block beyond its valid prefix to -inf
// (padding keys never enter the softmax).
__device__ __forceinline__ void mask_sub_block(uint32_t (&r0)[32], uint32_t (&r1)[32], int valid) {
#pragma unroll
  for (int u = 0; u < 32; ++u) {
    if (u >= valid) r0[u] = 0xFF800000u;
    if (u + 32 >= valid) r1[u] = 0xFF800000u;
  }
}

struct __align__(8) Ctl {
  uint64_t q_full;
  uint64_t kv_full[kStages];
  uint64_t kv_empty[kStages];
  uint64_t s_full[kSBufs];   // S buffer b holds S of chunk c (c % 3 == b)
  uint64_t p_full[kSBufs];   // P of chunk c written into S buffer c % 3
  uint64_t o_done[2];        // PV of a chunk of group g (c % 2 == g) completed
  uint64_t o_full;
  uint64_t merge;            // the odd-chunk group posted its row statistics
  uint64_t mma_done;
  uint32_t tmem_base;
  int abort_flag;
  int n_entries;
  int pad;
  float odd_m[kRows];   // odd-chunk group: reference maximum (log2 domain) per row
  float odd_lr[kRows];  // odd-chunk group: sum of the bf16-rounded probabilities
};

__host__ __device__ inline int words_for(int nb) { return (nb + 31) >> 5; }

size_t attn_smem_bytes(int nb) {
  return 1024 + kQBytes + kStages * kStageBytes + sizeof(Ctl) +
         sizeof(uint32_t) * (2 * (size_t)words_for(nb) + (size_t)nb);
}

// Entry of the sorted list: bits 0..13 the key block (nb <= 16,383), bits
// 30..31 which row halves use it (bit 0: rows 0..63, bit 1: rows 64..127);
// with a layout, bits 14..20 the valid (non-padding) tokens of the block's
// first 64 and bits 21..27 of its second 64 (128-token blocks).
constexpr uint32_t kEntryBlock = 0x3FFFu;
constexpr int kMaxAttnBlocks = 16383;

// Chunk c of the sorted entry list -> token starts of its two 64-key
// sub-blocks and, per sub-block, which row halves use it.
__device__ __forceinline__ void chunk_info(const uint32_t* list, int n_entries, int block, int c,
                                           int& t0, int& t1, uint32_t& m0, uint32_t& m1) {
  if (block == 64) {
    const uint32_t e0 = list[2 * c];
    t0 = (int)(e0 & kEntryBlock) * 64;
    m0 = e0 >> 30;
    if (2 * c + 1 < n_entries) {
      const uint32_t e1 = list[2 * c + 1];
      t1 = (int)(e1 & kEntryBlock) * 64;
      m1 = e1 >> 30;
    } else {  // odd count: repeat a valid sub-block, masked for every row
      t1 = t0;
      m1 = 0;
    }
  } else {
    const uint32_t e0 = list[c];
    t0 = (int)(e0 & kEntryBlock) * 128;
    t1 = t0 + 64;
    m0 = m1 = 3u;
  }
}

// Valid-token prefixes of chunk c's two sub-blocks (layouts only).
__device__ __forceinline__ void chunk_valid(const uint32_t* list, int n_entries, int block, int c,
                                            int& vk0, int& vk1) {
  if (block == 64) {
    vk0 = (int)((list[2 * c] >> 14) & 0x7Fu);
    vk1 = (2 * c + 1 < n_entries) ? (int)((list[2 * c + 1] >> 14) & 0x7Fu) : vk0;
  } else {
    const uint32_t e0 = list[c];
    vk0 = (int)((e0 >> 14) & 0x7Fu);
    vk1 = (int)((e0 >> 21) & 0x7Fu);
  }
}

__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                          DeviceError* err, int detail) {
  const bool ok = mbar_wait(bar, parity, abort_flag, err, detail);
  return __all_sync(0xffffffffu, ok);
}

template <typename OutT>
__device__ __forceinline__ void store_half_row(OutT* dst, const float* o, float inv);

template <>
__device__ __forceinline__ void store_half_row<__nv_bfloat16>(__nv_bfloat16* dst, const float* o,
                                                              float inv) {
  uint4* d4 = reinterpret_cast<uint4*>(dst);
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    uint4 v;
    v.x = pack_bf16x2(o[8 * u + 0] * inv, o[8 * u + 1] * inv);
    v.y = pack_bf16x2(o[8 * u + 2] * inv, o[8 * u + 3] * inv);
    v.z = pack_bf16x2(o[8 * u + 4] * inv, o[8 * u + 5] * inv);
    v.w = pack_bf16x2(o[8 * u + 6] * inv, o[8 * u + 7] * inv);
    d4[u] = v;
  }
}

template <>
__device__ __forceinline__ void store_half_row<float>(float* dst, const float* o, float inv) {
  float4* d4 = reinterpret_cast<float4*>(dst);
#pragma unroll
  for (int u = 0; u < 8; ++u)
    d4[u] = make_float4(o[4 * u] * inv, o[4 * u + 1] * inv, o[4 * u + 2] * inv,
                        o[4 * u + 3] * inv);
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

// 10 warps: three of them share an SM sub-partition's 16,384 registers, so
// the launch bound caps the kernel at 168 registers per thread.
template <typename OutT, bool kLayout>
__global__ void __launch_bounds__(kThreads, 1)
    block_sparse_attn_kernel(const __grid_constant__ CUtensorMap tm_q,
                             const __grid_constant__ CUtensorMap tm_k,
                             const __grid_constant__ CUtensorMap tm_v, const AttnParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024_shared(smem_raw);
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
  const uint32_t bar_s0 = smem_addr(&ctl->s_full[0]);
  const uint32_t bar_p0 = smem_addr(&ctl->p_full[0]);
  const uint32_t bar_od0 = smem_addr(&ctl->o_done[0]);
  const uint32_t bar_o = smem_addr(&ctl->o_full);
  const uint32_t bar_merge = smem_addr(&ctl->merge);
  const uint32_t bar_done = smem_addr(&ctl->mma_done);
  volatile int* abortf = &ctl->abort_flag;

  if (threadIdx.x == 0) {
    mbar_init(bar_q, 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(smem_addr(&ctl->kv_full[s]), 1);
      mbar_init(smem_addr(&ctl->kv_empty[s]), 1);
    }
    for (int b = 0; b < kSBufs; ++b) {
      mbar_init(bar_s0 + 8 * b, 1);
      mbar_init(bar_p0 + 8 * b, 128);
    }
    mbar_init(bar_od0, 1);
    mbar_init(bar_od0 + 8, 1);
    mbar_init(bar_o, 1);
    mbar_init(bar_merge, 128);
    mbar_init(bar_done, 1);
    ctl->abort_flag = 0;
    fence_mbarrier_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_addr(&ctl->tmem_base), kTmemCols);
    tmem_relinquish();
  }
  // Dense pass: every key block, for both query blocks of the tile.
  for (int w = threadIdx.x; w < 2 * W; w += kThreads) {
    const int ww = w < W ? w : w - W;
    bmA[w] = (kLayout && p.dense) ? ((ww < p.nb >> 5) ? 0xFFFFFFFFu : ((1u << (p.nb & 31)) - 1u))
                                  : 0u;
  }
  __syncthreads();

  // Kept sets of the tile's query blocks as bitmaps (duplicates collapse,
  // out-of-range entries are skipped and flagged).
  for (int e = threadIdx.x; e < ((kLayout && p.dense) ? 0 : nsets * p.budget); e += kThreads) {
    const int s = e / p.budget;
    const int r = e - s * p.budget;
    const int qb = qb0 + s;
    if (qb >= p.nbq) continue;
    const int j = p.idx[((size_t)h * p.nbq + qb) * p.budget + r];
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
        uint32_t e = (uint32_t)(w * 32 + bit) | (mem << 30);
        if (kLayout) {   // valid prefixes, once per block instead of once per chunk and thread
          const int tb = (w * 32 + bit) * p.block;
          e |= (uint32_t)layout_valid(p.lay_t, p.lay_r, tb, 64) << 14;
          if (p.block == 128) e |= (uint32_t)layout_valid(p.lay_t, p.lay_r, tb + 64, 64) << 21;
        }
        list[pos++] = e;
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
    // ---------------- TMA producer (whole warp; one elected lane issues) ----------------
    if (n_chunks > 0) {
      if (elect_one()) {
        tma_prefetch_desc(&tm_q);
        tma_prefetch_desc(&tm_k);
        tma_prefetch_desc(&tm_v);
        mbar_arrive_expect_tx(bar_q, kQBytes);
        tma_load_3d(smem_addr(sQ), &tm_q, bar_q, 0, h, row0);
      }
      __syncwarp();
      int issued = 0;
      for (int c = 0; c < n_chunks; ++c) {
        const int s = c % kStages;
        if (c >= kStages &&
            !warp_wait(smem_addr(&ctl->kv_empty[s]), ((c / kStages) - 1) & 1, abortf, p.err, 10))
          break;
        int t0, t1;
        uint32_t m0, m1;
        chunk_info(list, n_entries, p.block, c, t0, t1, m0, m1);
        const uint32_t st = smem_addr(sKV) + (uint32_t)s * kStageBytes;
        const uint32_t bar = smem_addr(&ctl->kv_full[s]);
        if (elect_one()) {
          mbar_arrive_expect_tx(bar, kStageBytes);
          tma_load_3d(st, &tm_k, bar, 0, h, t0);
          tma_load_3d(st + kSubBytes, &tm_k, bar, 0, h, t1);
          tma_load_3d(st + 2 * kSubBytes, &tm_v, bar, 0, h, t0);
          tma_load_3d(st + 3 * kSubBytes, &tm_v, bar, 0, h, t1);
        }
        __syncwarp();
        issued = c + 1;
      }
      // Copies still in flight must land before the CTA can exit.
      for (int c = issued > kStages ? issued - kStages : 0; c < issued; ++c)
        mbar_wait_drain(smem_addr(&ctl->kv_full[c % kStages]), (c / kStages) & 1, p.err, 11);
      mbar_wait_drain(bar_q, 0, p.err, 12);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ---------------- MMA issuer (whole warp; one elected lane issues) ----------------
    if (n_chunks > 0) {
      constexpr uint32_t idS = idesc_bf16_f32(128, 128, false);
      constexpr uint32_t idPV = idesc_bf16_f32(128, 64, true);
      const uint32_t tS = tmem + kColS;
      const uint32_t tO = tmem + kColO;
      const uint64_t dq = smem_desc_sw128(smem_addr(sQ), 16, 1024);
      // Stage s: K at +s*kStageBytes, V at +2*kSubBytes; one 16-key step of V
      // is 2048 bytes (128 units of 16 bytes in the descriptor's address field).
      const uint64_t dk0 = smem_desc_sw128(smem_addr(sKV), 16, 1024);
      const uint64_t dv0 = smem_desc_sw128(smem_addr(sKV) + 2 * kSubBytes, 16384, 1024);
      constexpr uint64_t kStageDesc = kStageBytes >> 4;
      bool ok = warp_wait(bar_q, 0, abortf, p.err, 20);
      auto issue_s = [&](int c) -> bool {
        const int s = c % kStages;
        const int b = c % kSBufs;
        if (!warp_wait(smem_addr(&ctl->kv_full[s]), (c / kStages) & 1, abortf, p.err, 22))
          return false;
        tc_fence_after();
        const uint64_t dk = dk0 + (uint64_t)s * kStageDesc;
        const uint32_t tSb = tS + 128u * (uint32_t)b;
        if (elect_one()) {
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_ss(tSb, dq + (uint64_t)(kk * 2), dk + (uint64_t)(kk * 2), idS, kk > 0 ? 1u : 0u);
          mma_commit(bar_s0 + 8u * (uint32_t)b);
        }
        __syncwarp();
        return true;
      };
      auto issue_pv = [&](int c) {
        const int sp = c % kStages;
        const uint64_t dv = dv0 + (uint64_t)sp * kStageDesc;
        const uint32_t tP = tS + 128u * (uint32_t)(c % kSBufs);
        const uint32_t tOp = tO + 64u * (uint32_t)(c & 1);
        const uint32_t acc0 = c > 1 ? 1u : 0u;
        if (elect_one()) {
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            mma_ts(tOp, tP + kk * 8, dv + (uint64_t)(kk * 128), idPV, kk > 0 ? 1u : acc0);
          mma_commit(smem_addr(&ctl->kv_empty[sp]));
          mma_commit(bar_od0 + 8u * (uint32_t)(c & 1));
        }
        __syncwarp();
      };
      for (int c = 0; ok && c < n_chunks && c < kSBufs; ++c) ok = issue_s(c);
      for (int c = 0; ok && c < n_chunks; ++c) {
        if (!warp_wait(bar_p0 + 8u * (uint32_t)(c % kSBufs), (c / kSBufs) & 1, abortf, p.err, 21)) {
          ok = false;
          break;
        }
        tc_fence_after();
        issue_pv(c);
        // S(c+3) reuses the buffer of P(c); the tensor core runs the MMAs in
        // issue order, so PV(c) has read P(c) before S(c+3) overwrites it.
        if (c + kSBufs < n_chunks && !(ok = issue_s(c + kSBufs))) break;
      }
      if (elect_one()) {
        if (ok) mma_commit(bar_o);
        mma_commit(bar_done);
      }
      __syncwarp();
      mbar_wait_drain(bar_done, 0, p.err, 24);
    }
    __syncwarp();
  } else {
    // ---------------- softmax + epilogue (warps 2..9) ----------------
    const int quad = warp & 3;             // TMEM lanes 32*quad .. 32*quad+31
    const int par = (warp - 2) >> 2;       // 0: even chunks, 1: odd chunks
    const int row = quad * 32 + lane;
    const int half = row >> 6;
    const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
    const uint32_t tS0 = tmem + kColS + lane_off;
    const uint32_t tO = tmem + kColO + lane_off + 64u * (uint32_t)par;
    const uint32_t bar_od = bar_od0 + 8u * (uint32_t)par;
    const float kScaleLog2 = 1.4426950408889634f * 0.125f;   // log2(e) / sqrt(64)
    const float2 scale2 = make_float2(kScaleLog2, kScaleLog2);
    float m_ref = -INFINITY;
    // Sums of the bf16-rounded probabilities that enter P V: the normaliser
    // of O and the sum behind lse (two independent accumulators per row).
    float lr_lo = 0.f, lr_hi = 0.f;
    bool ok = true;
    for (int c = par, it = 0; c < n_chunks; c += 2, ++it) {
      const int b = c % kSBufs;
      const uint32_t tS = tS0 + 128u * (uint32_t)b;
      const uint32_t bar_p = bar_p0 + 8u * (uint32_t)b;
      if (!warp_wait(bar_s0 + 8u * (uint32_t)b, (c / kSBufs) & 1, abortf, p.err, 30)) {
        ok = false;
        break;
      }
      tc_fence_after();
      int t0, t1;
      uint32_t m0, m1;
      chunk_info(list, n_entries, p.block, c, t0, t1, m0, m1);
      // Valid (non-padding) prefix of each 64-key sub-block.
      int vk0 = 64, vk1 = 64;
      if (kLayout) chunk_valid(list, n_entries, p.block, c, vk0, vk1);
      const bool use0 = ((m0 >> half) & 1u) && vk0 > 0;
      const bool use1 = ((m1 >> half) & 1u) && vk1 > 0;
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
      tmem_ld_wait_regs(r[0]);
      tmem_tie_regs(r[1]);
      tmem_tie_regs(r[2]);
      tmem_tie_regs(r[3]);
      if (kLayout) {
        if (vk0 < 64) mask_sub_block(r[0], r[1], vk0);
        if (vk1 < 64) mask_sub_block(r[2], r[3], vk1);
      }
      // Chunk maximum over eight independent chains (short dependency).
      float mxa[8];
#pragma unroll
      for (int q = 0; q < 8; ++q) mxa[q] = -INFINITY;
      if (use0) {
#pragma unroll
        for (int u = 0; u < 8; ++u) {
#pragma unroll
          for (int g = 0; g < 2; ++g) {
            mxa[2 * g] = fmax3(mxa[2 * g], __uint_as_float(r[g][4 * u]), __uint_as_float(r[g][4 * u + 1]));
            mxa[2 * g + 1] =
                fmax3(mxa[2 * g + 1], __uint_as_float(r[g][4 * u + 2]), __uint_as_float(r[g][4 * u + 3]));
          }
        }
      }
      if (use1) {
#pragma unroll
        for (int u = 0; u < 8; ++u) {
#pragma unroll
          for (int g = 2; g < 4; ++g) {
            mxa[2 * g] = fmax3(mxa[2 * g], __uint_as_float(r[g][4 * u]), __uint_as_float(r[g][4 * u + 1]));
            mxa[2 * g + 1] =
                fmax3(mxa[2 * g + 1], __uint_as_float(r[g][4 * u + 2]), __uint_as_float(r[g][4 * u + 3]));
          }
        }
      }
      const float mx = fmaxf(fmaxf(fmax3(mxa[0], mxa[1], mxa[2]), fmax3(mxa[3], mxa[4], mxa[5])),
                             fmaxf(mxa[6], mxa[7]));
      // Lazy rescale: a row moves its reference maximum only when the chunk's
      // maximum exceeds it by more than 8 (a factor 2^8 in p); O and its row
      // sums are rescaled after P is written (below).
      const float m_new = mx * kScaleLog2;
      const bool grow = m_new > m_ref + 8.0f;
      const bool rescale_o = __any_sync(0xffffffffu, grow) && it > 0;
      float alpha = 1.0f;
      if (grow) {
        alpha = fast_exp2(m_ref - m_new);   // 0 on the row's first kept chunk
        lr_lo *= alpha;
        lr_hi *= alpha;
        m_ref = m_new;
      }
      const float2 neg_m2 = make_float2(-m_ref, -m_ref);
#pragma unroll
      for (int g = 0; g < 4; ++g) {
        const bool use = (g < 2) ? use0 : use1;
        uint32_t pk[16];
        if (use) {
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const float2 sv = make_float2(__uint_as_float(r[g][2 * e]), __uint_as_float(r[g][2 * e + 1]));
            const float2 x = ffma2(sv, scale2, neg_m2);
            // One pair in four goes to the FMA pipe, the rest to MUFU.
            const float2 pe = ((e & 3) == 3) ? exp2_poly2(x)
                                             : make_float2(fast_exp2(x.x), fast_exp2(x.y));
            pk[e] = pack_bf16x2(pe.x, pe.y);
            lr_lo = add_bf16_lo(pk[e], lr_lo);
            lr_hi = add_bf16_hi(pk[e], lr_hi);
          }
        } else {
#pragma unroll
          for (int e = 0; e < 16; ++e) pk[e] = 0u;
        }
        tmem_st16(tS + 16 * g, pk);
      }
      if (rescale_o) {
        // This group's O holds its previous chunk (c - 2) once that PV has
        // completed (its commit is this group's o_done phase it - 1; the PV
        // before it completed before S(c) was signalled, so the parity is
        // unambiguous).  O is rescaled before this chunk's PV may start.  The
        // TMEM accesses are warp-collective, so the decision is per warp and
        // rows that keep their reference use alpha = 1.
        if (!warp_wait(bar_od, (it - 1) & 1, abortf, p.err, 32)) {
          ok = false;
          break;
        }
        tc_fence_after();
        uint32_t o[32];
#pragma unroll
        for (int g = 0; g < 2; ++g) {
          tmem_ld32(tO + 32 * g, o);
          tmem_ld_wait_regs(o);
#pragma unroll
          for (int u = 0; u < 32; ++u) o[u] = __float_as_uint(__uint_as_float(o[u]) * alpha);
          tmem_st32(tO + 32 * g, o);
        }
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(bar_p);
    }
    const float lr_sum = lr_lo + lr_hi;
    // Epilogue: the odd-chunk group posts its row statistics; the even-chunk
    // group merges both partial results and writes the row.
    const int tok = row0 + row;
    const bool query_pad = kLayout && !p.dense && (tok % p.lay_t) >= p.lay_r;
    if (par == 1) {
      ctl->odd_m[row] = m_ref;
      ctl->odd_lr[row] = lr_sum;
      mbar_arrive(bar_merge);
    } else if (n_chunks == 0) {
      // No kept key: output 0, lse -inf.
      if (tok < p.nq) {
        float zero[64];
#pragma unroll
        for (int u = 0; u < 64; ++u) zero[u] = 0.f;
        store_row(reinterpret_cast<OutT*>(p.out) + ((size_t)tok * p.heads + h) * kHeadDim, zero,
                  0.f);
        if (p.lse) p.lse[(size_t)h * p.nq + tok] = -INFINITY;
      }
    } else if (ok && warp_wait(bar_o, 0, abortf, p.err, 31) &&
               warp_wait(bar_merge, 0, abortf, p.err, 33)) {
      tc_fence_after();
      const bool two = n_chunks > 1;   // the odd group ran (its TMEM columns hold data)
      const float m1v = two ? ctl->odd_m[row] : -INFINITY;
      const float lr1 = two ? ctl->odd_lr[row] : 0.f;
      const float m = fmaxf(m_ref, m1v);
      const float a0 = fast_exp2(m_ref - m);    // 0 when this group never saw the row
      const float a1 = two ? fast_exp2(m1v - m) : 0.f;
      const float lr = fmaf(a1, lr1, a0 * lr_sum);
      // lr == 0 only when every kept key of the row is padding; a padding
      // query (its lanes diverge only here, after the warp-wide TMEM reads)
      // outputs 0 as well, with lse -inf.
      const bool zero_row = query_pad || !(lr > 0.f);
      const float inv = zero_row ? 0.f : 1.0f / lr;
      OutT* dst = reinterpret_cast<OutT*>(p.out) + ((size_t)tok * p.heads + h) * kHeadDim;
#pragma unroll
      for (int hc = 0; hc < 2; ++hc) {
        uint32_t oa[32], ob[32];
        tmem_ld32(tO + 32 * hc, oa);
        if (two) tmem_ld32(tO + 64 + 32 * hc, ob);
        tmem_ld_wait_regs(oa);
        tmem_tie_regs(ob);
        float of[32];
#pragma unroll
        for (int u = 0; u < 32; ++u) {
          of[u] = a0 * __uint_as_float(oa[u]);
          if (two) of[u] = fmaf(a1, __uint_as_float(ob[u]), of[u]);
          if (zero_row) of[u] = 0.f;
        }
        if (tok < p.nq) store_half_row(dst + 32 * hc, of, inv);
      }
      if (tok < p.nq && p.lse)
        p.lse[(size_t)h * p.nq + tok] =
            zero_row ? -INFINITY : (m + __log2f(lr)) * 0.6931471805599453f;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

__global__ void exp2_poly_test_kernel(const float* __restrict__ x, float* __restrict__ y, int n) {
  const int i = 2 * (blockIdx.x * blockDim.x + threadIdx.x);
  if (i + 1 < n) {
    const float2 r = exp2_poly2(make_float2(x[i], x[i + 1]));
    y[i] = r.x;
    y[i + 1] = r.y;
  } else if (i < n) {
    y[i] = exp2_poly2(make_float2(x[i], 0.f)).x;
  }
}

}  // namespace

ress_status launch_exp2_poly_test(const float* x, float* y, int n, cudaStream_t st) {
  if (n <= 0) return RESS_OK;
  const int pairs = (n + 1) / 2;
  exp2_poly_test_kernel<<<(pairs + 255) / 256, 256, 0, st>>>(x, y, n);
  return record_cuda(cudaGetLastError());
}

bool make_token_map(CUtensorMap* map, const void* base, const Geometry& g, int rows);

template <typename OutT, bool kLayout>
ress_status launch_attn_kernel(dim3 grid, size_t smem, const CUtensorMap& tq,
                               const CUtensorMap& tk, const CUtensorMap& tv, const AttnParams& p,
                               cudaStream_t st) {
  if (ress_status s = record_cuda(cudaFuncSetAttribute(block_sparse_attn_kernel<OutT, kLayout>,
                                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                       (int)smem)))
    return s;
  block_sparse_attn_kernel<OutT, kLayout><<<grid, kThreads, smem, st>>>(tq, tk, tv, p);
  return record_cuda(cudaGetLastError());
}

ress_status launch_attn_rows(const Geometry& g, const void* q, int64_t nq, bool dense,
                             const void* k, const void* v, int budget, const int32_t* idx,
                             void* out, bool out_f32, float* lse, cudaStream_t st) {
  Geometry gq = g;
  gq.n = nq;
  CUtensorMap tq, tk, tv;
  if (!make_token_map(&tq, q, gq, 128) || !make_token_map(&tk, k, g, 64) ||
      !make_token_map(&tv, v, g, 64))
    return RESS_ERR_CUDA;
  AttnParams p{};
  p.err = device_error_ptr();
  if (p.err == nullptr) return RESS_ERR_CUDA;
  p.n = (int)g.n;
  p.nq = (int)nq;
  p.heads = g.heads;
  p.nb = g.nb;
  p.nbq = (int)(nq / g.block);
  p.block = g.block;
  p.budget = budget;
  p.dense = dense ? 1 : 0;
  p.lay_t = g.lay_t;
  p.lay_r = g.lay_r;
  p.lay_s = g.lay_s;
  p.tiles_per_head = (g.block == 64) ? (p.nbq + 1) / 2 : p.nbq;
  p.idx = idx;
  p.out = out;
  p.lse = lse;
  const size_t smem = attn_smem_bytes(g.nb);
  if (smem > 227 * 1024 || g.nb > kMaxAttnBlocks)
    return RESS_ERR_UNSUPPORTED;   // kept-block lists no longer fit
  const dim3 grid((unsigned)(g.heads * p.tiles_per_head));
  // The plain path is compiled without any of the layout's checks.
  const bool lay = g.lay_t != 0 || dense;
  if (out_f32)
    return lay ? launch_attn_kernel<float, true>(grid, smem, tq, tk, tv, p, st)
               : launch_attn_kernel<float, false>(grid, smem, tq, tk, tv, p, st);
  return lay ? launch_attn_kernel<__nv_bfloat16, true>(grid, smem, tq, tk, tv, p, st)
             : launch_attn_kernel<__nv_bfloat16, false>(grid, smem, tq, tk, tv, p, st);
}

ress_status launch_attn(const Geometry& g, const void* q, const void* k, const void* v,
                        int budget, const int32_t* idx, void* out, bool out_f32, float* lse,
                        cudaStream_t st) {
  return launch_attn_rows(g, q, g.n, false, k, v, budget, idx, out, out_f32, lse, st);
}

}  // namespace ress
