// Stage 3: per-dropped-block drift on tcgen05 tensor cores.
//
// For a 128-row query tile (two 64-token query blocks, or one 128-token block)
// the CTA visits the union of the tile's dropped key blocks in ascending order.
// Per 128-key chunk:
//   S = Q K^T                          (M=128, N=128, K=64) into TMEM
//   P = exp(S / 8 - lse)  as bf16     (softmax warps; the kept-set lse of the
//                                      sparse pass; 0 where the row keeps the block)
//   C_j = P[:, block j] V[block j]    (one fresh TMEM accumulator per dropped block)
//   T  += P V                         (running sum of every C_j of the row)
// and the softmax warps reduce ||C_j||_F over the block's rows, writing
// drift[h][i][r] (r = rank of j among the dropped blocks of query block i);
// at the end set_drift[h][i] = ||T||_F.
//
// Source: ReSS (thelatestinai.com) Abstract, Fig. 1 and Fig. 3: masking a block
// shifts what attention writes into the residual stream; the drift score
// measures that shift per block, and the drift of a drop set depends on the
// directions of the contributions, so the set drift is the norm of their sum.
//
// Two kernels share this design.  With 64-token blocks (two contributions per
// chunk, all 512 TMEM columns) block_drift_kernel runs the chunk chain
// S -> P -> C_j -> ||C_j|| serially with warps 0 TMA, 1 TMEM + MMA and 2-5
// exponentials and reductions.  With 128-token blocks drift128_kernel (below)
// splits the chunks over two softmax groups, so that one group's exponentials
// overlap the other's contribution MMA and reduction.
#include "ress_common.cuh"
#include "ress_internal.h"

namespace ress {

namespace {

constexpr int kRows = 128;
constexpr int kStages = 2;
constexpr int kThreads = 192;
constexpr uint32_t kQBytes = 128 * 128;
constexpr uint32_t kSubBytes = 64 * 128;
constexpr uint32_t kStageBytes = 4 * kSubBytes;
constexpr uint32_t kColS = 0;     // S (fp32) / P (bf16, cols 0..63)
constexpr uint32_t kColC0 = 128;  // contribution of sub-block 0 (or the whole 128-key block)
constexpr uint32_t kColC1 = 192;  // contribution of sub-block 1 (block 64 only)
constexpr uint32_t kColT = 256;   // running sum T (block_drift_kernel)
constexpr size_t kOneCtaSmem = 116 * 1024;

struct DriftParams {
  DeviceError* err;
  int n;
  int heads;
  int nb;
  int block;
  int budget;
  int tiles_per_head;
  const int32_t* idx;
  const float* lse;
  float* drift;
  float* set_drift;
  int lay_t, lay_r, lay_s;   // per-view layout (lay_t == 0: none)
};

struct __align__(8) Ctl {
  uint64_t q_full;
  uint64_t kv_full[kStages];
  uint64_t kv_empty[kStages];
  uint64_t s_full;
  uint64_t p_full;
  uint64_t c_full;
  uint64_t c_free;
  uint64_t t_full;
  uint64_t mma_done;
  uint64_t red_full;    // the four softmax warps posted this chunk's partial sums
  uint64_t tred_full;   // ... and their partial sums of the running total
  uint32_t tmem_base;
  int abort_flag;
  int n_entries;
  int pad;
  float partial[2][4][2];   // [chunk parity][quad][sub-block] sums of squares
  float tpartial[4];
};

__host__ __device__ inline int words_for(int nb) { return (nb + 31) >> 5; }

size_t drift_smem_bytes(int nb) {
  return 1024 + kQBytes + kStages * kStageBytes + sizeof(Ctl) +
         sizeof(uint32_t) * (4 * (size_t)words_for(nb) + (size_t)nb);
}

__device__ __forceinline__ void chunk_info(const uint32_t* list, int n_entries, int block, int c,
                                           int& t0, int& t1, uint32_t& j0, uint32_t& j1,
                                           uint32_t& m0, uint32_t& m1) {
  if (block == 64) {
    const uint32_t e0 = list[2 * c];
    j0 = e0 & 0x3FFFFFFFu;
    t0 = (int)j0 * 64;
    m0 = e0 >> 30;
    if (2 * c + 1 < n_entries) {
      const uint32_t e1 = list[2 * c + 1];
      j1 = e1 & 0x3FFFFFFFu;
      t1 = (int)j1 * 64;
      m1 = e1 >> 30;
    } else {
      j1 = j0;
      t1 = t0;
      m1 = 0;
    }
  } else {
    const uint32_t e0 = list[c];
    j0 = j1 = e0 & 0x3FFFFFFFu;
    t0 = (int)j0 * 128;
    t1 = t0 + 64;
    m0 = m1 = 3u;
  }
}

__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                          DeviceError* err, int detail) {
  const bool ok = mbar_wait(bar, parity, abort_flag, err, detail);
  return __all_sync(0xffffffffu, ok);
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Rank of block j among the blocks NOT set in `kept` (bitmap) below j.
__device__ __forceinline__ int dropped_rank(const uint32_t* kept, const uint32_t* prefix, int j) {
  const uint32_t below = kept[j >> 5] & ((1u << (j & 31)) - 1u);
  return j - (int)(prefix[j >> 5] + __popc(below));
}

__global__ void __launch_bounds__(kThreads, 1)
    block_drift_kernel(const __grid_constant__ CUtensorMap tm_q,
                       const __grid_constant__ CUtensorMap tm_k,
                       const __grid_constant__ CUtensorMap tm_v, const DriftParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024_shared(smem_raw);
  uint8_t* sQ = smem;
  uint8_t* sKV = smem + kQBytes;
  Ctl* ctl = reinterpret_cast<Ctl*>(sKV + kStages * kStageBytes);
  const int W = words_for(p.nb);
  uint32_t* keptA = reinterpret_cast<uint32_t*>(ctl + 1);
  uint32_t* keptB = keptA + W;
  uint32_t* prefA = keptB + W;
  uint32_t* prefB = prefA + W;
  uint32_t* list = prefB + W;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int h = blockIdx.x / p.tiles_per_head;
  const int tile = blockIdx.x % p.tiles_per_head;
  const int row0 = tile * kRows;
  const int nsets = (p.block == 64) ? 2 : 1;
  const int qb0 = (p.block == 64) ? 2 * tile : tile;
  const bool validB = (p.block == 64) && (qb0 + 1 < p.nb);
  const int n_drop = p.nb - p.budget;

  const uint32_t bar_q = smem_addr(&ctl->q_full);
  const uint32_t bar_s = smem_addr(&ctl->s_full);
  const uint32_t bar_p = smem_addr(&ctl->p_full);
  const uint32_t bar_c = smem_addr(&ctl->c_full);
  const uint32_t bar_cf = smem_addr(&ctl->c_free);
  const uint32_t bar_t = smem_addr(&ctl->t_full);
  const uint32_t bar_done = smem_addr(&ctl->mma_done);
  const uint32_t bar_red = smem_addr(&ctl->red_full);
  const uint32_t bar_tred = smem_addr(&ctl->tred_full);
  volatile int* abortf = &ctl->abort_flag;

  if (threadIdx.x == 0) {
    mbar_init(bar_q, 1);
    mbar_init(bar_red, 128);
    mbar_init(bar_tred, 128);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(smem_addr(&ctl->kv_full[s]), 1);
      mbar_init(smem_addr(&ctl->kv_empty[s]), 1);
    }
    mbar_init(bar_s, 1);
    mbar_init(bar_p, 128);
    mbar_init(bar_c, 1);
    mbar_init(bar_cf, 128);
    mbar_init(bar_t, 1);
    mbar_init(bar_done, 1);
    ctl->abort_flag = 0;
    fence_mbarrier_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_addr(&ctl->tmem_base), 512);
    tmem_relinquish();
  }
  for (int w = threadIdx.x; w < 2 * W; w += kThreads) keptA[w] = 0u;
  __syncthreads();

  for (int e = threadIdx.x; e < nsets * p.budget; e += kThreads) {
    const int s = e / p.budget;
    const int r = e - s * p.budget;
    const int qb = qb0 + s;
    if (qb >= p.nb) continue;
    const int j = p.idx[((size_t)h * p.nb + qb) * p.budget + r];
    if (j < 0 || j >= p.nb) {
      raise_device_error(p.err, RESS_ERR_BAD_INDEX, 2);
      continue;
    }
    // A block named twice leaves more than nb - budget blocks dropped.
    if (atomicOr(&(s ? keptB : keptA)[j >> 5], 1u << (j & 31)) & (1u << (j & 31)))
      raise_device_error(p.err, RESS_ERR_BAD_INDEX, 5);
  }
  __syncthreads();

  // Prefix popcounts of the kept bitmaps and the union of the dropped sets.
  if (warp == 0) {
    int base = 0, baseA = 0, baseB = 0;
    for (int w0 = 0; w0 < W; w0 += 32) {
      const int w = w0 + lane;
      uint32_t valid = 0u;
      if (w < W) valid = (w == W - 1 && (p.nb & 31)) ? ((1u << (p.nb & 31)) - 1u) : 0xffffffffu;
      const uint32_t ka = (w < W) ? keptA[w] : 0u;
      const uint32_t kb = (w < W) ? keptB[w] : 0u;
      const uint32_t a = ~ka & valid;
      const uint32_t b = (nsets == 2) ? (validB ? (~kb & valid) : 0u) : a;
      int ca = __popc(ka), cb = __popc(kb);
      int ia = ca, ib = cb;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int ya = __shfl_up_sync(0xffffffffu, ia, o);
        const int yb = __shfl_up_sync(0xffffffffu, ib, o);
        if (lane >= o) {
          ia += ya;
          ib += yb;
        }
      }
      if (w < W) {
        prefA[w] = (uint32_t)(baseA + ia - ca);
        prefB[w] = (uint32_t)(baseB + ib - cb);
      }
      baseA += __shfl_sync(0xffffffffu, ia, 31);
      baseB += __shfl_sync(0xffffffffu, ib, 31);
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
    // TMA producer: the whole warp follows, one elected lane issues.
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
            !warp_wait(smem_addr(&ctl->kv_empty[s]), ((c / kStages) - 1) & 1, abortf, p.err, 40))
          break;
        int t0, t1;
        uint32_t j0, j1, m0, m1;
        chunk_info(list, n_entries, p.block, c, t0, t1, j0, j1, m0, m1);
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
      for (int c = issued > kStages ? issued - kStages : 0; c < issued; ++c)
        mbar_wait_drain(smem_addr(&ctl->kv_full[c % kStages]), (c / kStages) & 1, p.err, 41);
      mbar_wait_drain(bar_q, 0, p.err, 42);
    }
    __syncwarp();
  } else if (warp == 1) {
    // MMA issuer: the whole warp follows, one elected lane issues.
    if (n_chunks > 0) {
      constexpr uint32_t idS = idesc_bf16_f32(128, 128, false);
      constexpr uint32_t idPV = idesc_bf16_f32(128, 64, true);
      const uint32_t tS = tmem + kColS;
      const uint64_t dq = smem_desc_sw128(smem_addr(sQ), 16, 1024);
      const uint64_t dk0 = smem_desc_sw128(smem_addr(sKV), 16, 1024);
      const uint64_t dv0 = smem_desc_sw128(smem_addr(sKV) + 2 * kSubBytes, 16384, 1024);
      constexpr uint64_t kStageDesc = kStageBytes >> 4;
      constexpr uint64_t kSubDesc = kSubBytes >> 4;
      bool ok = warp_wait(bar_q, 0, abortf, p.err, 50);
      for (int c = 0; ok && c < n_chunks; ++c) {
        const int s = c % kStages;
        if (!warp_wait(smem_addr(&ctl->kv_full[s]), (c / kStages) & 1, abortf, p.err, 51)) break;
        tc_fence_after();
        const uint64_t dk = dk0 + (uint64_t)s * kStageDesc;
        const uint64_t dv = dv0 + (uint64_t)s * kStageDesc;
        if (elect_one()) {
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_ss(tS, dq + (uint64_t)(kk * 2), dk + (uint64_t)(kk * 2), idS, kk > 0 ? 1u : 0u);
          mma_commit(bar_s);
        }
        __syncwarp();
        if (!warp_wait(bar_p, c & 1, abortf, p.err, 52)) break;
        if (c > 0 && !warp_wait(bar_cf, (c - 1) & 1, abortf, p.err, 53)) break;
        tc_fence_after();
        if (elect_one()) {
          if (p.block == 64) {
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
              mma_ts(tmem + kColC0, tS + kk * 8, dv + (uint64_t)(kk * 128), idPV, kk > 0 ? 1u : 0u);
              mma_ts(tmem + kColC1, tS + 32 + kk * 8, dv + kSubDesc + (uint64_t)(kk * 128), idPV,
                     kk > 0 ? 1u : 0u);
            }
          } else {
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)
              mma_ts(tmem + kColC0, tS + kk * 8, dv + (uint64_t)(kk * 128), idPV, kk > 0 ? 1u : 0u);
          }
          // The contributions are signalled as soon as they are done (a commit
          // tracks the MMAs issued before it), so their norms overlap the
          // running sum below and the next chunk's S.
          mma_commit(bar_c);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            mma_ts(tmem + kColT, tS + kk * 8, dv + (uint64_t)(kk * 128), idPV,
                   (c > 0 || kk > 0) ? 1u : 0u);
          mma_commit(smem_addr(&ctl->kv_empty[s]));
          if (c == n_chunks - 1) mma_commit(bar_t);
        }
        __syncwarp();
      }
      if (elect_one()) mma_commit(bar_done);
      __syncwarp();
      mbar_wait_drain(bar_done, 0, p.err, 54);
    }
    __syncwarp();
  } else {
    const int quad = warp & 3;
    const int row = quad * 32 + lane;
    const int half = row >> 6;
    const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
    const uint32_t tS = tmem + kColS + lane_off;
    const float kScaleLog2 = 1.4426950408889634f * 0.125f;
    const int tok = row0 + row;
    // Layout: only the valid, non-special queries drop anything.
    const int pos = p.lay_t != 0 ? tok % p.lay_t : 0;
    const bool live_q = p.lay_t == 0 || (pos < p.lay_r && pos >= p.lay_s);
    const bool all_live = __all_sync(0xffffffffu, live_q);
    const float lse2 =
        (tok < p.n && live_q) ? p.lse[(size_t)h * p.n + tok] * 1.4426950408889634f : 0.f;
    const float neg_l = -lse2;
    const float2 neg_l2 = make_float2(neg_l, neg_l);
    const float2 scale2 = make_float2(kScaleLog2, kScaleLog2);
    const int sub_tid = threadIdx.x - 64;   // 0..127 among the softmax warps
    bool ok = true;
    for (int c = 0; c < n_chunks; ++c) {
      if (!warp_wait(bar_s, c & 1, abortf, p.err, 60)) { ok = false; break; }
      tc_fence_after();
      int t0, t1;
      uint32_t j0, j1, m0, m1;
      chunk_info(list, n_entries, p.block, c, t0, t1, j0, j1, m0, m1);
      const bool use0 = (m0 >> half) & 1u;
      const bool use1 = (m1 >> half) & 1u;
      const int vk0 = layout_valid(p.lay_t, p.lay_r, t0, 64);   // valid keys of each sub-block
      const int vk1 = layout_valid(p.lay_t, p.lay_r, t1, 64);
      if (use0 || use1) {
        // Two halves of 64 columns; P (bf16, two per column) of half hf goes
        // to columns 32 hf .. 32 hf + 31, below the S columns still unread.
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
          uint32_t r[2][32];
          tmem_ld32(tS + 64 * hf, r[0]);
          tmem_ld32(tS + 64 * hf + 32, r[1]);
          tmem_ld_wait_regs(r[0]);
          tmem_tie_regs(r[1]);
#pragma unroll
          for (int g = 0; g < 2; ++g) {
            const bool use = hf == 0 ? use0 : use1;
            uint32_t pk[16];
            const int vk = hf == 0 ? vk0 : vk1;
            if (use && vk == 64 && all_live) {
              // One pair in four on the FMA pipe (polynomial), the rest on MUFU.
#pragma unroll
              for (int e = 0; e < 16; ++e) {
                const float2 x = ffma2(make_float2(__uint_as_float(r[g][2 * e]), __uint_as_float(r[g][2 * e + 1])),
                                       scale2, neg_l2);
                const float2 pe = ((e & 3) == 3) ? exp2_poly2(x)
                                                 : make_float2(fast_exp2(x.x), fast_exp2(x.y));
                pk[e] = pack_bf16x2(pe.x, pe.y);
              }
            } else {
              // Layout: padding keys (columns beyond the sub-block's valid
              // prefix) and the rows of padding and special queries add nothing.
#pragma unroll
              for (int e = 0; e < 16; ++e) {
                const int col = 32 * g + 2 * e;
                float p0 = fast_exp2(fmaf(__uint_as_float(r[g][2 * e]), kScaleLog2, neg_l));
                float p1 = fast_exp2(fmaf(__uint_as_float(r[g][2 * e + 1]), kScaleLog2, neg_l));
                if (!use || !live_q || col >= vk) p0 = 0.f;
                if (!use || !live_q || col + 1 >= vk) p1 = 0.f;
                pk[e] = pack_bf16x2(p0, p1);
              }
            }
            tmem_st16(tS + 32 * hf + 16 * g, pk);
          }
        }
      } else {
        uint32_t z[32];
#pragma unroll
        for (int u = 0; u < 32; ++u) z[u] = 0u;
        tmem_st32(tS, z);
        tmem_st32(tS + 32, z);
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(bar_p);

      if (!warp_wait(bar_c, c & 1, abortf, p.err, 61)) { ok = false; break; }
      tc_fence_after();
      float ss0 = 0.f, ss1 = 0.f;
      {
        // Sum of squares over the 64 columns of a contribution: packed pairs
        // into four independent accumulators (a short dependency chain).
        auto sumsq64 = [&](uint32_t col) -> float {
          uint32_t cv[2][32];
          tmem_ld32(tmem + col + lane_off, cv[0]);
          tmem_ld32(tmem + col + lane_off + 32, cv[1]);
          tmem_ld_wait_regs(cv[0]);
          tmem_tie_regs(cv[1]);
          float2 acc[4];
#pragma unroll
          for (int q = 0; q < 4; ++q) acc[q] = make_float2(0.f, 0.f);
#pragma unroll
          for (int g = 0; g < 2; ++g) {
#pragma unroll
            for (int u = 0; u < 16; ++u) {
              const float2 x = make_float2(__uint_as_float(cv[g][2 * u]), __uint_as_float(cv[g][2 * u + 1]));
              acc[u & 3] = ffma2(x, x, acc[u & 3]);
            }
          }
          return ((acc[0].x + acc[0].y) + (acc[1].x + acc[1].y)) +
                 ((acc[2].x + acc[2].y) + (acc[3].x + acc[3].y));
        };
        ss0 = sumsq64(kColC0);
        if (p.block == 64) ss1 = sumsq64(kColC1);
      }
      tc_fence_before();
      mbar_arrive(bar_cf);
      ss0 = warp_sum(ss0);
      ss1 = warp_sum(ss1);
      if (lane == 0) {
        ctl->partial[c & 1][quad][0] = ss0;
        ctl->partial[c & 1][quad][1] = ss1;
      }
      __syncwarp();
      mbar_arrive(bar_red);
      // Writers: sub_tid 0..3 -> (half, sub-block) for block 64; sub_tid 0 for
      // block 128.  A slot is rewritten two chunks later at the earliest, and
      // no warp can run two chunks ahead of the writers (every chunk's PV
      // waits for all 128 softmax threads).
      const bool writer = (p.block == 64) ? (sub_tid < 4) : (sub_tid == 0);
      const bool have = writer && mbar_wait(bar_red, c & 1, abortf, p.err, 63);
      if (!have) {
        // not a writer (or the wait gave up)
      } else if (p.block == 64) {
        {
          const int hf = sub_tid >> 1, sb = sub_tid & 1;
          const uint32_t mem = sb ? m1 : m0;
          const int qb = qb0 + hf;
          if (((mem >> hf) & 1u) && qb < p.nb) {
            const int j = (int)(sb ? j1 : j0);
            const float ss = ctl->partial[c & 1][2 * hf][sb] + ctl->partial[c & 1][2 * hf + 1][sb];
            const int rnk = dropped_rank(hf ? keptB : keptA, hf ? prefB : prefA, j);
            if (rnk >= 0 && rnk < n_drop)
              p.drift[((size_t)h * p.nb + qb) * n_drop + rnk] = sqrtf(ss);
            else
              raise_device_error(p.err, RESS_ERR_BAD_INDEX, 3);
          }
        }
      } else if (sub_tid == 0) {
        const float ss = ctl->partial[c & 1][0][0] + ctl->partial[c & 1][1][0] +
                         ctl->partial[c & 1][2][0] + ctl->partial[c & 1][3][0];
        const int rnk = dropped_rank(keptA, prefA, (int)j0);
        if (rnk >= 0 && rnk < n_drop)
          p.drift[((size_t)h * p.nb + qb0) * n_drop + rnk] = sqrtf(ss);
        else
          raise_device_error(p.err, RESS_ERR_BAD_INDEX, 3);
      }
      __syncwarp();
    }
    // Drop-set drift J = ||sum_j C_j||_F.
    float tss = 0.f;
    if (ok && n_chunks > 0) {
      if (warp_wait(bar_t, 0, abortf, p.err, 62)) {
        tc_fence_after();
        uint32_t tv[32];
#pragma unroll
        for (int g = 0; g < 2; ++g) {
          tmem_ld32(tmem + kColT + lane_off + 32 * g, tv);
          tmem_ld_wait_regs(tv);
#pragma unroll
          for (int u = 0; u < 32; ++u) {
            const float x = __uint_as_float(tv[u]);
            tss = fmaf(x, x, tss);
          }
        }
      }
    }
    tss = warp_sum(tss);
    if (lane == 0) ctl->tpartial[quad] = tss;
    __syncwarp();
    mbar_arrive(bar_tred);
    const bool twriter = (p.block == 64) ? (sub_tid < 2) : (sub_tid == 0);
    if (p.set_drift && twriter && mbar_wait(bar_tred, 0, abortf, p.err, 64)) {
      if (p.block == 64) {
        if (sub_tid < 2) {
          const int qb = qb0 + sub_tid;
          if (qb < p.nb)
            p.set_drift[(size_t)h * p.nb + qb] =
                sqrtf(ctl->tpartial[2 * sub_tid] + ctl->tpartial[2 * sub_tid + 1]);
        }
      } else if (sub_tid == 0) {
        p.set_drift[(size_t)h * p.nb + qb0] = sqrtf(ctl->tpartial[0] + ctl->tpartial[1] +
                                                    ctl->tpartial[2] + ctl->tpartial[3]);
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


// ---------------------------------------------------------------------------
// 128-token blocks: one CTA per SM, two softmax groups on alternate chunks.
//
// The chunk chain S -> P -> C -> ||C|| of one 128-row tile is split over two
// groups of four softmax warps (warps 2-5 the even chunks, warps 6-9 the odd
// ones), each with its own S buffer (P written over its first 64 columns) and
// its own contribution accumulator in TMEM.  While one group waits for its
// contribution's MMA and reduces it, the other computes exponentials.  The
// running sum T is the sum of the contributions the softmax threads read
// anyway: each thread adds its row of every C_j into registers, and the two
// groups' partial sums meet in shared memory at the end (no running-sum MMA).
// TMEM: S0 0..127, S1 128..255, C0 256..319, C1 320..383.
// ---------------------------------------------------------------------------
constexpr int kThreads2 = 320;
constexpr int kStages2 = 4;
constexpr uint32_t kColC2 = 256;
constexpr int kTStride = 68;   // floats per row of the shared running-sum exchange (padded)

struct __align__(8) Ctl2 {
  uint64_t q_full;
  uint64_t kv_full[kStages2];
  uint64_t kv_empty[kStages2];
  uint64_t s_full[2];
  uint64_t p_full[2];
  uint64_t c_full[2];
  uint64_t c_free[2];
  uint64_t red_full[2];
  uint64_t t_post;      // group 1 wrote its running sums
  uint64_t tred_full;
  uint64_t mma_done;
  uint32_t tmem_base;
  int abort_flag;
  int n_entries;
  int pad;
  float partial[2][2][4];   // [group][chunk parity][quad]
  float tpartial[4];
};

size_t drift128_smem_bytes(int nb) {
  return 1024 + kQBytes + kStages2 * kStageBytes + sizeof(float) * kRows * kTStride + sizeof(Ctl2) +
         sizeof(uint32_t) * (2 * (size_t)words_for(nb) + (size_t)nb);
}

__global__ void __launch_bounds__(kThreads2, 1)
    drift128_kernel(const __grid_constant__ CUtensorMap tm_q,
                    const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const DriftParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024_shared(smem_raw);
  uint8_t* sQ = smem;
  uint8_t* sKV = smem + kQBytes;
  float* sT = reinterpret_cast<float*>(sKV + kStages2 * kStageBytes);   // [128][kTStride]
  Ctl2* ctl = reinterpret_cast<Ctl2*>(sT + kRows * kTStride);
  const int W = words_for(p.nb);
  uint32_t* kept = reinterpret_cast<uint32_t*>(ctl + 1);
  uint32_t* pref = kept + W;
  uint32_t* list = pref + W;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int h = blockIdx.x / p.tiles_per_head;
  const int qb = blockIdx.x % p.tiles_per_head;
  const int row0 = qb * kRows;
  const int n_drop = p.nb - p.budget;

  const uint32_t bar_q = smem_addr(&ctl->q_full);
  const uint32_t bar_s0 = smem_addr(&ctl->s_full[0]);
  const uint32_t bar_p0 = smem_addr(&ctl->p_full[0]);
  const uint32_t bar_c0 = smem_addr(&ctl->c_full[0]);
  const uint32_t bar_cf0 = smem_addr(&ctl->c_free[0]);
  const uint32_t bar_r0 = smem_addr(&ctl->red_full[0]);
  const uint32_t bar_tp = smem_addr(&ctl->t_post);
  const uint32_t bar_tred = smem_addr(&ctl->tred_full);
  const uint32_t bar_done = smem_addr(&ctl->mma_done);
  volatile int* abortf = &ctl->abort_flag;

  if (threadIdx.x == 0) {
    mbar_init(bar_q, 1);
    for (int s = 0; s < kStages2; ++s) {
      mbar_init(smem_addr(&ctl->kv_full[s]), 1);
      mbar_init(smem_addr(&ctl->kv_empty[s]), 1);
    }
    for (int g = 0; g < 2; ++g) {
      mbar_init(bar_s0 + 8 * g, 1);
      mbar_init(bar_p0 + 8 * g, 128);
      mbar_init(bar_c0 + 8 * g, 1);
      mbar_init(bar_cf0 + 8 * g, 128);
      mbar_init(bar_r0 + 8 * g, 128);
    }
    mbar_init(bar_tp, 128);
    mbar_init(bar_tred, 128);
    mbar_init(bar_done, 1);
    ctl->abort_flag = 0;
    fence_mbarrier_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_addr(&ctl->tmem_base), 512);
    tmem_relinquish();
  }
  for (int w = threadIdx.x; w < W; w += kThreads2) kept[w] = 0u;
  __syncthreads();

  for (int r = threadIdx.x; r < p.budget; r += kThreads2) {
    const int j = p.idx[((size_t)h * p.nb + qb) * p.budget + r];
    if (j < 0 || j >= p.nb) {
      raise_device_error(p.err, RESS_ERR_BAD_INDEX, 2);
      continue;
    }
    // A block named twice leaves more than nb - budget blocks dropped.
    if (atomicOr(&kept[j >> 5], 1u << (j & 31)) & (1u << (j & 31)))
      raise_device_error(p.err, RESS_ERR_BAD_INDEX, 5);
  }
  __syncthreads();

  // Prefix popcounts of the kept bitmap and the list of dropped blocks.
  if (warp == 0) {
    int base = 0, basek = 0;
    for (int w0 = 0; w0 < W; w0 += 32) {
      const int w = w0 + lane;
      uint32_t valid = 0u;
      if (w < W) valid = (w == W - 1 && (p.nb & 31)) ? ((1u << (p.nb & 31)) - 1u) : 0xffffffffu;
      const uint32_t k = (w < W) ? kept[w] : 0u;
      uint32_t u = ~k & valid;
      const int ck = __popc(k), cu = __popc(u);
      int ik = ck, iu = cu;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int yk = __shfl_up_sync(0xffffffffu, ik, o);
        const int yu = __shfl_up_sync(0xffffffffu, iu, o);
        if (lane >= o) {
          ik += yk;
          iu += yu;
        }
      }
      if (w < W) pref[w] = (uint32_t)(basek + ik - ck);
      basek += __shfl_sync(0xffffffffu, ik, 31);
      int pos = base + iu - cu;
      while (u) {
        const int bit = __ffs(u) - 1;
        u &= u - 1u;
        list[pos++] = (uint32_t)(w * 32 + bit);
      }
      base += __shfl_sync(0xffffffffu, iu, 31);
    }
    if (lane == 0) ctl->n_entries = base;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();

  const uint32_t tmem = ctl->tmem_base;
  const int n_chunks = ctl->n_entries;

  if (warp == 0) {
    // TMA producer: K and V of one dropped 128-token block per stage.
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
        const int s = c % kStages2;
        if (c >= kStages2 &&
            !warp_wait(smem_addr(&ctl->kv_empty[s]), ((c / kStages2) - 1) & 1, abortf, p.err, 40))
          break;
        const int t0 = (int)list[c] * 128;
        const uint32_t st = smem_addr(sKV) + (uint32_t)s * kStageBytes;
        const uint32_t bar = smem_addr(&ctl->kv_full[s]);
        if (elect_one()) {
          mbar_arrive_expect_tx(bar, kStageBytes);
          tma_load_3d(st, &tm_k, bar, 0, h, t0);
          tma_load_3d(st + kSubBytes, &tm_k, bar, 0, h, t0 + 64);
          tma_load_3d(st + 2 * kSubBytes, &tm_v, bar, 0, h, t0);
          tma_load_3d(st + 3 * kSubBytes, &tm_v, bar, 0, h, t0 + 64);
        }
        __syncwarp();
        issued = c + 1;
      }
      for (int c = issued > kStages2 ? issued - kStages2 : 0; c < issued; ++c)
        mbar_wait_drain(smem_addr(&ctl->kv_full[c % kStages2]), (c / kStages2) & 1, p.err, 41);
      mbar_wait_drain(bar_q, 0, p.err, 42);
    }
    __syncwarp();
  } else if (warp == 1) {
    // MMA issuer.  Per chunk c of group g = c & 1: C(c) into C_g once P(c) is
    // written and C(c - 2) has been read, then S(c + 2) into S_g (the tensor
    // core runs the MMAs in issue order, so C(c) has read P(c) before
    // S(c + 2) overwrites it).
    if (n_chunks > 0) {
      constexpr uint32_t idS = idesc_bf16_f32(128, 128, false);
      constexpr uint32_t idPV = idesc_bf16_f32(128, 64, true);
      const uint64_t dq = smem_desc_sw128(smem_addr(sQ), 16, 1024);
      const uint64_t dk0 = smem_desc_sw128(smem_addr(sKV), 16, 1024);
      const uint64_t dv0 = smem_desc_sw128(smem_addr(sKV) + 2 * kSubBytes, 16384, 1024);
      constexpr uint64_t kStageDesc = kStageBytes >> 4;
      bool ok = warp_wait(bar_q, 0, abortf, p.err, 50);
      auto issue_s = [&](int c) -> bool {
        const int s = c % kStages2;
        if (!warp_wait(smem_addr(&ctl->kv_full[s]), (c / kStages2) & 1, abortf, p.err, 51))
          return false;
        tc_fence_after();
        const uint64_t dk = dk0 + (uint64_t)s * kStageDesc;
        if (elect_one()) {
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_ss(tmem + 128u * (uint32_t)(c & 1), dq + (uint64_t)(kk * 2), dk + (uint64_t)(kk * 2),
                   idS, kk > 0 ? 1u : 0u);
          mma_commit(bar_s0 + 8u * (uint32_t)(c & 1));
        }
        __syncwarp();
        return true;
      };
      for (int c = 0; ok && c < n_chunks && c < 2; ++c) ok = issue_s(c);
      for (int c = 0; ok && c < n_chunks; ++c) {
        const int g = c & 1, it = c >> 1;
        if (!warp_wait(bar_p0 + 8u * (uint32_t)g, (uint32_t)it & 1u, abortf, p.err, 52)) break;
        if (it > 0 && !warp_wait(bar_cf0 + 8u * (uint32_t)g, (uint32_t)(it - 1) & 1u, abortf, p.err, 53))
          break;
        tc_fence_after();
        const int s = c % kStages2;
        const uint64_t dv = dv0 + (uint64_t)s * kStageDesc;
        const uint32_t tP = tmem + 128u * (uint32_t)g;
        if (elect_one()) {
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            mma_ts(tmem + kColC2 + 64u * (uint32_t)g, tP + kk * 8, dv + (uint64_t)(kk * 128), idPV,
                   kk > 0 ? 1u : 0u);
          mma_commit(bar_c0 + 8u * (uint32_t)g);
          mma_commit(smem_addr(&ctl->kv_empty[s]));
        }
        __syncwarp();
        if (c + 2 < n_chunks && !(ok = issue_s(c + 2))) break;
      }
      if (elect_one()) mma_commit(bar_done);
      __syncwarp();
      mbar_wait_drain(bar_done, 0, p.err, 54);
    }
    __syncwarp();
  } else {
    const int quad = warp & 3;
    const int grp = (warp - 2) >> 2;
    const int row = quad * 32 + lane;
    const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
    const uint32_t tS = tmem + 128u * (uint32_t)grp + lane_off;
    const uint32_t tC = tmem + kColC2 + 64u * (uint32_t)grp + lane_off;
    const uint32_t bar_s = bar_s0 + 8u * (uint32_t)grp;
    const uint32_t bar_p = bar_p0 + 8u * (uint32_t)grp;
    const uint32_t bar_c = bar_c0 + 8u * (uint32_t)grp;
    const uint32_t bar_cf = bar_cf0 + 8u * (uint32_t)grp;
    const uint32_t bar_red = bar_r0 + 8u * (uint32_t)grp;
    const float kScaleLog2 = 1.4426950408889634f * 0.125f;
    const int tok = row0 + row;
    // Layout: only the valid, non-special queries drop anything.
    const int pos = p.lay_t != 0 ? tok % p.lay_t : 0;
    const bool live_q = p.lay_t == 0 || (pos < p.lay_r && pos >= p.lay_s);
    const bool all_live = __all_sync(0xffffffffu, live_q);
    const float lse2 =
        (tok < p.n && live_q) ? p.lse[(size_t)h * p.n + tok] * 1.4426950408889634f : 0.f;
    const float2 neg_l2 = make_float2(-lse2, -lse2);
    const float2 scale2 = make_float2(kScaleLog2, kScaleLog2);
    const int gtid = threadIdx.x - 64 - 128 * grp;   // 0..127 within the group
    bool ok = true;
    float2 tsum[32];   // this row's share of T = sum of the group's contributions
#pragma unroll
    for (int u = 0; u < 32; ++u) tsum[u] = make_float2(0.f, 0.f);
    for (int c = grp, it = 0; c < n_chunks; c += 2, ++it) {
      const uint32_t ph = (uint32_t)it & 1u;
      if (!warp_wait(bar_s, ph, abortf, p.err, 60)) { ok = false; break; }
      tc_fence_after();
      const int j = (int)list[c];
      const int t0 = j * 128;
      // Two halves of 64 columns; P (bf16, two per column) of half hf goes
      // to columns 32 hf .. 32 hf + 31, below the S columns still unread.
#pragma unroll
      for (int hf = 0; hf < 2; ++hf) {
        const int vk = layout_valid(p.lay_t, p.lay_r, t0 + 64 * hf, 64);
        uint32_t r[2][32];
        tmem_ld32(tS + 64 * hf, r[0]);
        tmem_ld32(tS + 64 * hf + 32, r[1]);
        tmem_ld_wait_regs(r[0]);
        tmem_tie_regs(r[1]);
#pragma unroll
        for (int g = 0; g < 2; ++g) {
          uint32_t pk[16];
          if (vk == 64 && all_live) {
            // One pair in four on the FMA pipe (polynomial), the rest on MUFU.
#pragma unroll
            for (int e = 0; e < 16; ++e) {
              const float2 x = ffma2(make_float2(__uint_as_float(r[g][2 * e]), __uint_as_float(r[g][2 * e + 1])),
                                     scale2, neg_l2);
              const float2 pe = ((e & 3) == 3) ? exp2_poly2(x)
                                               : make_float2(fast_exp2(x.x), fast_exp2(x.y));
              pk[e] = pack_bf16x2(pe.x, pe.y);
            }
          } else {
            // Layout: padding keys (columns beyond the sub-block's valid
            // prefix) and the rows of padding and special queries add nothing.
#pragma unroll
            for (int e = 0; e < 16; ++e) {
              const int col = 32 * g + 2 * e;
              float p0 = fast_exp2(fmaf(__uint_as_float(r[g][2 * e]), kScaleLog2, neg_l2.x));
              float p1 = fast_exp2(fmaf(__uint_as_float(r[g][2 * e + 1]), kScaleLog2, neg_l2.x));
              if (!live_q || col >= vk) p0 = 0.f;
              if (!live_q || col + 1 >= vk) p1 = 0.f;
              pk[e] = pack_bf16x2(p0, p1);
            }
          }
          tmem_st16(tS + 32 * hf + 16 * g, pk);
        }
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(bar_p);

      if (!warp_wait(bar_c, ph, abortf, p.err, 61)) { ok = false; break; }
      tc_fence_after();
      float ss;
      {
        // Sum of squares of the row's 64 contribution columns: packed pairs
        // into four independent accumulators.
        uint32_t cv[2][32];
        tmem_ld32(tC, cv[0]);
        tmem_ld32(tC + 32, cv[1]);
        tmem_ld_wait_regs(cv[0]);
        tmem_tie_regs(cv[1]);
        tc_fence_before();
        mbar_arrive(bar_cf);
        float2 acc[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) acc[q] = make_float2(0.f, 0.f);
#pragma unroll
        for (int g = 0; g < 2; ++g) {
#pragma unroll
          for (int u = 0; u < 16; ++u) {
            const float2 x = make_float2(__uint_as_float(cv[g][2 * u]), __uint_as_float(cv[g][2 * u + 1]));
            acc[u & 3] = ffma2(x, x, acc[u & 3]);
            tsum[16 * g + u] = fadd2(tsum[16 * g + u], x);
          }
        }
        ss = ((acc[0].x + acc[0].y) + (acc[1].x + acc[1].y)) +
             ((acc[2].x + acc[2].y) + (acc[3].x + acc[3].y));
      }
      ss = warp_sum(ss);
      if (lane == 0) ctl->partial[grp][ph][quad] = ss;
      __syncwarp();
      mbar_arrive(bar_red);
      // One writer per group.  A slot is rewritten two of the group's chunks
      // later at the earliest, and no warp of the group runs that far ahead
      // of the writer (each chunk's C waits for all 128 threads of the group).
      if (gtid == 0 && mbar_wait(bar_red, ph, abortf, p.err, 63)) {
        const float tot = ctl->partial[grp][ph][0] + ctl->partial[grp][ph][1] +
                          ctl->partial[grp][ph][2] + ctl->partial[grp][ph][3];
        const int rnk = dropped_rank(kept, pref, j);
        if (rnk >= 0 && rnk < n_drop)
          p.drift[((size_t)h * p.nb + qb) * n_drop + rnk] = sqrtf(tot);
        else
          raise_device_error(p.err, RESS_ERR_BAD_INDEX, 3);
      }
      __syncwarp();
    }
    // Drop-set drift J = ||sum_j C_j||_F: group 1 posts its running sums,
    // group 0 adds its own and reduces.
    float* trow = sT + row * kTStride;
    if (grp == 1) {
#pragma unroll
      for (int u = 0; u < 16; ++u)
        *reinterpret_cast<float4*>(trow + 4 * u) =
            make_float4(tsum[2 * u].x, tsum[2 * u].y, tsum[2 * u + 1].x, tsum[2 * u + 1].y);
      mbar_arrive(bar_tp);
    } else {
      float tss = 0.f;
      if (mbar_wait(bar_tp, 0, abortf, p.err, 62)) {
        float2 acc[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) acc[q] = make_float2(0.f, 0.f);
#pragma unroll
        for (int u = 0; u < 16; ++u) {
          const float4 o = *reinterpret_cast<const float4*>(trow + 4 * u);
          const float2 a = fadd2(tsum[2 * u], make_float2(o.x, o.y));
          const float2 b = fadd2(tsum[2 * u + 1], make_float2(o.z, o.w));
          acc[u & 3] = ffma2(a, a, acc[u & 3]);
          acc[u & 3] = ffma2(b, b, acc[u & 3]);
        }
        tss = ((acc[0].x + acc[0].y) + (acc[1].x + acc[1].y)) +
              ((acc[2].x + acc[2].y) + (acc[3].x + acc[3].y));
      }
      tss = warp_sum(tss);
      if (lane == 0) ctl->tpartial[quad] = tss;
      __syncwarp();
      mbar_arrive(bar_tred);
      if (p.set_drift && gtid == 0 && mbar_wait(bar_tred, 0, abortf, p.err, 64))
        p.set_drift[(size_t)h * p.nb + qb] = sqrtf(ctl->tpartial[0] + ctl->tpartial[1] +
                                                   ctl->tpartial[2] + ctl->tpartial[3]);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace

ress_status launch_drift(const Geometry& g, const void* q, const void* k, const void* v,
                         int budget, const int32_t* idx, const float* lse, float* drift,
                         float* set_drift, cudaStream_t st) {
  CUtensorMap tq, tk, tv;
  if (!make_token_map(&tq, q, g, 128) || !make_token_map(&tk, k, g, 64) ||
      !make_token_map(&tv, v, g, 64))
    return RESS_ERR_CUDA;
  DriftParams p{};
  p.err = device_error_ptr();
  if (p.err == nullptr) return RESS_ERR_CUDA;
  p.n = (int)g.n;
  p.heads = g.heads;
  p.nb = g.nb;
  p.block = g.block;
  p.budget = budget;
  p.tiles_per_head = (g.block == 64) ? (g.nb + 1) / 2 : g.nb;
  p.idx = idx;
  p.lse = lse;
  p.drift = drift;
  p.set_drift = set_drift;
  p.lay_t = g.lay_t;
  p.lay_r = g.lay_r;
  p.lay_s = g.lay_s;
  const size_t smem = drift_smem_bytes(g.nb);
  if (smem > 227 * 1024) return RESS_ERR_UNSUPPORTED;   // block lists no longer fit
  const unsigned grid = (unsigned)(g.heads * p.tiles_per_head);
  if (g.block == 128) {
    const size_t smem2 = drift128_smem_bytes(g.nb);
    if (smem2 > 227 * 1024) return RESS_ERR_UNSUPPORTED;
    if (ress_status st_ = record_cuda(cudaFuncSetAttribute(
            drift128_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem2)))
      return st_;
    drift128_kernel<<<grid, kThreads2, smem2, st>>>(tq, tk, tv, p);
  } else {
    // All 512 TMEM columns per CTA: at least 116 KB of shared memory keeps a
    // second CTA (which would only wait in its TMEM allocation) off the SM.
    const size_t smem1 = smem > kOneCtaSmem ? smem : kOneCtaSmem;
    if (ress_status st_ = record_cuda(cudaFuncSetAttribute(
            block_drift_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem1)))
      return st_;
    block_drift_kernel<<<grid, kThreads, smem1, st>>>(tq, tk, tv, p);
  }
  return record_cuda(cudaGetLastError());
}

}  // namespace ress
