// Stage 1 on tcgen05: the fixed-budget top-k of the pooled scores
// s_ij = Qbar_i . Kbar_j (lambda == 0; the 1/sqrt(d) scale does not change a
// row's order), without ever storing a score row.
//
// A CTA takes one head and 128 query blocks: the TMEM lanes, one row per
// lane.  Qbar sits in TMEM as the A operand, split into tf32 high and low
// parts; the pooled keys stream through shared memory in 128-key chunks (TMA,
// 128-byte swizzle), also as tf32 high and low planes, and each chunk's
// 128 x 128 scores land in one of three TMEM accumulators.  Each row is owned
// by two worker threads (warps w and w + 4 share the TMEM lanes), one per
// 64-column half of every chunk.  Three passes over the keys, all reading
// the scores straight from TMEM:
//
//   sample   128 evenly spaced keys, approximate scores (Qhi . Khi): the
//            row's range [bot, top].
//   pass A   every key, approximate scores: a histogram of 256 bins of width
//            (top - bot) / 256 counted from the top (values outside the range
//            fall in the end bins); bin b* holds the budget-th largest
//            approximate score.
//   pass B   every key, the full product Qhi.Khi + Qhi.Klo + Qlo.Khi (about
//            float32 accuracy): a score above b*'s upper edge plus the
//            allowance delta for the approximate pass is kept outright, a
//            score within delta of b* is a candidate, anything else is
//            dropped.
//
// The candidates of a row (a few dozen at most) are then ranked by their
// full products (larger first, lower index first on equal scores), and the
// best budget - (kept outright) join the row's bitmap, which the worker warps
// write out in ascending block order, one row per warp at a time.  A row whose
// band turns out not to hold the budget-th score (delta is an allowance
// sized from the measured tf32 error, not a proof), or holds more candidates
// than fit, is handed to the exact fallback kernel, which recomputes it.
//
// Sources: ReSS (thelatestinai.com) Table S5, SpargeAttn row - selection by
// pooled query/key inner products; Table 1 - a fused scoring kernel;
// VASC (paperlayer.ai) A.2 - an exact-capacity binary Top-K.
//
// Warp roles (320 threads, one CTA per SM): warp 0 TMA, warp 1 TMEM owner and
// MMA issuer (one elected lane), warps 2-9 workers.  Every mbarrier wait is
// bounded; after a timeout the workers skip the remaining work but still pass
// every named barrier, and the CTA frees TMEM and exits.
#include "ress_common.cuh"
#include "ress_internal.h"

namespace ress {

namespace {

constexpr int kTcRows = 128;
constexpr int kTcThreads = 320;
constexpr int kTcWorkers = 256;
constexpr int kTcStages = 2;
constexpr uint32_t kTcBox = 128 * 32 * 4;     // 128 keys x 32 d of float32 = one swizzle span
constexpr uint32_t kTcPlane = 2 * kTcBox;     // 128 keys x 64 d
constexpr uint32_t kTcStage = 2 * kTcPlane;   // tf32 high and low planes
constexpr int kTcAcc = 3;
constexpr uint32_t kTcColQhi = 0, kTcColQlo = 64, kTcColAcc = 128;
constexpr int kTcCand = 32;                   // candidates per worker thread
constexpr int kTcWords = kMaxBlocksTc / 32;   // bitmap words per row
// Worker scratch: during pass A the row histograms, [128 words][128 rows]
// u32 (two u16 bin counts per word); afterwards the kept-block bitmaps
// [kTcWords][128 rows] u32, the candidate indices [kTcCand][256] u16 and
// their exact scores [kTcCand][256] f32.
constexpr uint32_t kTcHistBytes = 128 * kTcRows * 4;
constexpr uint32_t kTcBitmapBytes = kTcWords * kTcRows * 4;
constexpr uint32_t kTcCandJBytes = kTcCand * kTcWorkers * 2;
constexpr uint32_t kTcCandSBytes = kTcCand * kTcWorkers * 4;
constexpr uint32_t kTcRegion = (kTcBitmapBytes + kTcCandJBytes + kTcCandSBytes) > kTcHistBytes
                                   ? (kTcBitmapBytes + kTcCandJBytes + kTcCandSBytes)
                                   : kTcHistBytes;
constexpr uint32_t kMagicBits = 0x4B400000u;  // bits of 1.5 * 2^23
constexpr float kMagic = 12582912.0f;

struct TcArgs {
  DeviceError* err;
  const float* qbar;      // [H][nb][64]
  const float* khi;       // [H][nb_pad][64]
  const float* klo;       // [H][nb_pad][64]
  const float* knorm;     // [H][nb]
  int32_t* idx;           // [H][nb][budget]
  int32_t* fb_count;      // rows handed to the fallback
  int32_t* fb_list;       // [H * nb] codes h * nb + i
  int nb, nb_pad, budget, tiles_per_head, n_chunks;
};

struct __align__(8) TcCtl {
  uint64_t kv_full[kTcStages];
  uint64_t kv_empty[kTcStages];
  uint64_t acc_full[kTcAcc];
  uint64_t acc_empty[kTcAcc];
  uint64_t a_ready;
  uint64_t mma_done;
  uint32_t tmem_base;
  int abort_flag;
  uint32_t kmax_bits;
  int pad;
  float xa[2][kTcRows];
  float xb[2][kTcRows];
  int xc[2][kTcRows];
  int xd[2][kTcRows];
  int rstate[kTcRows];   // 1: the row's bitmap is its result; 0: dead row or handed over
};

size_t tc_smem_bytes() { return 1024 + kTcStages * kTcStage + kTcRegion + sizeof(TcCtl); }

__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                          DeviceError* err, int detail) {
  const bool ok = mbar_wait(bar, parity, abort_flag, err, detail);
  return __all_sync(0xffffffffu, ok);
}

// Shared-memory histogram increment; the result is not returned.
__device__ __forceinline__ void red_add_shared_u32(uint32_t addr, uint32_t v) {
  asm volatile("red.shared.add.u32 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
}

__device__ __forceinline__ float to_tf32(float x) {
  return __uint_as_float((__float_as_uint(x) + 0x1000u) & 0xFFFFE000u);
}

// Histogram bin of a pair of approximate scores: t = (top - s) * scale
// (off = top * scale), rounded to the nearest integer by adding 1.5 * 2^23
// in a separate step (a constant that folded both would lose t's fraction to
// the ulp of 1 at 2^23), clamped to [0, 255]; then one increment of the u16
// count of that bin in the row's histogram.
__device__ __forceinline__ void hist_pair(float s0, float s1, float2 neg_scale2, float2 off2,
                                          uint32_t hist_row) {
  const float2 t = ffma2(make_float2(s0, s1), neg_scale2, off2);
  const float2 f = fadd2(t, make_float2(kMagic, kMagic));
  const int b0 = min(max((int)(__float_as_uint(f.x) - kMagicBits), 0), 255);
  const int b1 = min(max((int)(__float_as_uint(f.y) - kMagicBits), 0), 255);
  red_add_shared_u32(hist_row + (uint32_t)(b0 >> 1) * (kTcRows * 4), 1u + (uint32_t)(b0 & 1) * 0xFFFFu);
  red_add_shared_u32(hist_row + (uint32_t)(b1 >> 1) * (kTcRows * 4), 1u + (uint32_t)(b1 & 1) * 0xFFFFu);
}

// r[u] for a run-time u without indexing the register array (which would
// place it in local memory): a tree of selects on the bits of u.
__device__ __forceinline__ uint32_t select32(const uint32_t (&r)[32], int u) {
  uint32_t l1[16], l2[8], l3[4], l4[2];
#pragma unroll
  for (int e = 0; e < 16; ++e) l1[e] = (u & 1) ? r[2 * e + 1] : r[2 * e];
#pragma unroll
  for (int e = 0; e < 8; ++e) l2[e] = (u & 2) ? l1[2 * e + 1] : l1[2 * e];
#pragma unroll
  for (int e = 0; e < 4; ++e) l3[e] = (u & 4) ? l2[2 * e + 1] : l2[2 * e];
#pragma unroll
  for (int e = 0; e < 2; ++e) l4[e] = (u & 8) ? l3[2 * e + 1] : l3[2 * e];
  return (u & 16) ? l4[1] : l4[0];
}

__global__ void __launch_bounds__(kTcThreads, 1)
    topk_tc_kernel(const __grid_constant__ CUtensorMap tm_khi,
                   const __grid_constant__ CUtensorMap tm_klo,
                   const __grid_constant__ CUtensorMap tm_ks, const TcArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* stages = smem;
  uint8_t* region = smem + kTcStages * kTcStage;
  TcCtl* ctl = reinterpret_cast<TcCtl*>(region + kTcRegion);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int h = blockIdx.x / a.tiles_per_head;
  const int i0 = (blockIdx.x % a.tiles_per_head) * kTcRows;
  const int C = a.n_chunks;
  const int n_seq = 2 * C + 1;   // the sample, C approximate chunks, C full-product chunks
  volatile int* abortf = &ctl->abort_flag;
  const uint32_t st0 = smem_addr(stages);

  if (threadIdx.x == 0) {
    for (int s = 0; s < kTcStages; ++s) {
      mbar_init(smem_addr(&ctl->kv_full[s]), 1);
      mbar_init(smem_addr(&ctl->kv_empty[s]), 1);
    }
    for (int b = 0; b < kTcAcc; ++b) {
      mbar_init(smem_addr(&ctl->acc_full[b]), 1);
      mbar_init(smem_addr(&ctl->acc_empty[b]), kTcWorkers);
    }
    mbar_init(smem_addr(&ctl->a_ready), kTcWorkers);
    mbar_init(smem_addr(&ctl->mma_done), 1);
    ctl->abort_flag = 0;
    ctl->kmax_bits = 0u;
    fence_mbarrier_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_addr(&ctl->tmem_base), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ctl->tmem_base;

  if (warp == 0) {
    // ---------------- TMA producer ----------------
    if (elect_one()) {
      tma_prefetch_desc(&tm_khi);
      tma_prefetch_desc(&tm_klo);
      tma_prefetch_desc(&tm_ks);
    }
    __syncwarp();
    int issued = 0;
    for (int seq = 0; seq < n_seq; ++seq) {
      const int s = seq % kTcStages;
      if (seq >= kTcStages &&
          !warp_wait(smem_addr(&ctl->kv_empty[s]), ((seq / kTcStages) - 1) & 1, abortf, a.err, 90))
        break;
      const bool full = seq > C;
      const uint32_t st = st0 + (uint32_t)s * kTcStage;
      const uint32_t bar = smem_addr(&ctl->kv_full[s]);
      if (elect_one()) {
        mbar_arrive_expect_tx(bar, full ? kTcStage : kTcPlane);
        if (seq == 0) {
          tma_load_3d(st, &tm_ks, bar, 0, 0, h);
          tma_load_3d(st + kTcBox, &tm_ks, bar, 32, 0, h);
        } else {
          const int c = full ? seq - C - 1 : seq - 1;
          tma_load_3d(st, &tm_khi, bar, 0, 128 * c, h);
          tma_load_3d(st + kTcBox, &tm_khi, bar, 32, 128 * c, h);
          if (full) {
            tma_load_3d(st + kTcPlane, &tm_klo, bar, 0, 128 * c, h);
            tma_load_3d(st + kTcPlane + kTcBox, &tm_klo, bar, 32, 128 * c, h);
          }
        }
      }
      __syncwarp();
      issued = seq + 1;
    }
    for (int seq = issued > kTcStages ? issued - kTcStages : 0; seq < issued; ++seq)
      mbar_wait_drain(smem_addr(&ctl->kv_full[seq % kTcStages]), (seq / kTcStages) & 1, a.err, 91);
    __syncwarp();
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    constexpr uint32_t id = idesc_tf32_f32(128, 128);
    bool ok = warp_wait(smem_addr(&ctl->a_ready), 0, abortf, a.err, 92);
    for (int seq = 0; ok && seq < n_seq; ++seq) {
      const int s = seq % kTcStages;
      const int b = seq % kTcAcc;
      if (!warp_wait(smem_addr(&ctl->kv_full[s]), (seq / kTcStages) & 1, abortf, a.err, 93)) break;
      if (seq >= kTcAcc &&
          !warp_wait(smem_addr(&ctl->acc_empty[b]), ((seq / kTcAcc) - 1) & 1, abortf, a.err, 94))
        break;
      tc_fence_after();
      const uint32_t st = st0 + (uint32_t)s * kTcStage;
      const uint32_t d = tmem + kTcColAcc + 128u * (uint32_t)b;
      const bool full = seq > C;
      if (elect_one()) {
        // K-step kk covers d = 8 kk .. 8 kk + 7: span kk / 4 of the plane,
        // 32 bytes per step inside the 128-byte swizzled rows.
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t off = (uint32_t)(kk >> 2) * kTcBox + (uint32_t)(kk & 3) * 32u;
          mma_ts_tf32(d, tmem + kTcColQhi + 8u * kk, smem_desc_sw128(st + off, 16, 1024), id,
                      kk > 0 ? 1u : 0u);
        }
        if (full) {
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint32_t off = (uint32_t)(kk >> 2) * kTcBox + (uint32_t)(kk & 3) * 32u;
            mma_ts_tf32(d, tmem + kTcColQhi + 8u * kk,
                        smem_desc_sw128(st + kTcPlane + off, 16, 1024), id, 1u);
          }
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint32_t off = (uint32_t)(kk >> 2) * kTcBox + (uint32_t)(kk & 3) * 32u;
            mma_ts_tf32(d, tmem + kTcColQlo + 8u * kk, smem_desc_sw128(st + off, 16, 1024), id,
                        1u);
          }
        }
        mma_commit(smem_addr(&ctl->kv_empty[s]));
        mma_commit(smem_addr(&ctl->acc_full[b]));
      }
      __syncwarp();
    }
    if (elect_one()) mma_commit(smem_addr(&ctl->mma_done));
    __syncwarp();
    mbar_wait_drain(smem_addr(&ctl->mma_done), 0, a.err, 95);
    __syncwarp();
  } else {
    // ---------------- workers ----------------
    const int wt = threadIdx.x - 64;            // 0 .. 255
    const int quad = warp & 3;                  // TMEM lanes 32 quad .. 32 quad + 31
    const int half = (warp - 2) >> 2;           // columns 64 half .. 64 half + 63 of a chunk
    const int row = quad * 32 + lane;
    const int i = i0 + row;
    const bool live = i < a.nb;
    const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
    const int nb = a.nb;
    const float* qrow = a.qbar + ((size_t)h * nb + (live ? i : 0)) * kHeadDim;
    bool ok = true;

    // Zero the histograms (64 KB over the 256 workers).
    {
      uint4* z = reinterpret_cast<uint4*>(region);
      for (int e = wt; e < (int)(kTcHistBytes / 16); e += kTcWorkers) z[e] = make_uint4(0u, 0u, 0u, 0u);
    }
    // Qbar row into TMEM: half 0 writes the tf32 high parts, half 1 the low.
    float qn2 = 0.f;
#pragma unroll
    for (int g = 0; g < 2; ++g) {
      uint32_t part[32];
#pragma unroll
      for (int u4 = 0; u4 < 8; ++u4) {
        float4 x = live ? *reinterpret_cast<const float4*>(qrow + 32 * g + 4 * u4)
                        : make_float4(0.f, 0.f, 0.f, 0.f);
        const float xs[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float hi = to_tf32(xs[e]);
          part[4 * u4 + e] = __float_as_uint(half ? to_tf32(xs[e] - hi) : hi);
          qn2 = fmaf(xs[e], xs[e], qn2);
        }
      }
      tmem_st32(tmem + (half ? kTcColQlo : kTcColQhi) + lane_off + 32u * (uint32_t)g, part);
    }
    // Largest key norm of the head.
    {
      float km = 0.f;
      for (int j = wt; j < nb; j += kTcWorkers) km = fmaxf(km, a.knorm[(size_t)h * nb + j]);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) km = fmaxf(km, __shfl_xor_sync(0xffffffffu, km, o));
      if (lane == 0) atomicMax(&ctl->kmax_bits, __float_as_uint(km));
    }
    tmem_st_wait();
    tc_fence_before();
    mbar_arrive(smem_addr(&ctl->a_ready));
    named_bar_sync(1, kTcWorkers);
    const float kmax = __uint_as_float(ctl->kmax_bits);
    // Allowance for the tf32 (high parts only) scores of the sample and of
    // pass A: 2^-11 |Qbar_i| max_j |Kbar_j|, about 2.6x the largest error
    // measured on the clustered workloads (the rigorous bound is 2^-10).
    const float delta = sqrtf(qn2) * kmax * (1.0f / 2048.0f);

    // ---- sample: the row's range ----
    float top = 0.f, bot = 0.f;
    {
      float mx = -INFINITY, mn = INFINITY;
      if (ok) ok = warp_wait(smem_addr(&ctl->acc_full[0]), 0, abortf, a.err, 96);
      if (ok) {
        tc_fence_after();
        const uint32_t tA = tmem + kTcColAcc + lane_off + 64u * (uint32_t)half;
        uint32_t r2[2][32];
        tmem_ld32(tA, r2[0]);
        tmem_ld32(tA + 32u, r2[1]);
        tmem_ld_wait_regs(r2[0]);
        tmem_ld_wait_regs(r2[1]);
#pragma unroll
        for (int g = 0; g < 2; ++g) {
          const uint32_t (&r)[32] = r2[g];
#pragma unroll
          for (int u = 0; u < 16; ++u) {
            const float s0 = __uint_as_float(r[2 * u]), s1 = __uint_as_float(r[2 * u + 1]);
            mx = fmax3(mx, s0, s1);
            mn = fminf(mn, fminf(s0, s1));
          }
        }
        tc_fence_before();
        mbar_arrive(smem_addr(&ctl->acc_empty[0]));
      }
      ctl->xa[half][row] = mx;
      ctl->xb[half][row] = mn;
    }
    named_bar_sync(1, kTcWorkers);
    top = fmaxf(ctl->xa[0][row], ctl->xa[1][row]);
    bot = fminf(ctl->xb[0][row], ctl->xb[1][row]);
    float scale = 256.0f / (top - bot);
    if (!(scale < INFINITY)) scale = 0.f;           // constant range: one bin
    const float2 neg_scale2 = make_float2(-scale, -scale);
    const float off = top * scale;
    const float2 off2 = make_float2(off, off);

    // ---- pass A: histogram of the approximate scores ----
    const uint32_t hist_row = smem_addr(region) + (uint32_t)row * 4u;
    for (int c = 0; c < C && ok; ++c) {
      const int seq = 1 + c;
      const int b = seq % kTcAcc;
      ok = warp_wait(smem_addr(&ctl->acc_full[b]), (seq / kTcAcc) & 1, abortf, a.err, 97);
      if (!ok) break;
      tc_fence_after();
      const uint32_t tA = tmem + kTcColAcc + 128u * (uint32_t)b + lane_off + 64u * (uint32_t)half;
      uint32_t r2[2][32];
      tmem_ld32(tA, r2[0]);
      tmem_ld32(tA + 32u, r2[1]);
      tmem_ld_wait_regs(r2[0]);
      tmem_ld_wait_regs(r2[1]);
#pragma unroll
      for (int g = 0; g < 2; ++g) {
        const uint32_t (&r)[32] = r2[g];
        const int j0 = 128 * c + 64 * half + 32 * g;
        if (j0 + 32 <= nb) {
#pragma unroll
          for (int u = 0; u < 16; ++u)
            hist_pair(__uint_as_float(r[2 * u]), __uint_as_float(r[2 * u + 1]), neg_scale2, off2,
                      hist_row);
        } else {
#pragma unroll
          for (int u = 0; u < 32; ++u) {
            if (j0 + u < nb) {
              const float t = fmaf(__uint_as_float(r[u]), neg_scale2.x, off2.x);
              const int b0 = min(max((int)(__float_as_uint(t + kMagic) - kMagicBits), 0), 255);
              red_add_shared_u32(hist_row + (uint32_t)(b0 >> 1) * (kTcRows * 4),
                                 1u + (uint32_t)(b0 & 1) * 0xFFFFu);
            }
          }
        }
      }
      tc_fence_before();
      mbar_arrive(smem_addr(&ctl->acc_empty[b]));
    }
    named_bar_sync(1, kTcWorkers);

    // ---- the bin b* of the budget-th largest approximate score ----
    // Both threads of a row scan the same counts, so they agree without an
    // exchange.  Bin 0 is the top of the range.
    float hiT = INFINITY, loT = -INFINITY;
    {
      const uint32_t* hist = reinterpret_cast<const uint32_t*>(region);
      int cum = 0, bstar = 255;
      for (int w = 0; w < 128; ++w) {
        const uint32_t v = hist[w * kTcRows + row];
        const int c0 = (int)(v & 0xFFFFu), c1 = (int)(v >> 16);
        if (cum + c0 >= a.budget) { bstar = 2 * w; break; }
        cum += c0;
        if (cum + c1 >= a.budget) { bstar = 2 * w + 1; break; }
        cum += c1;
      }
      // Bin b holds the approximate scores s with (top - s) * scale within
      // 1/2 of b (bin 0 everything above, bin 255 everything below the
      // range), up to rounding; the exact budget-th score lies within delta
      // of b*.
      const float eps = 1e-6f * (fabsf(top) + fabsf(bot)) + 1e-30f;
      if (scale > 0.f) {
        if (bstar > 0) hiT = top - ((float)bstar - 0.5f) / scale + delta + eps;
        if (bstar < 255) loT = top - ((float)bstar + 0.5f) / scale - delta - eps;
      }
    }
    named_bar_sync(1, kTcWorkers);   // the histograms are no longer read

    // ---- pass B: full products; keep, candidate or drop ----
    uint32_t* bitmap = reinterpret_cast<uint32_t*>(region);                           // [words][128]
    uint16_t* cand_j = reinterpret_cast<uint16_t*>(region + kTcBitmapBytes);          // [cap][256]
    float* cand_s = reinterpret_cast<float*>(region + kTcBitmapBytes + kTcCandJBytes); // [cap][256]
    int kept = 0, nc = 0;
    for (int c = 0; c < C && ok; ++c) {
      const int seq = C + 1 + c;
      const int b = seq % kTcAcc;
      ok = warp_wait(smem_addr(&ctl->acc_full[b]), (seq / kTcAcc) & 1, abortf, a.err, 98);
      if (!ok) break;
      tc_fence_after();
      const uint32_t tA = tmem + kTcColAcc + 128u * (uint32_t)b + lane_off + 64u * (uint32_t)half;
      uint32_t r2[2][32];
      tmem_ld32(tA, r2[0]);
      tmem_ld32(tA + 32u, r2[1]);
      tmem_ld_wait_regs(r2[0]);
      tmem_ld_wait_regs(r2[1]);
#pragma unroll
      for (int g = 0; g < 2; ++g) {
        const uint32_t (&r)[32] = r2[g];
        uint32_t kw = 0u, gw = 0u;
#pragma unroll
        for (int u = 0; u < 32; ++u) {
          const float sv = __uint_as_float(r[u]);
          kw |= (sv > hiT) ? (1u << u) : 0u;
          gw |= (sv >= loT) ? (1u << u) : 0u;
        }
        const int j0 = 128 * c + 64 * half + 32 * g;
        if (j0 + 32 > nb) {
          const uint32_t valid = j0 >= nb ? 0u : ((1u << (nb - j0)) - 1u);
          kw &= valid;
          gw &= valid;
        }
        if (j0 < nb) bitmap[(j0 >> 5) * kTcRows + row] = kw;
        kept += __popc(kw);
        uint32_t cw = gw & ~kw;
        while (cw != 0u) {
          const int u = __ffs(cw) - 1;
          cw &= cw - 1u;
          if (nc < kTcCand) {
            cand_j[nc * kTcWorkers + wt] = (uint16_t)(j0 + u);
            cand_s[nc * kTcWorkers + wt] = __uint_as_float(select32(r, u));
          }
          ++nc;
        }
      }
      tc_fence_before();
      mbar_arrive(smem_addr(&ctl->acc_empty[b]));
    }
    ctl->xc[half][row] = kept;
    ctl->xd[half][row] = ok ? nc : kTcCand + 1;
    named_bar_sync(1, kTcWorkers);

    // ---- rank the candidates; winners join the bitmap ----
    const int kept_all = ctl->xc[0][row] + ctl->xc[1][row];
    const int n0 = ctl->xd[0][row], n1 = ctl->xd[1][row];
    const int need = a.budget - kept_all;
    const bool row_ok = ok && n0 <= kTcCand && n1 <= kTcCand && need >= 0 && need <= n0 + n1;
    if (row_ok && live && need > 0) {
      const int wt_other = wt ^ 128;               // the row's other thread
      const int n_other = half ? n0 : n1;
      for (int n = 0; n < nc; ++n) {
        const int jx = cand_j[n * kTcWorkers + wt];
        const float sx = cand_s[n * kTcWorkers + wt];
        int rank = 0;
        for (int m = 0; m < nc; ++m) {
          const float sy = cand_s[m * kTcWorkers + wt];
          const int jy = cand_j[m * kTcWorkers + wt];
          rank += (sy > sx || (sy == sx && jy < jx)) ? 1 : 0;
        }
        for (int m = 0; m < n_other; ++m) {
          const float sy = cand_s[m * kTcWorkers + wt_other];
          const int jy = cand_j[m * kTcWorkers + wt_other];
          rank += (sy > sx || (sy == sx && jy < jx)) ? 1 : 0;
        }
        // The word of block jx belongs to this thread's half of the chunk.
        if (rank < need) bitmap[(jx >> 5) * kTcRows + row] |= 1u << (jx & 31);
      }
    }
    named_bar_sync(1, kTcWorkers);

    // ---- hand failed rows over; write the others in ascending order ----
    if (half == 0) {
      ctl->rstate[row] = (live && ok && row_ok) ? 1 : 0;
      if (live && ok && !row_ok) {
        const int slot = atomicAdd(a.fb_count, 1);
        a.fb_list[slot] = h * nb + i;
      }
    }
    named_bar_sync(1, kTcWorkers);
    // Each worker warp writes 16 rows, a row at a time: lanes take the
    // bitmap words, a warp prefix sum places their kept blocks, and the row's
    // output (contiguous in idx) is written by the whole warp.
    {
      const int ww = wt >> 5;
      const int words = (nb + 31) >> 5;
      for (int rr = ww; rr < kTcRows; rr += kTcWorkers / 32) {
        if (ctl->rstate[rr] == 0) continue;                 // warp-uniform
        int32_t* out = a.idx + ((size_t)h * nb + i0 + rr) * a.budget;
        int base = 0;
        for (int w0 = 0; w0 < words; w0 += 32) {
          const int w = w0 + lane;
          uint32_t m = w < words ? bitmap[w * kTcRows + rr] : 0u;
          const int cnt = __popc(m);
          int incl = cnt;
#pragma unroll
          for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += y;
          }
          int at = base + incl - cnt;
          while (m != 0u) {
            const int u = __ffs(m) - 1;
            m &= m - 1u;
            if (at < a.budget) out[at] = 32 * w + u;
            ++at;
          }
          base += __shfl_sync(0xffffffffu, incl, 31);
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

}  // namespace

ress_status launch_topk_tc(const Geometry& g, int budget, int32_t* idx, uint8_t* ws,
                           const SelectLayout& lay, cudaStream_t st) {
  CUtensorMap tm_khi, tm_klo, tm_ks;
  const size_t plane_head = (size_t)g.nb_pad * kHeadDim * 4;
  if (!make_f32_rows_map(&tm_khi, ws + lay.tc_khi, g.nb, g.heads, plane_head) ||
      !make_f32_rows_map(&tm_klo, ws + lay.tc_klo, g.nb, g.heads, plane_head) ||
      !make_f32_rows_map(&tm_ks, ws + lay.tc_ksample, 128, g.heads, (size_t)128 * kHeadDim * 4))
    return RESS_ERR_CUDA;
  TcArgs a{};
  a.err = device_error_ptr();
  if (a.err == nullptr) return RESS_ERR_CUDA;
  a.qbar = reinterpret_cast<const float*>(ws + lay.qbar);
  a.khi = reinterpret_cast<const float*>(ws + lay.tc_khi);
  a.klo = reinterpret_cast<const float*>(ws + lay.tc_klo);
  a.knorm = reinterpret_cast<const float*>(ws + lay.tc_knorm);
  a.idx = idx;
  a.fb_count = reinterpret_cast<int32_t*>(ws + lay.tc_fb_count);
  a.fb_list = reinterpret_cast<int32_t*>(ws + lay.tc_fb_list);
  a.nb = g.nb;
  a.nb_pad = g.nb_pad;
  a.budget = budget;
  a.tiles_per_head = (g.nb + kTcRows - 1) / kTcRows;
  a.n_chunks = (g.nb + 127) / 128;
  if (ress_status s = record_cuda(cudaMemsetAsync(a.fb_count, 0, sizeof(int32_t), st))) return s;
  const size_t smem = tc_smem_bytes();
  if (ress_status s = record_cuda(cudaFuncSetAttribute(
          topk_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem)))
    return s;
  topk_tc_kernel<<<g.heads * a.tiles_per_head, kTcThreads, smem, st>>>(tm_khi, tm_klo, tm_ks, a);
  return record_cuda(cudaGetLastError());
}

}  // namespace ress
