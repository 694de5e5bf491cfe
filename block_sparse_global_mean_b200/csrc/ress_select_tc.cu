// Stage 1 on tcgen05: the fixed-budget top-k of the pooled scores
// s_ij = Qbar_i . Kbar_j (lambda == 0; the 1/sqrt(d) scale does not change a
// row's order), without ever storing a score row.
//
// A CTA takes one head and 128 query blocks: the TMEM lanes, one row per
// lane.  Qbar sits in TMEM as the A operand, split into tf32 high and low
// parts; the pooled keys stream through shared memory in 128-key chunks (TMA,
// 128-byte swizzle), also as tf32 high and low planes, and each chunk's
// 128 x 128 scores land in one of three TMEM accumulators.  Each row is owned
// by four worker threads (the four warps that share its TMEM lane quadrant),
// one per 32-column quarter of every chunk.  Three passes over the keys, all
// reading the scores straight from TMEM:
//
//   sample   128 evenly spaced keys, approximate scores (Qhi . Khi): the
//            row's range [bot, top].
//   pass A   every key, approximate scores: a histogram of 128 bins of width
//            (top - bot) / 127 counted from the top (values outside the range
//            saturate into the end bins); bin b* holds the budget-th largest
//            approximate score.  The bin is formed by a saturating FMA and a
//            round-to-integer add of 1.5 * 2^23, whose bit pattern, times the
//            histogram's row stride, is the shared-memory address up to a
//            constant: about 3.5 instructions per score (the saturating FMA,
//            half a packed FMA, the address multiply-add and a shared
//            reduction).
//   pass B   every key, the full product Qhi.Khi + Qhi.Klo + Qlo.Khi (about
//            float32 accuracy): a score above b*'s upper edge plus the
//            allowance delta for the approximate pass is kept outright, a
//            score within delta of b* is a candidate (appended to the row's
//            list with its full-product score), anything else is dropped.
//
// Then one warp per row: the row's candidates are ranked by their full
// products (larger first, lower index first on equal scores), the best
// budget - (kept outright) join the row's bitmap, and the warp unpacks the
// bitmap in ascending block order into shared memory (sparse words by their
// lane, dense words by the whole warp) and copies the row out coalesced.  A row whose band turns out not to hold the budget-th score (delta is
// an allowance sized from the measured tf32 error, not a proof), or holds more
// candidates than fit, is handed to the exact fallback kernel, which
// recomputes it.
//
// Sources: ReSS (thelatestinai.com) Table S5, SpargeAttn row - selection by
// pooled query/key inner products; Table 1 - a fused scoring kernel;
// VASC (paperlayer.ai) A.2 - an exact-capacity binary Top-K.
//
// Warp roles (576 threads, one CTA per SM): warp 0 TMA, warp 1 TMEM owner and
// MMA issuer (one elected lane), warps 2-17 workers.  Every mbarrier wait is
// bounded; after a timeout the workers skip the remaining work but still pass
// every named barrier, and the CTA frees TMEM and exits.
#include "ress_common.cuh"
#include "ress_internal.h"

namespace ress {

namespace {

constexpr int kTcRows = 128;
constexpr int kTcThreads = 576;
constexpr int kTcWorkers = 512;
constexpr int kTcStages = 2;
constexpr uint32_t kTcBox = 128 * 32 * 4;     // 128 keys x 32 d of float32 = one swizzle span
constexpr uint32_t kTcPlane = 2 * kTcBox;     // 128 keys x 64 d
constexpr uint32_t kTcStage = 2 * kTcPlane;   // tf32 high and low planes
constexpr int kTcAcc = 3;
constexpr uint32_t kTcColQhi = 0, kTcColQlo = 64, kTcColAcc = 128;
constexpr int kTcBins = 128;
constexpr int kTcCand = 72;                   // candidates per row
constexpr int kTcWords = kMaxBlocksTc / 32;   // bitmap words per row
// Worker scratch: during pass A the row histograms, [kTcBins][128 rows] u32;
// afterwards the kept-block bitmaps [kTcWords][128 rows] u32, the candidate
// indices [kTcCand][128] u16 and their full-product scores [kTcCand][128] f32.
// Bitmap words and candidate slots are stored at row ^ (word or slot & 31), so
// that a warp touching 32 rows of one word, or 32 words of one row, hits 32
// different banks.
constexpr uint32_t kTcHistBytes = kTcBins * kTcRows * 4;
constexpr uint32_t kTcBitmapBytes = kTcWords * kTcRows * 4;
constexpr uint32_t kTcCandJBytes = kTcCand * kTcRows * 2;
constexpr uint32_t kTcCandSBytes = kTcCand * kTcRows * 4;
constexpr uint32_t kTcRegion = (kTcBitmapBytes + kTcCandJBytes + kTcCandSBytes) > kTcHistBytes
                                   ? (kTcBitmapBytes + kTcCandJBytes + kTcCandSBytes)
                                   : kTcHistBytes;
constexpr uint32_t kMagicBits = 0x4B400000u;  // bits of 1.5 * 2^23
constexpr float kMagic = 12582912.0f;
// The bin b of a score sits in the low bits of kMagicBits + b; times the
// histogram's row stride (512 bytes) that is b * 512 plus kMagicBits * 512,
// which is 2^31 modulo 2^32.
constexpr uint32_t kHistBias = kMagicBits * (uint32_t)(kTcRows * 4);

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
  float xa[4][kTcRows];     // per quarter: the sample's largest score
  float xb[4][kTcRows];     // per quarter: the sample's smallest score
  int kept[kTcRows];        // scores above the band
  int ncand[kTcRows];       // candidates appended (may exceed kTcCand)
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

// min(max(a * b + c, 0), 1) in one instruction.
__device__ __forceinline__ float fma_sat(float a, float b, float c) {
  float d;
  asm("fma.rn.sat.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// Histogram count of a pair of approximate scores: u = sat((top - s) / (top -
// bot)) (NaN saturates to 0), b = round(127 u) by adding 1.5 * 2^23 (so the
// float's bits are kMagicBits + b), and one increment of the row's bin b at
// hist_row + 512 b = hist_row - kHistBias + 512 * bits (modulo 2^32).
__device__ __forceinline__ void hist_pair(float s0, float s1, float neg_us, float off,
                                          uint32_t hist_base) {
  const float2 f = ffma2(make_float2(fma_sat(s0, neg_us, off), fma_sat(s1, neg_us, off)),
                         make_float2(127.0f, 127.0f), make_float2(kMagic, kMagic));
  red_add_shared_u32(hist_base + __float_as_uint(f.x) * (uint32_t)(kTcRows * 4), 1u);
  red_add_shared_u32(hist_base + __float_as_uint(f.y) * (uint32_t)(kTcRows * 4), 1u);
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

__device__ __forceinline__ uint32_t swz(int word_or_slot, int row) {
  return (uint32_t)(word_or_slot * kTcRows + (row ^ (word_or_slot & 31)));
}

__global__ void __launch_bounds__(kTcThreads, 1)
    topk_tc_kernel(const __grid_constant__ CUtensorMap tm_khi,
                   const __grid_constant__ CUtensorMap tm_klo,
                   const __grid_constant__ CUtensorMap tm_ks, const TcArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024_shared(smem_raw);
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
    const int wt = threadIdx.x - 64;            // 0 .. 511
    const int quad = warp & 3;                  // TMEM lanes 32 quad .. 32 quad + 31
    const int quarter = (warp - 2) >> 2;        // columns 32 quarter .. 32 quarter + 31 of a chunk
    const int row = quad * 32 + lane;
    const int i = i0 + row;
    const bool live = i < a.nb;
    const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
    const uint32_t col = 32u * (uint32_t)quarter;
    const int nb = a.nb;
    const float* qrow = a.qbar + ((size_t)h * nb + (live ? i : 0)) * kHeadDim;
    bool ok = true;

    // Zero the histograms (64 KB over the 512 workers) and the row counters.
    {
      uint4* z = reinterpret_cast<uint4*>(region);
      for (int e = wt; e < (int)(kTcHistBytes / 16); e += kTcWorkers) z[e] = make_uint4(0u, 0u, 0u, 0u);
      if (quarter == 0) {
        ctl->kept[row] = 0;
        ctl->ncand[row] = 0;
      }
    }
    // Qbar row into TMEM: quarter q writes d = 32 (q & 1) .. + 31 of the tf32
    // high (q < 2) or low (q >= 2) parts.  Every thread sums |Qbar_i|^2.
    float qn2 = 0.f;
    {
      const float* qown = qrow + 32 * (quarter & 1);
      uint32_t part[32];
#pragma unroll
      for (int u4 = 0; u4 < 8; ++u4) {
        const float4 x = live ? *reinterpret_cast<const float4*>(qown + 4 * u4)
                              : make_float4(0.f, 0.f, 0.f, 0.f);
        const float xs[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          qn2 = fmaf(xs[e], xs[e], qn2);
          const float hi = to_tf32(xs[e]);
          part[4 * u4 + e] = __float_as_uint(quarter >= 2 ? to_tf32(xs[e] - hi) : hi);
        }
      }
      tmem_st32(tmem + (quarter >= 2 ? kTcColQlo : kTcColQhi) + lane_off + 32u * (uint32_t)(quarter & 1),
                part);
      const float* qother = qrow + 32 * ((quarter & 1) ^ 1);
#pragma unroll 1
      for (int u4 = 0; u4 < 8; ++u4) {
        const float4 x = live ? *reinterpret_cast<const float4*>(qother + 4 * u4)
                              : make_float4(0.f, 0.f, 0.f, 0.f);
        qn2 = fmaf(x.x, x.x, fmaf(x.y, x.y, fmaf(x.z, x.z, fmaf(x.w, x.w, qn2))));
      }
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
    {
      float mx = -INFINITY, mn = INFINITY;
      if (ok) ok = warp_wait(smem_addr(&ctl->acc_full[0]), 0, abortf, a.err, 96);
      if (ok) {
        tc_fence_after();
        uint32_t r[32];
        tmem_ld32(tmem + kTcColAcc + lane_off + col, r);
        tmem_ld_wait_regs(r);
#pragma unroll
        for (int u = 0; u < 16; ++u) {
          const float s0 = __uint_as_float(r[2 * u]), s1 = __uint_as_float(r[2 * u + 1]);
          mx = fmax3(mx, s0, s1);
          mn = fminf(mn, fminf(s0, s1));
        }
        tc_fence_before();
        mbar_arrive(smem_addr(&ctl->acc_empty[0]));
      }
      ctl->xa[quarter][row] = mx;
      ctl->xb[quarter][row] = mn;
    }
    named_bar_sync(1, kTcWorkers);
    const float top = fmaxf(fmaxf(ctl->xa[0][row], ctl->xa[1][row]),
                            fmaxf(ctl->xa[2][row], ctl->xa[3][row]));
    const float bot = fminf(fminf(ctl->xb[0][row], ctl->xb[1][row]),
                            fminf(ctl->xb[2][row], ctl->xb[3][row]));
    // t = (top - s) * scale in [0, 127] across the sample's range.
    float scale = (float)(kTcBins - 1) / (top - bot);
    if (!(scale < INFINITY)) scale = 0.f;           // constant range: one bin
    const float us = 1.0f / (top - bot) < INFINITY ? 1.0f / (top - bot) : 0.f;
    const float neg_us = -us, off = top * us;

    // ---- pass A: histogram of the approximate scores ----
    // Every column is counted, the last chunk's padding too: TMA fills the
    // key rows past nb with zeros, whose score is exactly 0, so the scan
    // below takes their count (pad) back out of the bin that 0 falls in.
    const uint32_t hist_base = smem_addr(region) + (uint32_t)row * 4u - kHistBias;
    auto load_chunk = [&](int seq, uint32_t (&r)[32], int detail) -> bool {
      const int b = seq % kTcAcc;
      if (!warp_wait(smem_addr(&ctl->acc_full[b]), (seq / kTcAcc) & 1, abortf, a.err, detail))
        return false;
      tc_fence_after();
      tmem_ld32(tmem + kTcColAcc + 128u * (uint32_t)b + lane_off + col, r);
      tmem_ld_wait_regs(r);
      tc_fence_before();
      mbar_arrive(smem_addr(&ctl->acc_empty[b]));
      return true;
    };
    for (int c = 0; c < C && ok; ++c) {
      uint32_t r[32];
      ok = load_chunk(1 + c, r, 97);
      if (!ok) break;
#pragma unroll
      for (int u = 0; u < 16; ++u)
        hist_pair(__uint_as_float(r[2 * u]), __uint_as_float(r[2 * u + 1]), neg_us, off, hist_base);
    }
    named_bar_sync(1, kTcWorkers);

    // ---- the bin b* of the budget-th largest approximate score ----
    // The four threads of a row scan the same counts, so they agree without
    // an exchange.  Bin 0 is the top of the range.
    float hiT = INFINITY, loT = -INFINITY;
    {
      const uint32_t* hist = reinterpret_cast<const uint32_t*>(region);
      const int pad = 128 * C - nb;
      const int bin0 = (int)(__float_as_uint(fmaf(fma_sat(0.0f, neg_us, off), 127.0f, kMagic)) -
                             kMagicBits);
      int cum = 0, bstar = kTcBins - 1;
      for (int b0 = 0; b0 < kTcBins; b0 += 8) {
        int v[8], s8 = 0;
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          v[e] = (int)hist[(b0 + e) * kTcRows + row] - (b0 + e == bin0 ? pad : 0);
          s8 += v[e];
        }
        if (cum + s8 >= a.budget) {
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            if (cum + v[e] >= a.budget) {
              bstar = b0 + e;
              break;
            }
            cum += v[e];
          }
          break;
        }
        cum += s8;
      }
      // Bin b holds the approximate scores s with (top - s) * scale within
      // 1/2 of b (bin 0 everything above, the last bin everything below the
      // range), up to rounding; the exact budget-th score lies within delta
      // of b*.
      const float eps = 1e-6f * (fabsf(top) + fabsf(bot)) + 1e-30f;
      if (scale > 0.f) {
        if (bstar > 0) hiT = top - ((float)bstar - 0.5f) / scale + delta + eps;
        if (bstar < kTcBins - 1) loT = top - ((float)bstar + 0.5f) / scale - delta - eps;
      }
    }
    named_bar_sync(1, kTcWorkers);   // the histograms are no longer read

    // ---- pass B: full products; keep, candidate or drop ----
    uint32_t* bitmap = reinterpret_cast<uint32_t*>(region);                           // [words][128]
    uint16_t* cand_j = reinterpret_cast<uint16_t*>(region + kTcBitmapBytes);          // [cap][128]
    float* cand_s = reinterpret_cast<float*>(region + kTcBitmapBytes + kTcCandJBytes); // [cap][128]
    int kept = 0;
    for (int c = 0; c < C && ok; ++c) {
      uint32_t r[32];
      ok = load_chunk(C + 1 + c, r, 98);
      if (!ok) break;
      uint32_t kw = 0u, gw = 0u;
#pragma unroll
      for (int u = 0; u < 32; ++u) {
        const float sv = __uint_as_float(r[u]);
        kw |= (sv > hiT) ? (1u << u) : 0u;
        gw |= (sv >= loT) ? (1u << u) : 0u;
      }
      const int j0 = 128 * c + (int)col;
      if (j0 + 32 > nb) {
        const uint32_t valid = j0 >= nb ? 0u : ((1u << (nb - j0)) - 1u);
        kw &= valid;
        gw &= valid;
      }
      if (j0 < nb) bitmap[swz(j0 >> 5, row)] = kw;
      kept += __popc(kw);
      uint32_t cw = gw & ~kw;
      while (cw != 0u) {
        const int u = __ffs(cw) - 1;
        cw &= cw - 1u;
        const int slot = atomicAdd(&ctl->ncand[row], 1);
        if (slot < kTcCand) {
          cand_j[swz(slot, row)] = (uint16_t)(j0 + u);
          cand_s[swz(slot, row)] = __uint_as_float(select32(r, u));
        }
      }
    }
    if (kept > 0) atomicAdd(&ctl->kept[row], kept);
    named_bar_sync(1, kTcWorkers);

    // ---- one warp per row: rank the candidates, then write the row ----
    const bool aborted = *abortf != 0;
    const int ww = wt >> 5;
    const int words = (nb + 31) >> 5;
    const uint32_t lt_mask = (1u << lane) - 1u;
    // Output staging of this warp (the key stages are free once pass B is
    // done): 1,024 entries per warp, a row segment at a time.
    constexpr int kSeg = 1024;
    int32_t* stg = reinterpret_cast<int32_t*>(stages) + ww * kSeg;
    for (int rr = ww; rr < kTcRows; rr += kTcWorkers / 32) {
      if (aborted || i0 + rr >= nb) break;
      const int total = ctl->ncand[rr];
      const int need = a.budget - ctl->kept[rr];
      if (!(total <= kTcCand && need >= 0 && need <= total)) {
        if (lane == 0) {
          const int slot = atomicAdd(a.fb_count, 1);
          a.fb_list[slot] = h * nb + i0 + rr;
        }
        continue;
      }
      // Rank: the number of candidates with a larger full-product score, or
      // an equal score and a lower block index; the best `need` win.
      if (need > 0 && total <= 32) {
        const float sx = lane < total ? cand_s[swz(lane, rr)] : -INFINITY;
        const int jx = lane < total ? (int)cand_j[swz(lane, rr)] : 0xFFFF;
        int rank = 0;
#pragma unroll 4
        for (int m = 0; m < total; ++m) {
          const float sy = __shfl_sync(0xffffffffu, sx, m);
          const int jy = __shfl_sync(0xffffffffu, jx, m);
          rank += (sy > sx || (sy == sx && jy < jx)) ? 1 : 0;
        }
        if (lane < total && rank < need) atomicOr(&bitmap[swz(jx >> 5, rr)], 1u << (jx & 31));
      } else if (need > 0) {
        float sx[3];
        int jx[3], rank[3] = {0, 0, 0};
#pragma unroll
        for (int t = 0; t < 3; ++t) {
          const int cx = 32 * t + lane;
          sx[t] = cx < total ? cand_s[swz(cx, rr)] : -INFINITY;
          jx[t] = cx < total ? (int)cand_j[swz(cx, rr)] : 0xFFFF;
        }
#pragma unroll 2
        for (int m = 0; m < total; ++m) {
          const float sy = cand_s[swz(m, rr)];
          const int jy = cand_j[swz(m, rr)];
#pragma unroll
          for (int t = 0; t < 3; ++t)
            rank[t] += (sy > sx[t] || (sy == sx[t] && jy < jx[t])) ? 1 : 0;
        }
#pragma unroll
        for (int t = 0; t < 3; ++t)
          if (32 * t + lane < total && rank[t] < need)
            atomicOr(&bitmap[swz(jx[t] >> 5, rr)], 1u << (jx[t] & 31));
      }
      __syncwarp();
      // Write: lane l holds bitmap words l, l + 32 and l + 64; a warp scan
      // gives every word's first output position.  Words with at most 8
      // blocks are unpacked by their lane; denser words (whole views kept)
      // by the whole warp, one word at a time.  Both go through the staging
      // buffer, which the warp then copies out in 128-byte rows.
      uint32_t mw[3];
      int base[3], run = 0;
#pragma unroll
      for (int t = 0; t < 3; ++t) {
        const int w = 32 * t + lane;
        mw[t] = w < words ? bitmap[swz(w, rr)] : 0u;
        const int c = __popc(mw[t]);
        int incl = c;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int y = __shfl_up_sync(0xffffffffu, incl, o);
          if (lane >= o) incl += y;
        }
        base[t] = run + incl - c;
        run += __shfl_sync(0xffffffffu, incl, 31);
      }
      const int n_out = min(run, a.budget);
      int32_t* out = a.idx + ((size_t)h * nb + i0 + rr) * a.budget;
      for (int s0 = 0; s0 < n_out; s0 += kSeg) {
#pragma unroll
        for (int t = 0; t < 3; ++t) {
          const int wbase = 32 * (32 * t + lane);
          if (__popc(mw[t]) <= 8) {
            uint32_t m = mw[t];
            int pos = base[t] - s0;
            while (m != 0u) {
              const int u = __ffs(m) - 1;
              m &= m - 1u;
              if (pos >= 0 && pos < kSeg) stg[pos] = wbase + u;
              ++pos;
            }
          }
          uint32_t dense = __ballot_sync(0xffffffffu, __popc(mw[t]) > 8);
          while (dense != 0u) {
            const int src = __ffs(dense) - 1;
            dense &= dense - 1u;
            const uint32_t word = __shfl_sync(0xffffffffu, mw[t], src);
            const int pos = __shfl_sync(0xffffffffu, base[t], src) + __popc(word & lt_mask) - s0;
            if (((word >> lane) & 1u) && pos >= 0 && pos < kSeg)
              stg[pos] = 32 * (32 * t + src) + lane;
          }
        }
        __syncwarp();
        const int n_seg = min(n_out - s0, kSeg);
        for (int e = lane; e < n_seg; e += 32) out[s0 + e] = stg[e];
        __syncwarp();
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
