// Host-side declarations shared by the library's translation units.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "../../include/ress.h"

namespace ress {

// Validated problem geometry.
struct Geometry {
  int64_t n;     // tokens
  int heads;     // H
  int block;     // B
  int nb;        // N / B
  int nb_pad;    // nb rounded up to 256
  bool f32;      // inputs are float32
  // Per-view layout of the layout-aware entry points (lay_t == 0: none):
  // every view is lay_t consecutive tokens, positions < lay_r carry data (the
  // rest is padding) and positions < lay_s are special tokens.  lay_t is a
  // multiple of the block size, so a block's valid and special tokens are
  // prefixes of it.
  int lay_t = 0, lay_r = 0, lay_s = 0;
};

// Valid and special tokens among the `len` tokens from token t0 (both
// prefixes of the range; all of them valid when there is no layout).
__host__ __device__ inline int layout_valid(int lay_t, int lay_r, long long t0, int len) {
  if (lay_t == 0) return len;
  const int v = lay_r - (int)(t0 % lay_t);
  return v < 0 ? 0 : (v > len ? len : v);
}
// The same for a token index below 2^31 (a 32-bit remainder).
__host__ __device__ inline int layout_valid(int lay_t, int lay_r, int t0, int len) {
  if (lay_t == 0) return len;
  const int v = lay_r - (int)((unsigned)t0 % (unsigned)lay_t);
  return v < 0 ? 0 : (v > len ? len : v);
}

constexpr int kHeadDim = 64;
constexpr int kMaxHeads = 64;
constexpr int kMaxBlocksSelect = 4096;

inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// Selection workspace layout (byte offsets).  The shared-memory kernel uses
// qbar, kbar_t (and vbar, contrast when lambda > 0); the tensor-core kernel
// (lambda == 0) uses qbar and the tc_* arrays, placed after qbar.
struct SelectLayout {
  size_t qbar, kbar_t, vbar, contrast;
  size_t tc_khi, tc_klo, tc_ksample, tc_knorm, tc_fb_count, tc_fb_list;
  size_t total;
};
SelectLayout select_layout(const Geometry& g, bool with_v);

// The tensor-core selection handles lambda == 0, a fixed budget below nb and
// nb <= kMaxBlocksTc.
constexpr int kMaxBlocksTc = 2304;
bool select_uses_tc(const Geometry& g, int budget, bool with_v, bool cdf);

// Builds a 3-D TMA map over float32 rows [heads][rows][64] (row stride 256
// bytes) with a box of 32 floats x 128 rows x 1 head, 128-byte swizzle; rows
// beyond `rows` read as zero.
bool make_f32_rows_map(CUtensorMap* map, const void* base, int rows, int heads,
                       size_t head_stride_bytes);

// Builds a 3-D TMA map over a token-major [N][H][64] bf16 tensor with a box
// of 64 (d) x 1 (head) x `rows` (tokens), 128-byte swizzle.
bool make_token_map(CUtensorMap* map, const void* base, const Geometry& g, int rows);

// Records `err` as this thread's last CUDA error (for ress_last_cuda_error)
// and returns RESS_ERR_CUDA, or RESS_OK for cudaSuccess.
ress_status record_cuda(cudaError_t err);

struct DeviceError;
// Device address of the error flag on the current device (null on failure).
DeviceError* device_error_ptr();

// Launchers (argument checks are done by the caller).
// CDF-threshold selection: per row, the count of top blocks whose pooled
// probabilities reach tau goes to counts[H][nb]; idx rows hold the top
// min(count, budget) blocks, padded with the last kept block.
struct CdfSelect {
  float tau;
  int32_t* counts;
};
ress_status launch_select(const Geometry& g, const void* q, const void* k, const void* v,
                          int budget, float lambda, int32_t* idx, void* ws, cudaStream_t st,
                          const CdfSelect* cdf = nullptr);
// Tensor-core top-k over pooled scores, then the exact fallback for the rows
// it hands over (both after the pooling pass that fills the tc_* arrays).
ress_status launch_topk_tc(const Geometry& g, int budget, int32_t* idx, uint8_t* ws,
                           const SelectLayout& lay, cudaStream_t st);
ress_status launch_topk_fallback(const Geometry& g, int budget, int32_t* idx, uint8_t* ws,
                                 const SelectLayout& lay, cudaStream_t st);
ress_status launch_attn(const Geometry& g, const void* q, const void* k, const void* v,
                        int budget, const int32_t* idx, void* out, bool out_f32, float* lse,
                        cudaStream_t st);
// Attention for nq query rows of q (tiles of the same block size) against the
// keys of g; with `dense` every key block is kept for every row (idx unused).
ress_status launch_attn_rows(const Geometry& g, const void* q, int64_t nq, bool dense,
                             const void* k, const void* v, int budget, const int32_t* idx,
                             void* out, bool out_f32, float* lse, cudaStream_t st);
ress_status launch_drift(const Geometry& g, const void* q, const void* k, const void* v,
                         int budget, const int32_t* idx, const float* lse, float* drift,
                         float* set_drift, cudaStream_t st);
// Pooling pass alone: Qbar [H][nb][64], Kbar^T and Vbar^T [H][64][nb_pad]
// (Vbar^T only when v is not null).
ress_status launch_pool(const Geometry& g, const void* q, const void* k, const void* v,
                        float* qbar, float* kbar_t, float* vbar_t, cudaStream_t st);

// Workspace of the restoration-based selection (byte offsets).
struct RestoreLayout {
  size_t qbar, kbar_t, vbar_t, total;
};
RestoreLayout restore_layout(const Geometry& g);
ress_status launch_restore(const Geometry& g, const void* q, const void* k, const void* v,
                           int budget, int rounds, int cand, int32_t* idx, float* j_init,
                           float* j_final, uint8_t* ws, cudaStream_t st);

// VASC selection (value-aware demand with cross-layer memory).
// Pairs of adjacent key blocks: (nb + 1) / 2 per head, the last a singleton
// when nb is odd.
inline int vasc_pairs(int nb) { return (nb + 1) / 2; }
// Inputs of the score kernel's VASC mode: c_h per head (host array of H),
// the pair contrast and the memory's ranking copy [H][pairs], and the demand
// (units of 2^-32) and service sums [H][pairs] it adds to (zeroed before).
struct VascSelect {
  const int32_t* budgets;
  const float* rho;
  const float* mhat;
  unsigned long long* dsum;
  uint32_t* ssum;
};
ress_status launch_score_vasc(const Geometry& g, const float* qbar, const float* kbar_t,
                              int capacity, int32_t* idx, const VascSelect& vs,
                              cudaStream_t st);
// Workspace of ress_select_blocks_vasc (byte offsets): the pooled Q, K^T, V^T
// as for the restoration, then rho, mhat [H][pairs] float32, the demand sums
// [H][pairs] uint64 and the service counts [H][pairs] uint32.
struct VascLayout {
  size_t qbar, kbar_t, vbar_t, rho, mhat, dsum, ssum, total;
};
VascLayout vasc_layout(const Geometry& g);
ress_status launch_vasc(const Geometry& g, const void* q, const void* k, const void* v,
                        const int32_t* budgets, int capacity, bool value_aware, bool reset,
                        float* memory, int32_t* idx, float* demand, float* service, uint8_t* ws,
                        cudaStream_t st);

// Workspace of the special (camera, register) rows of the layout-aware
// attention: the gathered queries [rows_pad][H][64] bf16, their outputs and
// lse (byte offsets; total 0 when there are no special tokens).
struct SpecialLayout {
  int64_t rows, rows_pad;
  size_t q, out, lse, total;
};
SpecialLayout special_layout(const Geometry& g, bool out_f32);
// Gathers the special queries, runs them densely over every valid key and
// scatters their rows into out and lse.
ress_status launch_special_rows(const Geometry& g, const void* q, const void* k, const void* v,
                                void* out, bool out_f32, float* lse, uint8_t* ws,
                                cudaStream_t st);
ress_status launch_exp2_poly_test(const float* x, float* y, int n, cudaStream_t st);
ress_status launch_cast_bf16(const float* src, __nv_bfloat16* dst, size_t count, cudaStream_t st);

}  // namespace ress
