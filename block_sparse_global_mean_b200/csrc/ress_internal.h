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
};

constexpr int kHeadDim = 64;
constexpr int kMaxHeads = 64;
constexpr int kMaxBlocksSelect = 4096;

inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// Selection workspace layout (byte offsets).
struct SelectLayout {
  size_t qbar, kbar_t, vbar, contrast, total;
};
SelectLayout select_layout(const Geometry& g, bool with_v);

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
ress_status launch_attn(const Geometry& g, const void* q, const void* k, const void* v,
                        int budget, const int32_t* idx, void* out, bool out_f32, float* lse,
                        cudaStream_t st);
ress_status launch_drift(const Geometry& g, const void* q, const void* k, const void* v,
                         int budget, const int32_t* idx, const float* lse, float* drift,
                         float* set_drift, cudaStream_t st);
ress_status launch_exp2_poly_test(const float* x, float* y, int n, cudaStream_t st);
ress_status launch_cast_bf16(const float* src, __nv_bfloat16* dst, size_t count, cudaStream_t st);

}  // namespace ress
