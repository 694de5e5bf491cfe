// C ABI of the library: host-side argument checks, workspace queries, the
// float32 -> bf16 staging kernel, TMA descriptor encoding and the device
// error flag.  Every entry point validates before its first CUDA call.
#include <cudaTypedefs.h>

#include <cmath>
#include <cstdio>
#include <mutex>

#include "ress_common.cuh"
#include "ress_internal.h"

namespace ress {

__device__ DeviceError g_device_error = {0, 0};

namespace {

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

ress_status check_shape(const ress_shape* s, Geometry* g) {
  if (s == nullptr) return RESS_ERR_INVALID_ARG;
  if (s->n < 0 || s->heads <= 0 || s->head_dim <= 0 || s->block <= 0) return RESS_ERR_INVALID_ARG;
  if (s->dtype != RESS_BF16 && s->dtype != RESS_F32) return RESS_ERR_INVALID_ARG;
  if (s->head_dim != kHeadDim) return RESS_ERR_UNSUPPORTED;
  if (s->block != 64 && s->block != 128) return RESS_ERR_UNSUPPORTED;
  if (s->heads > kMaxHeads) return RESS_ERR_UNSUPPORTED;
  if (s->n % s->block != 0) return RESS_ERR_INVALID_ARG;
  // Token offsets and TMA coordinates are 32-bit.
  if (s->n > (int64_t)1 << 30) return RESS_ERR_UNSUPPORTED;
  g->n = s->n;
  g->heads = s->heads;
  g->block = s->block;
  g->nb = (int)(s->n / s->block);
  g->nb_pad = (g->nb + 255) & ~255;
  g->f32 = s->dtype == RESS_F32;
  return RESS_OK;
}

ress_status check_layout(const ress_layout* lay, Geometry* g) {
  if (lay == nullptr) return RESS_ERR_INVALID_ARG;
  const int t = lay->tokens_per_view, r = lay->real_tokens, sp = lay->special_tokens;
  if (t <= 0 || t % g->block != 0 || g->n % t != 0) return RESS_ERR_INVALID_ARG;
  if (r < 1 || r > t || sp < 0 || sp > r) return RESS_ERR_INVALID_ARG;
  g->lay_t = t;
  g->lay_r = r;
  g->lay_s = sp;
  return RESS_OK;
}

ress_status check_budget(const Geometry& g, int32_t budget) {
  if (g.nb == 0) return RESS_OK;
  return (budget >= 1 && budget <= g.nb) ? RESS_OK : RESS_ERR_INVALID_ARG;
}

__global__ void cast_bf16_kernel(const float4* __restrict__ src, uint2* __restrict__ dst,
                                 size_t n4) {
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n4;
       i += (size_t)gridDim.x * blockDim.x) {
    const float4 v = src[i];
    uint2 o;
    o.x = pack_bf16x2(v.x, v.y);
    o.y = pack_bf16x2(v.z, v.w);
    dst[i] = o;
  }
}

// One warp per (h, i) row of idx: every entry in [0, nb), strictly ascending.
__global__ void __launch_bounds__(256) validate_idx_kernel(const int32_t* __restrict__ idx,
                                                           int rows, int nb, int budget,
                                                           DeviceError* err) {
  const int row = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  const int32_t* r = idx + (size_t)row * budget;
  bool out_of_range = false, repeat = false, descending = false;
  for (int e = lane; e < budget; e += 32) {
    const int j = r[e];
    out_of_range |= j < 0 || j >= nb;
    if (e + 1 < budget) {
      const int nx = r[e + 1];
      repeat |= nx == j;
      descending |= nx < j;
    }
  }
  const unsigned any_range = __ballot_sync(0xffffffffu, out_of_range);
  const unsigned any_repeat = __ballot_sync(0xffffffffu, repeat);
  const unsigned any_desc = __ballot_sync(0xffffffffu, descending);
  if (lane == 0) {
    if (any_range) raise_device_error(err, RESS_ERR_BAD_INDEX, 80);
    else if (any_repeat) raise_device_error(err, RESS_ERR_BAD_INDEX, 81);
    else if (any_desc) raise_device_error(err, RESS_ERR_BAD_INDEX, 82);
  }
}

PFN_cuTensorMapEncodeTiled_v12000 get_encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  });
  return fn;
}

}  // namespace

namespace {
thread_local char g_last_cuda_error[256] = "";
}  // namespace

ress_status record_cuda(cudaError_t err) {
  if (err == cudaSuccess) return RESS_OK;
  snprintf(g_last_cuda_error, sizeof(g_last_cuda_error), "%s: %s", cudaGetErrorName(err),
           cudaGetErrorString(err));
  return RESS_ERR_CUDA;
}

DeviceError* device_error_ptr() {
  // One address per device; looked up with that device current.
  static DeviceError* cache[64] = {};
  static std::mutex mu;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> lock(mu);
  if (cache[dev] == nullptr) {
    void* ptr = nullptr;
    if (record_cuda(cudaGetSymbolAddress(&ptr, g_device_error)) != RESS_OK) return nullptr;
    cache[dev] = static_cast<DeviceError*>(ptr);
  }
  return cache[dev];
}

bool make_token_map(CUtensorMap* map, const void* base, const Geometry& g, int rows) {
  PFN_cuTensorMapEncodeTiled_v12000 encode = get_encode_fn();
  if (encode == nullptr) return false;
  const cuuint64_t dims[3] = {(cuuint64_t)kHeadDim, (cuuint64_t)g.heads, (cuuint64_t)g.n};
  const cuuint64_t strides[2] = {(cuuint64_t)kHeadDim * 2, (cuuint64_t)g.heads * kHeadDim * 2};
  const cuuint32_t box[3] = {(cuuint32_t)kHeadDim, 1u, (cuuint32_t)rows};
  const cuuint32_t estr[3] = {1u, 1u, 1u};
  const CUresult r = encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims,
                            strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                            CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS)
    snprintf(g_last_cuda_error, sizeof(g_last_cuda_error),
             "cuTensorMapEncodeTiled failed (CUresult %d)", (int)r);
  return r == CUDA_SUCCESS;
}

bool make_f32_rows_map(CUtensorMap* map, const void* base, int rows, int heads,
                       size_t head_stride_bytes) {
  PFN_cuTensorMapEncodeTiled_v12000 encode = get_encode_fn();
  if (encode == nullptr) return false;
  const cuuint64_t dims[3] = {(cuuint64_t)kHeadDim, (cuuint64_t)rows, (cuuint64_t)heads};
  const cuuint64_t strides[2] = {(cuuint64_t)kHeadDim * 4, (cuuint64_t)head_stride_bytes};
  const cuuint32_t box[3] = {32u, 128u, 1u};
  const cuuint32_t estr[3] = {1u, 1u, 1u};
  const CUresult r = encode(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<void*>(base), dims,
                            strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                            CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS)
    snprintf(g_last_cuda_error, sizeof(g_last_cuda_error),
             "cuTensorMapEncodeTiled failed (CUresult %d)", (int)r);
  return r == CUDA_SUCCESS;
}

ress_status launch_cast_bf16(const float* src, __nv_bfloat16* dst, size_t count, cudaStream_t st) {
  const size_t n4 = count / 4;   // count is a multiple of 64
  if (n4 == 0) return RESS_OK;
  const unsigned blocks = (unsigned)((n4 + 255) / 256 < 148 * 16 ? (n4 + 255) / 256 : 148 * 16);
  cast_bf16_kernel<<<blocks, 256, 0, st>>>(reinterpret_cast<const float4*>(src),
                                           reinterpret_cast<uint2*>(dst), n4);
  return record_cuda(cudaGetLastError());
}

}  // namespace ress

using namespace ress;

extern "C" {

int ress_version(void) { return (1 << 16) | 0; }

const char* ress_status_string(ress_status status) {
  switch (status) {
    case RESS_OK: return "ok";
    case RESS_ERR_INVALID_ARG: return "invalid argument";
    case RESS_ERR_UNSUPPORTED: return "unsupported configuration";
    case RESS_ERR_WORKSPACE: return "workspace too small";
    case RESS_ERR_CUDA: return "CUDA error";
    case RESS_ERR_TIMEOUT: return "device wait timed out";
    case RESS_ERR_BAD_INDEX: return "block index out of range";
  }
  return "unknown status";
}

size_t ress_select_workspace_bytes(const ress_shape* shape, float lambda) {
  Geometry g;
  if (check_shape(shape, &g) != RESS_OK) return 0;
  return select_layout(g, lambda != 0.f).total;
}

ress_status ress_select_blocks(const ress_shape* shape, const void* q, const void* k,
                               const void* v, int32_t budget, float lambda, int32_t* idx,
                               void* workspace, size_t workspace_bytes, void* stream) {
  Geometry g;
  ress_status s = check_shape(shape, &g);
  if (s != RESS_OK) return s;
  if (!(lambda >= 0.f) || std::isinf(lambda)) return RESS_ERR_INVALID_ARG;
  if ((s = check_budget(g, budget)) != RESS_OK) return s;
  if (g.nb == 0) return RESS_OK;
  if (g.nb > kMaxBlocksSelect) return RESS_ERR_UNSUPPORTED;
  const bool with_v = lambda != 0.f;
  if (!q || !k || !idx || (with_v && !v) || !workspace) return RESS_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || (with_v && !aligned16(v)) ||
      (reinterpret_cast<uintptr_t>(workspace) & 255u) || (reinterpret_cast<uintptr_t>(idx) & 3u))
    return RESS_ERR_INVALID_ARG;
  if (workspace_bytes < select_layout(g, with_v).total) return RESS_ERR_WORKSPACE;
  return launch_select(g, q, k, with_v ? v : nullptr, budget, lambda, idx, workspace,
                       static_cast<cudaStream_t>(stream));
}

ress_status ress_select_blocks_layout(const ress_shape* shape, const ress_layout* layout,
                                      const void* q, const void* k, int32_t budget,
                                      int32_t* idx, void* workspace, size_t workspace_bytes,
                                      void* stream) {
  Geometry g;
  ress_status s = check_shape(shape, &g);
  if (s != RESS_OK) return s;
  if ((s = check_layout(layout, &g)) != RESS_OK) return s;
  if ((s = check_budget(g, budget)) != RESS_OK) return s;
  if (g.nb == 0) return RESS_OK;
  if (g.nb > kMaxBlocksSelect) return RESS_ERR_UNSUPPORTED;
  if (!q || !k || !idx || !workspace) return RESS_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || (reinterpret_cast<uintptr_t>(workspace) & 255u) ||
      (reinterpret_cast<uintptr_t>(idx) & 3u))
    return RESS_ERR_INVALID_ARG;
  if (workspace_bytes < select_layout(g, false).total) return RESS_ERR_WORKSPACE;
  return launch_select(g, q, k, nullptr, budget, 0.f, idx, workspace,
                       static_cast<cudaStream_t>(stream));
}

ress_status ress_select_blocks_cdf(const ress_shape* shape, const void* q, const void* k,
                                   float tau, int32_t capacity, int32_t* counts, int32_t* idx,
                                   void* workspace, size_t workspace_bytes, void* stream) {
  Geometry g;
  ress_status s = check_shape(shape, &g);
  if (s != RESS_OK) return s;
  if (!(tau > 0.f && tau <= 1.f)) return RESS_ERR_INVALID_ARG;
  if ((s = check_budget(g, capacity)) != RESS_OK) return s;
  if (g.nb == 0) return RESS_OK;
  if (g.nb > kMaxBlocksSelect) return RESS_ERR_UNSUPPORTED;
  if (!q || !k || !counts || !idx || !workspace) return RESS_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || (reinterpret_cast<uintptr_t>(workspace) & 255u) ||
      (reinterpret_cast<uintptr_t>(idx) & 3u) || (reinterpret_cast<uintptr_t>(counts) & 3u))
    return RESS_ERR_INVALID_ARG;
  if (workspace_bytes < select_layout(g, false).total) return RESS_ERR_WORKSPACE;
  const CdfSelect cdf{tau, counts};
  return launch_select(g, q, k, nullptr, capacity, 0.f, idx, workspace,
                       static_cast<cudaStream_t>(stream), &cdf);
}

size_t ress_restore_workspace_bytes(const ress_shape* shape) {
  Geometry g;
  if (check_shape(shape, &g) != RESS_OK) return 0;
  return restore_layout(g).total;
}

ress_status ress_select_blocks_restore(const ress_shape* shape, const void* q, const void* k,
                                       const void* v, int32_t budget, int32_t rounds,
                                       int32_t candidates, int32_t* idx, float* drift_init,
                                       float* drift_final, void* workspace,
                                       size_t workspace_bytes, void* stream) {
  Geometry g;
  ress_status s = check_shape(shape, &g);
  if (s != RESS_OK) return s;
  if ((s = check_budget(g, budget)) != RESS_OK) return s;
  if (rounds < 0 || rounds > 64 || candidates < 1 || candidates > 16) return RESS_ERR_INVALID_ARG;
  if (g.nb == 0) return RESS_OK;
  if (g.nb > kMaxBlocksSelect) return RESS_ERR_UNSUPPORTED;
  if (!q || !k || !v || !idx || !workspace) return RESS_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) ||
      (reinterpret_cast<uintptr_t>(workspace) & 255u) || (reinterpret_cast<uintptr_t>(idx) & 3u) ||
      (reinterpret_cast<uintptr_t>(drift_init) & 3u) ||
      (reinterpret_cast<uintptr_t>(drift_final) & 3u))
    return RESS_ERR_INVALID_ARG;
  if (workspace_bytes < restore_layout(g).total) return RESS_ERR_WORKSPACE;
  return launch_restore(g, q, k, v, budget, rounds, candidates, idx, drift_init, drift_final,
                        static_cast<uint8_t*>(workspace), static_cast<cudaStream_t>(stream));
}

size_t ress_vasc_workspace_bytes(const ress_shape* shape) {
  Geometry g;
  if (check_shape(shape, &g) != RESS_OK) return 0;
  return vasc_layout(g).total;
}

ress_status ress_select_blocks_vasc(const ress_shape* shape, const void* q, const void* k,
                                    const void* v, const int32_t* budgets, int32_t capacity,
                                    int32_t value_aware, int32_t reset, float* memory,
                                    int32_t* idx, float* demand, float* service,
                                    void* workspace, size_t workspace_bytes, void* stream) {
  Geometry g;
  ress_status s = check_shape(shape, &g);
  if (s != RESS_OK) return s;
  if ((s = check_budget(g, capacity)) != RESS_OK) return s;
  if ((value_aware != 0 && value_aware != 1) || (reset != 0 && reset != 1))
    return RESS_ERR_INVALID_ARG;
  if (g.nb == 0) return RESS_OK;
  if (budgets == nullptr) return RESS_ERR_INVALID_ARG;
  for (int h = 0; h < g.heads; ++h)
    if (budgets[h] < 1 || budgets[h] > capacity) return RESS_ERR_INVALID_ARG;
  if (g.nb > kMaxBlocksSelect) return RESS_ERR_UNSUPPORTED;
  if (!q || !k || (value_aware && !v) || !memory || !idx || !workspace) return RESS_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || (v && !aligned16(v)) ||
      (reinterpret_cast<uintptr_t>(workspace) & 255u) || (reinterpret_cast<uintptr_t>(idx) & 3u) ||
      (reinterpret_cast<uintptr_t>(memory) & 3u) || (reinterpret_cast<uintptr_t>(demand) & 3u) ||
      (reinterpret_cast<uintptr_t>(service) & 3u))
    return RESS_ERR_INVALID_ARG;
  if (workspace_bytes < vasc_layout(g).total) return RESS_ERR_WORKSPACE;
  return launch_vasc(g, q, k, v, budgets, capacity, value_aware != 0, reset != 0, memory, idx,
                     demand, service, static_cast<uint8_t*>(workspace),
                     static_cast<cudaStream_t>(stream));
}

size_t ress_attn_workspace_bytes(const ress_shape* shape) {
  Geometry g;
  if (check_shape(shape, &g) != RESS_OK) return 0;
  return g.f32 ? 3 * align256((size_t)g.n * g.heads * kHeadDim * 2) : 0;
}

namespace {

// Stages float32 inputs as bf16 copies in the workspace (no-op for bf16).
ress_status stage_inputs(const Geometry& g, const void*& q, const void*& k, const void*& v,
                         void* workspace, size_t workspace_bytes, cudaStream_t st) {
  if (!g.f32) return RESS_OK;
  const size_t count = (size_t)g.n * g.heads * kHeadDim;
  const size_t each = align256(count * 2);
  if (!workspace || workspace_bytes < 3 * each) return RESS_ERR_WORKSPACE;
  if (reinterpret_cast<uintptr_t>(workspace) & 255u) return RESS_ERR_INVALID_ARG;
  uint8_t* w = static_cast<uint8_t*>(workspace);
  const void* src[3] = {q, k, v};
  for (int t = 0; t < 3; ++t) {
    const ress_status s = launch_cast_bf16(static_cast<const float*>(src[t]),
                                           reinterpret_cast<__nv_bfloat16*>(w + t * each), count, st);
    if (s != RESS_OK) return s;
  }
  q = w;
  k = w + each;
  v = w + 2 * each;
  return RESS_OK;
}

}  // namespace

ress_status ress_block_sparse_attn(const ress_shape* shape, const void* q, const void* k,
                                   const void* v, int32_t budget, const int32_t* idx,
                                   void* out, int32_t out_dtype, float* lse, void* workspace,
                                   size_t workspace_bytes, void* stream) {
  Geometry g;
  ress_status s = check_shape(shape, &g);
  if (s != RESS_OK) return s;
  if ((s = check_budget(g, budget)) != RESS_OK) return s;
  if (g.nb == 0) return RESS_OK;
  if (!q || !k || !v || !idx || !out) return RESS_ERR_INVALID_ARG;
  if (out_dtype != RESS_BF16 && out_dtype != RESS_F32) return RESS_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) ||
      (reinterpret_cast<uintptr_t>(idx) & 3u) || (reinterpret_cast<uintptr_t>(lse) & 3u))
    return RESS_ERR_INVALID_ARG;
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (g.f32 && (!workspace || workspace_bytes < ress_attn_workspace_bytes(shape)))
    return RESS_ERR_WORKSPACE;
  if ((s = stage_inputs(g, q, k, v, workspace, workspace_bytes, st)) != RESS_OK) return s;
  return launch_attn(g, q, k, v, budget, idx, out, out_dtype == RESS_F32, lse, st);
}

size_t ress_attn_layout_workspace_bytes(const ress_shape* shape, const ress_layout* layout,
                                        int32_t out_dtype) {
  Geometry g;
  if (check_shape(shape, &g) != RESS_OK || check_layout(layout, &g) != RESS_OK) return 0;
  if (out_dtype != RESS_BF16 && out_dtype != RESS_F32) return 0;
  return ress_attn_workspace_bytes(shape) + special_layout(g, out_dtype == RESS_F32).total;
}

ress_status ress_block_sparse_attn_layout(const ress_shape* shape, const ress_layout* layout,
                                          const void* q, const void* k, const void* v,
                                          int32_t budget, const int32_t* idx, void* out,
                                          int32_t out_dtype, float* lse, void* workspace,
                                          size_t workspace_bytes, void* stream) {
  Geometry g;
  ress_status s = check_shape(shape, &g);
  if (s != RESS_OK) return s;
  if ((s = check_layout(layout, &g)) != RESS_OK) return s;
  if ((s = check_budget(g, budget)) != RESS_OK) return s;
  if (g.nb == 0) return RESS_OK;
  if (!q || !k || !v || !idx || !out) return RESS_ERR_INVALID_ARG;
  if (out_dtype != RESS_BF16 && out_dtype != RESS_F32) return RESS_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) ||
      (reinterpret_cast<uintptr_t>(idx) & 3u) || (reinterpret_cast<uintptr_t>(lse) & 3u))
    return RESS_ERR_INVALID_ARG;
  const size_t stage = ress_attn_workspace_bytes(shape);
  const SpecialLayout sl = special_layout(g, out_dtype == RESS_F32);
  if (stage + sl.total > 0) {
    if (!workspace || workspace_bytes < stage + sl.total) return RESS_ERR_WORKSPACE;
    if (reinterpret_cast<uintptr_t>(workspace) & 255u) return RESS_ERR_INVALID_ARG;
  }
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  if ((s = stage_inputs(g, q, k, v, workspace, workspace_bytes, st)) != RESS_OK) return s;
  if ((s = launch_attn(g, q, k, v, budget, idx, out, out_dtype == RESS_F32, lse, st)) != RESS_OK)
    return s;
  return launch_special_rows(g, q, k, v, out, out_dtype == RESS_F32, lse,
                             static_cast<uint8_t*>(workspace) + stage, st);
}

namespace {
ress_status drift_checked(Geometry& g, const ress_shape* shape, const void* q, const void* k,
                          const void* v, int32_t budget, const int32_t* idx, const float* lse,
                          float* drift, float* set_drift, void* workspace, size_t workspace_bytes,
                          void* stream);
}  // namespace

ress_status ress_block_drift(const ress_shape* shape, const void* q, const void* k,
                             const void* v, int32_t budget, const int32_t* idx,
                             const float* lse, float* drift, float* set_drift,
                             void* workspace, size_t workspace_bytes, void* stream) {
  Geometry g;
  ress_status s = check_shape(shape, &g);
  if (s != RESS_OK) return s;
  return drift_checked(g, shape, q, k, v, budget, idx, lse, drift, set_drift, workspace,
                       workspace_bytes, stream);
}

ress_status ress_block_drift_layout(const ress_shape* shape, const ress_layout* layout,
                                    const void* q, const void* k, const void* v, int32_t budget,
                                    const int32_t* idx, const float* lse, float* drift,
                                    float* set_drift, void* workspace, size_t workspace_bytes,
                                    void* stream) {
  Geometry g;
  ress_status s = check_shape(shape, &g);
  if (s != RESS_OK) return s;
  if ((s = check_layout(layout, &g)) != RESS_OK) return s;
  return drift_checked(g, shape, q, k, v, budget, idx, lse, drift, set_drift, workspace,
                       workspace_bytes, stream);
}

namespace {
ress_status drift_checked(Geometry& g, const ress_shape* shape, const void* q, const void* k,
                          const void* v, int32_t budget, const int32_t* idx, const float* lse,
                          float* drift, float* set_drift, void* workspace, size_t workspace_bytes,
                          void* stream) {
  ress_status s;
  if ((s = check_budget(g, budget)) != RESS_OK) return s;
  if (g.nb == 0) return RESS_OK;
  if (!q || !k || !v || !idx || !lse || (budget < g.nb && !drift)) return RESS_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) ||
      (reinterpret_cast<uintptr_t>(idx) & 3u) || (reinterpret_cast<uintptr_t>(lse) & 3u) ||
      (reinterpret_cast<uintptr_t>(drift) & 3u) || (reinterpret_cast<uintptr_t>(set_drift) & 3u))
    return RESS_ERR_INVALID_ARG;
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (g.f32 && (!workspace || workspace_bytes < ress_attn_workspace_bytes(shape)))
    return RESS_ERR_WORKSPACE;
  if ((s = stage_inputs(g, q, k, v, workspace, workspace_bytes, st)) != RESS_OK) return s;
  return launch_drift(g, q, k, v, budget, idx, lse, drift, set_drift, st);
}
}  // namespace

ress_status ress_validate_idx(const ress_shape* shape, int32_t budget, const int32_t* idx,
                              void* stream) {
  Geometry g;
  ress_status s = check_shape(shape, &g);
  if (s != RESS_OK) return s;
  if ((s = check_budget(g, budget)) != RESS_OK) return s;
  if (g.nb == 0) return RESS_OK;
  if (!idx || (reinterpret_cast<uintptr_t>(idx) & 3u)) return RESS_ERR_INVALID_ARG;
  DeviceError* err = device_error_ptr();
  if (err == nullptr) return RESS_ERR_CUDA;
  const int rows = g.heads * g.nb;
  validate_idx_kernel<<<(rows + 7) / 8, 256, 0, static_cast<cudaStream_t>(stream)>>>(
      idx, rows, g.nb, budget, err);
  return record_cuda(cudaGetLastError());
}

ress_status ress_check_device_errors(void* stream, int32_t* detail) {
  if (detail) *detail = 0;
  if (ress_status s = record_cuda(cudaStreamSynchronize(static_cast<cudaStream_t>(stream))))
    return s;
  DeviceError e{0, 0};
  if (ress_status s = record_cuda(cudaMemcpyFromSymbol(&e, g_device_error, sizeof(e)))) return s;
  if (e.code != 0) {
    const DeviceError zero{0, 0};
    if (ress_status s = record_cuda(cudaMemcpyToSymbol(g_device_error, &zero, sizeof(zero))))
      return s;
  }
  if (detail) *detail = e.detail;
  return static_cast<ress_status>(e.code);
}

const char* ress_last_cuda_error(void) { return g_last_cuda_error; }

ress_status ress_test_exp2(const float* x, float* y, int32_t n, void* stream) {
  if (n < 0 || (n > 0 && (!x || !y))) return RESS_ERR_INVALID_ARG;
  return launch_exp2_poly_test(x, y, n, static_cast<cudaStream_t>(stream));
}

}  // extern "C"
