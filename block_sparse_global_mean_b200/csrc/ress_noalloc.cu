// Block selection for callers that cannot allocate device memory.
//
// ress_select_blocks takes its scratch (pooled Q, K and V, value contrast)
// from a caller-provided workspace.  Some callers cannot obtain one: a plugin
// that runs inside another framework and must not call cudaMalloc behind that
// framework's allocator, or a latency-critical loop in which an allocation
// (which may synchronise the device) is not allowed.  This entry point runs
// the same selection kernels with their scratch in a fixed array in device
// global memory that the library owns.  The array occupies
// kStaticScratchBytes on every GPU that loads the library, until the process
// exits.
#include "ress_internal.h"

#include <mutex>

namespace ress {
namespace {

// 32 MiB: enough for H = 16 heads and nb <= 2,200 blocks with the value
// contrast (100 or 200 views of 1,408 tokens at block 64 / 128).
constexpr size_t kStaticScratchBytes = size_t(32) << 20;

static __device__ __align__(256) unsigned char g_select_scratch[kStaticScratchBytes];

// Device address of g_select_scratch on the current device.  In host code the
// symbol itself is only a host-side stand-in, so the address is looked up once
// per device, with that device current, and cached.
void* static_scratch_address() {
  static void* cache[64] = {};
  static std::mutex mu;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> lock(mu);
  if (cache[dev] == nullptr) {
    void* ptr = nullptr;
    if (record_cuda(cudaGetSymbolAddress(&ptr, g_select_scratch)) != RESS_OK) return nullptr;
    cache[dev] = ptr;
  }
  return cache[dev];
}

}  // namespace
}  // namespace ress

extern "C" ress_status ress_select_blocks_noalloc(const ress_shape* shape, const void* q,
                                                  const void* k, const void* v, int32_t budget,
                                                  float lambda, int32_t* idx, void* stream) {
  // Argument checks first, with no CUDA call: the workspace entry point checks
  // everything else before the workspace size, so a non-null, aligned
  // placeholder with zero bytes yields RESS_ERR_WORKSPACE exactly when all the
  // other arguments are valid (or RESS_OK for an empty input, with no launch).
  const ress_status pre = ress_select_blocks(shape, q, k, v, budget, lambda, idx,
                                             reinterpret_cast<void*>(uintptr_t(256)), 0, stream);
  if (pre != RESS_ERR_WORKSPACE) return pre;
  if (ress_select_workspace_bytes(shape, lambda) > ress::kStaticScratchBytes)
    return RESS_ERR_WORKSPACE;   // the problem needs more scratch than the fixed array holds
  void* scratch = ress::static_scratch_address();
  if (scratch == nullptr) return RESS_ERR_CUDA;
  return ress_select_blocks(shape, q, k, v, budget, lambda, idx, scratch,
                            ress::kStaticScratchBytes, stream);
}
