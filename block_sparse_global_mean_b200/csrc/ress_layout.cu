// Layout-aware attention and drift: padding and the special (camera,
// register) tokens of every view.
//
// Source: VASC (paperlayer.ai) 4.2 and A.5: camera and register queries keep
// dense attention, key blocks made only of special tokens are always kept,
// and the selection's mask is otherwise passed to the sparse kernel as is;
// padding (the tokens that round a 1,374-token view up to a whole number of
// blocks) takes part in nothing.
//
//   - The sparse pass runs every query row against its kept blocks with the
//     padding keys masked (each block's valid tokens are a prefix of it,
//     since a view is a whole number of blocks); padding queries write 0
//     and lse -inf.
//   - The special queries of all views are gathered into a compact [Ns][H][64]
//     array, attend densely to every valid key (the same kernel, every key
//     block kept), and their rows are scattered over the sparse pass's.
//   - Drift counts only the valid non-special queries and the valid keys.
#include "ress_common.cuh"
#include "ress_internal.h"

namespace ress {

namespace {

// dst[r][h][:] = q[(r / S) * T + r % S][h][:] for r < V * S, zero rows up to
// rows_pad.  One 16-byte word per thread.
__global__ void gather_special_kernel(const uint4* __restrict__ q, uint4* __restrict__ dst,
                                      int words_per_row, int t, int sp, int views, int rows_pad) {
  const size_t total = (size_t)rows_pad * words_per_row;
  for (size_t e = blockIdx.x * (size_t)blockDim.x + threadIdx.x; e < total;
       e += (size_t)gridDim.x * blockDim.x) {
    const int r = (int)(e / words_per_row);
    const int w = (int)(e - (size_t)r * words_per_row);
    uint4 v = make_uint4(0u, 0u, 0u, 0u);
    if (r < views * sp) v = q[((size_t)(r / sp) * t + r % sp) * words_per_row + w];
    dst[e] = v;
  }
}

// out rows of the special tokens <- the dense pass's rows; lse likewise.
__global__ void scatter_special_kernel(const uint4* __restrict__ src, uint4* __restrict__ out,
                                       const float* __restrict__ lse_src, float* __restrict__ lse,
                                       int words_per_row, int heads, int64_t n, int rows_pad, int t,
                                       int sp, int views) {
  const int rows = views * sp;
  const size_t total = (size_t)rows * words_per_row;
  for (size_t e = blockIdx.x * (size_t)blockDim.x + threadIdx.x; e < total;
       e += (size_t)gridDim.x * blockDim.x) {
    const int r = (int)(e / words_per_row);
    const int w = (int)(e - (size_t)r * words_per_row);
    out[((size_t)(r / sp) * t + r % sp) * words_per_row + w] = src[e];
  }
  if (lse != nullptr) {
    for (size_t e = blockIdx.x * (size_t)blockDim.x + threadIdx.x; e < (size_t)heads * rows;
         e += (size_t)gridDim.x * blockDim.x) {
      const int h = (int)(e / rows);
      const int r = (int)(e - (size_t)h * rows);
      lse[(size_t)h * n + (size_t)(r / sp) * t + r % sp] = lse_src[(size_t)h * rows_pad + r];
    }
  }
}

unsigned grid_for(size_t items) {
  const size_t b = (items + 255) / 256;
  return (unsigned)(b < 148 * 8 ? (b > 0 ? b : 1) : 148 * 8);
}

}  // namespace

SpecialLayout special_layout(const Geometry& g, bool out_f32) {
  SpecialLayout l{};
  const int views = g.lay_t > 0 ? (int)(g.n / g.lay_t) : 0;
  l.rows = (int64_t)views * g.lay_s;
  l.rows_pad = (l.rows + 127) / 128 * 128;
  size_t off = 0;
  l.q = off;
  off += align256((size_t)l.rows_pad * g.heads * kHeadDim * 2);
  l.out = off;
  off += align256((size_t)l.rows_pad * g.heads * kHeadDim * (out_f32 ? 4 : 2));
  l.lse = off;
  off += align256((size_t)l.rows_pad * g.heads * 4);
  l.total = l.rows > 0 ? off : 0;
  return l;
}

ress_status launch_special_rows(const Geometry& g, const void* q, const void* k, const void* v,
                                void* out, bool out_f32, float* lse, uint8_t* ws,
                                cudaStream_t st) {
  const SpecialLayout l = special_layout(g, out_f32);
  if (l.rows == 0) return RESS_OK;
  const int views = (int)(g.n / g.lay_t);
  const int qwords = g.heads * kHeadDim * 2 / 16;
  gather_special_kernel<<<grid_for((size_t)l.rows_pad * qwords), 256, 0, st>>>(
      static_cast<const uint4*>(q), reinterpret_cast<uint4*>(ws + l.q), qwords, g.lay_t, g.lay_s,
      views, (int)l.rows_pad);
  if (ress_status s = record_cuda(cudaGetLastError())) return s;
  float* lse_s = reinterpret_cast<float*>(ws + l.lse);
  if (ress_status s = launch_attn_rows(g, ws + l.q, l.rows_pad, true, k, v, 1, nullptr,
                                       ws + l.out, out_f32, lse_s, st))
    return s;
  const int owords = g.heads * kHeadDim * (out_f32 ? 4 : 2) / 16;
  scatter_special_kernel<<<grid_for((size_t)l.rows * owords), 256, 0, st>>>(
      reinterpret_cast<const uint4*>(ws + l.out), static_cast<uint4*>(out), lse_s, lse, owords,
      g.heads, g.n, (int)l.rows_pad, g.lay_t, g.lay_s, views);
  return record_cuda(cudaGetLastError());
}

}  // namespace ress
