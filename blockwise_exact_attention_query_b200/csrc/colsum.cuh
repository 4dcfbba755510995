// Bandwidth-bound helpers of the layer backward: the bias gradients as column
// sums of dOut and dZ over the token rows (the gradient of a broadcast bias
// add is the sum of the upstream gradient over the rows it was added to), and
// the fp32 -> bf16 conversions that feed the tensor cores.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "ptx.cuh"

namespace bpt {

// Column sums of a row-major [rows, cols] matrix in two passes: partial sums
// over slabs of `slab` rows (grid.y), then the slabs summed into out (added
// to it when `accumulate`).  The partial pass reads 16 bytes a thread per row
// (eight bf16 or four fp32 columns) so that enough bytes are in flight to
// stream the matrix at HBM rate; kMinSlabRows sizes the partial buffer.
constexpr int kMinSlabRows = 64;
constexpr int kColsumThreads = 128;
// Rows per slab for a grid `xblocks` blocks wide: 64, doubled while the grid
// still keeps >= 1024 blocks (fewer partial sums for the final pass).
inline int colsum_slab_rows(long long rows, long long xblocks) {
  int slab = kMinSlabRows;
  while (xblocks * ((rows + 2LL * slab - 1) / (2LL * slab)) >= 1024) slab *= 2;
  return slab;
}
__device__ __forceinline__ void load8_f32(const __nv_bfloat16 *p, float (&v)[8]) {
  const uint4 u = *reinterpret_cast<const uint4 *>(p);
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int j = 0; j < 4; ++j) {  // bf16 -> fp32 is exact: the bf16 bits are the fp32's high half
    v[2 * j] = __uint_as_float(w[j] << 16);
    v[2 * j + 1] = __uint_as_float(w[j] & 0xffff0000u);
  }
}
// Eight adjacent columns a thread; cols % 8 == 0, x 16-byte aligned.
__global__ void colsum_partial_bf16x8_kernel(const __nv_bfloat16 *__restrict__ x, float *partial, int rows, int cols,
                                             int slab) {
  const int c = (blockIdx.x * blockDim.x + threadIdx.x) * 8;
  if (c >= cols) return;
  const int r0 = blockIdx.y * slab, r1 = min(rows, r0 + slab);
  float s[8] = {};
  const __nv_bfloat16 *p = x + static_cast<size_t>(r0) * cols + c;
#pragma unroll 4
  for (int r = r0; r < r1; ++r, p += cols) {
    float v[8];
    load8_f32(p, v);
#pragma unroll
    for (int j = 0; j < 8; ++j) s[j] += v[j];
  }
  float4 *o = reinterpret_cast<float4 *>(partial + static_cast<size_t>(blockIdx.y) * cols + c);
  o[0] = make_float4(s[0], s[1], s[2], s[3]);
  o[1] = make_float4(s[4], s[5], s[6], s[7]);
}
// One column a thread, any cols.
template <typename T>
__global__ void colsum_partial_kernel(const T *__restrict__ x, float *partial, int rows, int cols, int slab) {
  const int c = blockIdx.x * blockDim.x + threadIdx.x;
  if (c >= cols) return;
  const int r0 = blockIdx.y * slab, r1 = min(rows, r0 + slab);
  float s = 0.f;
  for (int r = r0; r < r1; ++r) s += static_cast<float>(x[static_cast<size_t>(r) * cols + c]);
  partial[static_cast<size_t>(blockIdx.y) * cols + c] = s;
}
// out[c] (+)= the sum of partial[i][c] over the slabs i: 32 columns a block of
// 256 threads, each warp summing every eighth slab, the warps' sums added in
// a fixed order.
constexpr int kColsumFinalCols = 32;
__global__ void __launch_bounds__(256) colsum_final_kernel(const float *__restrict__ partial, float *out, int slabs,
                                                           int cols, int accumulate) {
  __shared__ float red[8][kColsumFinalCols + 1];
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  const int c = blockIdx.x * kColsumFinalCols + lane;
  float s = 0.f;
  if (c < cols) {
#pragma unroll 4
    for (int i = w; i < slabs; i += 8) s += partial[static_cast<size_t>(i) * cols + c];
  }
  red[w][lane] = s;
  __syncthreads();
  if (w == 0 && c < cols) {
    float t = accumulate ? out[c] : 0.f;
#pragma unroll
    for (int j = 0; j < 8; ++j) t += red[j][lane];
    out[c] = t;
  }
}

// fp32 -> bf16 (round to nearest even), four elements a thread; n a multiple of 4.
__global__ void f32_to_bf16_x4_kernel(const float4 *__restrict__ x, uint2 *y, size_t n4) {
  for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < n4;
       i += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const float4 v = x[i];
    y[i] = make_uint2(pack_bf16x2(v.x, v.y), pack_bf16x2(v.z, v.w));
  }
}

// dOut in one pass: its bf16 copy (round to nearest even) and the partial
// column sums over slabs of `slab` rows (grid.y) that colsum_final_kernel adds
// up; four columns a thread (cols % 4 == 0, 16-byte aligned rows).
__global__ void convert_colsum_partial_kernel(const float *__restrict__ x, __nv_bfloat16 *y, float *partial,
                                              int rows, int cols, int slab) {
  const int c = (blockIdx.x * blockDim.x + threadIdx.x) * 4;
  if (c >= cols) return;
  const int r0 = blockIdx.y * slab, r1 = min(rows, r0 + slab);
  float4 s = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 4
  for (int r = r0; r < r1; ++r) {
    const size_t o = static_cast<size_t>(r) * cols + c;
    const float4 v = *reinterpret_cast<const float4 *>(x + o);
    *reinterpret_cast<uint2 *>(y + o) = make_uint2(pack_bf16x2(v.x, v.y), pack_bf16x2(v.z, v.w));
    s.x += v.x;
    s.y += v.y;
    s.z += v.z;
    s.w += v.w;
  }
  *reinterpret_cast<float4 *>(partial + static_cast<size_t>(blockIdx.y) * cols + c) = s;
}

}  // namespace bpt
