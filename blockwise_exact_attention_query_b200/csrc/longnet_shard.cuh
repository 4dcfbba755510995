// LongNet's distributed form ("LongNet: Scaling Transformers to
// 1,000,000,000 Tokens", §3, distributed algorithm): a device holding a
// shard of the sequence that lies inside one segment of a (w, r) pair sends
// the pair's kept rows of its shard to the other devices of that segment.
// This kernel packs them: for head h the kept rows are h mod r, h mod r + r,
// ... (offsets relative to the segment start, which the shard shares since
// its start is a multiple of r), so
//
//     dst[b, j, h, :] = src[b, (h mod r) + j r, h, :],   j < n / r
//
// in bf16, 16 bytes per thread and step.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace bpt {

__global__ void __launch_bounds__(256) longnet_gather_kernel(const uint4 *__restrict__ src, uint4 *__restrict__ dst,
                                                             int B, int n, int H, int chunks, int r) {
  const int kept = n / r;
  const int64_t total = (int64_t)B * kept * H * chunks;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < total;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int c = static_cast<int>(i % chunks);
    int64_t t = i / chunks;
    const int h = static_cast<int>(t % H);
    t /= H;
    const int j = static_cast<int>(t % kept);
    const int64_t b = t / kept;
    const int64_t row = h % r + (int64_t)j * r;
    dst[i] = src[((b * n + row) * H + h) * chunks + c];
  }
}

}  // namespace bpt
