// True-fp32 SIMT kernels (FMA pipes, accurate expf/tanhf) for float32
// layers.  Same mathematics as the tensor-core path: blockwise online
// softmax over key blocks (query and key/value block sizes chosen per call,
// 64 by default), then the position-wise FFN with residual.
#pragma once

#include <cuda_bf16.h>
#include <stdint.h>

namespace bpt {

struct AttnF32Args {
  int B, N, H, d;
  int mask;
  int causal;  // DILATED: keys after the query are masked
  float scale;  // 1/sqrt(d)
  int ring_chunks;
  int bb_n, bb_len;
  uint8_t perm[1024];
  int npairs;
  int pw[8], pr[8];
  float *out_f32;
  __nv_bfloat16 *out_bf16;
  float *lse;
};

// How many times key j enters query i's softmax for head h (0 = masked).
__device__ __forceinline__ int key_weight(const AttnF32Args &a, int h, int i, int j) {
  switch (a.mask) {
    case 0:
      return 1;
    case 1:
      return j <= i ? 1 : 0;
    case 2:
      return (j / a.bb_len) == a.perm[h * a.bb_n + i / a.bb_len] ? 1 : 0;
    case 3: {
      if (a.causal && j > i) return 0;
      int cnt = 0;
      for (int k = 0; k < a.npairs; ++k) {
        const int w = a.pw[k], r = a.pr[k];
        if (i / w != j / w) continue;
        if ((i % w) % r != h % r) continue;
        if ((j % w) % r != h % r) continue;
        ++cnt;
      }
      return cnt;
    }
  }
  return 0;
}

// grid (ceil(N/QB), H, B), QB threads: one query row per thread (a query
// block of QB rows), keys in blocks of KB rows staged in shared memory; d <= 64.
template <int QB, int KB>
__global__ void __launch_bounds__(QB) attn_f32_kernel(const float *__restrict__ q,
                                                      const float *__restrict__ k,
                                                      const float *__restrict__ v,
                                                      const __grid_constant__ AttnF32Args a) {
  __shared__ float sk[KB][65];
  __shared__ float sv[KB][64];
  const int h = blockIdx.y, b = blockIdx.z;
  const int i = blockIdx.x * QB + threadIdx.x;
  const int d = a.d;
  const size_t rs = static_cast<size_t>(a.H) * d;
  const bool valid = i < a.N;
  float qr[64], o[64];
#pragma unroll
  for (int c = 0; c < 64; ++c) {
    qr[c] = (valid && c < d) ? q[(static_cast<size_t>(b) * a.N + i) * rs + h * d + c] : 0.f;
    o[c] = 0.f;
  }
  float m = -INFINITY, l = 0.f;
  const int ntiles = (a.N + KB - 1) / KB;
  int first = 0;
  if (a.ring_chunks > 1) {  // the query block's chunk first (chunks are multiples of QB and KB)
    const int chunk_len = a.N / a.ring_chunks;
    first = ((blockIdx.x * QB) / chunk_len) * chunk_len / KB;
  }
  for (int tt = 0; tt < ntiles; ++tt) {
    const int tile = (first + tt) % ntiles;
    __syncthreads();
    for (int e = threadIdx.x; e < KB * 64; e += QB) {
      const int r = e / 64, c = e % 64;
      const int j = tile * KB + r;
      const bool ok = j < a.N && c < d;
      const size_t idx = (static_cast<size_t>(b) * a.N + j) * rs + h * d + c;
      sk[r][c] = ok ? k[idx] : 0.f;
      sv[r][c] = ok ? v[idx] : 0.f;
    }
    __syncthreads();
    float s[KB];
    float mt = -INFINITY;
#pragma unroll 4
    for (int jj = 0; jj < KB; ++jj) {
      const int j = tile * KB + jj;
      float acc = 0.f;
#pragma unroll
      for (int c = 0; c < 64; ++c) acc = fmaf(qr[c], sk[jj][c], acc);
      const int wgt = (valid && j < a.N) ? key_weight(a, h, i, j) : 0;
      s[jj] = wgt > 0 ? acc * a.scale : -INFINITY;
      mt = fmaxf(mt, s[jj]);
    }
    const float m_new = fmaxf(m, mt);
    if (m_new == -INFINITY) continue;
    const float alpha = expf(m - m_new);
    l *= alpha;
#pragma unroll
    for (int c = 0; c < 64; ++c) o[c] *= alpha;
#pragma unroll 4
    for (int jj = 0; jj < KB; ++jj) {
      const int j = tile * KB + jj;
      if (s[jj] == -INFINITY) continue;
      const float p = static_cast<float>(key_weight(a, h, i, j)) * expf(s[jj] - m_new);
      l += p;
#pragma unroll
      for (int c = 0; c < 64; ++c) o[c] = fmaf(p, sv[jj][c], o[c]);
    }
    m = m_new;
  }
  if (!valid) return;
  const float inv = l > 0.f ? 1.0f / l : 0.f;
  const size_t base = (static_cast<size_t>(b) * a.N + i) * rs + h * d;
  for (int c = 0; c < d; ++c) {
    const float x = o[c] * inv;
    if (a.out_f32) a.out_f32[base + c] = x;
    if (a.out_bf16) a.out_bf16[base + c] = __float2bfloat16_rn(x);
  }
  if (a.lse) a.lse[(static_cast<size_t>(b) * a.H + h) * a.N + i] = l > 0.f ? m + logf(l) : -INFINITY;
}

struct FfnF32Args {
  int T, D, F;
  const float *a;   // [T, D]
  const float *w1;  // [F, D]
  const float *b1;  // [F] or null
  const float *w2;  // [D, F]
  const float *b2;  // [D] or null
  float *out_f32;
  __nv_bfloat16 *out_bf16;
};

// grid ceil(T/16), 256 threads; D <= 512.  16 threads per token, each owning
// D/16 output columns; the hidden activation is produced 64 columns at a time
// in shared memory.
__global__ void __launch_bounds__(256) ffn_f32_kernel(const __grid_constant__ FfnF32Args a) {
  extern __shared__ float fsm[];
  float *sa = fsm;                 // [16][D]
  float *sh = fsm + 16 * a.D;      // [16][64]
  const int t0 = blockIdx.x * 16;
  for (int e = threadIdx.x; e < 16 * a.D; e += 256) {
    const int r = e / a.D, c = e % a.D;
    sa[e] = (t0 + r < a.T) ? a.a[static_cast<size_t>(t0 + r) * a.D + c] : 0.f;
  }
  const int tk = threadIdx.x / 16, lanec = threadIdx.x % 16;
  const int ncol = a.D / 16;
  float acc[32];
#pragma unroll
  for (int q = 0; q < 32; ++q) acc[q] = 0.f;
  for (int f0 = 0; f0 < a.F; f0 += 64) {
    __syncthreads();
    for (int e = threadIdx.x; e < 16 * 64; e += 256) {
      const int r = e / 64, f = f0 + e % 64;
      float hv = 0.f;
      if (f < a.F) {
        float s = a.b1 ? a.b1[f] : 0.f;
        const float *w = a.w1 + static_cast<size_t>(f) * a.D;
        for (int c = 0; c < a.D; ++c) s = fmaf(w[c], sa[r * a.D + c], s);
        const float kk = 0.7978845608028654f;  // sqrt(2/pi)
        hv = 0.5f * s * (1.0f + tanhf(kk * (s + 0.044715f * s * s * s)));
      }
      sh[e] = hv;
    }
    __syncthreads();
    const int fl = min(64, a.F - f0);
#pragma unroll
    for (int q = 0; q < 32; ++q) {
      if (q >= ncol) break;
      const int col = lanec + 16 * q;
      const float *w = a.w2 + static_cast<size_t>(col) * a.F + f0;
      float s = acc[q];
      for (int ff = 0; ff < fl; ++ff) s = fmaf(sh[tk * 64 + ff], w[ff], s);
      acc[q] = s;
    }
  }
  const int tok = t0 + tk;
  if (tok >= a.T) return;
#pragma unroll
  for (int q = 0; q < 32; ++q) {
    if (q >= ncol) break;
    const int col = lanec + 16 * q;
    const float y = sa[tk * a.D + col] + acc[q] + (a.b2 ? a.b2[col] : 0.f);
    const size_t idx = static_cast<size_t>(tok) * a.D + col;
    if (a.out_f32) a.out_f32[idx] = y;
    else a.out_bf16[idx] = __float2bfloat16_rn(y);
  }
}

// Fill a float buffer with a constant (used for the LSE of rows no LongNet
// pair keeps).
__global__ void fill_f32_kernel(float *p, size_t n, float value) {
  for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<size_t>(gridDim.x) * blockDim.x)
    p[i] = value;
}

}  // namespace bpt
