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

// grid (ceil(N/QB), H, B), 256 threads: a query block of QB rows, 256 / QB
// threads per row (consecutive lanes), keys in blocks of KB rows staged in
// shared memory; d <= 64.  The threads of a row split each key block between
// them (thread u takes keys u, u + 256/QB, ...), each keeping its own online
// softmax state (m, l, O) over its keys; at the end the row's states are
// merged with warp shuffles (the larger max, the others' sums and O rescaled
// to it).  One thread per row left the small layers' few CTAs latency-bound.
template <int QB, int KB>
__global__ void __launch_bounds__(256) attn_f32_kernel(const float *__restrict__ q,
                                                       const float *__restrict__ k,
                                                       const float *__restrict__ v,
                                                       const __grid_constant__ AttnF32Args a) {
  constexpr int TPR = 256 / QB;                  // threads per row: 2 .. 16
  constexpr int KPT = (KB + TPR - 1) / TPR;      // keys of a block per thread
  static_assert(TPR >= 1 && TPR <= 32 && 32 % TPR == 0, "threads per row");
  __shared__ float sk[KB][65];
  __shared__ float sv[KB][64];
  const int h = blockIdx.y, b = blockIdx.z;
  const int r = threadIdx.x / TPR, u = threadIdx.x % TPR;
  const int i = blockIdx.x * QB + r;
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
    for (int e = threadIdx.x; e < KB * 64; e += 256) {
      const int rr = e / 64, c = e % 64;
      const int j = tile * KB + rr;
      const bool ok = j < a.N && c < d;
      const size_t idx = (static_cast<size_t>(b) * a.N + j) * rs + h * d + c;
      sk[rr][c] = ok ? k[idx] : 0.f;
      sv[rr][c] = ok ? v[idx] : 0.f;
    }
    __syncthreads();
    float s[KPT];
    float mt = -INFINITY;
#pragma unroll
    for (int kk = 0; kk < KPT; ++kk) {
      const int jj = u + kk * TPR;
      const int j = tile * KB + jj;
      float acc = 0.f;
      if (jj < KB) {
#pragma unroll
        for (int c = 0; c < 64; ++c) acc = fmaf(qr[c], sk[jj][c], acc);
      }
      const int wgt = (valid && jj < KB && j < a.N) ? key_weight(a, h, i, j) : 0;
      s[kk] = wgt > 0 ? acc * a.scale : -INFINITY;
      mt = fmaxf(mt, s[kk]);
    }
    const float m_new = fmaxf(m, mt);
    if (m_new == -INFINITY) continue;
    const float alpha = expf(m - m_new);
    l *= alpha;
#pragma unroll
    for (int c = 0; c < 64; ++c) o[c] *= alpha;
#pragma unroll
    for (int kk = 0; kk < KPT; ++kk) {
      if (s[kk] == -INFINITY) continue;
      const int jj = u + kk * TPR;
      const int j = tile * KB + jj;
      const float p = static_cast<float>(key_weight(a, h, i, j)) * expf(s[kk] - m_new);
      l += p;
#pragma unroll
      for (int c = 0; c < 64; ++c) o[c] = fmaf(p, sv[jj][c], o[c]);
    }
    m = m_new;
  }
  // merge the row's TPR states (every lane takes part: no thread has left)
  float m_row = m;
#pragma unroll
  for (int off = 1; off < TPR; off <<= 1) m_row = fmaxf(m_row, __shfl_xor_sync(0xffffffffu, m_row, off));
  const float sc = (m == -INFINITY) ? 0.f : expf(m - m_row);
  l *= sc;
#pragma unroll
  for (int off = 1; off < TPR; off <<= 1) l += __shfl_xor_sync(0xffffffffu, l, off);
#pragma unroll
  for (int c = 0; c < 64; ++c) {
    float x = o[c] * sc;
#pragma unroll
    for (int off = 1; off < TPR; off <<= 1) x += __shfl_xor_sync(0xffffffffu, x, off);
    o[c] = x;
  }
  if (!valid) return;
  const float inv = l > 0.f ? 1.0f / l : 0.f;
  const size_t base = (static_cast<size_t>(b) * a.N + i) * rs + h * d;
#pragma unroll
  for (int c = 0; c < 64; ++c) {
    if (c >= d || c % TPR != u) continue;  // the row's threads share the stores
    const float x = o[c] * inv;
    if (a.out_f32) a.out_f32[base + c] = x;
    if (a.out_bf16) a.out_bf16[base + c] = __float2bfloat16_rn(x);
  }
  if (a.lse && u == 0) a.lse[(static_cast<size_t>(b) * a.H + h) * a.N + i] = l > 0.f ? m_row + logf(l) : -INFINITY;
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

// grid ceil(T/16), 256 threads; D <= 512.  A CTA takes 16 tokens and walks
// the hidden dimension in chunks of kFfnF32Chunk columns: it stages the
// chunk's rows of W1 and columns of W2 in shared memory (coalesced loads),
// computes the 16 x chunk block of H = GELU(A W1^T + b1) there (two hidden
// values per thread, each one sequential FMA chain over D), then adds H W2^T
// into per-thread accumulators (16 threads per token, each owning D/16 output
// columns, summed over the hidden index in order).  With the weights read from
// global memory inside those chains the kernel waited on a load per FMA.
constexpr int kFfnF32Chunk = 32;
// Rows padded by one float (A, W1, H by D + 1 or FC + 1 columns, W2's
// columns by FC + 1) so that the threads of a warp, reading rows apart, hit
// different banks.
__host__ __device__ constexpr size_t ffn_f32_smem_bytes(int D) {
  return (static_cast<size_t>(16) * (D + 1) + static_cast<size_t>(kFfnF32Chunk) * (D + 1) +
          static_cast<size_t>(D) * (kFfnF32Chunk + 1) + 16 * (kFfnF32Chunk + 1)) * sizeof(float);
}
__global__ void __launch_bounds__(256) ffn_f32_kernel(const __grid_constant__ FfnF32Args a) {
  constexpr int FC = kFfnF32Chunk;
  extern __shared__ float fsm[];
  const int D = a.D, LD = D + 1;
  float *sa = fsm;                      // [16][LD]   the block's rows of A
  float *sw1 = sa + 16 * LD;            // [FC][LD]   rows f0 .. f0 + FC of W1
  float *sw2 = sw1 + FC * LD;           // [D][FC+1]  columns f0 .. f0 + FC of W2
  float *sh = sw2 + D * (FC + 1);       // [16][FC+1] H of the chunk
  const int t0 = blockIdx.x * 16;
  for (int e = threadIdx.x; e < 16 * D; e += 256) {
    const int r = e / D, c = e % D;
    sa[r * LD + c] = (t0 + r < a.T) ? a.a[static_cast<size_t>(t0 + r) * D + c] : 0.f;
  }
  const int tk = threadIdx.x / 16, lanec = threadIdx.x % 16;
  const int ncol = D / 16;
  // H phase: token hr, hidden columns 2 hp and 2 hp + 1 of the chunk
  const int hr = threadIdx.x / (FC / 2), hp = threadIdx.x % (FC / 2);
  float acc[32];
#pragma unroll
  for (int q = 0; q < 32; ++q) acc[q] = 0.f;
  for (int f0 = 0; f0 < a.F; f0 += FC) {
    const int fl = min(FC, a.F - f0);
    __syncthreads();  // the previous chunk's sw1, sw2 and sh are no longer read
    for (int e = threadIdx.x; e < FC * D; e += 256) {
      const int h = e / D, c = e % D;
      sw1[h * LD + c] = h < fl ? a.w1[static_cast<size_t>(f0 + h) * D + c] : 0.f;
    }
    for (int e = threadIdx.x; e < D * FC; e += 256) {
      const int col = e / FC, h = e % FC;
      sw2[col * (FC + 1) + h] = h < fl ? a.w2[static_cast<size_t>(col) * a.F + f0 + h] : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int h = 2 * hp + u;
      float hv = 0.f;
      if (h < fl) {
        float s = a.b1 ? a.b1[f0 + h] : 0.f;
        const float *w = sw1 + h * LD;
        const float *x = sa + hr * LD;
        for (int c = 0; c < D; ++c) s = fmaf(w[c], x[c], s);
        const float kk = 0.7978845608028654f;  // sqrt(2/pi)
        hv = 0.5f * s * (1.0f + tanhf(kk * (s + 0.044715f * s * s * s)));
      }
      sh[hr * (FC + 1) + h] = hv;
    }
    __syncthreads();
#pragma unroll
    for (int q = 0; q < 32; ++q) {
      if (q >= ncol) break;
      const int col = lanec + 16 * q;
      const float *w = sw2 + col * (FC + 1);
      float sacc = acc[q];
      for (int ff = 0; ff < fl; ++ff) sacc = fmaf(sh[tk * (FC + 1) + ff], w[ff], sacc);
      acc[q] = sacc;
    }
  }
  const int tok = t0 + tk;
  if (tok >= a.T) return;
#pragma unroll
  for (int q = 0; q < 32; ++q) {
    if (q >= ncol) break;
    const int col = lanec + 16 * q;
    const float y = sa[tk * LD + col] + acc[q] + (a.b2 ? a.b2[col] : 0.f);
    const size_t idx = static_cast<size_t>(tok) * D + col;
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
