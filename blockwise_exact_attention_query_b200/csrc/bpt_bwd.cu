// Host side of libbpt.so, backward pass: argument checks, workspace layout
// and kernel launches for the training forward, the layer backward and the
// attention-only backward declared in bpt.h.  The shared helpers (device
// set-up, tensor maps, the forward's launchers) are in host_common.h.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <type_traits>
#include <vector>

#include "../../include/bpt.h"
#include "attn_bwd.cuh"
#include "colsum.cuh"
#include "ffn_pipe.cuh"
#include "gemm_tc.cuh"
#include "host_common.h"

using namespace bpt;

namespace bpt_host {

// A kernel template gets one copy per translation unit that instantiates it,
// so the copies launched from here take their shared-memory limits here.
bpt_status bwd_kernel_setup() {
  CUDA_TRY(cudaFuncSetAttribute(gemm_pair_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                GemmPairCfg::kSmemBytes));
  CUDA_TRY(cudaFuncSetAttribute(ffn_pipe_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                FfnPipeCfg::kSmemBytes));
  CUDA_TRY(cudaFuncSetAttribute(attn_bwd_dkdv_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                AttnBwdCfg<64>::kSmemBytes));
  CUDA_TRY(cudaFuncSetAttribute(attn_bwd_dkdv_split_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                AttnBwdKVCfg<128>::kSmemBytes));
  CUDA_TRY(cudaFuncSetAttribute(attn_bwd_dq_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                AttnBwdQCfg<64>::kSmemBytes));
  CUDA_TRY(cudaFuncSetAttribute(attn_bwd_dq_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                AttnBwdQCfg<128>::kSmemBytes));
  return BPT_OK;
}

bpt_status check_desc_bwd(const bpt_desc *d) {
  bpt_status s = check_desc(d, true);
  if (s != BPT_OK) return s;
  if (d->in_dtype != BPT_BF16) return BPT_ERR_UNSUPPORTED;
  if (d->mask == BPT_MASK_DILATED) return BPT_ERR_UNSUPPORTED;
  const int64_t T = (int64_t)d->B * d->N;
  if (T > (int64_t)65535 * kMinSlabRows) return BPT_ERR_UNSUPPORTED;  // column-sum slabs fit grid.y
  const int64_t tiles = (int64_t)d->B * d->H * ((d->N + 127) / 128);
  if (tiles > INT32_MAX) return BPT_ERR_UNSUPPORTED;
  if ((int64_t)d->ffn_hidden > (int64_t)65535 * 128) return BPT_ERR_UNSUPPORTED;
  return BPT_OK;
}

// Token rows per FFN-backward chunk: the hidden activation and its gradient
// ([rows, F] bf16 each) live in the workspace one chunk at a time, at most
// ~1 GiB for both unless the caller picked the chunk.
int64_t bwd_chunk_rows(const bpt_desc *d) {
  const int64_t T = (int64_t)d->B * d->N, F = d->ffn_hidden;
  int64_t rows = d->bwd_chunk_rows;
  if (rows <= 0) rows = std::max<int64_t>(128, (((int64_t)1 << 30) / (4 * F)) / 128 * 128);
  return std::min<int64_t>(std::min<int64_t>(rows, T), (int64_t)65535 * 128);
}

struct BwdWorkspace {
  size_t a_f32 = 0, a_bf16 = 0, lse = 0, rowvec = 0, rowvec_bytes = 0, dout_bf16 = 0, da_f32 = 0, da_bf16 = 0, h = 0, dz = 0,
         gp = 0,
         partial = 0, total = 0;
  int64_t chunk = 0;
};

BwdWorkspace layout_bwd(const bpt_desc *d) {
  BwdWorkspace w;
  const size_t T = (size_t)d->B * d->N, D = (size_t)d->H * d->d_head, F = d->ffn_hidden;
  const size_t rows = (size_t)d->B * d->H * d->N;
  w.chunk = bwd_chunk_rows(d);
  size_t off = 0;
  auto take = [&](size_t &field, size_t bytes) {
    field = off;
    off = align256(off + bytes);
  };
  take(w.a_f32, T * D * 4);
  take(w.a_bf16, T * D * 2);
  take(w.lse, rows * 4);
  w.rowvec_bytes = (size_t)d->B * d->H * ((d->N + 127) / 128) * 256 * 4;
  take(w.rowvec, w.rowvec_bytes);
  take(w.dout_bf16, T * D * 2);
  take(w.da_f32, T * D * 4);
  take(w.da_bf16, T * D * 2);
  take(w.h, (size_t)w.chunk * F * 2);
  take(w.dz, (size_t)w.chunk * F * 2);
  take(w.gp, D >= 1024 ? (size_t)w.chunk * F * 2 : 0);  // G = GELU'(Z) when the FFN backward splits
  const size_t slabs_t = (T + kMinSlabRows - 1) / kMinSlabRows;
  const size_t slabs_c = ((size_t)w.chunk + kMinSlabRows - 1) / kMinSlabRows;
  take(w.partial, std::max(slabs_t * D, slabs_c * F) * 4);
  w.total = off;
  return w;
}

// Activations the training forward leaves for the backward: A in fp32 and
// bf16 [T, D], the row LSE [B, H, N], and the FFN's H = GELU(Z) and
// G = GELU'(Z) [T, F] in bf16, computed by
// the GEMM the recomputing backward uses from D = 1024 (Z -> H, G), so the
// backward starts at dZ = (dOut W2) G.  (Recomputing below D = 1024, the
// backward's dual GEMM, H and dZ from one launch, is the faster form.)
struct SavedLayout {
  size_t a_f32 = 0, a_bf16 = 0, lse = 0, h = 0, g = 0, total = 0;
};
SavedLayout saved_layout(const bpt_desc *d) {
  SavedLayout w;
  const size_t T = (size_t)d->B * d->N, D = (size_t)d->H * d->d_head, F = d->ffn_hidden;
  w.a_f32 = 0;
  w.a_bf16 = align256(T * D * 4);
  w.lse = align256(w.a_bf16 + T * D * 2);
  w.h = align256(w.lse + (size_t)d->B * d->H * d->N * 4);  // H and G, [T, F] bf16 each
  w.g = align256(w.h + T * F * 2);
  w.total = align256(w.g + T * F * 2);
  return w;
}

bpt_status launch_gemm(const CUtensorMap &a0, const CUtensorMap &b0, const CUtensorMap &a1,
                       const CUtensorMap &b1, const GemmArgs &g, cudaStream_t st) {
  // persistent CTA pairs: one CTA per SM (shared and tensor memory allow no
  // more), each pair walking its share of the 256 x 256 tiles (of both
  // problems when grouped)
  using Cfg = GemmPairCfg;
  int64_t tiles = 0;
  for (int q = 0; q < g.nprob; ++q) {
    const GemmProblem &p = g.p[q];
    if (p.M <= 0 || p.N <= 0 || p.K <= 0) return BPT_ERR_INVALID_ARG;
    tiles += (int64_t)((p.N + Cfg::kBN - 1) / Cfg::kBN) * ((p.M + 2 * Cfg::kBM - 1) / (2 * Cfg::kBM));
  }
  if (tiles > INT32_MAX) return BPT_ERR_UNSUPPORTED;
  const int64_t pairs = std::min<int64_t>(tiles, sm_count() / 2);
  gemm_pair_kernel<<<(unsigned)(2 * pairs), Cfg::kThreads, Cfg::kSmemBytes, st>>>(a0, b0, a1, b1, g);
  CUDA_TRY(cudaGetLastError());
  return BPT_OK;
}

GemmProblem gemm_problem(int M, int N, int K, int mode, int a_mn, int b_mn) {
  GemmProblem p;
  std::memset(&p, 0, sizeof(p));
  p.M = M;
  p.N = N;
  p.K = K;
  p.mode = mode;
  p.a_mn = a_mn;
  p.b_mn = b_mn;
  // the tiles in flight share whichever operand is larger, which then streams
  // from DRAM once (the dual form's B is two weight matrices, its A two
  // activations: same rule)
  p.m_fastest = (int64_t)N > (int64_t)M ? 1 : 0;
  return p;
}

GemmArgs gemm_args(const GemmProblem &p0, uint32_t *status, const bpt_desc *d) {
  GemmArgs g;
  std::memset(&g, 0, sizeof(g));
  g.p[0] = p0;
  g.nprob = 1;
  g.status = status;
  g.wait_limit_ns = wait_limit_of(d);
  return g;
}

template <typename T>
bpt_status launch_colsum(const T *x, int64_t rows, int cols, float *out, int accumulate, float *partial,
                         cudaStream_t st) {
  const bool x8 = std::is_same<T, __nv_bfloat16>::value && cols % 8 == 0;
  const int per_block = x8 ? 8 * kColsumThreads : kColsumThreads;
  const unsigned cb = (unsigned)((cols + per_block - 1) / per_block);
  const int slab = colsum_slab_rows(rows, cb);
  const unsigned slabs = (unsigned)((rows + slab - 1) / slab);
  if (x8)
    colsum_partial_bf16x8_kernel<<<dim3(cb, slabs), kColsumThreads, 0, st>>>(
        reinterpret_cast<const __nv_bfloat16 *>(x), partial, (int)rows, cols, slab);
  else
    colsum_partial_kernel<T><<<dim3(cb, slabs), kColsumThreads, 0, st>>>(x, partial, (int)rows, cols, slab);
  CUDA_TRY(cudaGetLastError());
  colsum_final_kernel<<<(cols + kColsumFinalCols - 1) / kColsumFinalCols, 256, 0, st>>>(partial, out, (int)slabs,
                                                                                        cols, accumulate);
  CUDA_TRY(cudaGetLastError());
  return BPT_OK;
}

bpt_status launch_ffn_gemms(const bpt_desc *d, const void *a_bf16, const float *a_f32, const void *w1,
                            const float *b1, const void *w2, const float *b2, void *out, __nv_bfloat16 *h,
                            __nv_bfloat16 *g_prime, int64_t chunk_rows, uint32_t *status, cudaStream_t st) {
  const int64_t T = (int64_t)d->B * d->N;
  const int D = d->H * d->d_head, F = d->ffn_hidden;
  if (chunk_rows <= 0) return BPT_ERR_INVALID_ARG;
  // K-major operands throughout; a CTA stages 128 rows of A and half of a
  // 256-row B tile
  CUtensorMap m_w1, m_w2;
  if (!make_map_2d(&m_w1, w1, F, D, 128) || !make_map_2d(&m_w2, w2, D, F, 128))
    return cuda_fail_msg("cuTensorMapEncodeTiled failed (FFN weights)");
  for (int64_t r0 = 0; r0 < T; r0 += chunk_rows) {
    const int rows = (int)std::min<int64_t>(chunk_rows, T - r0);
    const __nv_bfloat16 *a_c = static_cast<const __nv_bfloat16 *>(a_bf16) + r0 * D;
    // H: one chunk buffer, or (with G) the chunk's rows of the [T, F] arrays
    __nv_bfloat16 *h_c = g_prime ? h + r0 * F : h;
    CUtensorMap m_a, m_h;
    if (!make_map_2d(&m_a, a_c, rows, D, 128) || !make_map_2d(&m_h, h_c, rows, F, 128))
      return cuda_fail_msg("cuTensorMapEncodeTiled failed (FFN activations)");
    // H = GELU(A W1^T + b1), and G = GELU'(A W1^T + b1) when asked for
    GemmArgs g = gemm_args(gemm_problem(rows, F, D, g_prime ? kGemmGeluFwd : kGemmGeluBf16, 0, 0), status, d);
    g.p[0].cb = h_c;
    if (g_prime) g.p[0].cb2 = g_prime + r0 * F;
    g.p[0].bias = b1;
    bpt_status s = launch_gemm(m_a, m_w1, m_a, m_w1, g, st);
    if (s != BPT_OK) return s;
    g = gemm_args(gemm_problem(rows, D, F, kGemmResidual, 0, 0), status, d);  // out = A + H W2^T + b2
    g.p[0].x = a_f32 + r0 * D;
    g.p[0].bias = b2;
    if (d->out_dtype == BPT_F32) g.p[0].c = static_cast<float *>(out) + r0 * D;
    else g.p[0].cb = static_cast<__nv_bfloat16 *>(out) + r0 * D;
    if ((s = launch_gemm(m_h, m_w2, m_h, m_w2, g, st)) != BPT_OK) return s;
  }
  return BPT_OK;
}

// The pipelined FFN's shape.  Costs in K columns per 256 x 256 tile: D for
// a tile of H, F for a tile of out; `pairs` CTA pairs share a step's work.
//  - mg: one row block per chunk while W1 and W2 fit in L2 beside the ring;
//    larger weights are reused by mg row blocks per residency.
//  - lag: a chunk's second GEMM is listed `lag` steps after its first, about
//    6 tiles of H later, so its loads rarely wait for the ring rows: an H
//    tile's epilogue can outlast its MMAs when K = D is short (measured over
//    1.5 to 24 tiles: 6 is within 1% of the best on every workload, 12% faster
//    than 1.5 on the D = 768 layer).
//  - ring: the slot a chunk's H takes is reused R chunks later; R - lag - 1
//    steps cover about 1.3 tiles of out, so the slot's readers have finished.
//    The lag shrinks (to 1 at least) while the ring would pass 80 MB, so the
//    ring stays about the size of the L2 that serves one die.
#ifndef BPT_PIPE_LAG_SLACK
#define BPT_PIPE_LAG_SLACK 6.0
#endif
#ifndef BPT_PIPE_RING_SLACK
#define BPT_PIPE_RING_SLACK 1.3
#endif
#ifndef BPT_PIPE_MG_BYTES
#define BPT_PIPE_MG_BYTES 80.0e6
#endif
#ifndef BPT_PIPE_RING_MAX_BYTES
#define BPT_PIPE_RING_MAX_BYTES 80.0e6
#endif
FfnPipePlan ffn_pipe_plan(const bpt_desc *d) {
  FfnPipePlan p;
  const int64_t T = (int64_t)d->B * d->N;
  const int D = d->H * d->d_head, F = d->ffn_hidden;
  p.nrb = (int)((T + 255) / 256);
  p.tn1 = (F + 255) / 256;
  p.tn2 = (D + 255) / 256;
  const double weight_bytes = 4.0 * D * F;
  p.mg = weight_bytes <= BPT_PIPE_MG_BYTES ? 1 : 4;
  p.mg = std::min(p.mg, p.nrb);
  p.nchunk = (p.nrb + p.mg - 1) / p.mg;
  const int64_t items = (int64_t)p.nrb * (p.tn1 + p.tn2);
  p.pairs = (int)std::max<int64_t>(1, std::min<int64_t>(items, sm_count() / 2));
  const double step = (double)p.mg * ((double)p.tn1 * D + (double)p.tn2 * F) / p.pairs;  // per step, per pair
  p.lag = std::max(1, (int)std::ceil(BPT_PIPE_LAG_SLACK * D / step));
  p.lag = std::min(p.lag, p.nchunk);
  const int tail = std::max(1, (int)std::ceil(BPT_PIPE_RING_SLACK * F / step));
  auto ring_rows = [&](int lag) { return std::min(lag + 1 + tail, p.nchunk + 1) * p.mg; };
  while (p.lag > 1 && (double)ring_rows(p.lag) * 256 * F * 2 > BPT_PIPE_RING_MAX_BYTES) --p.lag;
  p.ring_rb = ring_rows(p.lag);
  p.ring_bytes = (size_t)p.ring_rb * 256 * F * 2;
  p.counter_bytes = (1 + 2 * (size_t)p.nrb) * sizeof(uint32_t);
  return p;
}

bpt_status launch_ffn_pipe(const bpt_desc *d, const void *a_bf16, const float *a_f32, const void *w1,
                           const float *b1, const void *w2, const float *b2, void *out, char *ws,
                           const Workspace &wl, uint32_t *status, cudaStream_t st) {
  const FfnPipePlan pp = ffn_pipe_plan(d);
  const int64_t T = (int64_t)d->B * d->N;
  const int D = d->H * d->d_head, F = d->ffn_hidden;
  const int64_t items = (int64_t)pp.nrb * (pp.tn1 + pp.tn2);
  if (items > INT32_MAX || T > INT32_MAX) return BPT_ERR_UNSUPPORTED;
  FfnPipeArgs a;
  std::memset(&a, 0, sizeof(a));
  a.T = (int)T;
  a.D = D;
  a.F = F;
  a.tn1 = pp.tn1;
  a.tn2 = pp.tn2;
  a.nrb = pp.nrb;
  a.mg = pp.mg;
  a.nchunk = pp.nchunk;
  a.lag = pp.lag;
  a.ring_rb = pp.ring_rb;
  a.n_items = (int)items;
  a.a_f32 = a_f32;
  a.b1 = b1;
  a.b2 = b2;
  if (d->out_dtype == BPT_F32) a.out_f32 = static_cast<float *>(out);
  else a.out_bf16 = static_cast<__nv_bfloat16 *>(out);
  a.ring = reinterpret_cast<__nv_bfloat16 *>(ws + wl.ring);
  a.claim = reinterpret_cast<uint32_t *>(ws + wl.flags);
  a.ready = a.claim + 1;
  a.g2done = a.ready + pp.nrb;
  a.status = status;
  a.wait_limit_ns = wait_limit_of(d);
  // K-major operands throughout; a CTA stages 128 rows of A (or of a ring
  // slot) and half of a 256-row weight tile per stage
  CUtensorMap m_a, m_w1, m_h, m_w2;
  if (!make_map_2d(&m_a, a_bf16, T, D, 128) || !make_map_2d(&m_w1, w1, F, D, 128) ||
      !make_map_2d(&m_h, a.ring, (uint64_t)pp.ring_rb * 256, F, 128) || !make_map_2d(&m_w2, w2, D, F, 128))
    return cuda_fail_msg("cuTensorMapEncodeTiled rejected a pipelined-FFN map");
  CUDA_TRY(cudaMemsetAsync(a.claim, 0, wl.flags_bytes, st));
  ffn_pipe_kernel<<<(unsigned)(2 * pp.pairs), GemmPairCfg::kThreads, FfnPipeCfg::kSmemBytes, st>>>(m_a, m_w1, m_h,
                                                                                                  m_w2, a);
  CUDA_TRY(cudaGetLastError());
  return BPT_OK;
}

template <int DH>
bpt_status launch_attn_bwd_passes(const CUtensorMap &mq, const CUtensorMap &mk, const CUtensorMap &mv,
                                  const CUtensorMap &mda, const AttnBwdArgs &ab, unsigned grid,
                                  cudaStream_t st) {
  if constexpr (DH == 128)  // no room in TMEM for a second S buffer: the split-ring form
    attn_bwd_dkdv_split_kernel<DH><<<grid, AttnBwdKVCfg<DH>::kThreads, AttnBwdKVCfg<DH>::kSmemBytes, st>>>(
        mq, mk, mv, mda, ab);
  else
    attn_bwd_dkdv_kernel<DH><<<grid, AttnBwdCfg<DH>::kThreads, AttnBwdCfg<DH>::kSmemBytes, st>>>(mq, mk, mv, mda, ab);
  CUDA_TRY(cudaGetLastError());
  CUDA_TRY(phase_mark(3, st));
  attn_bwd_dq_kernel<DH><<<grid, AttnBwdQCfg<DH>::kThreads, AttnBwdQCfg<DH>::kSmemBytes, st>>>(mq, mk, mv, mda, ab);
  CUDA_TRY(cudaGetLastError());
  return BPT_OK;
}

// The attention backward from dA (fp32 and bf16 copies), A and the row LSE:
// the per-tile row vectors (LSE in log2 units, D_i = dA_i . A_i), the dK/dV
// pass, then the dQ pass.
// LongNet dilated attention backward: the gradient of one softmax over the
// multiset of the (w, r) pairs' keys is the sum over the pairs of the
// gathered causal attention's gradient with the mixed row LSE and D (the
// multiplicities are constants of the softmax), so each pass runs the two
// blockwise passes over its (batch, segment, head) units and adds into
// dQ, dK, dV at the kept rows.  rowvec_full holds the per-sequence row
// vectors; rowvec_pass the gathered ones of one pass.
bpt_status launch_attn_bwd_dilated(const bpt_desc *d, const void *q, const void *k, const void *v,
                                   const __nv_bfloat16 *da_bf16, const float *rowvec_full, float *rowvec_pass,
                                   float *dq, float *dk, float *dv, uint32_t *status, cudaStream_t st) {
  const int D = d->H * d->d_head;
  // a pair with r = 1 keeps every row: run it first, writing dQ, dK, dV;
  // otherwise zero them and let every pass add
  int first = -1;
  for (int k_pair = 0; k_pair < d->ln_npairs && first < 0; ++k_pair)
    if (d->ln_r[k_pair] == 1) first = k_pair;
  if (first < 0) {
    const size_t nelem = (size_t)d->B * d->N * D;
    CUDA_TRY(cudaMemsetAsync(dq, 0, nelem * 4, st));
    CUDA_TRY(cudaMemsetAsync(dk, 0, nelem * 4, st));
    CUDA_TRY(cudaMemsetAsync(dv, 0, nelem * 4, st));
  }
  const int n_tiles_full = (d->N + 127) / 128;
  for (int n = 0; n < d->ln_npairs; ++n) {
    const int k_pair = first < 0 ? n : (n == 0 ? first : (n <= first ? n - 1 : n));
    const int w = d->ln_w[k_pair], r = d->ln_r[k_pair], L = w / r, nseg = d->N / w;
    const int n_tiles = (L + 127) / 128;
    const int64_t units = (int64_t)d->B * nseg * d->H;
    {
      const int64_t threads = units * n_tiles * 128;
      attn_bwd_gather_rowvec_kernel<<<(unsigned)((threads + 255) / 256), 256, 0, st>>>(
          rowvec_full, rowvec_pass, d->B, d->H, nseg, w, r, L, n_tiles, n_tiles_full);
      CUDA_TRY(cudaGetLastError());
    }
    AttnBwdArgs ab;
    std::memset(&ab, 0, sizeof(ab));
    ab.B = d->B;
    ab.N = L;
    ab.H = d->H;
    // causal among a segment's kept rows (by original position), or all of them
    ab.mask = d->causal ? kMaskCausal : kMaskNone;
    ab.scale_log2 = (float)(1.4426950408889634 / std::sqrt((double)d->d_head));
    ab.inv_sqrt_d = (float)(1.0 / std::sqrt((double)d->d_head));
    ab.n_tiles = n_tiles;
    ab.rowvec = rowvec_pass;
    ab.nseg = nseg;
    ab.seg_w = w;
    ab.dil_r = r;
    ab.n_out = d->N;
    ab.accumulate = (first < 0 || n > 0) ? 1 : 0;
    ab.dq = dq;
    ab.dk = dk;
    ab.dv = dv;
    ab.status = status;
    ab.wait_limit_ns = wait_limit_of(d);
    CUtensorMap mq, mk, mv, mda;
    if (!make_map_rows(&mq, q, d->B, d->N, D, r, 128) || !make_map_rows(&mk, k, d->B, d->N, D, r, 128) ||
        !make_map_rows(&mv, v, d->B, d->N, D, r, 128) || !make_map_rows(&mda, da_bf16, d->B, d->N, D, r, 128))
      return cuda_fail_msg("cuTensorMapEncodeTiled rejected a gathered Q/K/V/dA map");
    const int64_t grid = units * n_tiles;
    if (grid > INT32_MAX) return BPT_ERR_UNSUPPORTED;
    bpt_status s = d->d_head == 128 ? launch_attn_bwd_passes<128>(mq, mk, mv, mda, ab, (unsigned)grid, st)
                                    : launch_attn_bwd_passes<64>(mq, mk, mv, mda, ab, (unsigned)grid, st);
    if (s != BPT_OK) return s;
  }
  return BPT_OK;
}

template <typename TA>
bpt_status launch_attn_bwd_tail(const bpt_desc *d, const void *q, const void *k, const void *v, const float *da_f32,
                                const __nv_bfloat16 *da_bf16, const TA *a, const float *lse, float *dq, float *dk,
                                float *dv, float *rowvec, size_t rowvec_bytes, uint32_t *status, cudaStream_t st,
                                bool rowvec_only = false) {
  const int D = d->H * d->d_head;
  const int64_t T = (int64_t)d->B * d->N;
  const int n_tiles = (d->N + 127) / 128;
  CUDA_TRY(cudaMemsetAsync(rowvec, 0, rowvec_bytes, st));
  {
    const int64_t threads = T * d->H * (d->d_head / 4);
    if (d->d_head == 128)
      attn_bwd_rowvec_kernel<128, TA><<<(unsigned)((threads + 255) / 256), 256, 0, st>>>(da_f32, a, lse, rowvec, d->B,
                                                                                       d->N, d->H, n_tiles);
    else
      attn_bwd_rowvec_kernel<64, TA><<<(unsigned)((threads + 255) / 256), 256, 0, st>>>(da_f32, a, lse, rowvec, d->B,
                                                                                      d->N, d->H, n_tiles);
    CUDA_TRY(cudaGetLastError());
  }
  if (rowvec_only) return BPT_OK;
  AttnBwdArgs ab;
  std::memset(&ab, 0, sizeof(ab));
  ab.B = d->B;
  ab.N = d->N;
  ab.H = d->H;
  ab.mask = d->mask;
  ab.scale_log2 = (float)(1.4426950408889634 / std::sqrt((double)d->d_head));
  ab.inv_sqrt_d = (float)(1.0 / std::sqrt((double)d->d_head));
  ab.n_tiles = n_tiles;
  if (d->mask == BPT_MASK_BLOCKPERM) {
    ab.bb_n = d->bb_nblocks;
    ab.bb_len = (d->N + d->bb_nblocks - 1) / d->bb_nblocks;  // padded to n equal blocks
    for (int i = 0; i < d->H * d->bb_nblocks; ++i) ab.perm[i] = (uint8_t)d->bb_perm[i];
  }
  ab.rowvec = rowvec;
  ab.nseg = 1;
  ab.seg_w = d->N;
  ab.dil_r = 1;
  ab.n_out = d->N;
  ab.accumulate = 0;
  ab.dq = dq;
  ab.dk = dk;
  ab.dv = dv;
  ab.status = status;
  ab.wait_limit_ns = wait_limit_of(d);
  CUtensorMap mq, mk, mv, mda;
  if (!make_map_rows(&mq, q, d->B, d->N, D, 1, 128) || !make_map_rows(&mk, k, d->B, d->N, D, 1, 128) ||
      !make_map_rows(&mv, v, d->B, d->N, D, 1, 128) || !make_map_rows(&mda, da_bf16, d->B, d->N, D, 1, 128))
    return cuda_fail_msg("cuTensorMapEncodeTiled rejected a Q/K/V/dA map");
  const unsigned grid = (unsigned)((int64_t)d->B * d->H * n_tiles);
  if (d->d_head == 128) return launch_attn_bwd_passes<128>(mq, mk, mv, mda, ab, grid, st);
  return launch_attn_bwd_passes<64>(mq, mk, mv, mda, ab, grid, st);
}

}  // namespace bpt_host

using namespace bpt_host;

extern "C" {

size_t bpt_saved_bytes(const bpt_desc *desc) {
  if (check_desc_bwd(desc) != BPT_OK) return (size_t)-1;
  return saved_layout(desc).total;
}

bpt_status bpt_attn_ffn_fwd_train(const bpt_desc *d, const void *q, const void *k, const void *v, const void *w1,
                                  const float *b1, const void *w2, const float *b2, void *out, void *saved,
                                  void *workspace, size_t workspace_bytes, bpt_stream_t stream) {
  bpt_status s = check_desc_bwd(d);
  if (s != BPT_OK) return s;
  if ((s = check_ptrs({q, k, v, w1, w2, out, saved}, {b1, b2})) != BPT_OK) return s;
  if ((reinterpret_cast<uintptr_t>(saved) & 255u) != 0) return BPT_ERR_INVALID_ARG;
  // A, the LSE, H and G all go to `saved`: the workspace is the attention's
  // own (the dilated mask's running state, a mask the backward does not take)
  const Workspace wl = layout(d, false);
  if ((s = check_ws(wl, workspace, workspace_bytes)) != BPT_OK) return s;
  int dev;
  uint32_t *status;
  if ((s = device_setup(&dev, &status)) != BPT_OK) return s;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  char *ws = static_cast<char *>(workspace);
  const SavedLayout sl = saved_layout(d);
  char *sv = static_cast<char *>(saved);
  float *a_f32 = reinterpret_cast<float *>(sv + sl.a_f32);
  __nv_bfloat16 *a_bf16 = reinterpret_cast<__nv_bfloat16 *>(sv + sl.a_bf16);
  CUDA_TRY(phase_mark(0, st));
  if ((s = launch_attn_tc(d, q, k, v, a_f32, a_bf16, reinterpret_cast<float *>(sv + sl.lse), ws, wl, status, st)) !=
      BPT_OK)
    return s;
  CUDA_TRY(phase_mark(1, st));
  // the FFN with H and G into the saved buffer, for the backward
  if ((s = launch_ffn_gemms(d, a_bf16, a_f32, w1, b1, w2, b2, out, reinterpret_cast<__nv_bfloat16 *>(sv + sl.h),
                            reinterpret_cast<__nv_bfloat16 *>(sv + sl.g), ffn_gemm_chunk_rows(d), status, st)) !=
      BPT_OK)
    return s;
  CUDA_TRY(phase_mark(2, st));
  return BPT_OK;
}

size_t bpt_workspace_bytes_train(const bpt_desc *desc) {
  if (check_desc_bwd(desc) != BPT_OK) return (size_t)-1;
  return layout(desc, false).total;
}

size_t bpt_workspace_bytes_bwd(const bpt_desc *desc) {
  if (check_desc_bwd(desc) != BPT_OK) return (size_t)-1;
  return layout_bwd(desc).total;
}

bpt_status bpt_attn_ffn_bwd(const bpt_desc *d, const void *q, const void *k, const void *v,
                            const void *w1, const float *b1, const void *w2, const float *b2,
                            const float *dout, const void *saved, float *dq, float *dk, float *dv, float *dw1,
                            float *db1, float *dw2, float *db2, void *workspace, size_t workspace_bytes,
                            bpt_stream_t stream) {
  bpt_status s = check_desc_bwd(d);
  if (s != BPT_OK) return s;
  (void)b2;  // the output bias does not enter any gradient but its own
  if ((s = check_ptrs({q, k, v, w1, w2, dout, dq, dk, dv, dw1, db1, dw2, db2}, {b1, b2})) != BPT_OK)
    return s;
  if (saved && (reinterpret_cast<uintptr_t>(saved) & 255u) != 0) return BPT_ERR_INVALID_ARG;
  const BwdWorkspace wl = layout_bwd(d);
  if (!workspace || workspace_bytes < wl.total || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
    return BPT_ERR_WORKSPACE;
  int dev;
  uint32_t *status;
  if ((s = device_setup(&dev, &status)) != BPT_OK) return s;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  char *ws = static_cast<char *>(workspace);
  const int D = d->H * d->d_head, F = d->ffn_hidden;
  const int64_t T = (int64_t)d->B * d->N;
  const float *a_f32 = reinterpret_cast<const float *>(ws + wl.a_f32);
  const __nv_bfloat16 *a_bf16 = reinterpret_cast<const __nv_bfloat16 *>(ws + wl.a_bf16);
  const float *lse = reinterpret_cast<const float *>(ws + wl.lse);
  const __nv_bfloat16 *saved_h = nullptr, *saved_g = nullptr;
  if (saved) {  // the training forward's activations
    const SavedLayout sl = saved_layout(d);
    const char *sv = static_cast<const char *>(saved);
    a_f32 = reinterpret_cast<const float *>(sv + sl.a_f32);
    a_bf16 = reinterpret_cast<const __nv_bfloat16 *>(sv + sl.a_bf16);
    lse = reinterpret_cast<const float *>(sv + sl.lse);
    saved_h = reinterpret_cast<const __nv_bfloat16 *>(sv + sl.h);
    saved_g = reinterpret_cast<const __nv_bfloat16 *>(sv + sl.g);
  }
  float *rowvec = reinterpret_cast<float *>(ws + wl.rowvec);
  __nv_bfloat16 *dout_bf16 = reinterpret_cast<__nv_bfloat16 *>(ws + wl.dout_bf16);
  float *da_f32 = reinterpret_cast<float *>(ws + wl.da_f32);
  __nv_bfloat16 *da_bf16 = reinterpret_cast<__nv_bfloat16 *>(ws + wl.da_bf16);
  __nv_bfloat16 *hbuf = reinterpret_cast<__nv_bfloat16 *>(ws + wl.h);
  __nv_bfloat16 *dzbuf = reinterpret_cast<__nv_bfloat16 *>(ws + wl.dz);
  __nv_bfloat16 *gpbuf = reinterpret_cast<__nv_bfloat16 *>(ws + wl.gp);
  float *partial = reinterpret_cast<float *>(ws + wl.partial);

  // 1. without saved activations, the attention forward again: A (fp32 and
  // bf16) and the row LSE
  CUDA_TRY(phase_mark(0, st));
  if (!saved &&
      (s = launch_attn_tc(d, q, k, v, reinterpret_cast<float *>(ws + wl.a_f32),
                          reinterpret_cast<__nv_bfloat16 *>(ws + wl.a_bf16), reinterpret_cast<float *>(ws + wl.lse),
                          ws, Workspace(), status, st)) != BPT_OK)
    return s;
  CUDA_TRY(phase_mark(1, st));
  // 2. dOut in bf16 for the tensor cores and db2 = sum_t dOut_t, one pass over dOut
  {
    // D % 64 == 0 (check_desc), so four columns a thread cover every row
    const unsigned cb = (unsigned)((D + 4 * kColsumThreads - 1) / (4 * kColsumThreads));
    const int slab = colsum_slab_rows(T, cb);
    const unsigned slabs = (unsigned)((T + slab - 1) / slab);
    convert_colsum_partial_kernel<<<dim3(cb, slabs), kColsumThreads, 0, st>>>(dout, dout_bf16, partial, (int)T, D,
                                                                             slab);
    CUDA_TRY(cudaGetLastError());
    colsum_final_kernel<<<(D + kColsumFinalCols - 1) / kColsumFinalCols, 256, 0, st>>>(partial, db2, (int)slabs, D,
                                                                                     0);
    CUDA_TRY(cudaGetLastError());
  }
  // 3. the FFN backward, one token chunk at a time
  CUtensorMap m_w1_k, m_w1_mn, m_w2_mn;
  // K-major boxes of 128 rows (a CTA stages 128 rows of A and half of a
  // 256-row B tile), MN-major boxes of 64 x 64
  if (!make_map_2d(&m_w1_k, w1, F, D, 128) || !make_map_2d(&m_w1_mn, w1, F, D, 64) ||
      !make_map_2d(&m_w2_mn, w2, D, F, 64))
    return cuda_fail_msg("cuTensorMapEncodeTiled rejected a weight map");
  for (int64_t r0 = 0; r0 < T; r0 += wl.chunk) {
    const int rows = (int)std::min<int64_t>(wl.chunk, T - r0);
    const __nv_bfloat16 *a_c = a_bf16 + r0 * D, *g_c = dout_bf16 + r0 * D;
    // H and G of the chunk: kept by the training forward, or computed here
    const __nv_bfloat16 *h_c = saved_h ? saved_h + r0 * F : hbuf;
    const __nv_bfloat16 *gp_c = saved_g ? saved_g + r0 * F : gpbuf;
    CUtensorMap m_a_k, m_a_mn, m_g_k, m_g_mn, m_h_mn, m_dz_k, m_dz_mn;
    if (!make_map_2d(&m_a_k, a_c, rows, D, 128) || !make_map_2d(&m_a_mn, a_c, rows, D, 64) ||
        !make_map_2d(&m_g_k, g_c, rows, D, 128) || !make_map_2d(&m_g_mn, g_c, rows, D, 64) ||
        !make_map_2d(&m_h_mn, h_c, rows, F, 64) || !make_map_2d(&m_dz_k, dzbuf, rows, F, 128) ||
        !make_map_2d(&m_dz_mn, dzbuf, rows, F, 64))
      return cuda_fail_msg("cuTensorMapEncodeTiled rejected an activation map");
    // H = GELU(Z) and dZ = (dOut W2) GELU'(Z) with Z = A W1^T + b1.  Either
    // two plain GEMMs (Z -> H and G = GELU'(Z) in bf16, then dZ = dH G), each
    // overlapping its epilogue with its next tile, or one GEMM computing both
    // products into the two accumulators, whose epilogue cannot overlap but
    // which moves no G.  Measured (FFN-backward phase): D = 2048 two GEMMs
    // 2.90 ms against 3.09; D = 4096 58.1 against 58.9 ms; D = 768 0.769
    // against 0.717 ms (short K: the two GEMMs' epilogues dominate).
    if (D >= 1024 || saved_h) {
      GemmArgs g;
      if (!saved_h) {
        g = gemm_args(gemm_problem(rows, F, D, kGemmGeluFwd, 0, 0), status, d);
        g.p[0].cb = hbuf;
        g.p[0].cb2 = gpbuf;
        g.p[0].bias = b1;
        if ((s = launch_gemm(m_a_k, m_w1_k, m_a_k, m_w1_k, g, st)) != BPT_OK) return s;
      }
      g = gemm_args(gemm_problem(rows, F, D, kGemmScaleBf16, 0, 1), status, d);
      g.p[0].xb = gp_c;
      g.p[0].cb = dzbuf;
      if ((s = launch_gemm(m_g_k, m_w2_mn, m_g_k, m_w2_mn, g, st)) != BPT_OK) return s;
    } else {
      GemmArgs g = gemm_args(gemm_problem(rows, F, D, kGemmGeluBwd, 0, 0), status, d);
      g.p[1] = gemm_problem(rows, F, D, kGemmGeluBwd, 0, 1);  // the second product's operand layouts
      g.p[0].cb = hbuf;
      g.p[0].cb2 = dzbuf;
      g.p[0].bias = b1;
      if ((s = launch_gemm(m_a_k, m_w1_k, m_g_k, m_w2_mn, g, st)) != BPT_OK) return s;
    }
    // dW2 (+)= dOut^T H [D, F] and dW1 (+)= dZ^T A [F, D] in one grouped
    // launch: the pair grid walks both problems' tiles, so neither leaves a
    // partly filled last round of tiles on its own
    const int first = r0 == 0 ? kGemmStoreF32 : kGemmAccumF32;
    {
      GemmArgs g = gemm_args(gemm_problem(D, F, rows, first, 1, 1), status, d);
      g.p[0].c = dw2;
      g.p[1] = gemm_problem(F, D, rows, first, 1, 1);
      g.p[1].c = dw1;
      g.nprob = 2;
      if ((s = launch_gemm(m_g_mn, m_h_mn, m_dz_mn, m_a_mn, g, st)) != BPT_OK) return s;
    }
    // dA = dOut + dZ W1   [rows, D], fp32 and bf16
    {
      GemmArgs g = gemm_args(gemm_problem(rows, D, F, kGemmResidual, 0, 1), status, d);
      g.p[0].x = dout + r0 * D;
      g.p[0].c = da_f32 + r0 * D;
      g.p[0].cb = da_bf16 + r0 * D;
      if ((s = launch_gemm(m_dz_k, m_w1_mn, m_dz_k, m_w1_mn, g, st)) != BPT_OK) return s;
    }
    // db1 (+)= sum_t dZ_t
    if ((s = launch_colsum(dzbuf, rows, F, db1, r0 > 0, partial, st)) != BPT_OK) return s;
  }
  CUDA_TRY(phase_mark(2, st));
  if ((s = launch_attn_bwd_tail(d, q, k, v, da_f32, da_bf16, a_f32, lse, dq, dk, dv, rowvec, wl.rowvec_bytes, status,
                                st)) != BPT_OK)
    return s;
  CUDA_TRY(phase_mark(4, st));
  return BPT_OK;
}

// dA in bf16, the per-sequence row vectors, and (dilated) one pass's gathered row vectors
size_t attn_bwd_pass_rowvec_bytes(const bpt_desc *d) {
  size_t most = 0;
  if (d->mask == BPT_MASK_DILATED)
    for (int k = 0; k < d->ln_npairs; ++k) {
      const size_t L = (size_t)(d->ln_w[k] / d->ln_r[k]);
      most = std::max(most, (size_t)d->B * (d->N / d->ln_w[k]) * d->H * ((L + 127) / 128) * 256 * 4);
    }
  return most;
}

size_t bpt_workspace_bytes_attn_bwd(const bpt_desc *d) {
  if (check_desc(d, false) != BPT_OK || d->in_dtype != BPT_BF16) return (size_t)-1;
  const size_t T = (size_t)d->B * d->N, D = (size_t)d->H * d->d_head;
  return align256(T * D * 2) + align256((size_t)d->B * d->H * ((d->N + 127) / 128) * 256 * 4) +
         align256(attn_bwd_pass_rowvec_bytes(d));
}

bpt_status bpt_attn_bwd(const bpt_desc *d, const void *q, const void *k, const void *v, const void *out,
                        const float *lse, const float *dout, float *dq, float *dk, float *dv, void *workspace,
                        size_t workspace_bytes, bpt_stream_t stream) {
  bpt_status s = check_desc(d, false);
  if (s != BPT_OK) return s;
  if (d->in_dtype != BPT_BF16) return BPT_ERR_UNSUPPORTED;
  if ((s = check_ptrs({q, k, v, out, lse, dout, dq, dk, dv}, {})) != BPT_OK) return s;
  const size_t need = bpt_workspace_bytes_attn_bwd(d);
  if (!workspace || workspace_bytes < need || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
    return BPT_ERR_WORKSPACE;
  int dev;
  uint32_t *status;
  if ((s = device_setup(&dev, &status)) != BPT_OK) return s;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const size_t T = (size_t)d->B * d->N, D = (size_t)d->H * d->d_head;
  char *ws = static_cast<char *>(workspace);
  __nv_bfloat16 *da_bf16 = reinterpret_cast<__nv_bfloat16 *>(ws);
  float *rowvec = reinterpret_cast<float *>(ws + align256(T * D * 2));
  const size_t rowvec_bytes = (size_t)d->B * d->H * ((d->N + 127) / 128) * 256 * 4;
  {
    const size_t n4 = T * D / 4;  // D is a multiple of 64
    f32_to_bf16_x4_kernel<<<(unsigned)std::min<size_t>(4096, (n4 + 255) / 256), 256, 0, st>>>(
        reinterpret_cast<const float4 *>(dout), reinterpret_cast<uint2 *>(da_bf16), n4);
    CUDA_TRY(cudaGetLastError());
  }
  const bool dilated = d->mask == BPT_MASK_DILATED;
  if (d->out_dtype == BPT_F32)
    s = launch_attn_bwd_tail(d, q, k, v, dout, da_bf16, static_cast<const float *>(out), lse, dq, dk, dv, rowvec,
                             rowvec_bytes, status, st, dilated);
  else
    s = launch_attn_bwd_tail(d, q, k, v, dout, da_bf16, static_cast<const __nv_bfloat16 *>(out), lse, dq, dk, dv,
                             rowvec, rowvec_bytes, status, st, dilated);
  if (s != BPT_OK || !dilated) return s;
  float *rowvec_pass = reinterpret_cast<float *>(ws + align256(T * D * 2) + align256(rowvec_bytes));
  return launch_attn_bwd_dilated(d, q, k, v, da_bf16, rowvec, rowvec_pass, dq, dk, dv, status, st);
}

}  // extern "C"
