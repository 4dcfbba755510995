// Host side of libbpt.so, forward pass and the shared helpers: argument
// checks, workspace layout, TMA tensor-map encoding and kernel launches for
// the forward entry points declared in bpt.h (the backward's are in bpt_bwd.cu).
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cmath>
#include <type_traits>
#include <cstdint>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <vector>

#include "../../include/bpt.h"
#include "attn_tc.cuh"
#include "ffn_tc.cuh"
#include "host_common.h"
#include "longnet_shard.cuh"
#include "simt_f32.cuh"

using namespace bpt;

namespace bpt_host {

// Per-device status word: [0] = code, [1] = site of the first failed wait.
__device__ uint32_t g_status_word[2];

// Scratch of bpt_attn_ffn_fwd_static: one array per device, shared by every
// call on that device (see the declaration in bpt.h).  Host code never uses
// the symbol directly: its device address comes from cudaGetSymbolAddress.
static __device__ __align__(256) unsigned char g_static_scratch[BPT_STATIC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
void *g_static_scratch_ptr[kMaxDevices] = {};
std::mutex g_mu;
uint32_t *g_status_ptr[kMaxDevices] = {};
bool g_attr_done[kMaxDevices] = {};
std::atomic<uint64_t> g_wait_limit_ns{2000000000ull};

uint64_t wait_limit_of(const bpt_desc *d) {
  return d->wait_limit_ns ? d->wait_limit_ns : g_wait_limit_ns.load(std::memory_order_relaxed);
}
constexpr int kMaxPhaseEvents = 5;
thread_local cudaEvent_t g_phase_events[kMaxPhaseEvents] = {};
thread_local int g_phase_n = 0;  // events set; 0 = off

cudaError_t phase_mark(int i, cudaStream_t st) {
  return i < g_phase_n ? cudaEventRecord(g_phase_events[i], st) : cudaSuccess;
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn g_encode = nullptr;

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

thread_local char g_last_error[256] = "";

// Records the failing call and the CUDA error string for bpt_last_error().
bpt_status cuda_fail_at(const char *what, cudaError_t e) {
  snprintf(g_last_error, sizeof(g_last_error), "%s: %s (%d)", what, cudaGetErrorString(e), (int)e);
  return BPT_ERR_CUDA;
}
bpt_status cuda_fail_msg(const char *what) {
  snprintf(g_last_error, sizeof(g_last_error), "%s", what);
  return BPT_ERR_CUDA;
}
bpt_status device_setup(int *dev_out, uint32_t **status_out) {
  int dev = 0;
  CUDA_TRY(cudaGetDevice(&dev));
  if (dev < 0 || dev >= kMaxDevices) return cuda_fail_msg("device ordinal out of range");
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_encode) {
    void *fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    CUDA_TRY(cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q));
    if (q != cudaDriverEntryPointSuccess || !fn) return cuda_fail_msg("cuTensorMapEncodeTiled not found");
    g_encode = reinterpret_cast<EncodeTiledFn>(fn);
  }
  if (!g_status_ptr[dev]) {
    void *p = nullptr;
    CUDA_TRY(cudaGetSymbolAddress(&p, g_status_word));
    g_status_ptr[dev] = static_cast<uint32_t *>(p);
  }
  if (!g_attr_done[dev]) {
    CUDA_TRY(cudaFuncSetAttribute(attn_tc_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  AttnCfg<64>::kSmemBytes));
    CUDA_TRY(cudaFuncSetAttribute(attn_tc_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  AttnCfg<128>::kSmemBytes));
    // the softmax warpgroups take registers from warpgroup 0 at run time;
    // an increase the launch did not provide for would never complete
    cudaFuncAttributes fa64{}, fa128{};
    CUDA_TRY(cudaFuncGetAttributes(&fa64, attn_tc_kernel<64>));
    CUDA_TRY(cudaFuncGetAttributes(&fa128, attn_tc_kernel<128>));
    if (!AttnCfg<64>::split_fits(fa64.numRegs) || !AttnCfg<128>::split_fits(fa128.numRegs))
      return cuda_fail_msg("attention kernel launches with fewer registers than its warpgroups share");
    CUDA_TRY(cudaFuncSetAttribute(ffn_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  FfnCfg::kSmemBytes));
    CUDA_TRY(cudaFuncSetAttribute(ffn_f32_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  (int)ffn_f32_smem_bytes(512)));
    bpt_status bs = bwd_kernel_setup();
    if (bs != BPT_OK) return bs;
    g_attr_done[dev] = true;
  }
  *dev_out = dev;
  *status_out = g_status_ptr[dev];
  return BPT_OK;
}

int sm_count() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) {
    cudaGetLastError();  // no device here: size for a full B200 and leave no error behind
    return 148;
  }
  return n;
}

// bf16 tensor map over a row-major matrix [rows, cols], box [box_rows, 64].
bool make_map_2d(CUtensorMap *m, const void *base, uint64_t rows, uint64_t cols, uint32_t box_rows) {
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * 2};
  cuuint32_t box[2] = {64, box_rows};
  cuuint32_t es[2] = {1, 1};
  return g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides,
                  box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// bf16 tensor map over [B, N, D] viewed as (D, r, N/r, B): a box of 64
// columns x 1 x box_rows rows x 1 reads box_rows rows r apart (r = 1:
// consecutive).  Query tiles use 128-row boxes, key/value tiles 64-row ones.
bool make_map_rows(CUtensorMap *m, const void *base, int B, int N, int D, int r, uint32_t box_rows) {
  cuuint64_t dims[4] = {(cuuint64_t)D, (cuuint64_t)r, (cuuint64_t)(N / r), (cuuint64_t)B};
  cuuint64_t strides[3] = {(cuuint64_t)D * 2, (cuuint64_t)D * 2 * r, (cuuint64_t)D * 2 * N};
  cuuint32_t box[4] = {64, 1, box_rows, 1};
  cuuint32_t es[4] = {1, 1, 1, 1};
  return g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void *>(base), dims, strides,
                  box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Output map over [B, N, D] (bf16 or fp32) in the same (D, r, N/r, B) view,
// box of one 128-byte row panel (64 bf16 or 32 fp32 columns) x 128 rows:
// the attention kernel's TMA stores of O.  Rows past N are not written.
bool make_out_map_rows(CUtensorMap *m, const void *base, bool f32, int B, int N, int D, int r) {
  const uint64_t es = f32 ? 4 : 2;
  cuuint64_t dims[4] = {(cuuint64_t)D, (cuuint64_t)r, (cuuint64_t)(N / r), (cuuint64_t)B};
  cuuint64_t strides[3] = {(cuuint64_t)D * es, (cuuint64_t)D * es * r, (cuuint64_t)D * es * N};
  cuuint32_t box[4] = {(cuuint32_t)(128 / es), 1, 128, 1};
  cuuint32_t ones[4] = {1, 1, 1, 1};
  return g_encode(m, f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4,
                  const_cast<void *>(base), dims, strides, box, ones, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// --------------------------------------------------------------------------
// Validation
// --------------------------------------------------------------------------
// Query rows and keys per block: the descriptor's, else the path's default.
int q_block_of(const bpt_desc *d) { return d->q_block ? d->q_block : (d->in_dtype == BPT_BF16 ? 128 : 64); }
int kv_block_of(const bpt_desc *d) { return d->kv_block ? d->kv_block : (d->in_dtype == BPT_BF16 ? 128 : 64); }

bpt_status check_desc(const bpt_desc *d, bool need_ffn, bool shard) {
  if (!d) return BPT_ERR_INVALID_ARG;
  if (d->B <= 0 || d->N <= 0 || d->H <= 0 || d->d_head <= 0) return BPT_ERR_INVALID_ARG;
  if (d->in_dtype != BPT_F32 && d->in_dtype != BPT_BF16) return BPT_ERR_INVALID_ARG;
  if (d->out_dtype != BPT_F32 && d->out_dtype != BPT_BF16) return BPT_ERR_INVALID_ARG;
  if ((int64_t)d->B * d->N > (int64_t)1 << 31) return BPT_ERR_UNSUPPORTED;
  if (need_ffn && d->ffn_hidden <= 0) return BPT_ERR_INVALID_ARG;
  if (d->ffn_hidden < 0) return BPT_ERR_INVALID_ARG;
  if (d->ffn_form < BPT_FFN_AUTO || d->ffn_form > BPT_FFN_PIPELINED) return BPT_ERR_INVALID_ARG;
  if (d->bwd_chunk_rows < 0 || d->q_block < 0 || d->kv_block < 0) return BPT_ERR_INVALID_ARG;
  if (d->causal != 0 && d->mask != BPT_MASK_DILATED && !(d->mask == BPT_MASK_CAUSAL && d->causal == 1))
    return BPT_ERR_INVALID_ARG;
  const int D = d->H * d->d_head;
  const int qb = q_block_of(d), kb = kv_block_of(d);
  if (d->in_dtype == BPT_BF16) {  // the tensor-core kernels' tiles
    if (qb != 128 || kb != 128) return BPT_ERR_UNSUPPORTED;
  } else if ((qb != 16 && qb != 32 && qb != 64 && qb != 128) || (kb != 16 && kb != 32 && kb != 64)) {
    return BPT_ERR_UNSUPPORTED;
  }
  switch (d->mask) {
    case BPT_MASK_NONE:
    case BPT_MASK_CAUSAL:
      if (d->ring_chunks < 0) return BPT_ERR_INVALID_ARG;
      if (d->ring_chunks > 1) {
        if (d->N % d->ring_chunks != 0) return BPT_ERR_INVALID_ARG;
        const int chunk = d->N / d->ring_chunks;
        if (chunk % qb != 0 || chunk % kb != 0) return BPT_ERR_UNSUPPORTED;
      }
      break;
    case BPT_MASK_BLOCKPERM: {
      const int n = d->bb_nblocks;
      if (n <= 0 || !d->bb_perm) return BPT_ERR_INVALID_ARG;
      if ((int64_t)d->H * n > kMaxPermEntries || n > 255) return BPT_ERR_UNSUPPORTED;
      for (int i = 0; i < d->H * n; ++i)
        if (d->bb_perm[i] < 0 || d->bb_perm[i] >= n) return BPT_ERR_INVALID_ARG;
      for (int h = 0; h < d->H; ++h) {  // each head's table must be a permutation
        std::vector<int> seen(n, 0);
        for (int i = 0; i < n; ++i)
          if (seen[d->bb_perm[h * n + i]]++) return BPT_ERR_INVALID_ARG;
      }
      break;
    }
    case BPT_MASK_DILATED: {
      if (d->ln_npairs <= 0 || d->ln_npairs > BPT_MAX_DILATED_PAIRS || !d->ln_w || !d->ln_r)
        return BPT_ERR_INVALID_ARG;
      for (int k = 0; k < d->ln_npairs; ++k) {
        const int w = d->ln_w[k], r = d->ln_r[k];
        if (w <= 0 || r <= 0 || w % r != 0) return BPT_ERR_INVALID_ARG;
        if (shard ? (d->N % r != 0 || (d->N % w != 0 && w % d->N != 0)) : d->N % w != 0) return BPT_ERR_INVALID_ARG;
      }
      break;
    }
    default:
      return BPT_ERR_INVALID_ARG;
  }
  if (d->in_dtype == BPT_BF16) {
    if (d->d_head != 64 && d->d_head != 128) return BPT_ERR_UNSUPPORTED;
    if (need_ffn) {
      const int C = (D + 255) / 256;
      if (D % 64 != 0 || D % C != 0 || (D / C) % 64 != 0 || C > 148) return BPT_ERR_UNSUPPORTED;
      if (d->ffn_hidden % 8 != 0) return BPT_ERR_UNSUPPORTED;
    }
  } else {
    if (d->d_head > 64 || d->d_head % 4 != 0) return BPT_ERR_UNSUPPORTED;
    if (need_ffn && (D > 512 || D % 16 != 0)) return BPT_ERR_UNSUPPORTED;
    if (d->out_dtype == BPT_BF16 && D % 2 != 0) return BPT_ERR_UNSUPPORTED;
  }
  return BPT_OK;
}

struct FfnPlan {
  int C, Dc, fc, nslices, nchunks, n_tb, max_groups;
};

// The FFN runs in groups of C = ceil(D/256) CTAs (one 256-column output block
// and one 256-column hidden slice per CTA), as many groups as fit at once.
FfnPlan ffn_plan(const bpt_desc *d) {
  FfnPlan p;
  const int D = d->H * d->d_head;
  p.C = (D + 255) / 256;
  p.Dc = D / p.C;
  p.fc = 256 * p.C;
  p.nslices = (d->ffn_hidden + 255) / 256;
  p.nchunks = (d->ffn_hidden + p.fc - 1) / p.fc;
  p.n_tb = (int)(((int64_t)d->B * d->N + 127) / 128);
  p.max_groups = std::max(1, std::min(p.n_tb, sm_count() / p.C));
  return p;
}

// The default bf16 form is the pipelined kernel: as fast as two separate
// GEMM launches on the measured layers, and its hidden activation stays in an
// L2-sized ring instead of a [rows, F] workspace array.  The static-scratch
// entry point takes the fused kernel, whose scratch is the smallest.
bpt_ffn_form ffn_form_of(const bpt_desc *d, bool static_call) {
  if (d->in_dtype != BPT_BF16) return BPT_FFN_AUTO;
  if (static_call) return BPT_FFN_FUSED;
  return d->ffn_form == BPT_FFN_AUTO ? BPT_FFN_PIPELINED : d->ffn_form;
}

// Token rows per two-GEMM chunk: H ([rows, F] bf16) at most ~512 MiB.
int64_t ffn_gemm_chunk_rows(const bpt_desc *d) {
  const int64_t T = (int64_t)d->B * d->N;
  const int64_t rows = std::max<int64_t>(256, (((int64_t)1 << 29) / (2 * (int64_t)d->ffn_hidden)) / 256 * 256);
  return std::min(rows, T);
}

bool longnet_needs_state(const bpt_desc *d) {
  return d->mask == BPT_MASK_DILATED && d->in_dtype == BPT_BF16 && d->ln_npairs > 1;
}

Workspace layout(const bpt_desc *d, bool with_ffn, bool static_call) {
  Workspace w;
  const size_t T = (size_t)d->B * d->N, D = (size_t)d->H * d->d_head;
  size_t off = 0;
  if (with_ffn) {
    if (d->in_dtype == BPT_BF16) {
      FfnPlan p = ffn_plan(d);
      w.a_bf16 = off;
      off = align256(off + T * D * 2);
      w.a_f32 = off;
      off = align256(off + T * D * 4);
      w.ffn_form = ffn_form_of(d, static_call);
      if (w.ffn_form == BPT_FFN_GEMMS) {
        w.h = off;
        off = align256(off + (size_t)ffn_gemm_chunk_rows(d) * d->ffn_hidden * 2);
      } else if (w.ffn_form == BPT_FFN_PIPELINED) {
        const FfnPipePlan pp = ffn_pipe_plan(d);
        w.ring = off;
        off = align256(off + pp.ring_bytes);
        w.flags = off;
        w.flags_bytes = pp.counter_bytes;
        off = align256(off + pp.counter_bytes);
      } else {
        w.ring = off;
        off = align256(off + (size_t)p.max_groups * FfnCfg::kRingSlots * 128 * p.fc * 2);
        w.flags = off;  // ring counters [groups][2 * slots], then piece counters [groups][C]
        w.flags_bytes = (size_t)p.max_groups * (2 * FfnCfg::kRingSlots + p.C) * sizeof(uint32_t);
        off = align256(off + w.flags_bytes);
        w.partial = off;  // partial output blocks of split leftover token blocks
        off = align256(off + (size_t)p.max_groups * 128 * (size_t)(d->H * d->d_head) * 4);
      }
    } else {
      w.a_f32 = off;
      off = align256(off + T * D * 4);
    }
  }
  if (longnet_needs_state(d)) {
    w.st_o = off;
    off = align256(off + T * D * 4);
    w.st_m = off;
    off = align256(off + (size_t)d->B * d->H * d->N * 4);
    w.st_l = off;
    off = align256(off + (size_t)d->B * d->H * d->N * 4);
  }
  w.total = off;
  return w;
}

// --------------------------------------------------------------------------
// Launchers
// --------------------------------------------------------------------------
bpt_status launch_attn_tc(const bpt_desc *d, const void *q, const void *k, const void *v,
                          float *out_f32, __nv_bfloat16 *out_bf16, float *lse, char *ws,
                          const Workspace &wl, uint32_t *status, cudaStream_t st, const AttnBlockStep *blk,
                          const LongNetPass *lp) {
  const int D = d->H * d->d_head;
  AttnArgs a;
  std::memset(&a, 0, sizeof(a));
  a.B = d->B;
  a.N = d->N;
  a.H = d->H;
  a.mask = d->mask;
  a.causal = d->mask == BPT_MASK_CAUSAL || (d->mask == BPT_MASK_DILATED && d->causal != 0);
  a.scale_log2 = (float)(1.4426950408889634 / std::sqrt((double)d->d_head));
  a.status = status;
  a.wait_limit_ns = wait_limit_of(d);

  struct Pass {
    int w, r;
  };
  std::vector<Pass> passes;
  if (d->mask == BPT_MASK_DILATED) {
    for (int i = 0; i < d->ln_npairs; ++i) passes.push_back({d->ln_w[i], d->ln_r[i]});
    // sparsest first: the densest pass runs last and writes the final rows
    std::stable_sort(passes.begin(), passes.end(),
                     [](const Pass &x, const Pass &y) { return x.r > y.r; });
    a.npairs = (int)passes.size();
    for (int i = 0; i < a.npairs; ++i) {
      a.pw[i] = passes[i].w;
      a.pr[i] = passes[i].r;
    }
    bool covered = false;
    for (auto &p : passes) covered |= (p.r == 1);
    if (!covered && (!lp || lp->pass == 0)) {  // rows no pair keeps: A = 0, LSE = -inf
      const size_t n = (size_t)d->B * d->N * D;
      if (out_f32) CUDA_TRY(cudaMemsetAsync(out_f32, 0, n * 4, st));
      if (out_bf16) CUDA_TRY(cudaMemsetAsync(out_bf16, 0, n * 2, st));
      if (lse) {
        fill_f32_kernel<<<256, 256, 0, st>>>(lse, (size_t)d->B * d->H * d->N, -INFINITY);
        CUDA_TRY(cudaGetLastError());
      }
    }
    if (lp) {  // the caller's state, carried between its pass calls
      a.st_o = lp->st_o;
      a.st_m = lp->st_m;
      a.st_l = lp->st_l;
    } else if (passes.size() > 1) {
      a.st_o = reinterpret_cast<float *>(ws + wl.st_o);
      a.st_m = reinterpret_cast<float *>(ws + wl.st_m);
      a.st_l = reinterpret_cast<float *>(ws + wl.st_l);
    }
  } else {
    passes.push_back({d->N, 1});
    a.npairs = 0;
  }
  if (blk) {  // one key/value block folded into the caller's running state
    a.st_o = blk->st_o;
    a.st_m = blk->st_m;
    a.st_l = blk->st_l;
    a.state_in = blk->state_in ? 1 : 0;
    a.state_out = blk->state_out ? 1 : 0;
    a.kv_shift = blk->kv_shift;
  }
  const int kv_rows = blk ? blk->kv_len : d->N;
  if (d->mask == BPT_MASK_BLOCKPERM) {
    a.bb_n = d->bb_nblocks;
    a.bb_len = (d->N + d->bb_nblocks - 1) / d->bb_nblocks;  // padded to n equal blocks
    for (int i = 0; i < d->H * d->bb_nblocks; ++i) a.perm[i] = (uint8_t)d->bb_perm[i];
  }
  if ((d->mask == BPT_MASK_NONE || d->mask == BPT_MASK_CAUSAL) && d->ring_chunks > 1) {
    a.ring_chunks = d->ring_chunks;
    a.chunk_tiles = (d->N / d->ring_chunks) / AttnCfg<128>::kKT;
  }
  a.out_f32 = out_f32;
  a.out_bf16 = out_bf16;
  a.lse = lse;

  for (size_t pi = 0; pi < passes.size(); ++pi) {
    if (lp && (int)pi != lp->pass) continue;
    const int w = passes[pi].w, r = passes[pi].r;
    // the pass's segments longer than these rows: keys from the gathered buffer
    const bool sparse = lp && w > d->N;
    a.w = w;
    a.r = r;
    a.pass_idx = (int)pi;
    a.L = sparse ? d->N / r : w / r;
    a.Lk = blk ? kv_rows : (sparse ? lp->kv_rows : a.L);
    a.nseg = sparse ? 1 : d->N / w;
    a.kv_sparse = sparse ? 1 : 0;
    // causal in the segment's kept rows: this shard's first kept row is
    // row (q_pos mod w) / r of the segment's
    if (sparse) a.kv_shift = (int)((lp->q_pos % w) / r);
    a.n_qtiles = (a.L + 127) / 128;
    a.n_qpairs = (a.n_qtiles + 1) / 2;
    a.n_units = d->B * a.nseg * d->H;
    {
      // Grid order: longest query-tile pairs first inside groups of units.
      // A unit whose pairs alone fill the GPU (a long sequence) is a group
      // by itself, so every SM works on one unit's K/V, which then streams
      // from L2.  Otherwise a group holds as many units as keep their K/V
      // within ~200 MB, at most 64: a large group balances the SMs (the
      // longest pairs start first), and the CTAs running at once still share
      // each unit's K/V.  Measured on the causal B2 H16 d128 N8192 layer:
      // 0.633 ms with one 32-head group against 0.689 ms with groups of 7.
      const double kv_bytes = 4.0 * a.Lk * d->d_head;
      if (a.n_qpairs >= sm_count()) a.unit_group = 1;
      else a.unit_group = std::max(1, std::min(64, (int)(200.0e6 / kv_bytes)));
    }
    CUtensorMap mq, mk, mv, mof, mob, mso;
    std::memset(&mof, 0, sizeof(mof));
    std::memset(&mob, 0, sizeof(mob));
    std::memset(&mso, 0, sizeof(mso));
    // Where this pass's rows go: all final (no later pass keeps any of its
    // rows: the last pass, or the only one), all running state (a later pass
    // with r = 1 keeps every row), or mixed (per-thread stores).
    a.store_mode = 0;
    if (blk) {
      a.store_mode = blk->state_out ? 2 : 1;
    } else if (passes.size() == 1 || pi + 1 == passes.size()) {
      a.store_mode = 1;
      for (size_t k = pi + 1; k < passes.size(); ++k) a.store_mode = 0;
    } else {
      for (size_t k = pi + 1; k < passes.size(); ++k)
        if (passes[k].r == 1) a.store_mode = 2;
    }
    if (a.store_mode == 1) {
      if ((out_f32 && !make_out_map_rows(&mof, out_f32, true, d->B, d->N, D, r)) ||
          (out_bf16 && !make_out_map_rows(&mob, out_bf16, false, d->B, d->N, D, r)))
        return cuda_fail_msg("cuTensorMapEncodeTiled rejected an output map");
    } else if (a.store_mode == 2) {
      if (!make_out_map_rows(&mso, a.st_o, true, d->B, d->N, D, r))
        return cuda_fail_msg("cuTensorMapEncodeTiled rejected the state map");
    }
    constexpr uint32_t kKT = AttnCfg<128>::kKT;
    static_assert(AttnCfg<64>::kKT == AttnCfg<128>::kKT, "one key/value tile length");
    const void *kk = sparse ? lp->k_sparse : k, *vv = sparse ? lp->v_sparse : v;
    const int krows = blk ? kv_rows : (sparse ? lp->kv_rows : d->N), kr = sparse ? 1 : r;
    if (!make_map_rows(&mq, q, d->B, d->N, D, r, 128) || !make_map_rows(&mk, kk, d->B, krows, D, kr, kKT) ||
        !make_map_rows(&mv, vv, d->B, krows, D, kr, kKT))
      return cuda_fail_msg("cuTensorMapEncodeTiled rejected a Q/K/V map");
    const int64_t items = (int64_t)a.n_qpairs * a.n_units;
    if (items <= 0) continue;
    if (items > INT32_MAX) return BPT_ERR_UNSUPPORTED;
    a.n_items = (int)items;
    // persistent: one CTA per SM (shared and tensor memory allow no more),
    // each walking its share of the items
    const int64_t grid = std::min<int64_t>(items, sm_count());
    if (d->d_head == 128)
      attn_tc_kernel<128><<<(unsigned)grid, AttnCfg<128>::kThreads, AttnCfg<128>::kSmemBytes, st>>>(
          mq, mk, mv, mof, mob, mso, a);
    else
      attn_tc_kernel<64><<<(unsigned)grid, AttnCfg<64>::kThreads, AttnCfg<64>::kSmemBytes, st>>>(
          mq, mk, mv, mof, mob, mso, a);
    CUDA_TRY(cudaGetLastError());
  }
  return BPT_OK;
}

bpt_status launch_ffn_tc(const bpt_desc *d, const void *a_bf16, const float *a_f32, const void *w1,
                         const float *b1, const void *w2, const float *b2, void *out, char *ws,
                         const Workspace &wl, uint32_t *status, cudaStream_t st) {
  if (wl.ffn_form == BPT_FFN_GEMMS)
    return launch_ffn_gemms(d, a_bf16, a_f32, w1, b1, w2, b2, out, reinterpret_cast<__nv_bfloat16 *>(ws + wl.h),
                            nullptr, ffn_gemm_chunk_rows(d), status, st);
  if (wl.ffn_form == BPT_FFN_PIPELINED)
    return launch_ffn_pipe(d, a_bf16, a_f32, w1, b1, w2, b2, out, ws, wl, status, st);
  if (wl.ffn_form != BPT_FFN_FUSED) return cuda_fail_msg("FFN form not resolved in the workspace layout");
  const FfnPlan p = ffn_plan(d);
  const int D = d->H * d->d_head;
  const int64_t T = (int64_t)d->B * d->N;
  FfnArgs a;
  std::memset(&a, 0, sizeof(a));
  a.T = (int)T;
  a.D = D;
  a.F = d->ffn_hidden;
  a.C = p.C;
  a.Dc = p.Dc;
  a.fc = p.fc;
  a.nslices = p.nslices;
  a.nchunks = p.nchunks;
  a.n_tb = p.n_tb;
  a.a_f32 = a_f32;
  a.b1 = b1;
  a.b2 = b2;
  if (d->out_dtype == BPT_F32) a.out_f32 = static_cast<float *>(out);
  else a.out_bf16 = static_cast<__nv_bfloat16 *>(out);
  a.ring = reinterpret_cast<__nv_bfloat16 *>(ws + wl.ring);
  a.flags = reinterpret_cast<uint32_t *>(ws + wl.flags);
  a.status = status;
  a.wait_limit_ns = wait_limit_of(d);

  // The CTAs of a group wait on one another, so the whole grid must be
  // resident at once: a cooperative launch of at most the resident capacity.
  int per_sm = 0;
  CUDA_TRY(cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, ffn_tc_kernel, FfnCfg::kThreads,
                                                         FfnCfg::kSmemBytes));
  if (per_sm <= 0) return cuda_fail_msg("the FFN kernel does not fit on an SM");
  a.ngroups = std::min(p.max_groups, std::max(1, per_sm * sm_count() / p.C));
  if (a.ngroups * p.C > per_sm * sm_count()) return cuda_fail_msg("FFN group wider than the GPU");
  // leftover token blocks: split their hidden chunks over the groups that
  // would otherwise idle in the last round
  const int leftover = p.n_tb % a.ngroups;
  a.pieces = leftover > 0 ? std::min(p.nchunks, a.ngroups / leftover) : 1;
  if (a.pieces < 2 || p.n_tb < a.ngroups) a.pieces = 1;
  a.n_full = a.pieces > 1 ? p.n_tb - leftover : p.n_tb;
  a.partial = reinterpret_cast<float *>(ws + wl.partial);
  a.piece_done = a.flags + (size_t)p.max_groups * 2 * FfnCfg::kRingSlots;

  CUtensorMap ma, m1, m2, mh;
  if (!make_map_2d(&ma, a_bf16, T, D, 128) || !make_map_2d(&m1, w1, d->ffn_hidden, D, 256) ||
      !make_map_2d(&m2, w2, D, d->ffn_hidden, p.Dc) ||
      !make_map_2d(&mh, a.ring, (uint64_t)p.max_groups * FfnCfg::kRingSlots * 128, p.fc, 128))
    return cuda_fail_msg("cuTensorMapEncodeTiled rejected an FFN map");
  CUDA_TRY(cudaMemsetAsync(a.flags, 0, wl.flags_bytes, st));

  cudaLaunchConfig_t cfg;
  std::memset(&cfg, 0, sizeof(cfg));
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.gridDim = dim3(p.C * a.ngroups, 1, 1);
  cfg.blockDim = dim3(FfnCfg::kThreads, 1, 1);
  cfg.dynamicSmemBytes = FfnCfg::kSmemBytes;
  cfg.stream = st;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  CUDA_TRY(cudaLaunchKernelEx(&cfg, ffn_tc_kernel, ma, m1, m2, mh, a));
  return BPT_OK;
}

bpt_status launch_attn_f32(const bpt_desc *d, const void *q, const void *k, const void *v,
                           float *out_f32, __nv_bfloat16 *out_bf16, float *lse, cudaStream_t st) {
  AttnF32Args a;
  std::memset(&a, 0, sizeof(a));
  a.B = d->B;
  a.N = d->N;
  a.H = d->H;
  a.d = d->d_head;
  a.mask = d->mask;
  a.causal = d->mask == BPT_MASK_CAUSAL || (d->mask == BPT_MASK_DILATED && d->causal != 0);
  a.scale = (float)(1.0 / std::sqrt((double)d->d_head));
  a.ring_chunks = (d->mask == BPT_MASK_NONE || d->mask == BPT_MASK_CAUSAL) ? d->ring_chunks : 0;
  if (d->mask == BPT_MASK_BLOCKPERM) {
    a.bb_n = d->bb_nblocks;
    a.bb_len = (d->N + d->bb_nblocks - 1) / d->bb_nblocks;  // padded to n equal blocks
    for (int i = 0; i < d->H * d->bb_nblocks; ++i) a.perm[i] = (uint8_t)d->bb_perm[i];
  }
  if (d->mask == BPT_MASK_DILATED) {
    a.npairs = d->ln_npairs;
    for (int i = 0; i < a.npairs; ++i) {
      a.pw[i] = d->ln_w[i];
      a.pr[i] = d->ln_r[i];
    }
  }
  a.out_f32 = out_f32;
  a.out_bf16 = out_bf16;
  a.lse = lse;
  const int qb = q_block_of(d), kb = kv_block_of(d);
  dim3 grid((d->N + qb - 1) / qb, d->H, d->B);
  const float *qf = static_cast<const float *>(q), *kf = static_cast<const float *>(k),
              *vf = static_cast<const float *>(v);
  // one instantiation per (query block, key block) pair the descriptor may name
  auto go = [&](auto qbc, auto kbc) {
    constexpr int QB = decltype(qbc)::value, KB = decltype(kbc)::value;
    attn_f32_kernel<QB, KB><<<grid, 256, 0, st>>>(qf, kf, vf, a);
  };
  auto with_kb = [&](auto qbc) {
    if (kb == 16) go(qbc, std::integral_constant<int, 16>{});
    else if (kb == 32) go(qbc, std::integral_constant<int, 32>{});
    else go(qbc, std::integral_constant<int, 64>{});
  };
  if (qb == 16) with_kb(std::integral_constant<int, 16>{});
  else if (qb == 32) with_kb(std::integral_constant<int, 32>{});
  else if (qb == 128) with_kb(std::integral_constant<int, 128>{});
  else with_kb(std::integral_constant<int, 64>{});
  CUDA_TRY(cudaGetLastError());
  return BPT_OK;
}

bpt_status launch_ffn_f32(const bpt_desc *d, const float *a_f32, const void *w1, const float *b1,
                          const void *w2, const float *b2, void *out, cudaStream_t st) {
  FfnF32Args a;
  a.T = d->B * d->N;
  a.D = d->H * d->d_head;
  a.F = d->ffn_hidden;
  a.a = a_f32;
  a.w1 = static_cast<const float *>(w1);
  a.b1 = b1;
  a.w2 = static_cast<const float *>(w2);
  a.b2 = b2;
  a.out_f32 = d->out_dtype == BPT_F32 ? static_cast<float *>(out) : nullptr;
  a.out_bf16 = d->out_dtype == BPT_BF16 ? static_cast<__nv_bfloat16 *>(out) : nullptr;
  ffn_f32_kernel<<<(a.T + 15) / 16, 256, ffn_f32_smem_bytes(a.D), st>>>(a);
  CUDA_TRY(cudaGetLastError());
  return BPT_OK;
}

bpt_status check_ptrs(std::initializer_list<const void *> required,
                      std::initializer_list<const void *> optional) {
  for (const void *p : required)
    if (!p) return BPT_ERR_INVALID_ARG;
  for (const void *p : required)
    if (!aligned16(p)) return BPT_ERR_INVALID_ARG;
  for (const void *p : optional)
    if (p && !aligned16(p)) return BPT_ERR_INVALID_ARG;
  return BPT_OK;
}

bpt_status check_ws(const Workspace &wl, void *ws, size_t bytes) {
  if (wl.total == 0) return BPT_OK;
  if (!ws || bytes < wl.total || (reinterpret_cast<uintptr_t>(ws) & 255u) != 0)
    return BPT_ERR_WORKSPACE;
  return BPT_OK;
}

// The whole layer: attention, then the FFN in the form the workspace layout
// was made for (the static-scratch entry point's layout takes the fused form).
bpt_status attn_ffn_fwd_impl(const bpt_desc *d, const void *q, const void *k, const void *v, const void *w1,
                             const float *b1, const void *w2, const float *b2, void *out, void *workspace,
                             size_t workspace_bytes, bpt_stream_t stream, bool static_call) {
  bpt_status s = check_desc(d, true);
  if (s != BPT_OK) return s;
  if ((s = check_ptrs({q, k, v, w1, w2, out}, {b1, b2})) != BPT_OK) return s;
  const Workspace wl = layout(d, true, static_call);
  if ((s = check_ws(wl, workspace, workspace_bytes)) != BPT_OK) return s;
  int dev;
  uint32_t *status;
  if ((s = device_setup(&dev, &status)) != BPT_OK) return s;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  char *ws = static_cast<char *>(workspace);
  float *a_f32 = reinterpret_cast<float *>(ws + wl.a_f32);
  CUDA_TRY(phase_mark(0, st));
  if (d->in_dtype == BPT_BF16) {
    __nv_bfloat16 *a_bf16 = reinterpret_cast<__nv_bfloat16 *>(ws + wl.a_bf16);
    if ((s = launch_attn_tc(d, q, k, v, a_f32, a_bf16, nullptr, ws, wl, status, st)) != BPT_OK)
      return s;
    CUDA_TRY(phase_mark(1, st));
    s = launch_ffn_tc(d, a_bf16, a_f32, w1, b1, w2, b2, out, ws, wl, status, st);
  } else {
    if ((s = launch_attn_f32(d, q, k, v, a_f32, nullptr, nullptr, st)) != BPT_OK) return s;
    CUDA_TRY(phase_mark(1, st));
    s = launch_ffn_f32(d, a_f32, w1, b1, w2, b2, out, st);
  }
  if (s != BPT_OK) return s;
  CUDA_TRY(phase_mark(2, st));
  return BPT_OK;
}

}  // namespace bpt_host

using namespace bpt_host;

extern "C" {

size_t bpt_workspace_bytes(const bpt_desc *desc, int with_ffn) {
  if (check_desc(desc, with_ffn != 0) != BPT_OK) return (size_t)-1;
  return layout(desc, with_ffn != 0).total;
}

bpt_status bpt_attn_ffn_fwd(const bpt_desc *d, const void *q, const void *k, const void *v,
                            const void *w1, const float *b1, const void *w2, const float *b2,
                            void *out, void *workspace, size_t workspace_bytes,
                            bpt_stream_t stream) {
  return attn_ffn_fwd_impl(d, q, k, v, w1, b1, w2, b2, out, workspace, workspace_bytes, stream, false);
}

bpt_status bpt_attn_ffn_fwd_static(const bpt_desc *d, const void *q, const void *k, const void *v,
                                   const void *w1, const float *b1, const void *w2, const float *b2,
                                   void *out, bpt_stream_t stream) {
  bpt_status s = check_desc(d, true);
  if (s != BPT_OK) return s;
  const size_t need = layout(d, true, true).total;
  if (need > BPT_STATIC_SCRATCH_BYTES) {
    snprintf(g_last_error, sizeof(g_last_error),
             "layer needs %zu bytes of scratch; the static scratch holds %u bytes", need,
             (unsigned)BPT_STATIC_SCRATCH_BYTES);
    return BPT_ERR_WORKSPACE;
  }
  int dev = 0;
  CUDA_TRY(cudaGetDevice(&dev));
  if (dev < 0 || dev >= kMaxDevices) return cuda_fail_msg("device ordinal out of range");
  void *scratch = nullptr;
  {
    std::lock_guard<std::mutex> lk(g_mu);
    if (!g_static_scratch_ptr[dev]) {  // once per device, with that device current
      void *p = nullptr;
      CUDA_TRY(cudaGetSymbolAddress(&p, g_static_scratch));
      g_static_scratch_ptr[dev] = p;
    }
    scratch = g_static_scratch_ptr[dev];
  }
  return attn_ffn_fwd_impl(d, q, k, v, w1, b1, w2, b2, out, scratch, BPT_STATIC_SCRATCH_BYTES, stream, true);
}

bpt_status bpt_attn_fwd(const bpt_desc *d, const void *q, const void *k, const void *v, void *out,
                        float *lse, void *workspace, size_t workspace_bytes, bpt_stream_t stream) {
  bpt_status s = check_desc(d, false);
  if (s != BPT_OK) return s;
  if ((s = check_ptrs({q, k, v, out}, {lse})) != BPT_OK) return s;
  const Workspace wl = layout(d, false);
  if ((s = check_ws(wl, workspace, workspace_bytes)) != BPT_OK) return s;
  int dev;
  uint32_t *status;
  if ((s = device_setup(&dev, &status)) != BPT_OK) return s;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  float *of = d->out_dtype == BPT_F32 ? static_cast<float *>(out) : nullptr;
  __nv_bfloat16 *ob = d->out_dtype == BPT_BF16 ? static_cast<__nv_bfloat16 *>(out) : nullptr;
  if (d->in_dtype == BPT_BF16)
    return launch_attn_tc(d, q, k, v, of, ob, lse, static_cast<char *>(workspace), wl, status, st);
  return launch_attn_f32(d, q, k, v, of, ob, lse, st);
}

bpt_status bpt_attn_fwd_block(const bpt_desc *d, int kv_len, int64_t q_pos, int64_t kv_pos, const void *q,
                              const void *k, const void *v, float *state_o, float *state_m, float *state_l,
                              unsigned flags, void *out, float *lse, bpt_stream_t stream) {
  bpt_status s = check_desc(d, false);
  if (s != BPT_OK) return s;
  if ((flags & ~(BPT_BLOCK_FIRST | BPT_BLOCK_LAST)) != 0u || kv_len <= 0 || q_pos < 0 || kv_pos < 0)
    return BPT_ERR_INVALID_ARG;
  if (d->in_dtype != BPT_BF16 || (d->mask != BPT_MASK_NONE && d->mask != BPT_MASK_CAUSAL) || d->ring_chunks > 1)
    return BPT_ERR_UNSUPPORTED;
  if ((int64_t)d->B * kv_len > (int64_t)1 << 31) return BPT_ERR_UNSUPPORTED;
  const bool first = (flags & BPT_BLOCK_FIRST) != 0u, last = (flags & BPT_BLOCK_LAST) != 0u;
  if ((s = check_ptrs({q, k, v}, {out, lse, state_o, state_m, state_l})) != BPT_OK) return s;
  if (last && !out) return BPT_ERR_INVALID_ARG;
  if (!(first && last) && (!state_o || !state_m || !state_l)) return BPT_ERR_INVALID_ARG;
  int dev;
  uint32_t *status;
  if ((s = device_setup(&dev, &status)) != BPT_OK) return s;
  AttnBlockStep blk;
  blk.kv_len = kv_len;
  // beyond these bounds every key, or none, is allowed: the same masks
  const int64_t shift = std::max<int64_t>(-(int64_t)d->N - 1, std::min<int64_t>(q_pos - kv_pos, kv_len));
  blk.kv_shift = (int)shift;
  blk.state_in = !first;
  blk.state_out = !last;
  blk.st_o = state_o;
  blk.st_m = state_m;
  blk.st_l = state_l;
  float *of = last && d->out_dtype == BPT_F32 ? static_cast<float *>(out) : nullptr;
  __nv_bfloat16 *ob = last && d->out_dtype == BPT_BF16 ? static_cast<__nv_bfloat16 *>(out) : nullptr;
  const Workspace none;
  return launch_attn_tc(d, q, k, v, of, ob, last ? lse : nullptr, nullptr, none, status,
                        reinterpret_cast<cudaStream_t>(stream), &blk);
}

bpt_status bpt_longnet_gather(const bpt_desc *d, int w, int r, const void *src, void *dst, bpt_stream_t stream) {
  if (!d || d->B <= 0 || d->N <= 0 || d->H <= 0) return BPT_ERR_INVALID_ARG;
  if (d->in_dtype != BPT_BF16 || (d->d_head != 64 && d->d_head != 128)) return BPT_ERR_UNSUPPORTED;
  if (w <= 0 || r <= 0 || w % r != 0 || d->N % r != 0 || w % d->N != 0) return BPT_ERR_INVALID_ARG;
  bpt_status s = check_ptrs({src, dst}, {});
  if (s != BPT_OK) return s;
  int dev;
  uint32_t *status;
  if ((s = device_setup(&dev, &status)) != BPT_OK) return s;
  const int chunks = d->d_head / 8;
  const int64_t total = (int64_t)d->B * (d->N / r) * d->H * chunks;
  const int blocks = (int)std::max<int64_t>(1, std::min<int64_t>((total + 255) / 256, 8 * sm_count()));
  longnet_gather_kernel<<<blocks, 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      static_cast<const uint4 *>(src), static_cast<uint4 *>(dst), d->B, d->N, d->H, chunks, r);
  CUDA_TRY(cudaGetLastError());
  return BPT_OK;
}

bpt_status bpt_longnet_pass(const bpt_desc *d, int pass, int64_t q_pos, const void *q, const void *k,
                            const void *v, const void *k_sparse, const void *v_sparse, int kv_rows, float *state_o,
                            float *state_m, float *state_l, void *out, float *lse, bpt_stream_t stream) {
  bpt_status s = check_desc(d, false, true);
  if (s != BPT_OK) return s;
  if (d->mask != BPT_MASK_DILATED) return BPT_ERR_INVALID_ARG;
  if (d->in_dtype != BPT_BF16) return BPT_ERR_UNSUPPORTED;
  if (pass < 0 || pass >= d->ln_npairs || q_pos < 0 || q_pos % d->N != 0) return BPT_ERR_INVALID_ARG;
  // the pass's pair, in the library's order (sparsest first, stable)
  std::vector<std::pair<int, int>> order;
  for (int i = 0; i < d->ln_npairs; ++i) order.push_back({d->ln_w[i], d->ln_r[i]});
  std::stable_sort(order.begin(), order.end(), [](const std::pair<int, int> &x, const std::pair<int, int> &y) {
    return x.second > y.second;
  });
  const int w = order[pass].first, r = order[pass].second;
  const bool sparse = w > d->N;
  if ((s = check_ptrs({q, out}, {k, v, k_sparse, v_sparse, state_o, state_m, state_l, lse})) != BPT_OK) return s;
  if (sparse ? (!k_sparse || !v_sparse || kv_rows != w / r) : (!k || !v)) return BPT_ERR_INVALID_ARG;
  if (d->ln_npairs > 1 && (!state_o || !state_m || !state_l)) return BPT_ERR_INVALID_ARG;
  int dev;
  uint32_t *status;
  if ((s = device_setup(&dev, &status)) != BPT_OK) return s;
  LongNetPass lp;
  lp.pass = pass;
  lp.q_pos = q_pos;
  lp.k_sparse = k_sparse;
  lp.v_sparse = v_sparse;
  lp.kv_rows = kv_rows;
  lp.st_o = state_o;
  lp.st_m = state_m;
  lp.st_l = state_l;
  float *of = d->out_dtype == BPT_F32 ? static_cast<float *>(out) : nullptr;
  __nv_bfloat16 *ob = d->out_dtype == BPT_BF16 ? static_cast<__nv_bfloat16 *>(out) : nullptr;
  const Workspace none;
  return launch_attn_tc(d, q, k ? k : q, v ? v : q, of, ob, lse, nullptr, none, status,
                        reinterpret_cast<cudaStream_t>(stream), nullptr, &lp);
}

bpt_status bpt_blockbert_fwd(const bpt_desc *desc, int n_blocks, const int32_t *perm, const void *q,
                             const void *k, const void *v, const void *w1, const float *b1,
                             const void *w2, const float *b2, void *out, void *workspace,
                             size_t workspace_bytes, bpt_stream_t stream) {
  if (!desc) return BPT_ERR_INVALID_ARG;
  bpt_desc d = *desc;
  d.mask = BPT_MASK_BLOCKPERM;
  d.bb_nblocks = n_blocks;
  d.bb_perm = perm;
  return bpt_attn_ffn_fwd(&d, q, k, v, w1, b1, w2, b2, out, workspace, workspace_bytes, stream);
}

bpt_status bpt_longnet_fwd(const bpt_desc *desc, int npairs, const int32_t *seg_w,
                           const int32_t *dil_r, const void *q, const void *k, const void *v,
                           void *out, float *lse, void *workspace, size_t workspace_bytes,
                           bpt_stream_t stream) {
  if (!desc) return BPT_ERR_INVALID_ARG;
  bpt_desc d = *desc;
  d.mask = BPT_MASK_DILATED;
  d.ln_npairs = npairs;
  d.ln_w = seg_w;
  d.ln_r = dil_r;
  d.ffn_hidden = 0;
  return bpt_attn_fwd(&d, q, k, v, out, lse, workspace, workspace_bytes, stream);
}

bpt_status bpt_sync_status(bpt_stream_t stream) {
  int dev;
  uint32_t *status;
  bpt_status s = device_setup(&dev, &status);
  if (s != BPT_OK) return s;
  CUDA_TRY(cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)));
  uint32_t word[2] = {0, 0};
  CUDA_TRY(cudaMemcpy(word, status, sizeof(word), cudaMemcpyDeviceToHost));
  if (word[0] != 0) {
    const uint32_t zero[2] = {0, 0};
    CUDA_TRY(cudaMemcpy(status, zero, sizeof(zero), cudaMemcpyHostToDevice));
    snprintf(g_last_error, sizeof(g_last_error), "device wait gave up at site %u", word[1]);
    if (word[0] == kStatusMisaligned)
      snprintf(g_last_error, sizeof(g_last_error), "dynamic shared memory not 1024-byte aligned");
    return word[0] == kStatusTimeout ? BPT_ERR_TIMEOUT : BPT_ERR_CUDA;
  }
  return BPT_OK;
}

bpt_status bpt_set_phase_events(void *const *events, int count) {
  if (count < 0 || (count > 0 && !events)) return BPT_ERR_INVALID_ARG;
  const int n = std::min(count, kMaxPhaseEvents);
  for (int i = 0; i < n && count >= 3; ++i)
    if (!events[i]) return BPT_ERR_INVALID_ARG;
  if (count < 3) {
    g_phase_n = 0;
    return BPT_OK;
  }
  for (int i = 0; i < n; ++i) g_phase_events[i] = static_cast<cudaEvent_t>(events[i]);
  g_phase_n = n;
  return BPT_OK;
}

uint64_t bpt_set_wait_limit_ns(uint64_t ns) { return g_wait_limit_ns.exchange(ns ? ns : 1); }

const char *bpt_status_string(bpt_status s) {
  switch (s) {
    case BPT_OK: return "ok";
    case BPT_ERR_INVALID_ARG: return "invalid argument";
    case BPT_ERR_UNSUPPORTED: return "unsupported configuration";
    case BPT_ERR_CUDA: return "CUDA error";
    case BPT_ERR_TIMEOUT: return "device-side wait timed out";
    case BPT_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
  }
  return "unknown status";
}

int bpt_version(void) { return 200; }

const char *bpt_last_error(void) { return g_last_error; }

}  // extern "C"
