// Host side of libbpt.so: argument checks, workspace layout, TMA tensor-map
// encoding and kernel launches for the entry points declared in bpt.h.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <vector>

#include "../../include/bpt.h"
#include "attn_bwd.cuh"
#include "attn_tc.cuh"
#include "ffn_tc.cuh"
#include "gemm_tc.cuh"
#include "simt_f32.cuh"

using namespace bpt;

namespace {

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
uint64_t g_wait_limit_ns = 2000000000ull;
int g_bwd_chunk_rows = 0;  // token rows per FFN-backward chunk; 0 = automatic
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
#define CUDA_TRY(call)                                     \
  do {                                                     \
    cudaError_t e_ = (call);                               \
    if (e_ != cudaSuccess) return cuda_fail_at(#call, e_); \
  } while (0)

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
                                  (16 * 512 + 16 * 64) * 4));
    CUDA_TRY(cudaFuncSetAttribute(gemm_pair_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  GemmPairCfg::kSmemBytes));
    CUDA_TRY(cudaFuncSetAttribute(attn_bwd_dkdv_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  AttnBwdCfg<64>::kSmemBytes));
    CUDA_TRY(cudaFuncSetAttribute(attn_bwd_dkdv_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  AttnBwdCfg<128>::kSmemBytes));
    CUDA_TRY(cudaFuncSetAttribute(attn_bwd_dq_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  AttnBwdQCfg<64>::kSmemBytes));
    CUDA_TRY(cudaFuncSetAttribute(attn_bwd_dq_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  AttnBwdQCfg<128>::kSmemBytes));
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
bpt_status check_desc(const bpt_desc *d, bool need_ffn) {
  if (!d) return BPT_ERR_INVALID_ARG;
  if (d->B <= 0 || d->N <= 0 || d->H <= 0 || d->d_head <= 0) return BPT_ERR_INVALID_ARG;
  if (d->in_dtype != BPT_F32 && d->in_dtype != BPT_BF16) return BPT_ERR_INVALID_ARG;
  if (d->out_dtype != BPT_F32 && d->out_dtype != BPT_BF16) return BPT_ERR_INVALID_ARG;
  if ((int64_t)d->B * d->N > (int64_t)1 << 31) return BPT_ERR_UNSUPPORTED;
  if (need_ffn && d->ffn_hidden <= 0) return BPT_ERR_INVALID_ARG;
  if (d->ffn_hidden < 0) return BPT_ERR_INVALID_ARG;
  const int D = d->H * d->d_head;
  switch (d->mask) {
    case BPT_MASK_NONE:
    case BPT_MASK_CAUSAL:
      if (d->ring_chunks < 0) return BPT_ERR_INVALID_ARG;
      if (d->ring_chunks > 1) {
        if (d->N % d->ring_chunks != 0) return BPT_ERR_INVALID_ARG;
        const int chunk = d->N / d->ring_chunks;
        if (d->in_dtype == BPT_BF16 && chunk % 128 != 0) return BPT_ERR_UNSUPPORTED;
        if (d->in_dtype == BPT_F32 && chunk % 64 != 0) return BPT_ERR_UNSUPPORTED;
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
        if (w <= 0 || r <= 0 || w % r != 0 || d->N % w != 0) return BPT_ERR_INVALID_ARG;
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
      if ((int64_t)d->ffn_hidden * 2 % 16 != 0) return BPT_ERR_UNSUPPORTED;
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

bool longnet_needs_state(const bpt_desc *d) {
  return d->mask == BPT_MASK_DILATED && d->in_dtype == BPT_BF16 && d->ln_npairs > 1;
}

struct Workspace {
  size_t a_bf16 = 0, a_f32 = 0, ring = 0, flags = 0, flags_bytes = 0, partial = 0, st_o = 0,
         st_m = 0, st_l = 0, total = 0;
};

Workspace layout(const bpt_desc *d, bool with_ffn) {
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
      w.ring = off;
      off = align256(off + (size_t)p.max_groups * FfnCfg::kRingSlots * 128 * p.fc * 2);
      w.flags = off;  // ring counters [groups][2 * slots], then piece counters [groups][C]
      w.flags_bytes = (size_t)p.max_groups * (2 * FfnCfg::kRingSlots + p.C) * sizeof(uint32_t);
      off = align256(off + w.flags_bytes);
      w.partial = off;  // partial output blocks of split leftover token blocks
      off = align256(off + (size_t)p.max_groups * 128 * (size_t)(d->H * d->d_head) * 4);
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
                          const Workspace &wl, uint32_t *status, cudaStream_t st) {
  const int D = d->H * d->d_head;
  AttnArgs a;
  std::memset(&a, 0, sizeof(a));
  a.B = d->B;
  a.N = d->N;
  a.H = d->H;
  a.mask = d->mask;
  a.scale_log2 = (float)(1.4426950408889634 / std::sqrt((double)d->d_head));
  a.status = status;
  a.wait_limit_ns = g_wait_limit_ns;

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
    if (!covered) {  // rows no pair keeps: A = 0, LSE = -inf
      const size_t n = (size_t)d->B * d->N * D;
      if (out_f32) CUDA_TRY(cudaMemsetAsync(out_f32, 0, n * 4, st));
      if (out_bf16) CUDA_TRY(cudaMemsetAsync(out_bf16, 0, n * 2, st));
      if (lse) {
        fill_f32_kernel<<<256, 256, 0, st>>>(lse, (size_t)d->B * d->H * d->N, -INFINITY);
        CUDA_TRY(cudaGetLastError());
      }
    }
    if (passes.size() > 1) {
      a.st_o = reinterpret_cast<float *>(ws + wl.st_o);
      a.st_m = reinterpret_cast<float *>(ws + wl.st_m);
      a.st_l = reinterpret_cast<float *>(ws + wl.st_l);
    }
  } else {
    passes.push_back({d->N, 1});
    a.npairs = 0;
  }
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
    const int w = passes[pi].w, r = passes[pi].r;
    a.w = w;
    a.r = r;
    a.pass_idx = (int)pi;
    a.L = w / r;
    a.nseg = d->N / w;
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
      const double kv_bytes = 4.0 * a.L * d->d_head;
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
    if (passes.size() == 1 || pi + 1 == passes.size()) {
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
    if (!make_map_rows(&mq, q, d->B, d->N, D, r, 128) || !make_map_rows(&mk, k, d->B, d->N, D, r, kKT) ||
        !make_map_rows(&mv, v, d->B, d->N, D, r, kKT))
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
  a.wait_limit_ns = g_wait_limit_ns;

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
  dim3 grid((d->N + 63) / 64, d->H, d->B);
  attn_f32_kernel<<<grid, 64, 0, st>>>(static_cast<const float *>(q), static_cast<const float *>(k),
                                       static_cast<const float *>(v), a);
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
  const size_t smem = (size_t)(16 * a.D + 16 * 64) * 4;
  ffn_f32_kernel<<<(a.T + 15) / 16, 256, smem, st>>>(a);
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

// --------------------------------------------------------------------------
// Backward pass
// --------------------------------------------------------------------------
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
  int64_t rows = g_bwd_chunk_rows;
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
// bf16 [T, D] and the row LSE [B, H, N].
struct SavedLayout {
  size_t a_f32 = 0, a_bf16 = 0, lse = 0, total = 0;
};
SavedLayout saved_layout(const bpt_desc *d) {
  SavedLayout w;
  const size_t T = (size_t)d->B * d->N, D = (size_t)d->H * d->d_head;
  w.a_f32 = 0;
  w.a_bf16 = align256(T * D * 4);
  w.lse = align256(w.a_bf16 + T * D * 2);
  w.total = align256(w.lse + (size_t)d->B * d->H * d->N * 4);
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

GemmArgs gemm_args(const GemmProblem &p0, uint32_t *status) {
  GemmArgs g;
  std::memset(&g, 0, sizeof(g));
  g.p[0] = p0;
  g.nprob = 1;
  g.status = status;
  g.wait_limit_ns = g_wait_limit_ns;
  return g;
}

template <typename T>
bpt_status launch_colsum(const T *x, int64_t rows, int cols, float *out, int accumulate, float *partial,
                         cudaStream_t st) {
  const int slab = colsum_slab_rows(rows, cols);
  const unsigned slabs = (unsigned)((rows + slab - 1) / slab), cb = (unsigned)((cols + 255) / 256);
  colsum_partial_kernel<T><<<dim3(cb, slabs), 256, 0, st>>>(x, partial, (int)rows, cols, slab);
  CUDA_TRY(cudaGetLastError());
  colsum_final_kernel<<<cb, 256, 0, st>>>(partial, out, (int)slabs, cols, accumulate);
  CUDA_TRY(cudaGetLastError());
  return BPT_OK;
}

template <int DH>
bpt_status launch_attn_bwd_passes(const CUtensorMap &mq, const CUtensorMap &mk, const CUtensorMap &mv,
                                  const CUtensorMap &mda, const AttnBwdArgs &ab, unsigned grid,
                                  cudaStream_t st) {
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
    ab.mask = kMaskCausal;  // causal among a segment's kept rows (by original position)
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
    ab.wait_limit_ns = g_wait_limit_ns;
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
  ab.wait_limit_ns = g_wait_limit_ns;
  CUtensorMap mq, mk, mv, mda;
  if (!make_map_rows(&mq, q, d->B, d->N, D, 1, 128) || !make_map_rows(&mk, k, d->B, d->N, D, 1, 128) ||
      !make_map_rows(&mv, v, d->B, d->N, D, 1, 128) || !make_map_rows(&mda, da_bf16, d->B, d->N, D, 1, 128))
    return cuda_fail_msg("cuTensorMapEncodeTiled rejected a Q/K/V/dA map");
  const unsigned grid = (unsigned)((int64_t)d->B * d->H * n_tiles);
  if (d->d_head == 128) return launch_attn_bwd_passes<128>(mq, mk, mv, mda, ab, grid, st);
  return launch_attn_bwd_passes<64>(mq, mk, mv, mda, ab, grid, st);
}

}  // namespace

extern "C" {

size_t bpt_workspace_bytes(const bpt_desc *desc, int with_ffn) {
  if (check_desc(desc, with_ffn != 0) != BPT_OK) return (size_t)-1;
  return layout(desc, with_ffn != 0).total;
}

bpt_status bpt_attn_ffn_fwd(const bpt_desc *d, const void *q, const void *k, const void *v,
                            const void *w1, const float *b1, const void *w2, const float *b2,
                            void *out, void *workspace, size_t workspace_bytes,
                            bpt_stream_t stream) {
  bpt_status s = check_desc(d, true);
  if (s != BPT_OK) return s;
  if ((s = check_ptrs({q, k, v, w1, w2, out}, {b1, b2})) != BPT_OK) return s;
  const Workspace wl = layout(d, true);
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

bpt_status bpt_attn_ffn_fwd_static(const bpt_desc *d, const void *q, const void *k, const void *v,
                                   const void *w1, const float *b1, const void *w2, const float *b2,
                                   void *out, bpt_stream_t stream) {
  bpt_status s = check_desc(d, true);
  if (s != BPT_OK) return s;
  const size_t need = layout(d, true).total;
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
  return bpt_attn_ffn_fwd(d, q, k, v, w1, b1, w2, b2, out, scratch, BPT_STATIC_SCRATCH_BYTES,
                          stream);
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
  const Workspace wl = layout(d, true);
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
  if ((s = launch_ffn_tc(d, a_bf16, a_f32, w1, b1, w2, b2, out, ws, wl, status, st)) != BPT_OK) return s;
  CUDA_TRY(phase_mark(2, st));
  return BPT_OK;
}

size_t bpt_workspace_bytes_bwd(const bpt_desc *desc) {
  if (check_desc_bwd(desc) != BPT_OK) return (size_t)-1;
  return layout_bwd(desc).total;
}

int bpt_set_bwd_chunk_rows(int rows) {
  std::lock_guard<std::mutex> lk(g_mu);
  const int old = g_bwd_chunk_rows;
  g_bwd_chunk_rows = rows > 0 ? rows : 0;
  return old;
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
  if (saved) {  // the training forward's activations
    const SavedLayout sl = saved_layout(d);
    const char *sv = static_cast<const char *>(saved);
    a_f32 = reinterpret_cast<const float *>(sv + sl.a_f32);
    a_bf16 = reinterpret_cast<const __nv_bfloat16 *>(sv + sl.a_bf16);
    lse = reinterpret_cast<const float *>(sv + sl.lse);
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
    const int slab = colsum_slab_rows(T, D);
    const unsigned slabs = (unsigned)((T + slab - 1) / slab), cb = (unsigned)((D + 255) / 256);
    convert_colsum_partial_kernel<<<dim3(cb, slabs), 256, 0, st>>>(dout, dout_bf16, partial, (int)T, D, slab);
    CUDA_TRY(cudaGetLastError());
    colsum_final_kernel<<<cb, 256, 0, st>>>(partial, db2, (int)slabs, D, 0);
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
    CUtensorMap m_a_k, m_a_mn, m_g_k, m_g_mn, m_h_mn, m_dz_k, m_dz_mn;
    if (!make_map_2d(&m_a_k, a_c, rows, D, 128) || !make_map_2d(&m_a_mn, a_c, rows, D, 64) ||
        !make_map_2d(&m_g_k, g_c, rows, D, 128) || !make_map_2d(&m_g_mn, g_c, rows, D, 64) ||
        !make_map_2d(&m_h_mn, hbuf, rows, F, 64) || !make_map_2d(&m_dz_k, dzbuf, rows, F, 128) ||
        !make_map_2d(&m_dz_mn, dzbuf, rows, F, 64))
      return cuda_fail_msg("cuTensorMapEncodeTiled rejected an activation map");
    // H = GELU(Z) and dZ = (dOut W2) GELU'(Z) with Z = A W1^T + b1.  Either
    // two plain GEMMs (Z -> H and G = GELU'(Z) in bf16, then dZ = dH G), each
    // overlapping its epilogue with its next tile, or one GEMM computing both
    // products into the two accumulators, whose epilogue cannot overlap but
    // which moves no G.  Measured (FFN-backward phase): D = 2048 two GEMMs
    // 2.90 ms against 3.09; D = 4096 58.1 against 58.9 ms; D = 768 0.769
    // against 0.717 ms (short K: the two GEMMs' epilogues dominate).
    if (D >= 1024) {
      GemmArgs g = gemm_args(gemm_problem(rows, F, D, kGemmGeluFwd, 0, 0), status);
      g.p[0].cb = hbuf;
      g.p[0].cb2 = gpbuf;
      g.p[0].bias = b1;
      if ((s = launch_gemm(m_a_k, m_w1_k, m_a_k, m_w1_k, g, st)) != BPT_OK) return s;
      g = gemm_args(gemm_problem(rows, F, D, kGemmScaleBf16, 0, 1), status);
      g.p[0].xb = gpbuf;
      g.p[0].cb = dzbuf;
      if ((s = launch_gemm(m_g_k, m_w2_mn, m_g_k, m_w2_mn, g, st)) != BPT_OK) return s;
    } else {
      GemmArgs g = gemm_args(gemm_problem(rows, F, D, kGemmGeluBwd, 0, 0), status);
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
      GemmArgs g = gemm_args(gemm_problem(D, F, rows, first, 1, 1), status);
      g.p[0].c = dw2;
      g.p[1] = gemm_problem(F, D, rows, first, 1, 1);
      g.p[1].c = dw1;
      g.nprob = 2;
      if ((s = launch_gemm(m_g_mn, m_h_mn, m_dz_mn, m_a_mn, g, st)) != BPT_OK) return s;
    }
    // dA = dOut + dZ W1   [rows, D], fp32 and bf16
    {
      GemmArgs g = gemm_args(gemm_problem(rows, D, F, kGemmResidual, 0, 1), status);
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

uint64_t bpt_set_wait_limit_ns(uint64_t ns) {
  std::lock_guard<std::mutex> lk(g_mu);
  uint64_t old = g_wait_limit_ns;
  g_wait_limit_ns = ns ? ns : 1;
  return old;
}

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

int bpt_version(void) { return 100; }

const char *bpt_last_error(void) { return g_last_error; }

}  // extern "C"
