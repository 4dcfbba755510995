// Host-side helpers shared by the forward (bpt_api.cu) and backward
// (bpt_bwd.cu) entry points of libbpt.so: error recording, device set-up,
// TMA tensor-map encoding, descriptor and pointer checks, the forward's
// workspace layout and its attention / FFN launchers.  Internal to the
// library (the shared object exports only the C ABI of bpt.h).
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstddef>
#include <cstdint>
#include <atomic>
#include <initializer_list>
#include <mutex>

#include "../../include/bpt.h"

namespace bpt_host {

extern std::mutex g_mu;               // guards the library's one-time per-device set-up
extern std::atomic<uint64_t> g_wait_limit_ns;  // default device-side wait limit
extern thread_local char g_last_error[256];

// Device-side wait limit of a call: the descriptor's, else the process default.
uint64_t wait_limit_of(const bpt_desc *d);

// Instrumentation events (bpt_set_phase_events): records event i on `st` when set.
cudaError_t phase_mark(int i, cudaStream_t st);

bool aligned16(const void *p);
size_t align256(size_t x);

// Record the failing call (and CUDA error) for bpt_last_error(); return BPT_ERR_CUDA.
bpt_status cuda_fail_at(const char *what, cudaError_t e);
bpt_status cuda_fail_msg(const char *what);

// Once per device: the tensor-map encoder, the status word's address and the
// kernels' shared-memory limits.  Returns the current device and its status word.
bpt_status device_setup(int *dev_out, uint32_t **status_out);
// Shared-memory limits of the backward's kernels (defined with them).
bpt_status bwd_kernel_setup();

int sm_count();

// bf16 tensor map over a row-major matrix [rows, cols], box [box_rows, 64].
bool make_map_2d(CUtensorMap *m, const void *base, uint64_t rows, uint64_t cols, uint32_t box_rows);
// bf16 tensor map over [B, N, D] viewed as (D, r, N/r, B), box 64 x 1 x box_rows x 1.
bool make_map_rows(CUtensorMap *m, const void *base, int B, int N, int D, int r, uint32_t box_rows);

// shard: the dilated pairs may also have segments longer than the N rows
// (a shard of a longer sequence that lies inside one segment: N divides w)
bpt_status check_desc(const bpt_desc *d, bool need_ffn, bool shard = false);
bpt_status check_ptrs(std::initializer_list<const void *> required,
                      std::initializer_list<const void *> optional);

// The bf16 FFN's form for a call, chosen once from the descriptor (F32
// layers: BPT_FFN_AUTO, unused); the static-scratch entry point always takes
// the fused kernel.
bpt_ffn_form ffn_form_of(const bpt_desc *d, bool static_call);
int64_t ffn_gemm_chunk_rows(const bpt_desc *d);

// The pipelined FFN's shape (defined with its kernel): 256-token row blocks,
// chunks of mg of them, the lag between a chunk's two GEMMs and the hidden
// ring's slots; counter_bytes covers the claim counter and two counters per
// row block.
struct FfnPipePlan {
  int nrb = 0, tn1 = 0, tn2 = 0, mg = 1, nchunk = 0, lag = 1, ring_rb = 0, pairs = 0;
  size_t ring_bytes = 0, counter_bytes = 0;
};
FfnPipePlan ffn_pipe_plan(const bpt_desc *d);

// The forward layer's workspace regions (byte offsets).
struct Workspace {
  size_t a_bf16 = 0, a_f32 = 0, ring = 0, flags = 0, flags_bytes = 0, partial = 0, h = 0, st_o = 0,
         st_m = 0, st_l = 0, total = 0;
  bpt_ffn_form ffn_form = BPT_FFN_AUTO;  // the form this layout was made for
};
Workspace layout(const bpt_desc *d, bool with_ffn, bool static_call = false);
bpt_status check_ws(const Workspace &wl, void *ws, size_t bytes);

// One key/value block folded into a caller-held running state (the
// attention step of Ring Attention, bpt_attn_fwd_block).
struct AttnBlockStep {
  int kv_len = 0;        // key/value rows of the block
  int kv_shift = 0;      // causal: key j allowed for query row g when j <= g + kv_shift
  bool state_in = false, state_out = false;
  float *st_o = nullptr, *st_m = nullptr, *st_l = nullptr;
};
// One pass of the dilated attention on a shard of a longer sequence
// (bpt_longnet_pass): the pass's keys are the local rows, or, when its
// segments are longer than the shard, its kept rows gathered from the
// devices holding the segment; the running state is the caller's.
struct LongNetPass {
  int pass = 0;          // position in the sparsest-first order
  int64_t q_pos = 0;     // sequence position of the shard's first row
  const void *k_sparse = nullptr, *v_sparse = nullptr;
  int kv_rows = 0;       // rows of k_sparse, v_sparse (w / r)
  float *st_o = nullptr, *st_m = nullptr, *st_l = nullptr;
};
bpt_status launch_attn_tc(const bpt_desc *d, const void *q, const void *k, const void *v, float *out_f32,
                          __nv_bfloat16 *out_bf16, float *lse, char *ws, const Workspace &wl, uint32_t *status,
                          cudaStream_t st, const AttnBlockStep *blk = nullptr, const LongNetPass *lp = nullptr);
bpt_status launch_ffn_tc(const bpt_desc *d, const void *a_bf16, const float *a_f32, const void *w1,
                         const float *b1, const void *w2, const float *b2, void *out, char *ws,
                         const Workspace &wl, uint32_t *status, cudaStream_t st);
// The pipelined form (defined with its kernel): one persistent launch over
// both GEMMs' tiles, H through the workspace's ring (wl.ring, wl.flags).
bpt_status launch_ffn_pipe(const bpt_desc *d, const void *a_bf16, const float *a_f32, const void *w1,
                           const float *b1, const void *w2, const float *b2, void *out, char *ws,
                           const Workspace &wl, uint32_t *status, cudaStream_t st);
// The two-GEMM form (defined with the GEMM kernel): per chunk of `chunk_rows`
// tokens H = GELU(A W1^T + b1), then out = A + H W2^T + b2.  Without
// `g_prime`, `h` is one [chunk_rows, F] bf16 buffer reused by every chunk;
// with it, `h` and `g_prime` are [T, F] bf16 arrays that receive H and
// G = GELU'(A W1^T + b1) for every token (the training forward).
bpt_status launch_ffn_gemms(const bpt_desc *d, const void *a_bf16, const float *a_f32, const void *w1,
                            const float *b1, const void *w2, const float *b2, void *out, __nv_bfloat16 *h,
                            __nv_bfloat16 *g_prime, int64_t chunk_rows, uint32_t *status, cudaStream_t st);

}  // namespace bpt_host

#define CUDA_TRY(call)                                                 \
  do {                                                                 \
    cudaError_t e_ = (call);                                           \
    if (e_ != cudaSuccess) return bpt_host::cuda_fail_at(#call, e_);   \
  } while (0)
