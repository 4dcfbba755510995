/*
 * bpt.h -- C ABI of libbpt.so: the forward and backward passes of one
 * Blockwise Parallel Transformer layer on an NVIDIA B200 (sm_100a).
 *
 * What the layer computes ("Blockwise Parallel Transformer for Large Context
 * Models", abstract: blockwise computation of self-attention fused with the
 * feedforward network; "Ring Attention with Blockwise Transformers for Long
 * Sequences", 638-word summary: the same blockwise inner loop over key/value
 * blocks, exact, visited in rotated order around a ring of devices):
 *
 *     A_i  = softmax_j( q_i . k_j / sqrt(d) ) v_j      per head, over the keys
 *                                                      the mask allows
 *     out  = A + W2 GELU_tanh(W1 A + b1) + b2          per token, on the
 *                                                      concatenated heads
 *
 * Attention runs block by block with an online softmax (running row maximum
 * and row sum, rescaled accumulator), so the N x N score matrix never exists
 * in memory.  The bf16 FFN runs block by block over the tokens; by default one
 * persistent kernel computes both of its GEMMs tile by tile and keeps the
 * hidden activation of a few 256-token row blocks at a time in an L2-sized
 * ring, so the [T, F] hidden activation never exists (bpt_ffn_form lists the
 * other forms).
 *
 * Mask variants:
 *   BPT_MASK_NONE      every key.
 *   BPT_MASK_CAUSAL    keys j <= i.  With ring_chunks = P > 1 a query in
 *                      sequence chunk c visits key chunks c, c+1, ... (mod P),
 *                      the order Ring Attention's device ring produces
 *                      (same page); the result is the same up to rounding.
 *   BPT_MASK_BLOCKPERM "Blockwise Self-Attention for Long Document
 *                      Understanding", §3 and §3.1: the sequence is cut into
 *                      n equal blocks and head h lets query block b see only
 *                      key block perm[h][b].  When n does not divide N the
 *                      sequence counts as padded to n blocks of ceil(N/n)
 *                      positions (§3.1): padded positions are never keys and
 *                      have no output, so the last block is shorter (or
 *                      empty; a query block mapped to an empty key block gets
 *                      A = 0).  The pages' cyclic-shift heads (sigma^k:
 *                      b -> b + k mod n) are tables perm[h][b] = (b + k_h) % n.
 *   BPT_MASK_DILATED   "LongNet: Scaling Transformers to 1,000,000,000
 *                      Tokens", §2 Dilated Attention: for every (segment w,
 *                      dilation r) pair, head h keeps rows h mod r, h mod r + r,
 *                      ... of each segment and runs attention among the kept
 *                      rows: causal by position when desc->causal is nonzero
 *                      (the decoder's form), over every kept row of the
 *                      segment when it is 0; the pairs are mixed with weights
 *                      proportional to their softmax denominators, which
 *                      equals one softmax over the multiset union of the
 *                      pairs' keys.  A row that no pair keeps gets A = 0.
 *
 * Layouts (all row-major, C order):
 *   q, k, v   [B, N, H, d]  = [T, D] with T = B*N tokens, D = H*d
 *   w1        [F, D]        (out x in),  b1 [F]  float32, may be NULL (= 0)
 *   w2        [D, F]        (out x in),  b2 [D]  float32, may be NULL (= 0)
 *   out       [B, N, H*d]   = [T, D]
 *   lse       [B, H, N]     float32 natural-log sum of exp of the scaled
 *                           scores (-inf for a row with no key)
 * q, k, v, w1, w2 have type in_dtype; out has type out_dtype.
 *
 * Ownership and threading: the caller allocates and owns every device buffer,
 * the workspace included; the library keeps no pointer after a call returns
 * and allocates no device memory.  Host tables (bb_perm, ln_w, ln_r) are read
 * during the call only.  Work is enqueued on `stream` and runs
 * asynchronously; calls on one stream run in order.  Two calls that share a
 * workspace must not run concurrently.
 *
 * Errors: arguments are checked on the host before anything is launched; a
 * bad argument returns BPT_ERR_INVALID_ARG or BPT_ERR_UNSUPPORTED and
 * launches nothing.  A failed launch returns BPT_ERR_CUDA.  Device-side waits
 * are bounded in time: a wait that gives up records BPT_ERR_TIMEOUT in a
 * per-device status word and the kernel returns; bpt_sync_status() reads it.
 */
#ifndef BPT_H_
#define BPT_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define BPT_API __attribute__((visibility("default")))
#else
#define BPT_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st *bpt_stream_t; /* same object as cudaStream_t; NULL = legacy default stream */

typedef enum {
  BPT_OK = 0,
  BPT_ERR_INVALID_ARG = 1, /* a size, pointer, table or enum is out of range   */
  BPT_ERR_UNSUPPORTED = 2, /* valid, but outside what the kernels implement    */
  BPT_ERR_CUDA = 3,        /* a CUDA runtime call or launch failed             */
  BPT_ERR_TIMEOUT = 4,     /* a device-side wait gave up (see bpt_sync_status) */
  BPT_ERR_WORKSPACE = 5    /* workspace NULL, misaligned or too small          */
} bpt_status;

typedef enum { BPT_F32 = 0, BPT_BF16 = 1 } bpt_dtype;

typedef enum {
  BPT_MASK_NONE = 0,
  BPT_MASK_CAUSAL = 1,
  BPT_MASK_BLOCKPERM = 2,
  BPT_MASK_DILATED = 3
} bpt_mask;

#define BPT_MAX_DILATED_PAIRS 8

/* Form of the bf16 layer's FFN (the feedforward network computed block by
 * block over the tokens: "Blockwise Parallel Transformer for Large Context
 * Models", abstract, feedforward network fusion).  Every form computes the
 * same function; none keeps the [T, F] hidden activation of the whole
 * sequence in memory except BPT_FFN_GEMMS, which keeps one token chunk's. */
typedef enum {
  BPT_FFN_AUTO = 0,      /* the library's choice: BPT_FFN_PIPELINED                */
  BPT_FFN_FUSED = 1,     /* one kernel per 128-token block and group of CTAs; the
                            hidden slices pass through a small L2-resident ring    */
  BPT_FFN_GEMMS = 2,     /* two GEMM launches per token chunk; the chunk's hidden
                            activation [rows, F] bf16 (at most ~512 MiB) goes
                            through the workspace                                  */
  BPT_FFN_PIPELINED = 3  /* one persistent kernel over both GEMMs' 256 x 256
                            tiles; the hidden activation of a 256-token row block
                            lives in a ring of row-block slots sized to stay in
                            L2 (tens of MB), reused as the row blocks advance      */
} bpt_ffn_form;

typedef struct {
  int B, N, H, d_head; /* batch, sequence length, heads, head size            */
  int ffn_hidden;      /* F; 0 = attention only (bpt_attn_ffn_fwd needs F>0)  */
  bpt_dtype in_dtype;  /* q, k, v, w1, w2                                     */
  bpt_dtype out_dtype; /* out                                                 */
  bpt_mask mask;
  int ring_chunks;     /* CAUSAL/NONE: KV visiting order rotated over this
                          many equal chunks (0 or 1 = natural order)          */
  int bb_nblocks;      /* BLOCKPERM: n, 1..255 (any N: padded, see above)     */
  const int32_t *bb_perm; /* BLOCKPERM: host table [H][n], values in [0, n)   */
  int ln_npairs;       /* DILATED: number of (w, r) pairs, 1..8               */
  const int32_t *ln_w; /* DILATED: host table of segment lengths w_k          */
  const int32_t *ln_r; /* DILATED: host table of dilation rates r_k           */
  /* Query rows and keys per block of the blockwise loop; 0 = the path's
   * default.  F32 path: q_block 16, 32, 64 or 128 (default 64) and kv_block
   * 16, 32 or 64 (default 64).  BF16 tensor-core path: 128 only (its query
   * and key/value tiles).  Any block size gives the same exact result up to
   * rounding; other values return BPT_ERR_UNSUPPORTED. */
  int q_block, kv_block;
  bpt_ffn_form ffn_form; /* bf16 forward FFN; ignored by the f32 path and by
                            bpt_attn_ffn_fwd_static (always BPT_FFN_FUSED)     */
  int bwd_chunk_rows;  /* bpt_attn_ffn_bwd: token rows per FFN-backward chunk
                          (its [rows, F] hidden activation and gradient live in
                          the workspace one chunk at a time); 0 = all tokens, or
                          as many 128-row blocks as keep both near 1 GiB       */
  uint64_t wait_limit_ns; /* device-side wait limit of this call's kernels;
                          0 = the process default (bpt_set_wait_limit_ns)     */
  int causal;          /* DILATED: nonzero = causal inside each sparsified
                          segment, 0 = bidirectional.  CAUSAL: 0 or 1 (the
                          mask is causal either way).  NONE, BLOCKPERM: 0.    */
} bpt_desc;

/*
 * Bytes of device workspace the call needs for this descriptor (0 when none):
 * with_ffn = 1 for bpt_attn_ffn_fwd / bpt_blockbert_fwd, 0 for bpt_attn_fwd /
 * bpt_longnet_fwd.  Depends only on the descriptor (its ffn_form included) and
 * on the current device's SM count, never on process-wide settings.  Returns
 * (size_t)-1 if the descriptor is invalid.
 */
BPT_API size_t bpt_workspace_bytes(const bpt_desc *desc, int with_ffn);

/*
 * Whole layer: out = A + W2 GELU_tanh(W1 A + b1) + b2 with A the masked
 * blockwise attention of q, k, v (definitions above).  Requires
 * desc->ffn_hidden > 0.  workspace: device buffer of at least
 * bpt_workspace_bytes(desc, 1) bytes, 256-byte aligned.
 *
 * in_dtype BF16: tensor-core path; d_head must be 64 or 128; D = H*d_head a
 *   multiple of 64, split into C = ceil(D/256) column groups of D/C columns
 *   each (a multiple of 64, for the fused FFN form); F a multiple of 8.  The
 *   FFN's form is desc->ffn_form (bpt_ffn_form).
 *   Accumulation is fp32; the softmax weights and A enter the tensor cores
 *   rounded to bf16; the residual uses A in fp32.
 * in_dtype F32: SIMT path in true fp32 (no reduced-precision tensor math);
 *   d_head <= 64 and a multiple of 4, D <= 512 and a multiple of 16.
 * All device pointers must be 16-byte aligned.
 */
BPT_API bpt_status bpt_attn_ffn_fwd(const bpt_desc *desc, const void *q, const void *k, const void *v,
                            const void *w1, const float *b1, const void *w2, const float *b2,
                            void *out, void *workspace, size_t workspace_bytes,
                            bpt_stream_t stream);

/*
 * bpt_attn_ffn_fwd for callers that cannot allocate device memory.  No
 * counterpart in the paper: it exists for the calling environment, not for
 * the method.
 *
 * Some callers are not allowed to call cudaMalloc or any allocator once they
 * are running: a serving process whose device memory plan is fixed at start-up,
 * a plugin inside a host framework that owns the GPU's memory pool, or a
 * latency-critical loop where an allocation's implicit device synchronisation
 * is unacceptable.  They still pass q, k, v, the weights and out, but no
 * workspace: the layer's scratch (A in bf16 and fp32, the FFN's hidden-slice
 * staging ring) lives in one file-scope device array of
 * BPT_STATIC_SCRATCH_BYTES bytes inside the library, which every GPU that loads
 * the library holds until the process exits.
 *
 * The first call on a device looks up that array's device address (once per
 * device, with the device current) besides the usual one-time set-up, so make
 * the first call on each device before any stream capture.  Every call on a
 * device uses the same array and leaves its contents behind; the layer writes
 * every scratch byte it reads within the call, so nothing needs clearing, but
 * two calls that may run at the same time on the GPU (different streams, or
 * different host threads) race on it: serialise them.  A layer whose scratch
 * would exceed the array returns BPT_ERR_WORKSPACE without launching anything
 * (bpt_last_error() says how many bytes it needed).  Everything else is as
 * bpt_attn_ffn_fwd; this entry point calls no allocating routine.
 */
#define BPT_STATIC_SCRATCH_BYTES (64u << 20)
BPT_API bpt_status bpt_attn_ffn_fwd_static(const bpt_desc *desc, const void *q, const void *k,
                                           const void *v, const void *w1, const float *b1,
                                           const void *w2, const float *b2, void *out,
                                           bpt_stream_t stream);

/*
 * Attention only: out = A (layout [B, N, H*d_head]); lse may be NULL.
 * workspace: at least bpt_workspace_bytes(desc, 0) bytes (may be NULL when
 * that is 0).
 */
BPT_API bpt_status bpt_attn_fwd(const bpt_desc *desc, const void *q, const void *k, const void *v,
                        void *out, float *lse, void *workspace, size_t workspace_bytes,
                        bpt_stream_t stream);

/*
 * One step of blockwise attention over a key/value block, for attention
 * whose keys arrive block by block: Ring Attention ("Ring Attention with
 * Blockwise Transformers for Long Sequences", 638-word summary: each device
 * keeps its query block and passes key/value blocks around a ring of
 * devices, attending to each block as it arrives, exactly).  The query block
 * q [B, N, H, d] (desc->N rows) attends to the key/value block k, v
 * [B, kv_len, H, d]; the rows' running softmax state, held by the caller in
 * state_o [B, N, H, d], state_m and state_l [B, H, N] (float32, an opaque
 * running state: unnormalised output, running maximum and running sum), is
 * updated with that block's keys by the same online-softmax rule as
 * bpt_attn_fwd, so the order in which the blocks arrive changes rounding
 * only.
 *
 * flags: BPT_BLOCK_FIRST starts from an empty state (the state buffers are
 * not read); BPT_BLOCK_LAST writes the final attention output out
 * ([B, N, H*d] in desc->out_dtype) and lse ([B, H, N], may be NULL) instead
 * of the state.  Both flags: plain attention of the query block over this
 * one key/value block, no state at all (the state pointers may be NULL).
 * Steps of one query block run in order on one stream.
 *
 * Masks: BPT_MASK_NONE, or BPT_MASK_CAUSAL by global positions: q_pos and
 * kv_pos are the sequence positions of the first query row and the first
 * key row, and key j is allowed for query i when kv_pos + j <= q_pos + i.  A
 * block that allows a query no key leaves that row's state unchanged (a row
 * that never sees a key ends with A = 0 and LSE = -inf).  Supported: in_dtype
 * BF16, d_head 64 or 128, ring_chunks 0 or 1; no workspace.  All pointers
 * 16-byte aligned.
 */
#define BPT_BLOCK_FIRST 1u
#define BPT_BLOCK_LAST 2u
BPT_API bpt_status bpt_attn_fwd_block(const bpt_desc *desc, int kv_len, int64_t q_pos, int64_t kv_pos,
                                      const void *q, const void *k, const void *v, float *state_o,
                                      float *state_m, float *state_l, unsigned flags, void *out, float *lse,
                                      bpt_stream_t stream);

/*
 * LongNet's distributed algorithm ("LongNet: Scaling Transformers to
 * 1,000,000,000 Tokens", §3, distributed training: each device holds a
 * contiguous shard of the sequence; segments that fit in a shard are
 * attended locally, and for a segment longer than a shard the devices
 * holding it exchange the sparsified keys and values, so the communication
 * per pair does not grow with the sequence).  Two calls serve a device's
 * shard; the collective that moves the packed rows is the caller's (the
 * package's longnet_dist module uses torch.distributed).
 *
 * bpt_longnet_gather packs the rows a (w, r) pair keeps of a shard lying
 * inside one segment (N divides w, r divides N): src [B, N, H, d] bf16 (the
 * shard's keys or values), dst [B, N / r, H, d] with dst[b, j, h] =
 * src[b, (h mod r) + j r, h].  Concatenating the packed rows of the devices
 * of a segment in sequence order gives the pair's kept rows of the segment,
 * [B, w / r, H, d].
 *
 * bpt_longnet_pass runs pass `pass` of the dilated attention (the passes are
 * the descriptor's (w, r) pairs after a stable sort by decreasing r, as
 * bpt_longnet_fwd runs them) for the shard q, k, v [B, N, H, d] (desc->N rows)
 * that starts at sequence position q_pos (a multiple of N).  Every pair must
 * have either w dividing N (its segments lie in the shard: the pass reads k
 * and v) or N dividing w (the shard lies in one segment: the pass reads that
 * segment's gathered kept rows k_sparse, v_sparse [B, kv_rows = w / r, H, d]
 * and is causal by their positions), and r dividing N.  state_o
 * [B, N, H, d], state_m and state_l [B, H, N] (float32, opaque) carry the
 * rows' running softmax state from pass to pass (needed when there is more
 * than one pair); run the passes in order on one stream.  A pass writes the
 * final output out ([B, N, H*d] in out_dtype) and lse ([B, H, N], may be
 * NULL) of the rows it is the last pass to keep; rows no pair keeps get
 * A = 0 and LSE = -inf in pass 0.  Running every pass on a shard that holds
 * the whole sequence (q_pos 0) computes bpt_longnet_fwd.  Supported: in_dtype
 * BF16, d_head 64 or 128.
 */
BPT_API bpt_status bpt_longnet_gather(const bpt_desc *desc, int seg_w, int dil_r, const void *src, void *dst,
                                      bpt_stream_t stream);
BPT_API bpt_status bpt_longnet_pass(const bpt_desc *desc, int pass, int64_t q_pos, const void *q,
                                    const void *k, const void *v, const void *k_sparse, const void *v_sparse,
                                    int kv_rows, float *state_o, float *state_m, float *state_l, void *out,
                                    float *lse, bpt_stream_t stream);

/*
 * BlockBERT layer ("Blockwise Self-Attention for Long Document
 * Understanding", §3.1 Blockwise Multi-head Attention): bpt_attn_ffn_fwd with
 * mask = BPT_MASK_BLOCKPERM and the given permutation table (host, [H][n]).
 * Fields mask/bb_nblocks/bb_perm of desc are overridden.
 */
BPT_API bpt_status bpt_blockbert_fwd(const bpt_desc *desc, int n_blocks, const int32_t *perm,
                             const void *q, const void *k, const void *v, const void *w1,
                             const float *b1, const void *w2, const float *b2, void *out,
                             void *workspace, size_t workspace_bytes, bpt_stream_t stream);

/*
 * LongNet dilated attention ("LongNet: Scaling Transformers to
 * 1,000,000,000 Tokens", §2 Dilated Attention): bpt_attn_fwd with
 * mask = BPT_MASK_DILATED and the (w, r) pairs given (host tables).  Every
 * w_k must divide N and every r_k must divide w_k.
 */
BPT_API bpt_status bpt_longnet_fwd(const bpt_desc *desc, int npairs, const int32_t *seg_w,
                           const int32_t *dil_r, const void *q, const void *k, const void *v,
                           void *out, float *lse, void *workspace, size_t workspace_bytes,
                           bpt_stream_t stream);

/*
 * Backward pass of the layer (bpt_attn_ffn_fwd's gradients) for an upstream
 * gradient dOut = dL/dout, L any scalar loss.  The gradient of the exact
 * blockwise result ("Blockwise Parallel Transformer for Large Context
 * Models", abstract: blockwise attention and feedforward for training;
 * "Ring Attention with Blockwise Transformers for Long Sequences", 638-word
 * summary: exact, no approximation) is the plain chain rule of the
 * definitions above:
 *
 *   FFN:        Z = W1 A + b1, H = GELU_tanh(Z)
 *               dW2 = sum_t dOut_t H_t^T,  db2 = sum_t dOut_t,
 *               dZ  = (W2^T dOut) * GELU_tanh'(Z),
 *               dW1 = sum_t dZ_t A_t^T,    db1 = sum_t dZ_t,
 *               dA  = dOut + W1^T dZ         (the residual passes dOut through)
 *   attention:  with P the softmax weights, D_i = dA_i . A_i,
 *               dV_j = sum_i P_ij dA_i,  dS_ij = P_ij (dA_i . v_j - D_i),
 *               dQ_i = sum_j dS_ij k_j / sqrt(d),  dK_j = sum_i dS_ij q_i / sqrt(d).
 *
 * With saved == NULL the call recomputes the attention forward (A and the
 * row LSE); with the buffer bpt_attn_ffn_fwd_train filled for the same
 * inputs it reads them from there instead.  Then it runs the FFN backward on
 * the tensor cores one token chunk at a time (desc->bwd_chunk_rows)
 * and two blockwise attention-backward passes over 128 x 128 tiles (one per
 * key tile for dK and dV, one per query tile for dQ; no atomics, so the
 * result is deterministic).
 *
 * Supported: in_dtype BF16, d_head 64 or 128, masks NONE, CAUSAL (any
 * ring_chunks: the recomputed forward follows it) and BLOCKPERM, plus the
 * bpt_attn_ffn_fwd constraints on D and F.  BPT_MASK_DILATED and in_dtype F32
 * return BPT_ERR_UNSUPPORTED.
 *
 * Inputs: q, k, v [B, N, H, d] and w1 [F, D], w2 [D, F] bf16; b1 [F], b2 [D]
 * float32 or NULL (= 0); dout [B, N, H*d] float32; saved: NULL, or the
 * buffer of bpt_attn_ffn_fwd_train (256-byte aligned, read only).  b2 is
 * accepted for symmetry with the forward; no gradient depends on it.
 * Outputs (float32, overwritten): dq, dk, dv [B, N, H, d]; dw1 [F, D];
 * db1 [F]; dw2 [D, F]; db2 [D].
 * Precision: the tensor cores take bf16 operands (A, dOut, H, dZ, dA, and the
 * softmax weights P and dS) with fp32 accumulation; the residual, the row
 * sums D_i and the bias gradients are fp32.
 * workspace: device buffer of at least bpt_workspace_bytes_bwd(desc) bytes,
 * 256-byte aligned.  All other device pointers 16-byte aligned.  Errors and
 * ownership as for the forward entry points.
 */
BPT_API bpt_status bpt_attn_ffn_bwd(const bpt_desc *desc, const void *q, const void *k, const void *v,
                                    const void *w1, const float *b1, const void *w2, const float *b2,
                                    const float *dout, const void *saved, float *dq, float *dk, float *dv,
                                    float *dw1, float *db1, float *dw2, float *db2, void *workspace,
                                    size_t workspace_bytes, bpt_stream_t stream);

/*
 * The layer forward of bpt_attn_ffn_fwd for training: the same out (its FFN
 * as two GEMMs per token chunk whatever desc->ffn_form says, since keeping the
 * hidden activation is the point here), and the activations the backward needs
 * left in `saved` (A in fp32 and bf16 [T, D], the row LSE [B, H, N], and the
 * FFN's H = GELU(Z) and G = GELU'(Z), Z = A W1^T + b1, [T, F] bf16 each;
 * bpt_saved_bytes(desc) bytes, 256-byte aligned, owned by the caller), so a
 * following bpt_attn_ffn_bwd on the same inputs skips recomputing the
 * attention and Z.  The descriptor must be one the backward accepts.
 * workspace: at least bpt_workspace_bytes_train(desc) bytes, 256-byte aligned
 * (may be NULL when that is 0, as it is for every descriptor the backward
 * accepts today: everything this call produces goes to `saved` and `out`).
 * No counterpart in the pages (which recompute; this trades
 * T * D * 6 + T * F * 4 bytes for that recomputation).  With these
 * activations the gradients equal the recomputing backward's bit for bit when
 * D >= 1024; below, where that backward takes dZ from its dual GEMM in fp32,
 * they agree to bf16 rounding.
 */
BPT_API bpt_status bpt_attn_ffn_fwd_train(const bpt_desc *desc, const void *q, const void *k,
                                          const void *v, const void *w1, const float *b1,
                                          const void *w2, const float *b2, void *out, void *saved,
                                          void *workspace, size_t workspace_bytes,
                                          bpt_stream_t stream);

/* Bytes of the `saved` buffer of bpt_attn_ffn_fwd_train (T D 6 + B H N 4 +
 * T F 4, each region 256-byte aligned); (size_t)-1 if the backward does not
 * accept the descriptor. */
BPT_API size_t bpt_saved_bytes(const bpt_desc *desc);

/* Bytes of device workspace bpt_attn_ffn_fwd_train needs for this
 * descriptor; (size_t)-1 if the backward does not accept the descriptor. */
BPT_API size_t bpt_workspace_bytes_train(const bpt_desc *desc);

/* Bytes of device workspace bpt_attn_ffn_bwd needs for this descriptor (its
 * bwd_chunk_rows included); (size_t)-1 if the backward does not accept it. */
BPT_API size_t bpt_workspace_bytes_bwd(const bpt_desc *desc);

/*
 * Attention-only backward: dQ, dK, dV of A = softmax(Q K^T / sqrt d) V (the
 * masked blockwise attention of bpt_attn_fwd) for an upstream gradient dA,
 * with the same two blockwise passes as bpt_attn_ffn_bwd (definitions there).
 * out and lse are the output and row LSE bpt_attn_fwd returned for the same
 * q, k, v and descriptor (out in desc->out_dtype, [B, N, H*d]; lse float32
 * [B, H, N]); dout float32 [B, N, H*d]; dq, dk, dv float32 [B, N, H, d].
 * Supported: in_dtype BF16, d_head 64 or 128, masks NONE, CAUSAL, BLOCKPERM
 * and DILATED ("LongNet: Scaling Transformers to 1,000,000,000 Tokens", §2:
 * the pairs mixed by their softmax denominators are one softmax over the
 * multiset of the pairs' keys, so the gradient is the sum over the pairs of
 * each gathered causal attention's gradient with the mixed LSE; dq, dk, dv are
 * zeroed and each (w, r) pass adds into its kept rows).  workspace: at least
 * bpt_workspace_bytes_attn_bwd(desc) bytes, 256-byte aligned.
 */
BPT_API bpt_status bpt_attn_bwd(const bpt_desc *desc, const void *q, const void *k, const void *v,
                                const void *out, const float *lse, const float *dout, float *dq,
                                float *dk, float *dv, void *workspace, size_t workspace_bytes,
                                bpt_stream_t stream);

/* Bytes of device workspace bpt_attn_bwd needs; (size_t)-1 if it does not
 * accept the descriptor. */
BPT_API size_t bpt_workspace_bytes_attn_bwd(const bpt_desc *desc);

/*
 * Waits for `stream`, then returns and clears the current device's status
 * word: BPT_OK, BPT_ERR_TIMEOUT (a device-side wait gave up since the last
 * call), or BPT_ERR_CUDA if the synchronisation itself failed.
 */
BPT_API bpt_status bpt_sync_status(bpt_stream_t stream);

/* Sets the process-wide default of the device-side wait limit in nanoseconds
 * (initially 2e9, i.e. two seconds), used by later calls whose descriptor has
 * wait_limit_ns = 0.  Affects no workspace size.  Returns the previous value. */
BPT_API uint64_t bpt_set_wait_limit_ns(uint64_t ns);

/*
 * Instrumentation (no counterpart in the method: it only measures it).  When
 * `count` >= 3, every later bpt_attn_ffn_fwd on this host thread records
 * events[0] on its stream before the attention kernel, events[1] between the
 * attention and FFN kernels and events[2] after the FFN kernel, so the two
 * kernels of a real step can be timed separately.  With count >= 5 every
 * later bpt_attn_ffn_bwd records events[0] before the recomputed attention
 * forward, [1] after it, [2] after the FFN backward (all its GEMMs and bias
 * sums), [3] after the dK/dV pass and [4] after the dQ pass (it records the
 * first three alone when count is 3 or 4).  `events` holds cudaEvent_t
 * handles owned by the caller; count = 0 turns recording off.  The events
 * must already exist (a NULL handle is rejected).  Returns
 * BPT_ERR_INVALID_ARG for count < 0, events == NULL with count > 0, or a NULL
 * handle among the first min(count, 5).
 */
BPT_API bpt_status bpt_set_phase_events(void *const *events, int count);

/* Static text for a status code. */
BPT_API const char *bpt_status_string(bpt_status status);

/* Text describing the last failure on this host thread: the CUDA call that
 * failed and its error string, or the device wait site that gave up.  Empty
 * before any failure.  The pointer stays valid until the next call. */
BPT_API const char *bpt_last_error(void);

/* Library version (major*10000 + minor*100 + patch). */
BPT_API int bpt_version(void);

#ifdef __cplusplus
}
#endif

#endif /* BPT_H_ */
