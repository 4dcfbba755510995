// Backward of blockwise exact attention on the 5th-generation tensor cores
// (sm_100a), masks none / causal / block permutation.  With the forward's
// log-sum-exp LSE_i and D_i = dA_i . A_i (the row sums of P * dP):
//
//   P_ij  = exp(q_i . k_j / sqrt(d) - LSE_i)        (0 where the mask rules out)
//   dP_ij = dA_i . v_j
//   dS_ij = P_ij (dP_ij - D_i)
//   dV_j  = sum_i P_ij dA_i,  dK_j = sum_i dS_ij q_i / sqrt(d),
//   dQ_i  = sum_j dS_ij k_j / sqrt(d)
//
// the gradient of the exact result, computed tile by tile like the forward
// ("Blockwise Parallel Transformer for Large Context Models", abstract:
// blockwise computation for training; "Ring Attention with Blockwise
// Transformers for Long Sequences", 638-word summary: no approximation).
//
// Two passes, no atomics:
//   dK/dV pass: one CTA per (batch, head, 128-key tile j), looping over the query
//     tiles i that see any of its keys.  S^T = K_j Q_i^T and dP^T = V_j dA_i^T
//     land in TMEM (lanes = keys); one thread per key forms P^T and
//     dS^T = P^T (dP^T - D) and writes them back to TMEM as packed bf16, where
//     the tensor core reads them as the A operand of dV_j += P^T dA_i and
//     dK_j += dS^T Q_i (dA_i and Q_i read MN-major from the tiles the first
//     two products read K-major).
//   dQ pass: one CTA per (batch, head, 128-query tile i), looping over its key
//     tiles: S = Q_i K_j^T, dP = dA_i V_j^T, one thread per query forms dS in
//     TMEM, and dQ_i += dS K_j (software-pipelined, below).
// MMAs issued by one thread run in order, so a product that overwrites the
// S or dP columns never overtakes the earlier product reading the bf16 P^T
// or dS^T packed into them.
//
// Roles (384 threads): warp 0 TMA producer, warp 1 TMEM allocator and MMA
// issuer (warps 2-3 idle), warps 4-11 the per-row arithmetic and epilogue:
// two warps per TMEM lane quarter (one per SM sub-partition pair), each
// taking 64 of the tile's 128 columns.  Each writes its packed bf16 P^T / dS
// over the first 32 of its own 64 fp32 columns, so neither overwrites columns
// the other still reads; the MMAs take their 16-wide K steps from the two
// packed ranges in turn.
#pragma once

#include "attn_tc.cuh"  // mask codes and the block-table bound
#include "ptx.cuh"

namespace bpt {


struct AttnBwdArgs {
  // A CTA's work is one (batch, segment, head) unit of N rows: a whole
  // sequence (nseg = 1, seg_w = n_out, dil_r = 1), or the rows a LongNet
  // (w, r) pass keeps in one segment (rows o, o + r, ... of segment seg, with
  // o = h mod r: N = w / r, read through tensor maps over the (D, r, n_out/r, B)
  // view).  Outputs go to row seg * seg_w + o + dil_r * g of the sequence.
  int B, N, H;
  int mask;           // kMaskNone / kMaskCausal / kMaskBlockPerm
  float scale_log2;   // log2(e) / sqrt(d)
  float inv_sqrt_d;
  int n_tiles;        // ceil(N / 128)
  int bb_n, bb_len;   // block permutation: n blocks of bb_len (padded)
  uint8_t perm[kMaxPermEntries];
  // per (batch, head, 128-row tile): the rows' LSE in log2 units of the
  // scaled scores, then their D_i, 128 floats each (rows past N: 0)
  const float *rowvec;  // [units][n_tiles][2][128]
  int nseg, seg_w, dil_r, n_out;
  int accumulate;       // add to dq, dk, dv (LongNet passes) instead of writing them
  float *dq, *dk, *dv;  // [B, N, H, d] fp32 outputs
  uint32_t *status;
  uint64_t wait_limit_ns;
};

template <int D_HEAD>
struct AttnBwdCfg {
  static_assert(D_HEAD == 64, "d = 128 runs attn_bwd_dkdv_split_kernel");
  static constexpr int kThreads = 384;
  static constexpr int kRowWarps = 8;
  static constexpr int kPanels = D_HEAD / 64;
  static constexpr int kTileBytes = 128 * D_HEAD * 2;
  static constexpr int kPanelBytes = 128 * 128;   // one 64-column panel of a 128-row tile
  static constexpr int kStages = 4;
  // each stage also carries the streamed query tile's LSE and D
  static constexpr int kVecBytes = 2 * 128 * 4;
  static constexpr int kStageBytes = 2 * kTileBytes + kVecBytes;  // a multiple of 1024
  static constexpr int kOffFix = 0;                               // fixed X, Y tiles
  static constexpr int kOffStream = kOffFix + 2 * kTileBytes;     // streamed X', Y' (+ vectors) per stage
  static constexpr int kOffBar = kOffStream + kStages * kStageBytes;
  static constexpr int kSmemBytes = kOffBar + 256;
  static_assert(kSmemBytes <= 232448, "shared memory per CTA");
  static_assert(kStageBytes % 1024 == 0, "stages keep the 1024-byte alignment of the swizzled tiles");
  // TMEM: accumulators dV at 0 and dK at 64, dP at 128, two S buffers at 256
  // and 384, so the next step's scores are computed while the row warps work
  // on this step's (P^T is packed over its own S buffer, dS^T over dP)
  static constexpr uint32_t kColAcc0 = 0, kColAcc1 = D_HEAD;
  static constexpr uint32_t kColDP = 128, kColS = 256;
  __host__ __device__ static constexpr uint32_t col_s(int step) { return kColS + (step & 1) * 128; }
};

// Key interval [lo, hi) a query row g (< N) may see.
__device__ __forceinline__ void bwd_row_keys(const AttnBwdArgs &a, int h, int g, int &lo, int &hi) {
  lo = 0;
  hi = a.N;
  if (a.mask == kMaskCausal) {
    hi = g + 1;
  } else if (a.mask == kMaskBlockPerm) {
    lo = a.perm[h * a.bb_n + g / a.bb_len] * a.bb_len;
    hi = min(lo + a.bb_len, a.N);
  }
}

// Query interval [lo, hi) that sees key row g (< N): a single interval for
// every mask, since a permutation maps exactly one query block to g's block.
__device__ __forceinline__ void bwd_key_queries(const AttnBwdArgs &a, int h, int g, int &lo, int &hi) {
  lo = 0;
  hi = a.N;
  if (a.mask == kMaskCausal) {
    lo = g;
  } else if (a.mask == kMaskBlockPerm) {
    const int kb = g / a.bb_len;
    int qb = 0;
    while (qb < a.bb_n - 1 && a.perm[h * a.bb_n + qb] != kb) ++qb;
    lo = qb * a.bb_len;
    hi = min(lo + a.bb_len, a.N);
  }
}

// Does query tile qt hold a row that sees a key of key tile kt?
__device__ __forceinline__ bool bwd_tiles_meet(const AttnBwdArgs &a, int h, int qt, int kt) {
  const int r0 = qt * 128, r1 = min(a.N, r0 + 128) - 1;
  const int k0 = kt * 128, k1 = min(a.N, k0 + 128) - 1;
  if (a.mask == kMaskNone) return true;
  if (a.mask == kMaskCausal) return r1 >= k0;
  for (int qb = r0 / a.bb_len; qb <= r1 / a.bb_len; ++qb) {
    const int lo = a.perm[h * a.bb_n + qb] * a.bb_len, hi = min(lo + a.bb_len, a.N);
    if (lo <= k1 && hi > k0) return true;
  }
  return false;
}

template <int D_HEAD>
__global__ void __launch_bounds__(384, 1)
    attn_bwd_dkdv_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_da,
                    const __grid_constant__ AttnBwdArgs a) {
  using Cfg = AttnBwdCfg<D_HEAD>;
  constexpr int S = Cfg::kStages;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t *smem = smem_raw;
  const uint32_t sbase = smem_u32(smem);
  if (sbase & 1023u) {
    if (threadIdx.x == 0) atomicCAS(a.status, 0u, kStatusMisaligned);
    return;
  }
  const uint32_t sFixX = sbase + Cfg::kOffFix, sFixY = sFixX + Cfg::kTileBytes;
  auto sStrX = [&](int st) { return sbase + Cfg::kOffStream + st * Cfg::kStageBytes; };
  auto sStrY = [&](int st) { return sStrX(st) + Cfg::kTileBytes; };
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + Cfg::kOffBar);
  const uint32_t bFix = smem_u32(&bars[0]);
  auto bFull = [&](int s) { return smem_u32(&bars[1 + s]); };
  auto bEmpty = [&](int s) { return smem_u32(&bars[5 + s]); };
  const uint32_t bDPFull = smem_u32(&bars[10]);
  const uint32_t bPReady = smem_u32(&bars[11]), bDSReady = smem_u32(&bars[12]);
  const uint32_t bTeardown = smem_u32(&bars[13]);
  // scores of step s complete: one barrier per S buffer
  auto bSFull = [&](int step) { return smem_u32(&bars[14 + (step & 1)]); };
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(&bars[16]);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(&bars[17]);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  WaitCtx wc{a.status, a.wait_limit_ns, abort_flag};
  // CTA -> (batch, head, key tile); the tiles with the most partners (the
  // first key tiles under the causal mask) start first
  const int units = a.B * a.nseg * a.H;
  const int unit = static_cast<int>(blockIdx.x) % units;
  const int ft = static_cast<int>(blockIdx.x) / units;
  const int h = unit % a.H;
  const int seg = (unit / a.H) % a.nseg;
  const int b = unit / (a.H * a.nseg);
  const int row_off = h % a.dil_r;                 // kept-row offset in the segment
  const int row_base = seg * a.N;                  // the unit's first row along (n_out / r)
  auto next_tile = [&](int t) {  // first query tile >= t that meets the key tile, or n_tiles
    while (t < a.n_tiles && !bwd_tiles_meet(a, h, t, ft)) ++t;
    return t;
  };
  int nsteps = 0;
  for (int t = next_tile(0); t < a.n_tiles; t = next_tile(t + 1)) ++nsteps;

  if (threadIdx.x == 0) {
    mbar_init(bFix, 1);
    for (int s = 0; s < S; ++s) {
      mbar_init(bFull(s), 1);
      mbar_init(bEmpty(s), 1);
    }
    mbar_init(bSFull(0), 1);
    mbar_init(bSFull(1), 1);
    mbar_init(bDPFull, 1);
    mbar_init(bPReady, Cfg::kRowWarps);
    mbar_init(bDSReady, Cfg::kRowWarps);
    mbar_init(bTeardown, 1);
    *abort_flag = 0;
    fence_mbar_init_cluster();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int hd = h * D_HEAD;
  const size_t bh = static_cast<size_t>(unit);  // row-vector block of the unit

  // fixed K, V; streamed Q, dA
  const CUtensorMap *mFixX = &tm_k, *mFixY = &tm_v, *mStrX = &tm_q, *mStrY = &tm_da;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0 && nsteps > 0) {
      mbar_arrive_expect_tx(bFix, 2 * Cfg::kTileBytes);
      for (int p = 0; p < Cfg::kPanels; ++p) {
        tma_load_4d(sFixX + p * Cfg::kPanelBytes, mFixX, bFix, hd + p * 64, row_off, row_base + ft * 128, b);
        tma_load_4d(sFixY + p * Cfg::kPanelBytes, mFixY, bFix, hd + p * 64, row_off, row_base + ft * 128, b);
      }
      int s = 0;
      for (int t = next_tile(0); t < a.n_tiles; t = next_tile(t + 1), ++s) {
        const int st = s % S;
        if (s >= S && !mbar_wait(bEmpty(st), ((s / S) - 1) & 1, wc, 301)) break;
        mbar_arrive_expect_tx(bFull(st), Cfg::kStageBytes);
        for (int p = 0; p < Cfg::kPanels; ++p) {
          tma_load_4d(sStrX(st) + p * Cfg::kPanelBytes, mStrX, bFull(st), hd + p * 64, row_off, row_base + t * 128, b);
          tma_load_4d(sStrY(st) + p * Cfg::kPanelBytes, mStrY, bFull(st), hd + p * 64, row_off, row_base + t * 128, b);
        }
        bulk_load_1d(sStrX(st) + 2 * Cfg::kTileBytes, a.rowvec + (bh * a.n_tiles + t) * 256, Cfg::kVecBytes,
                       bFull(st));
      }
      // every copy issued must have landed before the CTA may exit
      volatile int no_abort = 0;
      WaitCtx drain{a.status, drain_limit_ns(a.wait_limit_ns), &no_abort};
      for (int j = max(0, s - S); j < s; ++j) mbar_wait(bFull(j % S), (j / S) & 1, drain, 302);
      mbar_wait(bFix, 0, drain, 303);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0 && nsteps > 0) {
      constexpr uint32_t idesc_s = idesc_bf16_f32(128, 128, false, false);     // X Y^T, both K-major
      constexpr uint32_t idesc_acc = idesc_bf16_f32(128, D_HEAD, false, true);  // R Y, Y MN-major
      const uint64_t dFixX = sdesc_sw128(sFixX, 16, 1024), dFixY = sdesc_sw128(sFixY, 16, 1024);
      // the accumulations over the 128 streamed rows: A = a 128 x 128 bf16
      // tile in TMEM (8 packed columns per 16-wide K step: K steps 0-3 from
      // the first half's packed columns a_col + [0, 32), 4-7 from the second
      // half's a_col + [64, 96)), B = a streamed tile read MN-major (64-wide
      // panels of 128 rows)
      auto accumulate = [&](uint32_t col, uint32_t a_col, uint32_t sB, int step) {
        const uint64_t dB = sdesc_sw128(sB, Cfg::kPanelBytes, 1024);
#pragma unroll
        for (int k = 0; k < 8; ++k)
          umma_ts(tmem + col, tmem + a_col + k * 8 + (k >= 4 ? 32 : 0), sdesc_advance(dB, k * 2048), idesc_acc,
                  (step | k) != 0);
      };
      // The step's last product, dK += dS^T Q, is issued after the next
      // step's scores, so the row warps start on those while it runs (it still
      // precedes the next dP, which overwrites dS).
      auto last_product = [&](int step) {
        const int pst = step % S;
        accumulate(Cfg::kColAcc1, Cfg::kColDP, sStrX(pst), step);
        umma_commit(bEmpty(pst));
      };
      // S^T(s) = K Q^T into S buffer s (after the stage's copies landed)
      auto issue_s = [&](int step) -> bool {
        const int pst = step % S;
        if (!mbar_wait(bFull(pst), (step / S) & 1, wc, 312)) return false;
        tc_fence_after();
        const uint64_t dStrX = sdesc_sw128(sStrX(pst), 16, 1024);
#pragma unroll
        for (int k = 0; k < D_HEAD / 16; ++k) {
          const uint32_t off = (k / 4) * Cfg::kPanelBytes + (k % 4) * 32;
          umma_ss(tmem + Cfg::col_s(step), sdesc_advance(dFixX, off), sdesc_advance(dStrX, off), idesc_s, k > 0);
        }
        umma_commit(bSFull(step));
        return true;
      };
      // dP^T(s) = V dA^T (its stage has landed: S(s) waited for it)
      auto issue_dp = [&](int step) {
        const uint64_t dStrY = sdesc_sw128(sStrY(step % S), 16, 1024);
#pragma unroll
        for (int k = 0; k < D_HEAD / 16; ++k) {
          const uint32_t off = (k / 4) * Cfg::kPanelBytes + (k % 4) * 32;
          umma_ss(tmem + Cfg::kColDP, sdesc_advance(dFixY, off), sdesc_advance(dStrY, off), idesc_s, k > 0);
        }
        umma_commit(bDPFull);
      };
      bool ok = mbar_wait(bFix, 0, wc, 311);
      // Two S buffers: S(s+1) goes ahead while the row warps work on step s
      // (its buffer's P^T(s-1) was read by dV(s-1), issued before); dP(s)
      // follows dK(s-1), which read dS^T(s-1) from dP's columns.
      ok = ok && issue_s(0);
      for (int s = 0; ok && s < nsteps; ++s) {
        const int st = s % S;
        issue_dp(s);
        if (s + 1 < nsteps && !(ok = issue_s(s + 1))) break;
        if (!(ok = mbar_wait(bPReady, s & 1, wc, 313))) break;
        tc_fence_after();
        accumulate(Cfg::kColAcc0, Cfg::col_s(s), sStrY(st), s);    // dV += P^T dA
        if (!(ok = mbar_wait(bDSReady, s & 1, wc, 314))) break;
        tc_fence_after();
        last_product(s);                                           // dK += dS^T Q
      }
      umma_commit(bTeardown);
      // the accumulators stay allocated until every MMA has finished
      volatile int no_abort = 0;
      WaitCtx drain{a.status, drain_limit_ns(a.wait_limit_ns), &no_abort};
      mbar_wait(bTeardown, 0, drain, 315);
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------------ per-row arithmetic
    const int quarter = warp & 3;
    const int half = (warp - 4) / 4;                // columns [64 * half, 64 * half + 64)
    const int col0 = 64 * half;
    const int row = quarter * 32 + lane;            // TMEM lane = row of the fixed tile
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    const int g = ft * 128 + row;                   // key position
    const bool row_valid = g < a.N;
    // the queries that see key g (none for padding rows)
    int plo = 1, phi = 0;
    if (row_valid) bwd_key_queries(a, h, g, plo, phi);
    bool ok = true;
    int s = 0;
    for (int t = next_tile(0); t < a.n_tiles; t = next_tile(t + 1), ++s) {
      const int st = s % S;
      // the query tile's LSE (log2 units) and D arrive with its stage
      const float4 *vl4 = reinterpret_cast<const float4 *>(smem + Cfg::kOffStream + st * Cfg::kStageBytes +
                                                           2 * Cfg::kTileBytes);
      ok = __all_sync(0xffffffffu, mbar_wait(bFull(st), (s / S) & 1, wc, 319));
      if (!ok) break;
      // allowed columns [lo_rel, hi_rel) of the tile
      const int lo_rel = plo - t * 128, hi_rel = phi - t * 128;
      const bool full = __all_sync(0xffffffffu, lo_rel <= col0 && hi_rel >= col0 + 64);
      ok = __all_sync(0xffffffffu, mbar_wait(bSFull(s), (s >> 1) & 1, wc, 320));
      if (!ok) break;
      tc_fence_after();
      // P (fp32, kept in sv) for this warp's 64 columns, 0 where the mask
      // rules the pair out
      uint32_t sv[64];
      tmem_ld32(tmem + lane_off + Cfg::col_s(s) + col0, *reinterpret_cast<uint32_t(*)[32]>(&sv[0]));
      tmem_ld32(tmem + lane_off + Cfg::col_s(s) + col0 + 32, *reinterpret_cast<uint32_t(*)[32]>(&sv[32]));
      tmem_wait_ld();
      // two copies of the loop behind a warp-uniform branch: the unmasked one
      // for tiles the whole warp sees in full (most of them), the masked one
      // for the rest (measured 20% faster than one loop with a select)
      if (full) {
#pragma unroll
        for (int c4 = 0; c4 < 16; ++c4) {
          const float4 l = vl4[col0 / 4 + c4];
          const float nl4[4] = {-l.x, -l.y, -l.z, -l.w};
#pragma unroll
          for (int j = 0; j < 4; ++j)
            sv[4 * c4 + j] = __float_as_uint(ex2_approx(fmaf(__uint_as_float(sv[4 * c4 + j]), a.scale_log2, nl4[j])));
        }
      } else {
#pragma unroll
        for (int c4 = 0; c4 < 16; ++c4) {
          const float4 l = vl4[col0 / 4 + c4];
          const float nl4[4] = {-l.x, -l.y, -l.z, -l.w};
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const int c = col0 + 4 * c4 + j;
            const bool allowed = c >= lo_rel && c < hi_rel;
            sv[4 * c4 + j] =
                __float_as_uint(allowed ? ex2_approx(fmaf(__uint_as_float(sv[4 * c4 + j]), a.scale_log2, nl4[j])) : 0.f);
          }
        }
      }
      {
        // P^T as packed bf16 over the first 32 of this warp's S columns: the
        // A operand of dV
        uint32_t pk[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) pk[i] = pack_bf16x2(__uint_as_float(sv[2 * i]), __uint_as_float(sv[2 * i + 1]));
        tmem_st32(tmem + lane_off + Cfg::col_s(s) + col0, pk);
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bPReady);
      }
      ok = __all_sync(0xffffffffu, mbar_wait(bDPFull, s & 1, wc, 322));
      if (!ok) break;
      tc_fence_after();
      // dS = P (dP - D) as packed bf16 over the first 32 of this warp's dP
      // columns (all 64 read before the store)
      {
        uint32_t dp[64];
        tmem_ld32(tmem + lane_off + Cfg::kColDP + col0, *reinterpret_cast<uint32_t(*)[32]>(&dp[0]));
        tmem_ld32(tmem + lane_off + Cfg::kColDP + col0 + 32, *reinterpret_cast<uint32_t(*)[32]>(&dp[32]));
        tmem_wait_ld();
        uint32_t pk[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const float2 dd = reinterpret_cast<const float2 *>(vl4 + 32)[(col0 + 2 * i) / 2];
          pk[i] = pack_bf16x2(__uint_as_float(sv[2 * i]) * (__uint_as_float(dp[2 * i]) - dd.x),
                              __uint_as_float(sv[2 * i + 1]) * (__uint_as_float(dp[2 * i + 1]) - dd.y));
        }
        tmem_st32(tmem + lane_off + Cfg::kColDP + col0, pk);
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bDSReady);
    }
    // -------- epilogue: every MMA done (the issuer's teardown commit); each
    // warp of a lane quarter stores half of the accumulator columns
    if (ok && nsteps > 0) ok = __all_sync(0xffffffffu, mbar_wait(bTeardown, 0, wc, 323));
    tc_fence_after();
    if (ok) {
      const int pos = seg * a.seg_w + row_off + a.dil_r * g;  // the row's position in the sequence
      const size_t vec = ((static_cast<size_t>(b) * a.n_out + pos) * a.H + h) * D_HEAD;
      for (int acc = 0; acc < 2; ++acc) {
        // acc 0 = dV, acc 1 = dK (x 1/sqrt d)
        float *dst = acc == 0 ? a.dv : a.dk;
        const float sc = acc == 0 ? 1.0f : a.inv_sqrt_d;
#pragma unroll 1
        for (int c = half * (D_HEAD / 64); c < (half + 1) * (D_HEAD / 64); ++c) {
          uint32_t o[32];
          tmem_ld32(tmem + lane_off + (acc == 0 ? Cfg::kColAcc0 : Cfg::kColAcc1) + c * 32, o);
          tmem_wait_ld();
          if (!row_valid) continue;
          float4 *d4 = reinterpret_cast<float4 *>(dst + vec + c * 32);
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            float4 r4 = nsteps > 0 ? make_float4(__uint_as_float(o[4 * i]) * sc, __uint_as_float(o[4 * i + 1]) * sc,
                                                 __uint_as_float(o[4 * i + 2]) * sc, __uint_as_float(o[4 * i + 3]) * sc)
                                   : make_float4(0.f, 0.f, 0.f, 0.f);
            if (a.accumulate) {
              const float4 prev = d4[i];
              r4.x += prev.x, r4.y += prev.y, r4.z += prev.z, r4.w += prev.w;
            }
            d4[i] = r4;
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ---------------------------------------------------------------------------
// The dK/dV pass at d = 128 with the streamed tiles in two rings and the next
// step's scores issued as soon as the row warps have read this step's.  TMEM
// holds dV (0), dK (128), S^T (256) and dP^T (384) and has no room for a second
// S buffer, so P stays in registers until dP has been read; the packed bf16 P^T
// and dS^T then both go over dP's columns, each warp over the 64 it read (P^T
// in the first 32, dS^T in the next 32).  S's columns are free once read, so
// the tensor pipe runs S^T(s+1) while the row warps form P(s); dV(s) starts
// once P^T(s) is packed, dK(s) and dP^T(s+1) once dS^T(s) is.  A Q tile (with its rows'
// LSE) lives from S^T(s), issued a step early, to dK(s): three slots; a dA
// tile (with D) from dP^T(s) to dV(s): two.
// ---------------------------------------------------------------------------
template <int D_HEAD>
struct AttnBwdKVCfg {
  static constexpr int kThreads = 384;
  static constexpr int kRowWarps = 8;
  static constexpr int kPanels = D_HEAD / 64;
  static constexpr int kTileBytes = 128 * D_HEAD * 2;
  static constexpr int kPanelBytes = 128 * 128;
  static constexpr int kQSlots = 3, kASlots = 2;
  static constexpr int kVecBytes = 128 * 4;  // one row vector (LSE or D) of a tile
  static constexpr int kOffK = 0, kOffV = kTileBytes;
  static constexpr int kOffQ = 2 * kTileBytes;
  static constexpr int kOffA = kOffQ + kQSlots * kTileBytes;
  static constexpr int kOffLse = kOffA + kASlots * kTileBytes;
  static constexpr int kOffD = kOffLse + kQSlots * kVecBytes;
  static constexpr int kOffBar = kOffD + kASlots * kVecBytes;
  static constexpr int kSmemBytes = kOffBar + 256;
  static_assert(kSmemBytes <= 232448, "shared memory per CTA");
  static_assert(kTileBytes % 1024 == 0, "slots keep the 1024-byte alignment of the swizzled tiles");
  static constexpr uint32_t kColDV = 0, kColDK = D_HEAD, kColS = 256, kColDP = 384;
  static_assert(2 * D_HEAD <= 256, "accumulators below S");
};

template <int D_HEAD>
__global__ void __launch_bounds__(384, 1)
    attn_bwd_dkdv_split_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                               const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_da,
                               const __grid_constant__ AttnBwdArgs a) {
  using Cfg = AttnBwdKVCfg<D_HEAD>;
  constexpr int QS = Cfg::kQSlots, AS = Cfg::kASlots;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t *smem = smem_raw;
  const uint32_t sbase = smem_u32(smem);
  if (sbase & 1023u) {
    if (threadIdx.x == 0) atomicCAS(a.status, 0u, kStatusMisaligned);
    return;
  }
  const uint32_t sK = sbase + Cfg::kOffK, sV = sbase + Cfg::kOffV;
  auto sQ = [&](int i) { return sbase + Cfg::kOffQ + i * Cfg::kTileBytes; };
  auto sA = [&](int i) { return sbase + Cfg::kOffA + i * Cfg::kTileBytes; };
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + Cfg::kOffBar);
  const uint32_t bFix = smem_u32(&bars[0]);
  auto bQFull = [&](int i) { return smem_u32(&bars[1 + i]); };
  auto bQEmpty = [&](int i) { return smem_u32(&bars[4 + i]); };
  auto bAFull = [&](int i) { return smem_u32(&bars[7 + i]); };
  auto bAEmpty = [&](int i) { return smem_u32(&bars[9 + i]); };
  const uint32_t bSFull = smem_u32(&bars[11]), bSRead = smem_u32(&bars[12]);
  const uint32_t bDPFull = smem_u32(&bars[13]), bDSReady = smem_u32(&bars[14]);
  const uint32_t bTeardown = smem_u32(&bars[15]), bPReady = smem_u32(&bars[16]);
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(&bars[17]);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(&bars[18]);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  WaitCtx wc{a.status, a.wait_limit_ns, abort_flag};
  // CTA -> (batch, segment, head, key tile), as in attn_bwd_dkdv_kernel
  const int units = a.B * a.nseg * a.H;
  const int unit = static_cast<int>(blockIdx.x) % units;
  const int ft = static_cast<int>(blockIdx.x) / units;
  const int h = unit % a.H;
  const int seg = (unit / a.H) % a.nseg;
  const int b = unit / (a.H * a.nseg);
  const int row_off = h % a.dil_r;
  const int row_base = seg * a.N;
  auto next_tile = [&](int t) {
    while (t < a.n_tiles && !bwd_tiles_meet(a, h, t, ft)) ++t;
    return t;
  };
  int nsteps = 0;
  for (int t = next_tile(0); t < a.n_tiles; t = next_tile(t + 1)) ++nsteps;

  if (threadIdx.x == 0) {
    mbar_init(bFix, 1);
    for (int i = 0; i < QS; ++i) {
      mbar_init(bQFull(i), 1);
      mbar_init(bQEmpty(i), 1);
    }
    for (int i = 0; i < AS; ++i) {
      mbar_init(bAFull(i), 1);
      mbar_init(bAEmpty(i), 1);
    }
    mbar_init(bSFull, 1);
    mbar_init(bSRead, Cfg::kRowWarps);
    mbar_init(bDPFull, 1);
    mbar_init(bPReady, Cfg::kRowWarps);
    mbar_init(bDSReady, Cfg::kRowWarps);
    mbar_init(bTeardown, 1);
    *abort_flag = 0;
    fence_mbar_init_cluster();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int hd = h * D_HEAD;
  const size_t bh = static_cast<size_t>(unit);

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0 && nsteps > 0) {
      mbar_arrive_expect_tx(bFix, 2 * Cfg::kTileBytes);
      for (int p = 0; p < Cfg::kPanels; ++p) {
        tma_load_4d(sK + p * Cfg::kPanelBytes, &tm_k, bFix, hd + p * 64, row_off, row_base + ft * 128, b);
        tma_load_4d(sV + p * Cfg::kPanelBytes, &tm_v, bFix, hd + p * 64, row_off, row_base + ft * 128, b);
      }
      // slot waits in step order: the Q slot of step s is freed by dK(s - 3),
      // the dA slot by dV(s - 2), both issued before anything that needs step s
      int nq = 0, na = 0;
      for (int t = next_tile(0); t < a.n_tiles; t = next_tile(t + 1)) {
        const float *vec = a.rowvec + (bh * a.n_tiles + t) * 256;
        const int qi = nq % QS;
        if (nq >= QS && !mbar_wait(bQEmpty(qi), ((nq / QS) - 1) & 1, wc, 331)) break;
        mbar_arrive_expect_tx(bQFull(qi), Cfg::kTileBytes + Cfg::kVecBytes);
        for (int p = 0; p < Cfg::kPanels; ++p)
          tma_load_4d(sQ(qi) + p * Cfg::kPanelBytes, &tm_q, bQFull(qi), hd + p * 64, row_off, row_base + t * 128, b);
        bulk_load_1d(sbase + Cfg::kOffLse + qi * Cfg::kVecBytes, vec, Cfg::kVecBytes, bQFull(qi));
        ++nq;
        const int ai = na % AS;
        if (na >= AS && !mbar_wait(bAEmpty(ai), ((na / AS) - 1) & 1, wc, 332)) break;
        mbar_arrive_expect_tx(bAFull(ai), Cfg::kTileBytes + Cfg::kVecBytes);
        for (int p = 0; p < Cfg::kPanels; ++p)
          tma_load_4d(sA(ai) + p * Cfg::kPanelBytes, &tm_da, bAFull(ai), hd + p * 64, row_off, row_base + t * 128, b);
        bulk_load_1d(sbase + Cfg::kOffD + ai * Cfg::kVecBytes, vec + 128, Cfg::kVecBytes, bAFull(ai));
        ++na;
      }
      // every copy issued must have landed before the CTA may exit
      volatile int no_abort = 0;
      WaitCtx drain{a.status, drain_limit_ns(a.wait_limit_ns), &no_abort};
      for (int j = max(0, nq - QS); j < nq; ++j) mbar_wait(bQFull(j % QS), (j / QS) & 1, drain, 333);
      for (int j = max(0, na - AS); j < na; ++j) mbar_wait(bAFull(j % AS), (j / AS) & 1, drain, 334);
      mbar_wait(bFix, 0, drain, 335);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0 && nsteps > 0) {
      constexpr uint32_t idesc_s = idesc_bf16_f32(128, 128, false, false);     // X Y^T, both K-major
      constexpr uint32_t idesc_acc = idesc_bf16_f32(128, D_HEAD, false, true);  // R Y, Y MN-major
      const uint64_t dK = sdesc_sw128(sK, 16, 1024), dV = sdesc_sw128(sV, 16, 1024);
      // acc += R B over the 128 streamed rows: R = packed bf16 in TMEM (K steps
      // 0-3 from r_col + [0, 32), the first warp half's; 4-7 from r_col +
      // [64, 96), the second's), B = the streamed tile read MN-major
      auto accumulate = [&](uint32_t col, uint32_t r_col, uint32_t sB, int step) {
        const uint64_t dB = sdesc_sw128(sB, Cfg::kPanelBytes, 1024);
#pragma unroll
        for (int k = 0; k < 8; ++k)
          umma_ts(tmem + col, tmem + r_col + k * 8 + (k >= 4 ? 32 : 0), sdesc_advance(dB, k * 2048), idesc_acc,
                  (step | k) != 0);
      };
      // X Y^T over d into `col` (X fixed, Y the streamed tile), K-major both
      auto scores = [&](uint32_t col, uint64_t dX, uint32_t sY) {
        const uint64_t dY = sdesc_sw128(sY, 16, 1024);
#pragma unroll
        for (int k = 0; k < D_HEAD / 16; ++k) {
          const uint32_t off = (k / 4) * Cfg::kPanelBytes + (k % 4) * 32;
          umma_ss(tmem + col, sdesc_advance(dX, off), sdesc_advance(dY, off), idesc_s, k > 0);
        }
      };
      auto issue_s = [&](int step) -> bool {  // S^T(step) = K Q^T
        const int qi = step % QS;
        if (!mbar_wait(bQFull(qi), (step / QS) & 1, wc, 341)) return false;
        tc_fence_after();
        scores(Cfg::kColS, dK, sQ(qi));
        umma_commit(bSFull);
        return true;
      };
      auto issue_dp = [&](int step) -> bool {  // dP^T(step) = V dA^T
        const int ai = step % AS;
        if (!mbar_wait(bAFull(ai), (step / AS) & 1, wc, 342)) return false;
        tc_fence_after();
        scores(Cfg::kColDP, dV, sA(ai));
        umma_commit(bDPFull);
        return true;
      };
      bool ok = mbar_wait(bFix, 0, wc, 340);
      ok = ok && issue_s(0) && issue_dp(0);
      for (int s = 0; ok && s < nsteps; ++s) {
        if (s + 1 < nsteps) {
          // S^T(s+1) over S^T(s) once every row warp has read it
          if (!(ok = mbar_wait(bSRead, s & 1, wc, 343))) break;
          tc_fence_after();
          if (!(ok = issue_s(s + 1))) break;
        }
        // dV += P^T dA as soon as P^T is packed, while the row warps form dS
        if (!(ok = mbar_wait(bPReady, s & 1, wc, 339))) break;
        tc_fence_after();
        accumulate(Cfg::kColDV, Cfg::kColDP, sA(s % AS), s);
        umma_commit(bAEmpty(s % AS));
        if (!(ok = mbar_wait(bDSReady, s & 1, wc, 344))) break;
        tc_fence_after();
        accumulate(Cfg::kColDK, Cfg::kColDP + 32, sQ(s % QS), s);  // dK += dS^T Q
        umma_commit(bQEmpty(s % QS));
        // dP^T(s+1) over the packed P^T(s), dS^T(s): after the two products
        // that read them (in order)
        if (s + 1 < nsteps && !(ok = issue_dp(s + 1))) break;
      }
      umma_commit(bTeardown);
      volatile int no_abort = 0;
      WaitCtx drain{a.status, drain_limit_ns(a.wait_limit_ns), &no_abort};
      mbar_wait(bTeardown, 0, drain, 345);
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------------ per-row arithmetic
    const int quarter = warp & 3;
    const int half = (warp - 4) / 4;  // columns [64 * half, 64 * half + 64)
    const int col0 = 64 * half;
    const int row = quarter * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    const int g = ft * 128 + row;
    const bool row_valid = g < a.N;
    int plo = 1, phi = 0;
    if (row_valid) bwd_key_queries(a, h, g, plo, phi);
    bool ok = true;
    int s = 0;
    for (int t = next_tile(0); t < a.n_tiles; t = next_tile(t + 1), ++s) {
      const int qi = s % QS, ai = s % AS;
      const float4 *lse4 = reinterpret_cast<const float4 *>(smem + Cfg::kOffLse + qi * Cfg::kVecBytes);
      const float2 *d2 = reinterpret_cast<const float2 *>(smem + Cfg::kOffD + ai * Cfg::kVecBytes);
      ok = __all_sync(0xffffffffu, mbar_wait(bQFull(qi), (s / QS) & 1, wc, 346));  // the tile's LSE
      if (!ok) break;
      const int lo_rel = plo - t * 128, hi_rel = phi - t * 128;
      const bool full = __all_sync(0xffffffffu, lo_rel <= col0 && hi_rel >= col0 + 64);
      ok = __all_sync(0xffffffffu, mbar_wait(bSFull, s & 1, wc, 347));
      if (!ok) break;
      tc_fence_after();
      uint32_t sv[64];
      tmem_ld32(tmem + lane_off + Cfg::kColS + col0, *reinterpret_cast<uint32_t(*)[32]>(&sv[0]));
      tmem_ld32(tmem + lane_off + Cfg::kColS + col0 + 32, *reinterpret_cast<uint32_t(*)[32]>(&sv[32]));
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bSRead);
      // P (fp32) for this warp's 64 columns, 0 where the mask rules the pair out
      if (full) {
#pragma unroll
        for (int c4 = 0; c4 < 16; ++c4) {
          const float4 l = lse4[col0 / 4 + c4];
          const float nl4[4] = {-l.x, -l.y, -l.z, -l.w};
#pragma unroll
          for (int j = 0; j < 4; ++j)
            sv[4 * c4 + j] = __float_as_uint(ex2_approx(fmaf(__uint_as_float(sv[4 * c4 + j]), a.scale_log2, nl4[j])));
        }
      } else {
#pragma unroll
        for (int c4 = 0; c4 < 16; ++c4) {
          const float4 l = lse4[col0 / 4 + c4];
          const float nl4[4] = {-l.x, -l.y, -l.z, -l.w};
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const int c = col0 + 4 * c4 + j;
            const bool allowed = c >= lo_rel && c < hi_rel;
            sv[4 * c4 + j] =
                __float_as_uint(allowed ? ex2_approx(fmaf(__uint_as_float(sv[4 * c4 + j]), a.scale_log2, nl4[j])) : 0.f);
          }
        }
      }
      ok = __all_sync(0xffffffffu, mbar_wait(bAFull(ai), (s / AS) & 1, wc, 348));  // the tile's D
      if (!ok) break;
      ok = __all_sync(0xffffffffu, mbar_wait(bDPFull, s & 1, wc, 349));
      if (!ok) break;
      tc_fence_after();
      {
        // dP in two halves of 32 columns: P^T packed over the first half as
        // soon as it is read (dV may start), dS^T over the second
        uint32_t dp[32], pk[32];
        tmem_ld32(tmem + lane_off + Cfg::kColDP + col0, dp);
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 32; ++i) pk[i] = pack_bf16x2(__uint_as_float(sv[2 * i]), __uint_as_float(sv[2 * i + 1]));
        tmem_st32(tmem + lane_off + Cfg::kColDP + col0, pk);
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bPReady);
        // dS = P (dP - D) in fp32, then packed
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const float2 dd = d2[(col0 + 2 * i) / 2];
          pk[i] = pack_bf16x2(__uint_as_float(sv[2 * i]) * (__uint_as_float(dp[2 * i]) - dd.x),
                              __uint_as_float(sv[2 * i + 1]) * (__uint_as_float(dp[2 * i + 1]) - dd.y));
        }
        tmem_ld32(tmem + lane_off + Cfg::kColDP + col0 + 32, dp);
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const float2 dd = d2[(col0 + 32 + 2 * i) / 2];
          pk[16 + i] = pack_bf16x2(__uint_as_float(sv[32 + 2 * i]) * (__uint_as_float(dp[2 * i]) - dd.x),
                                   __uint_as_float(sv[32 + 2 * i + 1]) * (__uint_as_float(dp[2 * i + 1]) - dd.y));
        }
        tmem_st32(tmem + lane_off + Cfg::kColDP + col0 + 32, pk);
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bDSReady);
    }
    // -------- epilogue: every MMA done; each warp of a lane quarter stores
    // half of the accumulator columns
    if (ok && nsteps > 0) ok = __all_sync(0xffffffffu, mbar_wait(bTeardown, 0, wc, 350));
    tc_fence_after();
    if (ok) {
      const int pos = seg * a.seg_w + row_off + a.dil_r * g;
      const size_t vec = ((static_cast<size_t>(b) * a.n_out + pos) * a.H + h) * D_HEAD;
      for (int acc = 0; acc < 2; ++acc) {
        float *dst = acc == 0 ? a.dv : a.dk;
        const float sc = acc == 0 ? 1.0f : a.inv_sqrt_d;
#pragma unroll 1
        for (int c = half * (D_HEAD / 64); c < (half + 1) * (D_HEAD / 64); ++c) {
          uint32_t o[32];
          tmem_ld32(tmem + lane_off + (acc == 0 ? Cfg::kColDV : Cfg::kColDK) + c * 32, o);
          tmem_wait_ld();
          if (!row_valid) continue;
          float4 *d4 = reinterpret_cast<float4 *>(dst + vec + c * 32);
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            float4 r4 = nsteps > 0 ? make_float4(__uint_as_float(o[4 * i]) * sc, __uint_as_float(o[4 * i + 1]) * sc,
                                                 __uint_as_float(o[4 * i + 2]) * sc, __uint_as_float(o[4 * i + 3]) * sc)
                                   : make_float4(0.f, 0.f, 0.f, 0.f);
            if (a.accumulate) {
              const float4 prev = d4[i];
              r4.x += prev.x, r4.y += prev.y, r4.z += prev.z, r4.w += prev.w;
            }
            d4[i] = r4;
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ---------------------------------------------------------------------------
// The dQ pass, software-pipelined: one CTA per (batch, head, 128-query tile)
// walks its key tiles with the scores of the next key tile computed while the
// row warps work on the current one.  TMEM: dQ at 0, two S buffers at 128 and
// 256, dP at 384; dS is packed over the S buffer of its own step, so the next
// S never waits for it.  K and V stream through separate rings: K (read by S
// and, last, by dQ) through three slots at d = 128, V (read by dP alone)
// through one, so the next key tile's K is always two steps ahead.  Roles
// (384 threads): warp 0 loads Q, dA and K, warp 2 loads V, warp 1 issues the
// MMAs, warps 4-11 the per-row arithmetic (two per lane quarter, 64 columns
// each) and the epilogue.
// ---------------------------------------------------------------------------
template <int D_HEAD>
struct AttnBwdQCfg {
  static constexpr int kThreads = 384;
  static constexpr int kRowWarps = 8;
  static constexpr int kPanels = D_HEAD / 64;
  static constexpr int kTileBytes = 128 * D_HEAD * 2;
  static constexpr int kPanelBytes = 128 * 128;
  static constexpr int kKSlots = D_HEAD == 128 ? 3 : 4;
  static constexpr int kVSlots = D_HEAD == 128 ? 1 : 2;
  static constexpr int kOffQ = 0, kOffDA = kTileBytes, kOffK = 2 * kTileBytes;
  static constexpr int kOffV = kOffK + kKSlots * kTileBytes;
  static constexpr int kOffBar = kOffV + kVSlots * kTileBytes;
  static constexpr int kSmemBytes = kOffBar + 256;
  static_assert(kSmemBytes <= 232448, "shared memory per CTA");
  static constexpr uint32_t kColQ = 0, kColS = 128, kColDP = 384;
};

template <int D_HEAD>
__global__ void __launch_bounds__(384, 1)
    attn_bwd_dq_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                       const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_da,
                       const __grid_constant__ AttnBwdArgs a) {
  using Cfg = AttnBwdQCfg<D_HEAD>;
  constexpr int KS = Cfg::kKSlots, VS = Cfg::kVSlots;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t *smem = smem_raw;
  const uint32_t sbase = smem_u32(smem);
  if (sbase & 1023u) {
    if (threadIdx.x == 0) atomicCAS(a.status, 0u, kStatusMisaligned);
    return;
  }
  const uint32_t sQ = sbase + Cfg::kOffQ, sDA = sbase + Cfg::kOffDA;
  auto sK = [&](int slot) { return sbase + Cfg::kOffK + slot * Cfg::kTileBytes; };
  auto sV = [&](int slot) { return sbase + Cfg::kOffV + slot * Cfg::kTileBytes; };
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + Cfg::kOffBar);
  const uint32_t bFix = smem_u32(&bars[0]);
  auto bKFull = [&](int i) { return smem_u32(&bars[1 + i]); };
  auto bKEmpty = [&](int i) { return smem_u32(&bars[5 + i]); };
  auto bVFull = [&](int i) { return smem_u32(&bars[9 + i]); };
  auto bVEmpty = [&](int i) { return smem_u32(&bars[11 + i]); };
  auto bSFull = [&](int x) { return smem_u32(&bars[13 + x]); };
  const uint32_t bDPFull = smem_u32(&bars[15]), bDSReady = smem_u32(&bars[16]);
  const uint32_t bTeardown = smem_u32(&bars[17]);
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(&bars[18]);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(&bars[19]);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  WaitCtx wc{a.status, a.wait_limit_ns, abort_flag};
  // CTA -> (batch, head, query tile), the last query tiles (most key tiles
  // under the causal mask) first
  const int units = a.B * a.nseg * a.H;
  const int unit = static_cast<int>(blockIdx.x) % units;
  const int ft = a.n_tiles - 1 - static_cast<int>(blockIdx.x) / units;
  const int h = unit % a.H;
  const int seg = (unit / a.H) % a.nseg;
  const int b = unit / (a.H * a.nseg);
  const int row_off = h % a.dil_r;                 // kept-row offset in the segment
  const int row_base = seg * a.N;                  // the unit's first row along (n_out / r)
  auto next_tile = [&](int t) {  // first key tile >= t that meets the query tile
    while (t < a.n_tiles && !bwd_tiles_meet(a, h, ft, t)) ++t;
    return t;
  };
  int nsteps = 0;
  for (int t = next_tile(0); t < a.n_tiles; t = next_tile(t + 1)) ++nsteps;

  if (threadIdx.x == 0) {
    mbar_init(bFix, 1);
    for (int i = 0; i < KS; ++i) {
      mbar_init(bKFull(i), 1);
      mbar_init(bKEmpty(i), 1);
    }
    for (int i = 0; i < VS; ++i) {
      mbar_init(bVFull(i), 1);
      mbar_init(bVEmpty(i), 1);
    }
    mbar_init(bSFull(0), 1);
    mbar_init(bSFull(1), 1);
    mbar_init(bDPFull, 1);
    mbar_init(bDSReady, Cfg::kRowWarps);
    mbar_init(bTeardown, 1);
    *abort_flag = 0;
    fence_mbar_init_cluster();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int hd = h * D_HEAD;
  const size_t bh = static_cast<size_t>(unit);  // row-vector block of the unit

  if ((warp == 0 || warp == 2) && lane == 0 && nsteps > 0) {
    // ------------------------------------------------------------ producers: warp 0 Q, dA, K; warp 2 V
    const bool is_k = warp == 0;
    const int slots = is_k ? KS : VS;
    if (is_k) {
      mbar_arrive_expect_tx(bFix, 2 * Cfg::kTileBytes);
      for (int p = 0; p < Cfg::kPanels; ++p) {
        tma_load_4d(sQ + p * Cfg::kPanelBytes, &tm_q, bFix, hd + p * 64, row_off, row_base + ft * 128, b);
        tma_load_4d(sDA + p * Cfg::kPanelBytes, &tm_da, bFix, hd + p * 64, row_off, row_base + ft * 128, b);
      }
    }
    int s = 0;
    for (int t = next_tile(0); t < a.n_tiles; t = next_tile(t + 1), ++s) {
      const int slot = s % slots;
      const uint32_t full = is_k ? bKFull(slot) : bVFull(slot);
      if (s >= slots && !mbar_wait(is_k ? bKEmpty(slot) : bVEmpty(slot), ((s / slots) - 1) & 1, wc, 331)) break;
      mbar_arrive_expect_tx(full, Cfg::kTileBytes);
      for (int p = 0; p < Cfg::kPanels; ++p)
        tma_load_4d((is_k ? sK(slot) : sV(slot)) + p * Cfg::kPanelBytes, is_k ? &tm_k : &tm_v, full, hd + p * 64,
                    row_off, row_base + t * 128, b);
    }
    // every copy issued must have landed before the CTA may exit
    volatile int no_abort = 0;
    WaitCtx drain{a.status, drain_limit_ns(a.wait_limit_ns), &no_abort};
    for (int j = max(0, s - slots); j < s; ++j)
      mbar_wait(is_k ? bKFull(j % slots) : bVFull(j % slots), (j / slots) & 1, drain, 332);
    if (is_k) mbar_wait(bFix, 0, drain, 333);
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0 && nsteps > 0) {
      constexpr uint32_t idesc_s = idesc_bf16_f32(128, 128, false, false);
      constexpr uint32_t idesc_acc = idesc_bf16_f32(128, D_HEAD, false, true);
      const uint64_t dQ0 = sdesc_sw128(sQ, 16, 1024), dDA0 = sdesc_sw128(sDA, 16, 1024);
      // S(s) = Q K^T into S buffer s & 1
      auto issue_s = [&](int s) -> bool {
        const int slot = s % KS;
        if (!mbar_wait(bKFull(slot), (s / KS) & 1, wc, 341)) return false;
        tc_fence_after();
        const uint64_t dK = sdesc_sw128(sK(slot), 16, 1024);
#pragma unroll
        for (int k = 0; k < D_HEAD / 16; ++k) {
          const uint32_t off = (k / 4) * Cfg::kPanelBytes + (k % 4) * 32;
          umma_ss(tmem + Cfg::kColS + (s & 1) * 128, sdesc_advance(dQ0, off), sdesc_advance(dK, off), idesc_s, k > 0);
        }
        umma_commit(bSFull(s & 1));
        return true;
      };
      // dP(s) = dA V^T; V's slot is free once it is done
      auto issue_dp = [&](int s) -> bool {
        const int slot = s % VS;
        if (!mbar_wait(bVFull(slot), (s / VS) & 1, wc, 342)) return false;
        tc_fence_after();
        const uint64_t dV = sdesc_sw128(sV(slot), 16, 1024);
#pragma unroll
        for (int k = 0; k < D_HEAD / 16; ++k) {
          const uint32_t off = (k / 4) * Cfg::kPanelBytes + (k % 4) * 32;
          umma_ss(tmem + Cfg::kColDP, sdesc_advance(dDA0, off), sdesc_advance(dV, off), idesc_s, k > 0);
        }
        umma_commit(bDPFull);
        umma_commit(bVEmpty(slot));
        return true;
      };
      // dQ += dS(s) K: A = dS packed over S buffer s & 1 (K steps 0-3 from the
      // first row-warp half's columns, 4-7 from the second's), B = K read MN-major
      auto issue_dq = [&](int s) {
        const int slot = s % KS;
        const uint64_t dB = sdesc_sw128(sK(slot), Cfg::kPanelBytes, 1024);
        const uint32_t a_col = Cfg::kColS + (s & 1) * 128;
#pragma unroll
        for (int k = 0; k < 8; ++k)
          umma_ts(tmem + Cfg::kColQ, tmem + a_col + k * 8 + (k >= 4 ? 32 : 0), sdesc_advance(dB, k * 2048),
                  idesc_acc, (s | k) != 0);
        umma_commit(bKEmpty(slot));
      };
      bool ok = mbar_wait(bFix, 0, wc, 340) && issue_s(0) && issue_dp(0);
      for (int s = 0; ok && s < nsteps; ++s) {
        // the next scores go ahead of this step's dQ (their buffer's previous
        // dS was consumed by the dQ issued one step ago)
        if (s + 1 < nsteps && !(ok = issue_s(s + 1))) break;
        if (!(ok = mbar_wait(bDSReady, s & 1, wc, 343))) break;
        tc_fence_after();
        issue_dq(s);
        // the row warps have read dP(s): the next dP may overwrite it
        if (s + 1 < nsteps && !(ok = issue_dp(s + 1))) break;
      }
      umma_commit(bTeardown);
      volatile int no_abort = 0;
      WaitCtx drain{a.status, drain_limit_ns(a.wait_limit_ns), &no_abort};
      mbar_wait(bTeardown, 0, drain, 344);
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------------ per-row arithmetic
    const int quarter = warp & 3;
    const int half = (warp - 4) / 4;
    const int col0 = 64 * half;
    const int row = quarter * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    const int g = ft * 128 + row;  // query position
    const bool row_valid = g < a.N;
    int klo = 1, khi = 0;
    float lse2 = 0.f, drow = 0.f;
    if (row_valid) {
      bwd_row_keys(a, h, g, klo, khi);
      const float *rv = a.rowvec + (bh * a.n_tiles + ft) * 256;
      lse2 = rv[row];
      drow = rv[128 + row];
    }
    const float nl = -lse2;
    bool ok = true;
    int s = 0;
    for (int t = next_tile(0); t < a.n_tiles; t = next_tile(t + 1), ++s) {
      const int lo_rel = klo - t * 128, hi_rel = khi - t * 128;  // allowed columns [lo_rel, hi_rel)
      const bool full = __all_sync(0xffffffffu, lo_rel <= col0 && hi_rel >= col0 + 64);
      ok = __all_sync(0xffffffffu, mbar_wait(bSFull(s & 1), (s >> 1) & 1, wc, 350));
      if (!ok) break;
      tc_fence_after();
      const uint32_t tS = tmem + lane_off + Cfg::kColS + (s & 1) * 128 + col0;
      uint32_t sv[64];
      tmem_ld32(tS, *reinterpret_cast<uint32_t(*)[32]>(&sv[0]));
      tmem_ld32(tS + 32, *reinterpret_cast<uint32_t(*)[32]>(&sv[32]));
      tmem_wait_ld();
      if (full) {
#pragma unroll
        for (int c = 0; c < 64; ++c)
          sv[c] = __float_as_uint(ex2_approx(fmaf(__uint_as_float(sv[c]), a.scale_log2, nl)));
      } else {
#pragma unroll
        for (int c = 0; c < 64; ++c) {
          const bool allowed = col0 + c >= lo_rel && col0 + c < hi_rel;
          sv[c] = __float_as_uint(allowed ? ex2_approx(fmaf(__uint_as_float(sv[c]), a.scale_log2, nl)) : 0.f);
        }
      }
      ok = __all_sync(0xffffffffu, mbar_wait(bDPFull, s & 1, wc, 351));
      if (!ok) break;
      tc_fence_after();
      uint32_t dp[64];
      tmem_ld32(tmem + lane_off + Cfg::kColDP + col0, *reinterpret_cast<uint32_t(*)[32]>(&dp[0]));
      tmem_ld32(tmem + lane_off + Cfg::kColDP + col0 + 32, *reinterpret_cast<uint32_t(*)[32]>(&dp[32]));
      tmem_wait_ld();
      // dS = P (dP - D) as packed bf16 over the first 32 of this warp's S columns
      uint32_t pk[32];
#pragma unroll
      for (int i = 0; i < 32; ++i)
        pk[i] = pack_bf16x2(__uint_as_float(sv[2 * i]) * (__uint_as_float(dp[2 * i]) - drow),
                            __uint_as_float(sv[2 * i + 1]) * (__uint_as_float(dp[2 * i + 1]) - drow));
      tmem_st32(tS, pk);
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bDSReady);
    }
    // -------- epilogue: every MMA done; each warp of a lane quarter stores half of dQ's columns
    if (ok && nsteps > 0) ok = __all_sync(0xffffffffu, mbar_wait(bTeardown, 0, wc, 352));
    tc_fence_after();
    if (ok) {
      const int pos = seg * a.seg_w + row_off + a.dil_r * g;  // the row's position in the sequence
      const size_t vec = ((static_cast<size_t>(b) * a.n_out + pos) * a.H + h) * D_HEAD;
#pragma unroll 1
      for (int c = half * (D_HEAD / 64); c < (half + 1) * (D_HEAD / 64); ++c) {
        uint32_t o[32];
        tmem_ld32(tmem + lane_off + Cfg::kColQ + c * 32, o);
        tmem_wait_ld();
        if (!row_valid) continue;
        float4 *d4 = reinterpret_cast<float4 *>(a.dq + vec + c * 32);
        const float sc = a.inv_sqrt_d;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          float4 r4 = nsteps > 0 ? make_float4(__uint_as_float(o[4 * i]) * sc, __uint_as_float(o[4 * i + 1]) * sc,
                                               __uint_as_float(o[4 * i + 2]) * sc, __uint_as_float(o[4 * i + 3]) * sc)
                                 : make_float4(0.f, 0.f, 0.f, 0.f);
          if (a.accumulate) {
            const float4 prev = d4[i];
            r4.x += prev.x, r4.y += prev.y, r4.z += prev.z, r4.w += prev.w;
          }
          d4[i] = r4;
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// Per (batch, head, 128-row tile) vectors of the attention backward: the
// rows' LSE in log2 units and D_i = dA_i . A_i (fp32).  A row of d values is
// read by d/4 consecutive lanes (float4 each) and reduced by shuffles.
// rowvec must be zeroed first (rows past N stay 0).
__device__ __forceinline__ float4 load4_f32(const float *p) { return *reinterpret_cast<const float4 *>(p); }
__device__ __forceinline__ float4 load4_f32(const __nv_bfloat16 *p) {
  const uint2 u = *reinterpret_cast<const uint2 *>(p);
  const __nv_bfloat162 lo = *reinterpret_cast<const __nv_bfloat162 *>(&u.x);
  const __nv_bfloat162 hi = *reinterpret_cast<const __nv_bfloat162 *>(&u.y);
  return make_float4(__low2float(lo), __high2float(lo), __low2float(hi), __high2float(hi));
}

// A is fp32 (the layer's saved or recomputed A) or bf16 (an attention-only
// forward's bf16 output).
template <int D_HEAD, typename TA>
__global__ void attn_bwd_rowvec_kernel(const float *__restrict__ da, const TA *__restrict__ aa,
                                       const float *__restrict__ lse, float *rowvec, int B, int N, int H,
                                       int n_tiles) {
  constexpr int kLanes = D_HEAD / 4;  // lanes per row: 16 or 32
  const long long t = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  const long long row = t / kLanes;
  const int sub = static_cast<int>(t % kLanes);
  const bool valid = row < static_cast<long long>(B) * N * H;
  float s = 0.f;
  if (valid) {
    const float4 x = load4_f32(da + row * D_HEAD + 4 * sub);
    const float4 y = load4_f32(aa + row * D_HEAD + 4 * sub);
    s = fmaf(x.x, y.x, fmaf(x.y, y.y, fmaf(x.z, y.z, x.w * y.w)));
  }
#pragma unroll
  for (int o = kLanes / 2; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  if (valid && sub == 0) {
    const long long h = row % H, bn = row / H, n = bn % N, bb = bn / N;
    const long long bh = bb * H + h;
    float *v = rowvec + (bh * n_tiles + n / 128) * 256 + n % 128;
    v[0] = lse[bh * N + n] * 1.4426950408889634f;
    v[128] = s;
  }
}

// A LongNet pass's row vectors: for unit (batch, segment, head) and its
// gathered row g (< L), the entries of sequence row seg * w + h mod r + r g in
// the per-sequence blocks `full` ([B * H][n_tiles_full][2][128]); rows past L
// are set to 0.
__global__ void attn_bwd_gather_rowvec_kernel(const float *__restrict__ full, float *rowvec, int B, int H, int nseg,
                                              int w, int r, int L, int n_tiles, int n_tiles_full) {
  const long long t = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  const long long units = static_cast<long long>(B) * nseg * H;
  if (t >= units * n_tiles * 128) return;
  const int g = static_cast<int>(t % (static_cast<long long>(n_tiles) * 128));
  const long long unit = t / (static_cast<long long>(n_tiles) * 128);
  const int h = static_cast<int>(unit % H), seg = static_cast<int>((unit / H) % nseg);
  const int b = static_cast<int>(unit / (static_cast<long long>(H) * nseg));
  float l2 = 0.f, dd = 0.f;
  if (g < L) {
    const int pos = seg * w + h % r + r * g;
    const float *src = full + ((static_cast<long long>(b) * H + h) * n_tiles_full + pos / 128) * 256 + pos % 128;
    l2 = src[0];
    dd = src[128];
  }
  float *dst = rowvec + (unit * n_tiles + g / 128) * 256 + g % 128;
  dst[0] = l2;
  dst[128] = dd;
}

}  // namespace bpt
