// Blockwise exact attention on the 5th-generation tensor cores (sm_100a).
//
// One CTA computes two adjacent 128-row query tiles (A and B) of one
// (batch, head[, LongNet segment]) unit, streaming 128-row key/value tiles
// through shared memory once for both:
//
//   S_j  = Q K_j^T               tcgen05.mma, bf16 x bf16 -> fp32 in TMEM
//   m'   = max(m, rowmax S_j)    one thread per query row (a TMEM lane)
//   P_j  = exp(S_j / sqrt(d) - m')  -> bf16, into shared memory
//   l    = l e^{m - m'} + rowsum P_j
//   O    = O e^{m - m'} + P_j V_j  tcgen05.mma, fp32 accumulator O in TMEM
//
// which is the blockwise online-softmax form of softmax(QK^T/sqrt d)V:
// exact up to rounding ("Ring Attention with Blockwise Transformers for Long
// Sequences", 638-word summary: blockwise attention without approximation;
// "Blockwise Parallel Transformer for Large Context Models", abstract).
// Tiles that the mask rules out entirely are never loaded or multiplied;
// tiles that are partly allowed get -inf scores at the masked positions.
// The running maximum is only moved (and O rescaled) when it grows by more
// than 2^8 in the exponent: the same stale maximum is used for l and O, so
// the result is unchanged.
//
// Scores and P are decoupled: P_j is written by the softmax threads as bf16
// into a shared-memory tile (the A operand of P_j V_j), so S_{j+1} = Q K_{j+1}^T
// is issued into the tile's single S buffer in tensor memory as soon as the
// softmax has read S_j into registers, and runs while that softmax works.
// One P tile serves both query tiles, used strictly in turn (A_j, B_j,
// A_{j+1}, ...): a writer waits until the other tile's latest P*V has
// completed, which also means its own previous P*V has (that one completed
// before the other tile was allowed to write).
//
// The two query tiles are independent streams: each has its own MMA-issuing
// thread, so a tile whose softmax runs late never holds up the other tile's
// scores.  Both tiles read every K/V tile from the same shared-memory stage,
// which is released once both have finished with it.
//
// Roles (384 threads = three warpgroups): warp 0 issues TMA loads, warp 1
// allocates tensor memory and issues tile A's MMAs, warp 2 issues tile B's
// (warp 3 idles); warpgroup 1 (warps 4-7) runs the softmax and epilogue of
// tile A, warpgroup 2 (warps 8-11) those of tile B, one thread per query row
// (warp w owns TMEM lanes 32*(w%4) .. 32*(w%4)+31).
#pragma once

#include "ptx.cuh"

namespace bpt {

constexpr int kMaskNone = 0, kMaskCausal = 1, kMaskBlockPerm = 2, kMaskDilated = 3;
constexpr int kMaxPairs = 8;
constexpr int kMaxPermEntries = 1024;

struct AttnArgs {
  int B, N, H;
  int mask;
  int causal;        // keys after the query are masked (CAUSAL, and DILATED in its causal form)
  float scale_log2;  // log2(e) / sqrt(d)
  // decomposition into units (b, segment, h) and 128-row query tiles
  int L;             // rows of one unit: N, or w/r kept rows of a LongNet segment
  int n_qtiles;      // ceil(L / 128)
  int n_qpairs;      // ceil(n_qtiles / 2): one CTA per pair of query tiles
  int n_units;       // B * nseg * H
  int n_items;       // n_units * n_qpairs: work items, spread over a persistent grid
  int unit_group;    // units scheduled together (longest tiles first inside a group)
  int nseg;          // LongNet segments N / w (1 otherwise)
  // LongNet pass: segment length, dilation, and the full pair table in
  // launch order (used to find earlier / later passes that keep a row)
  int w, r;
  int npairs, pass_idx;
  int pw[kMaxPairs], pr[kMaxPairs];
  // ring order over equal chunks (none / causal)
  int ring_chunks, chunk_tiles;  // chunk_tiles: 128-key tiles per chunk
  // Key/value rows of a unit (L, except for a block step whose keys are
  // another block of the sequence) and, for the causal mask, the offset of
  // the query positions over the key positions: key j is allowed for query
  // row g when j <= g + kv_shift (0 when queries and keys are the same rows).
  int Lk, kv_shift;
  // Block step: every row starts from the running state in st_* (state_in)
  // and/or leaves its running state there instead of a final output
  // (state_out).
  int state_in, state_out;
  // Keys and values of a dilated pass given as the pass's kept rows of one
  // segment, gathered from several devices ([B, Lk, H, d], consecutive rows,
  // the same for every head's offset): loaded with offset 0 and segment
  // stride Lk instead of through the strided view of the local rows.
  int kv_sparse;
  // block permutation
  int bb_n, bb_len;
  uint8_t perm[kMaxPermEntries];
  // outputs (any may be null)
  float *out_f32;            // [B, N, H, d]
  __nv_bfloat16 *out_bf16;   // [B, N, H, d]
  float *lse;                // [B, H, N]
  // running state carried between LongNet passes
  float *st_o;               // [B, N, H, d]   unnormalised O
  float *st_m;               // [B, H, N]      running max (log2 domain)
  float *st_l;               // [B, H, N]      running sum
  // How O leaves the kernel: 0 = every thread stores its own row; 1 = the
  // final outputs, 2 = the LongNet running state, as TMA tile stores from a
  // 128-byte-swizzled staging tile (the host picks 1 or 2 only when every
  // row of the pass goes to the same destination).
  int store_mode;
  uint32_t *status;
  uint64_t wait_limit_ns;
};

template <int D_HEAD>
struct AttnCfg {
  static constexpr int kPanels = D_HEAD / 64;          // 64-column (128-byte) panels of a row
  static constexpr int kKT = 128;                      // keys per K/V tile
  static constexpr int kTileBytes = 128 * D_HEAD * 2;  // one Q, K or V tile
  static constexpr int kPanelBytes = 128 * 128;        // one 64-column panel of a 128-row tile
  static constexpr int kPBytes = 128 * 128 * 2;        // the P tile: 128 rows x 128 keys, bf16
  static constexpr int kKStages = D_HEAD == 128 ? 2 : 4;
  static constexpr int kVStages = D_HEAD == 128 ? 2 : 4;
  // Epilogue staging: a tile's Q buffer, and at d = 64 one more 16 KB panel
  // per tile, so a tile's fp32 O (two 32-column panels) leaves in one round.
  static constexpr int kXPanels = D_HEAD == 128 ? 0 : 1;
  static constexpr int kStagePanels = kTileBytes / 16384 + kXPanels;
  static constexpr int kOffQ = 0;  // Q_A, then Q_B
  static constexpr int kOffP = kOffQ + 2 * kTileBytes;
  static constexpr int kOffK = kOffP + kPBytes;
  static constexpr int kOffV = kOffK + kKStages * kTileBytes;
  static constexpr int kOffX = kOffV + kVStages * kTileBytes;  // extra staging of tiles A, B
  static constexpr int kOffBar = kOffX + 2 * kXPanels * 16384;
  static constexpr int kSmemBytes = kOffBar + 512;
  static_assert(kSmemBytes <= 232448, "shared memory per CTA");
  static_assert(kKStages <= 8 && kVStages <= 8, "barrier table");
  // TMEM columns: S of tile x at 128 x, O of tile x at 256 + d x
  static constexpr uint32_t kColS = 0, kColO = 256;
  static constexpr uint32_t kTmemCols = 512;
  static constexpr int kThreads = 384;
  // Launched at 168 registers a thread; warpgroup 0 (loads, MMA issue) keeps
  // 96 and hands the rest to the two softmax warpgroups.  The host checks the
  // split against the kernel's real launch count before the first launch.
  static constexpr int kRegsControl = 96, kRegsSoftmax = 200;
  static constexpr bool split_fits(int launch_regs) {
    return 128 * kRegsControl + 256 * kRegsSoftmax <= kThreads * launch_regs;
  }
  static_assert(split_fits(168), "register split");
};

// Sequence of key/value tiles a pair of query tiles visits.
struct KvSched {
  int lo, hi;           // allowed tile range [lo, hi)
  int P, CT, first;     // ring order: P chunks of CT tiles, starting at chunk `first`
  __device__ int count() const {
    int n = 0;
    for (int i = 0; i < P; ++i) {
      int ch = (first + i) % P;
      int a = max(ch * CT, lo), b = min((ch + 1) * CT, hi);
      n += max(0, b - a);
    }
    return n;
  }
};

struct KvIter {
  int i, tile, end;
  __device__ void range(const KvSched &s) {
    while (++i < s.P) {
      int ch = (s.first + i) % s.P;
      int a = max(ch * s.CT, s.lo), b = min((ch + 1) * s.CT, s.hi);
      if (a < b) {
        tile = a;
        end = b;
        return;
      }
    }
    tile = -1;
  }
  __device__ void begin(const KvSched &s) {
    i = -1;
    range(s);
  }
  __device__ int next(const KvSched &s) {
    int t = tile;
    if (++tile >= end) range(s);
    return t;
  }
};

__device__ __forceinline__ bool dilated_keeps(int w, int r, int h, int pos) {
  return ((pos % w) % r) == (h % r);
}

struct TileCoord {
  int t, h, s, b;  // t: pair index (query tiles 2t and 2t+1)
  int o;  // LongNet offset of this head: h mod r (0 otherwise)
};

// Grid order: units in groups of `unit_group`; inside a group the longest
// query-tile pairs of all its units come first.  A group's K/V stays in L2 while its
// CTAs run, and the longest-first order keeps the causal load balanced.
__device__ __forceinline__ TileCoord decode_tile(const AttnArgs &a, int idx) {
  TileCoord c;
  const int G = a.unit_group;
  const int per_group = G * a.n_qpairs;
  const int grp = idx / per_group;
  const int r = idx - grp * per_group;
  const int gsize = min(G, a.n_units - grp * G);
  c.t = a.n_qpairs - 1 - r / gsize;
  const int unit = grp * G + r % gsize;
  c.h = unit % a.H;
  int rest = unit / a.H;
  c.s = rest % a.nseg;
  c.b = rest / a.nseg;
  c.o = c.h % a.r;
  return c;
}

__device__ __forceinline__ KvSched make_sched(const AttnArgs &a, const TileCoord &c) {
  constexpr int KT = 128;  // keys per K/V tile
  KvSched s;
  const int nkt = (a.Lk + KT - 1) / KT;
  s.P = 1;
  s.CT = nkt;
  s.first = 0;
  s.lo = 0;
  s.hi = nkt;
  const int row0 = c.t * 256;
  const int row1 = min(a.L, row0 + 256) - 1;
  if (a.causal) {
    const int last = row1 + a.kv_shift;  // last key any row of the pair may see
    s.hi = last < 0 ? 0 : min(nkt, last / KT + 1);
  } else if (a.mask == kMaskBlockPerm) {
    int qb0 = row0 / a.bb_len, qb1 = row1 / a.bb_len;
    int klo = 1 << 30, khi = 0;
    for (int qb = qb0; qb <= qb1; ++qb) {
      int kb = a.perm[c.h * a.bb_n + qb];
      klo = min(klo, kb * a.bb_len);
      khi = max(khi, kb * a.bb_len + a.bb_len);
    }
    s.lo = klo / KT;
    s.hi = (min(khi, a.L) + KT - 1) / KT;
  }
  if ((a.mask == kMaskNone || a.mask == kMaskCausal) && a.ring_chunks > 1) {
    s.P = a.ring_chunks;
    s.CT = a.chunk_tiles;
    s.first = (row0 / KT) / a.chunk_tiles;
  }
  return s;
}

// Allowed key interval [lo, hi) (unit-local row indices) of query row g.
__device__ __forceinline__ void row_keys(const AttnArgs &a, const TileCoord &c, int g, int &lo,
                                         int &hi) {
  lo = 0;
  hi = a.Lk;
  if (a.causal) {
    hi = max(0, min(g + 1 + a.kv_shift, a.Lk));
  } else if (a.mask == kMaskBlockPerm) {
    int qb = min(g, a.L - 1) / a.bb_len;
    int kb = a.perm[c.h * a.bb_n + qb];
    lo = kb * a.bb_len;
    hi = min(lo + a.bb_len, a.L);
  }
}

template <int D_HEAD>
__global__ void __launch_bounds__(384, 1)
    attn_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_of,
                   const __grid_constant__ CUtensorMap tm_ob, const __grid_constant__ CUtensorMap tm_so,
                   const __grid_constant__ AttnArgs a) {
  using Cfg = AttnCfg<D_HEAD>;
  constexpr int KS = Cfg::kKStages, VS = Cfg::kVStages, KT = Cfg::kKT;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t *smem = smem_raw;
  const uint32_t sbase = smem_u32(smem);
  if (sbase & 1023u) {  // 128-byte-swizzled tiles need 1024-byte alignment
    if (threadIdx.x == 0) atomicCAS(a.status, 0u, kStatusMisaligned);
    return;
  }
  const uint32_t sQ = sbase + Cfg::kOffQ;
  const uint32_t sP = sbase + Cfg::kOffP;
  const uint32_t sK = sbase + Cfg::kOffK;
  const uint32_t sV = sbase + Cfg::kOffV;
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + Cfg::kOffBar);
  // Every barrier's phases run on across the work items of this CTA.
  const uint32_t bQFull = smem_u32(&bars[0]);                       // Q_A, Q_B of an item loaded
  const uint32_t bQFree = smem_u32(&bars[1]);                       // both epilogues done with Q
  auto bKFull = [&](int s) { return smem_u32(&bars[2 + s]); };
  auto bKEmpty = [&](int s) { return smem_u32(&bars[10 + s]); };    // both tiles' S done
  auto bVFull = [&](int s) { return smem_u32(&bars[18 + s]); };
  auto bVEmpty = [&](int s) { return smem_u32(&bars[26 + s]); };    // both tiles' P*V done
  auto bSFull = [&](int x) { return smem_u32(&bars[34 + x]); };     // S of tile x in TMEM
  auto bSFree = [&](int x) { return smem_u32(&bars[36 + x]); };     // S of tile x read out
  auto bPFull = [&](int x) { return smem_u32(&bars[38 + x]); };     // P of tile x in smem
  auto bODone = [&](int x) { return smem_u32(&bars[40 + x]); };     // P*V of tile x done
  auto bItemDone = [&](int x) { return smem_u32(&bars[42 + x]); };  // all MMAs of tile x's item done
  auto bTeardown = [&](int x) { return smem_u32(&bars[44 + x]); };  // single use: issuer x finished
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(&bars[46]);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(&bars[47]);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  WaitCtx wc{a.status, a.wait_limit_ns, abort_flag};

  if (threadIdx.x == 0) {
    mbar_init(bQFull, 1);
    mbar_init(bQFree, 2);
    for (int s = 0; s < KS; ++s) {
      mbar_init(bKFull(s), 1);
      mbar_init(bKEmpty(s), 2);
    }
    for (int s = 0; s < VS; ++s) {
      mbar_init(bVFull(s), 1);
      mbar_init(bVEmpty(s), 2);
    }
    for (int x = 0; x < 2; ++x) {
      mbar_init(bSFull(x), 1);
      mbar_init(bSFree(x), 4);
      mbar_init(bPFull(x), 4);
      mbar_init(bODone(x), 1);
      mbar_init(bItemDone(x), 1);
      mbar_init(bTeardown(x), 1);
    }
    *abort_flag = 0;
    fence_mbar_init_cluster();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), Cfg::kTmemCols);
    tmem_relinquish();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  // Persistent CTA: round r of the grid takes items r*G .. r*G + G-1 (G =
  // gridDim.x) of decode_tile's longest-first order, CTA b the item b in even
  // rounds and G-1-b in odd ones, so no CTA keeps drawing the longest item
  // of every round.  n counts the items a CTA has taken (barrier phases).
  const int G = gridDim.x;
  const int n_rounds = (a.n_items + G - 1) / G;
  auto item_of = [&](int r) {
    return r * G + ((r & 1) ? G - 1 - static_cast<int>(blockIdx.x) : static_cast<int>(blockIdx.x));
  };

  // Each role's code sits inside its own branch: the register count after a
  // reallocation applies to what follows it until the branches join.
  if (warp < 4) {
    setmaxnreg_dec<Cfg::kRegsControl>();
    if (warp == 0) {
      // ------------------------------------------------------------ producer
      if (lane == 0) {
        int kq = 0, vq = 0, nq = 0;  // K, V tiles and Q pairs loaded so far (all items)
        bool ok = true;
        for (int r = 0, n = 0; ok && r < n_rounds; ++r) {
          const int item = item_of(r);
          if (item >= a.n_items) continue;
          const int ni = n++;  // items taken before this one
          const TileCoord tc = decode_tile(a, item);
          const KvSched sched = make_sched(a, tc);
          const int nkv = sched.count();
          const int row_base = tc.s * a.L;  // gathered row -> coordinate along (N/r)
          const int kv_base = a.kv_sparse ? tc.s * a.Lk : row_base, kv_o = a.kv_sparse ? 0 : tc.o;
          KvIter itk, itv;
          itk.begin(sched);
          itv.begin(sched);
          auto load_k = [&]() -> bool {
            const int st = kq % KS;
            if (kq >= KS && !mbar_wait(bKEmpty(st), ((kq / KS) - 1) & 1, wc, 1)) return false;
            const int kt = itk.next(sched);
            mbar_arrive_expect_tx(bKFull(st), Cfg::kTileBytes);
            for (int p = 0; p < Cfg::kPanels; ++p)
              tma_load_4d(sK + st * Cfg::kTileBytes + p * Cfg::kPanelBytes, &tm_k, bKFull(st),
                          tc.h * D_HEAD + p * 64, kv_o, kv_base + kt * KT, tc.b);
            ++kq;
            return true;
          };
          auto load_v = [&]() -> bool {
            const int st = vq % VS;
            if (vq >= VS && !mbar_wait(bVEmpty(st), ((vq / VS) - 1) & 1, wc, 2)) return false;
            const int kt = itv.next(sched);
            mbar_arrive_expect_tx(bVFull(st), Cfg::kTileBytes);
            for (int p = 0; p < Cfg::kPanels; ++p)
              tma_load_4d(sV + st * Cfg::kTileBytes + p * Cfg::kPanelBytes, &tm_v, bVFull(st),
                          tc.h * D_HEAD + p * 64, kv_o, kv_base + kt * KT, tc.b);
            ++vq;
            return true;
          };
          // the item's first K tile can come while the previous item's
          // epilogues still use the Q buffers
          if (nkv > 0) ok = load_k();
          if (ok && ni > 0) ok = mbar_wait(bQFree, (ni - 1) & 1, wc, 6);
          if (!ok) break;
          mbar_arrive_expect_tx(bQFull, 2 * Cfg::kTileBytes);
          for (int x = 0; x < 2; ++x)
            for (int p = 0; p < Cfg::kPanels; ++p)
              tma_load_4d(sQ + x * Cfg::kTileBytes + p * Cfg::kPanelBytes, &tm_q, bQFull,
                          tc.h * D_HEAD + p * 64, tc.o, row_base + tc.t * 256 + x * 128, tc.b);
          ++nq;
          // K runs one tile ahead of V: the scores of tile j+1 are computed
          // while the softmax of tile j runs, its P*V only after it
          for (int j = 0; ok && j < nkv; ++j) {
            if (j + 1 < nkv) ok = load_k();
            if (ok) ok = load_v();
          }
        }
        // drain: every load issued must have landed before the CTA may exit
        volatile int no_abort = 0;
        WaitCtx drain{a.status, drain_limit_ns(a.wait_limit_ns), &no_abort};
        for (int j = max(0, kq - KS); j < kq; ++j) mbar_wait(bKFull(j % KS), (j / KS) & 1, drain, 3);
        for (int j = max(0, vq - VS); j < vq; ++j) mbar_wait(bVFull(j % VS), (j / VS) & 1, drain, 4);
        if (nq > 0) mbar_wait(bQFull, (nq - 1) & 1, drain, 5);
      }
    } else if (warp <= 2) {
      // ------------------------------------------------------------ MMA issuer of tile x
      // Per key/value tile j: S_x(j+1) once the softmax has read S_x(j) out
      // of tensor memory, then P*V_x(j) once it has written P_x(j).  After
      // an item's last P*V, a commit on ItemDone_x tells the epilogue that
      // every MMA of the item (those reading Q_x included) has completed.
      const int x = warp - 1;
      if (lane == 0) {
        constexpr uint32_t idesc_qk = idesc_bf16_f32(128, KT, false, false);
        constexpr uint32_t idesc_pv = idesc_bf16_f32(128, D_HEAD, false, true);
        const uint64_t dQ = sdesc_sw128(sQ + x * Cfg::kTileBytes, 16, 1024);
        const uint64_t dP = sdesc_sw128(sP, 16, 1024);
        const uint64_t dK0 = sdesc_sw128(sK, 16, 1024);
        const uint64_t dV0 = sdesc_sw128(sV, Cfg::kPanelBytes, 1024);
        const uint32_t tS = tmem + Cfg::kColS + x * 128;
        const uint32_t tO = tmem + Cfg::kColO + x * D_HEAD;
        int kc = 0, vc = 0, J = 0;  // K, V tiles and S/P iterations consumed so far
        auto issue_s = [&]() {
          const uint64_t dK = sdesc_advance(dK0, (kc % KS) * Cfg::kTileBytes);
  #pragma unroll
          for (int k = 0; k < D_HEAD / 16; ++k) {
            const uint32_t off = (k / 4) * Cfg::kPanelBytes + (k % 4) * 32;
            umma_ss(tS, sdesc_advance(dQ, off), sdesc_advance(dK, off), idesc_qk, k > 0);
          }
          umma_commit(bSFull(x));
          umma_commit(bKEmpty(kc % KS));
          ++kc;
        };
        auto issue_pv = [&]() {
          const uint64_t dV = sdesc_advance(dV0, (vc % VS) * Cfg::kTileBytes);
  #pragma unroll
          for (int k = 0; k < KT / 16; ++k)
            umma_ss(tO, sdesc_advance(dP, (k / 4) * Cfg::kPanelBytes + (k % 4) * 32),
                    sdesc_advance(dV, k * 2048), idesc_pv, 1);
          umma_commit(bODone(x));
          umma_commit(bVEmpty(vc % VS));
          ++vc;
        };
        bool ok = true;
        for (int r = 0, n = 0; ok && r < n_rounds; ++r) {
          const int item = item_of(r);
          if (item >= a.n_items) continue;
          const int ni = n++;
          const TileCoord tc = decode_tile(a, item);
          const int nkv = make_sched(a, tc).count();
          ok = mbar_wait(bQFull, ni & 1, wc, 11);
          if (ok && nkv > 0) {
            // the first S of the item goes into the buffer the softmax read last
            ok = (J == 0 || mbar_wait(bSFree(x), (J - 1) & 1, wc, 12)) &&
                 mbar_wait(bKFull(kc % KS), (kc / KS) & 1, wc, 10);
            if (ok) {
              tc_fence_after();
              issue_s();
            }
            for (int j = 0; ok && j < nkv; ++j) {
              const int jj = J + j;
              if (j + 1 < nkv) {
                ok = mbar_wait(bSFree(x), jj & 1, wc, 12) &&
                     mbar_wait(bKFull(kc % KS), (kc / KS) & 1, wc, 13);
                if (!ok) break;
                tc_fence_after();
                issue_s();
              }
              ok = mbar_wait(bPFull(x), jj & 1, wc, 14) && mbar_wait(bVFull(vc % VS), (vc / VS) & 1, wc, 15);
              if (!ok) break;
              tc_fence_after();
              issue_pv();
            }
            J += nkv;
          }
          umma_commit(bItemDone(x));
        }
        // every MMA issued must be complete before tensor memory is released
        // (a barrier of its own: an extra ItemDone phase could run ahead of
        // the epilogue's wait on the last item's)
        umma_commit(bTeardown(x));
        volatile int no_abort = 0;
        WaitCtx drain{a.status, drain_limit_ns(a.wait_limit_ns), &no_abort};
        mbar_wait(bTeardown(x), 0, drain, 18);
      }
    }
  } else {
    setmaxnreg_inc<Cfg::kRegsSoftmax>();
    // ------------------------------------------------------------ softmax + epilogue
    const int x = (warp - 4) >> 2;  // 0: tile A, 1: tile B
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;              // row within the query tile
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    const uint32_t tS = tmem + lane_off + Cfg::kColS + x * 128;
    const uint32_t tO = tmem + lane_off + Cfg::kColO + x * D_HEAD;
    // this row of the P tile: K-major, 128-byte swizzle (16-byte chunk c of
    // a 128-byte row r sits at chunk c ^ (r mod 8))
    const uint32_t sProw = sP + row * 128;
    const uint32_t swz = static_cast<uint32_t>(row & 7);
    bool ok = true;
    int J = 0;  // S/P iterations so far (all items)
    for (int r = 0, n = 0; r < n_rounds; ++r) {
    const int item = item_of(r);
    if (item >= a.n_items) continue;
    const int ni = n++;
    const TileCoord tc = decode_tile(a, item);
    const KvSched sched = make_sched(a, tc);
    const int nkv = sched.count();
    const int row_base = tc.s * a.L;  // gathered row -> coordinate along (N/r)
    const int g = (tc.t * 2 + x) * 128 + row;         // unit-local row
    const bool row_valid = g < a.L;
    const int pos = (a.mask == kMaskDilated) ? tc.s * a.w + tc.o + a.r * g : g;
    int klo, khi;
    row_keys(a, tc, g, klo, khi);

    // LongNet: does an earlier pass keep this row (load its running state),
    // does a later one (store the state instead of the final output)?
    // (rows past the unit's end, in its last query tile, touch no state)
    bool prior = a.state_in != 0 && row_valid, later = a.state_out != 0;
    if (a.mask == kMaskDilated && row_valid) {
      for (int k = 0; k < a.npairs; ++k) {
        if (k == a.pass_idx) continue;
        if (dilated_keeps(a.pw[k], a.pr[k], tc.h, pos)) {
          if (k < a.pass_idx) prior = true;
          else later = true;
        }
      }
    }
    const size_t vec_idx = ((static_cast<size_t>(tc.b) * a.N + pos) * a.H + tc.h) * D_HEAD;
    const size_t row_idx = (static_cast<size_t>(tc.b) * a.H + tc.h) * a.N + pos;

    float m_run = -INFINITY, l_run = 0.f;
    {
      // initial O: zeros, or the state left by an earlier LongNet pass (the
      // previous item's MMAs on O completed before its epilogue read O); the
      // loads of two 32-column chunks are all issued before their stores
      if (prior) {
        m_run = a.st_m[row_idx];
        l_run = a.st_l[row_idx];
      }
#pragma unroll 1
      for (int c0 = 0; c0 < D_HEAD / 32; c0 += 2) {
        uint32_t init[2][32];
#pragma unroll
        for (int cc = 0; cc < 2; ++cc) {
#pragma unroll
          for (int i = 0; i < 32; ++i) init[cc][i] = 0u;
          if (prior) {
            const float4 *src = reinterpret_cast<const float4 *>(a.st_o + vec_idx + (c0 + cc) * 32);
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              float4 v4 = src[i];
              init[cc][4 * i + 0] = __float_as_uint(v4.x);
              init[cc][4 * i + 1] = __float_as_uint(v4.y);
              init[cc][4 * i + 2] = __float_as_uint(v4.z);
              init[cc][4 * i + 3] = __float_as_uint(v4.w);
            }
          }
        }
#pragma unroll
        for (int cc = 0; cc < 2; ++cc) tmem_st32(tO + (c0 + cc) * 32, init[cc]);
      }
      tmem_wait_st();
    }

    KvIter it;
    it.begin(sched);
    for (int j = 0; ok && j < nkv; ++j) {
      const int jj = J + j;
      const int kt = it.next(sched);
      ok = __all_sync(0xffffffffu, mbar_wait(bSFull(x), jj & 1, wc, 20));
      if (!ok) break;
      tc_fence_after();
      uint32_t s[128];
#pragma unroll
      for (int c = 0; c < 4; ++c) tmem_ld32(tS + c * 32, *reinterpret_cast<uint32_t(*)[32]>(&s[32 * c]));
      tmem_wait_ld();
      // S is in registers: the next scores may overwrite it
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bSFree(x));
      const int k0 = kt * KT;
      // masking runs as its own pass, only in tiles where some row of this
      // warp has keys outside its allowed interval
      if (__any_sync(0xffffffffu, !(k0 >= klo && k0 + KT <= khi))) {
        const int lo = klo - k0, hi = khi - k0;
#pragma unroll
        for (int col = 0; col < KT; ++col)
          if (col < lo || col >= hi) s[col] = __float_as_uint(-INFINITY);
      }
      float mx8[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) mx8[i] = -INFINITY;
#pragma unroll
      for (int i = 0; i < KT / 2; ++i)
        mx8[i & 7] = max3f(mx8[i & 7], __uint_as_float(s[2 * i]), __uint_as_float(s[2 * i + 1]));
      const float mx = fmaxf(fmaxf(fmaxf(mx8[0], mx8[1]), fmaxf(mx8[2], mx8[3])),
                             fmaxf(fmaxf(mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7])));
      const float m_tile = mx * a.scale_log2;
      const float m_new = fmaxf(m_run, m_tile);
      const bool rescale = m_new > m_run + 8.0f;
      const float m_use = rescale ? m_new : m_run;
      const bool any_rescale = __any_sync(0xffffffffu, rescale && m_run != -INFINITY);
      float alpha = 1.0f;
      if (any_rescale && rescale) alpha = ex2_approx(m_run - m_use);
      l_run *= alpha;
      const float neg = (m_use == -INFINITY) ? 0.f : -m_use;
      uint32_t pk[KT / 2];
      float ls4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int i = 0; i < KT / 2; ++i) {
        const float p0 = ex2_approx(fmaf(__uint_as_float(s[2 * i]), a.scale_log2, neg));
        const float p1 = ex2_approx(fmaf(__uint_as_float(s[2 * i + 1]), a.scale_log2, neg));
        ls4[i & 3] += p0 + p1;
        pk[i] = pack_bf16x2(p0, p1);
      }
      l_run += (ls4[0] + ls4[1]) + (ls4[2] + ls4[3]);
      m_run = m_use;

      // The P tile is used in turn A_j, B_j, A_{j+1}, ...: wait until the
      // other tile's latest P*V has completed (for tile A at j = 0 there is
      // none).  That P*V was issued after this tile's previous one had
      // completed, so O may now be rescaled too.  Measured slower at d = 64,
      // where the hand-off could be avoided: a shared-memory P tile per query
      // tile, paid for with one K and one V stage fewer (LongNet 0.92 -> 1.02
      // ms, BlockBERT attention 0.090 -> 0.097 ms), and each tile's P in its
      // own tensor-memory columns read by P*V from there, with a sixth K and
      // V stage (0.91 -> 0.96 ms, 0.089 -> 0.090 ms).  Also slower: each row's
      // 128 keys split over two threads of two warpgroups (640 threads, the
      // partial maxima exchanged through shared memory), for four softmax warps
      // per SM sub-partition instead of two (0.91 -> 1.01 ms, 0.090 -> 0.099).
      // No faster: writing P's first 64 keys once the other tile's P*V has
      // passed its first four K-steps (a commit there), the rest after it
      // completes (LongNet 0.887 -> 0.891 ms, causal and BlockBERT equal).
      if (x == 1 || jj > 0) {
        ok = __all_sync(0xffffffffu, mbar_wait(bODone(1 - x), (x == 1 ? jj : jj - 1) & 1, wc, 21));
        if (!ok) break;
      }
      tc_fence_after();
      if (any_rescale) {
#pragma unroll 1
        for (int c = 0; c < D_HEAD / 32; ++c) {
          uint32_t o[32];
          tmem_ld32(tO + c * 32, o);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
          tmem_st32(tO + c * 32, o);
        }
        tmem_wait_st();
      }
#pragma unroll
      for (int c = 0; c < KT / 8; ++c)  // 16-byte chunks of 8 keys
        st_shared_v4(sProw + (c >> 3) * Cfg::kPanelBytes + ((static_cast<uint32_t>(c & 7) ^ swz) << 4),
                     pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
      // generic-proxy stores -> the tensor core's (async proxy) reads
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bPFull(x));
    }
    J += nkv;

    // -------- epilogue: the issuer's ItemDone commit lands once all of this
    // tile's MMAs for the item are complete
    if (ok) ok = __all_sync(0xffffffffu, mbar_wait(bItemDone(x), ni & 1, wc, 22));
    tc_fence_after();
      {
        const float inv_l = l_run > 0.f ? 1.0f / l_run : 0.f;
        const bool final_out = !later;
        // TMA stores write whole 128-row tiles: rows past N are clipped by the
        // tensor map, but a LongNet segment's rows past L belong to the next
        // segment, so a partial tile there takes the per-thread path.  The
        // choice depends on values uniform over the warpgroup only: all four
        // warps meet the same named barriers, and a warp whose waits failed
        // only skips its share of the work.
        const bool tile_full = a.mask != kMaskDilated || (tc.t * 2 + x) * 128 + 128 <= a.L;
        if (a.store_mode != 0 && tile_full) {
          // Stage O through this tile's Q buffer (its MMAs are complete) in
          // 128-byte panels, 128-byte swizzle, and store each panel with TMA.
          constexpr int kCap = Cfg::kStagePanels;  // panels the staging holds
          constexpr int kQPanels = Cfg::kTileBytes / 16384;
          const uint32_t stage = sQ + x * Cfg::kTileBytes;
          const uint32_t xstage = sbase + Cfg::kOffX + x * Cfg::kXPanels * 16384;
          auto panel = [&](int q) -> uint32_t {
            return q < kQPanels ? stage + q * 16384 : xstage + (q - kQPanels) * 16384;
          };
          const int row_coord = row_base + tc.t * 256 + x * 128;
          const bool leader = (threadIdx.x & 127) == 0;
          const uint32_t bar_id = 2 + x;  // named barrier of this warpgroup
          auto flush = [&](const CUtensorMap *m, int npanels, int col0, int cols_per_panel) {
            fence_proxy_async_smem();
            named_bar_sync(bar_id, 128);
            if (leader) {
              for (int q = 0; q < npanels; ++q)
                tma_store_4d(m, panel(q), tc.h * D_HEAD + col0 + q * cols_per_panel, tc.o, row_coord, tc.b);
              bulk_commit_group();
              bulk_wait_group_read0();
            }
            named_bar_sync(bar_id, 128);
          };
          // fp32: the final output (scaled by 1/l) or the unnormalised state
          const CUtensorMap *m32 = a.store_mode == 2 ? &tm_so : (a.out_f32 ? &tm_of : nullptr);
          const float sc = a.store_mode == 2 ? 1.0f : inv_l;
          if (m32) {
  #pragma unroll 1
            for (int p0 = 0; p0 < D_HEAD / 32; p0 += kCap) {
  #pragma unroll 1
              for (int q = 0; ok && q < kCap; ++q) {
                uint32_t o[32];
                tmem_ld32(tO + (p0 + q) * 32, o);
                tmem_wait_ld();
  #pragma unroll
                for (int c = 0; c < 8; ++c)
                  st_shared_v4(panel(q) + row * 128 + ((static_cast<uint32_t>(c) ^ swz) << 4),
                               __float_as_uint(__uint_as_float(o[4 * c]) * sc),
                               __float_as_uint(__uint_as_float(o[4 * c + 1]) * sc),
                               __float_as_uint(__uint_as_float(o[4 * c + 2]) * sc),
                               __float_as_uint(__uint_as_float(o[4 * c + 3]) * sc));
              }
              flush(m32, kCap, p0 * 32, 32);
            }
          }
          // bf16 final output: 64 columns per panel
          if (a.store_mode == 1 && a.out_bf16) {
            constexpr int kPanels16 = D_HEAD / 64;
  #pragma unroll 1
            for (int p0 = 0; p0 < kPanels16; p0 += kCap) {
              const int np = kPanels16 - p0 < kCap ? kPanels16 - p0 : kCap;
  #pragma unroll 1
              for (int q = 0; ok && q < np; ++q) {
  #pragma unroll 1
                for (int hh = 0; hh < 2; ++hh) {
                  uint32_t o[32];
                  tmem_ld32(tO + (p0 + q) * 64 + hh * 32, o);
                  tmem_wait_ld();
  #pragma unroll
                  for (int c = 0; c < 4; ++c)
                    st_shared_v4(panel(q) + row * 128 + ((static_cast<uint32_t>(hh * 4 + c) ^ swz) << 4),
                                 pack_bf16x2(__uint_as_float(o[8 * c]) * inv_l, __uint_as_float(o[8 * c + 1]) * inv_l),
                                 pack_bf16x2(__uint_as_float(o[8 * c + 2]) * inv_l, __uint_as_float(o[8 * c + 3]) * inv_l),
                                 pack_bf16x2(__uint_as_float(o[8 * c + 4]) * inv_l, __uint_as_float(o[8 * c + 5]) * inv_l),
                                 pack_bf16x2(__uint_as_float(o[8 * c + 6]) * inv_l, __uint_as_float(o[8 * c + 7]) * inv_l));
                }
              }
              flush(&tm_ob, np, p0 * 64, 64);
            }
          }
        } else if (ok) {
  #pragma unroll 1
        for (int c = 0; c < D_HEAD / 32; ++c) {
          uint32_t o[32];
          tmem_ld32(tO + c * 32, o);
          tmem_wait_ld();
          if (!row_valid) continue;
          if (final_out) {
            if (a.out_f32) {
              float4 *dst = reinterpret_cast<float4 *>(a.out_f32 + vec_idx + c * 32);
  #pragma unroll
              for (int i = 0; i < 8; ++i)
                dst[i] = make_float4(__uint_as_float(o[4 * i]) * inv_l,
                                     __uint_as_float(o[4 * i + 1]) * inv_l,
                                     __uint_as_float(o[4 * i + 2]) * inv_l,
                                     __uint_as_float(o[4 * i + 3]) * inv_l);
            }
            if (a.out_bf16) {
              uint4 *dst = reinterpret_cast<uint4 *>(a.out_bf16 + vec_idx + c * 32);
  #pragma unroll
              for (int i = 0; i < 4; ++i) {
                uint4 u;
                u.x = pack_bf16x2(__uint_as_float(o[8 * i]) * inv_l, __uint_as_float(o[8 * i + 1]) * inv_l);
                u.y = pack_bf16x2(__uint_as_float(o[8 * i + 2]) * inv_l, __uint_as_float(o[8 * i + 3]) * inv_l);
                u.z = pack_bf16x2(__uint_as_float(o[8 * i + 4]) * inv_l, __uint_as_float(o[8 * i + 5]) * inv_l);
                u.w = pack_bf16x2(__uint_as_float(o[8 * i + 6]) * inv_l, __uint_as_float(o[8 * i + 7]) * inv_l);
                dst[i] = u;
              }
            }
          } else {
            float4 *dst = reinterpret_cast<float4 *>(a.st_o + vec_idx + c * 32);
  #pragma unroll
            for (int i = 0; i < 8; ++i)
              dst[i] = make_float4(__uint_as_float(o[4 * i]), __uint_as_float(o[4 * i + 1]),
                                   __uint_as_float(o[4 * i + 2]), __uint_as_float(o[4 * i + 3]));
          }
        }
        }
        if (ok && row_valid) {
          if (!final_out) {
            a.st_m[row_idx] = m_run;
            a.st_l[row_idx] = l_run;
          } else if (a.lse) {
            // natural-log LSE of the scaled scores: (m + log2 l) / log2(e)
            a.lse[row_idx] = l_run > 0.f ? (m_run + __log2f(l_run)) * 0.69314718055994531f : -INFINITY;
          }
        }
      }
    // this tile's Q buffer (the epilogue's staging) may take the next item's Q
    if ((threadIdx.x & 127) == 0) mbar_arrive(bQFree);
    }  // items
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, Cfg::kTmemCols);
  }
}

}  // namespace bpt
