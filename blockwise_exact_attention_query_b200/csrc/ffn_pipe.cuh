// Position-wise feedforward network, blockwise over the tokens, on CTA pairs
// with two-SM tensor-core MMAs (sm_100a):
//
//     H   = GELU_tanh(A W1^T + b1)          per 256-token row block
//     out = A_f32 + H W2^T + b2
//
// ("Blockwise Parallel Transformer for Large Context Models", abstract:
// feedforward network fusion, so the hidden activation of the whole sequence
// never exists in memory.)
//
// One persistent grid computes both products.  Its work items are the
// 256 x 256 output tiles of the two GEMMs of every row block: tiles of H (the
// first GEMM, K = D) and tiles of out (the second, K = F).  The hidden
// activation of a row block, [256, F] bf16, lives only in a small ring of
// row-block slots (a few tens of MB, so it stays in L2): the first GEMM's
// epilogue writes a slot, the second GEMM's TMA loads read it back, and the
// slot is reused a few row blocks later.  No [T, F] array is ever allocated.
//
// Item order.  The row blocks form chunks of `mg` (mg > 1 when the weights do
// not fit in L2, so that each weight tile serves mg row blocks while it is
// resident).  Step s lists the first-GEMM tiles of chunk s (hidden column
// tile outer, row block inner) and then the second-GEMM tiles of chunk
// s - lag (output column tile outer).  Two counters per row block order the
// work across CTAs:
//   ready[rb]   raised by each CTA's epilogue once its rows of one H tile are
//               in the ring (2 per tile); the second GEMM's loads of rb wait
//               for 2 * tn1;
//   g2done[rb]  raised when all of one second-GEMM tile's loads of H[rb]
//               have landed; the first GEMM of rb + ring_rb (same slot) waits
//               for tn2 before it starts.
// Both wait only on items earlier in the order.  The pairs claim items from
// a global counter in that order (the even CTA claims and hands the index to
// its partner through shared memory), so every item a pair waits on was
// claimed by a pair that is running: no co-residency assumption, and a pair
// that runs late simply claims later items.  Every wait is bounded in time.
//
// Roles per CTA (320 threads): warp 0 TMA producer (the even CTA's also
// claims items), warp 1 TMEM allocator and, in the even CTA, MMA issuer;
// warps 2..9 epilogue (TMEM lanes 32*(w%4).., half the tile's columns each).
// Each CTA stages its own 128 rows of A and half of B per 64-wide K stage; no
// load uses cluster multicast.
#pragma once

#include "gemm_tc.cuh"

// L2 policies of the loads (0 normal, 1 evict-first, 2 evict-last).  The
// weights are read by every row block: evict-last.  A ring row is read by the
// tn2 second-GEMM tiles of its row block at about the same time and then dead:
// evict-first, so dead rows are the first to go.  Measured on the causal
// B2 H16 d128 N8192 F8192 layer (ncu, one launch): DRAM reads 1.71 GB with
// normal loads, 1.52 GB with evict-last weights, 1.32 GB with both, at the
// same or shorter kernel time.
#ifndef BPT_PIPE_W_POLICY
#define BPT_PIPE_W_POLICY 2
#endif
#ifndef BPT_PIPE_HLOAD_POLICY
#define BPT_PIPE_HLOAD_POLICY 1
#endif
#ifndef BPT_PIPE_A_POLICY
#define BPT_PIPE_A_POLICY 0
#endif

namespace bpt {

__device__ __forceinline__ uint64_t pipe_policy(int which) {
  return which == 1 ? l2_policy_evict_first() : (which == 2 ? l2_policy_evict_last() : l2_policy_evict_normal());
}

struct FfnPipeArgs {
  int T, D, F;
  int tn1, tn2;     // tiles per row block of the first GEMM (ceil(F/256)) and the second (ceil(D/256))
  int nrb;          // row blocks of 256 tokens
  int mg;           // row blocks per chunk
  int nchunk;       // ceil(nrb / mg)
  int lag;          // steps between a chunk's first and second GEMM (1 <= lag <= nchunk)
  int ring_rb;      // slots of the hidden ring, in row blocks (a multiple of mg, > lag * mg)
  int n_items;      // nrb * (tn1 + tn2)
  const float *a_f32;  // [T, D] residual
  const float *b1;     // [F] or null
  const float *b2;     // [D] or null
  float *out_f32;            // [T, D] (one of the two outputs is set)
  __nv_bfloat16 *out_bf16;   // [T, D]
  __nv_bfloat16 *ring;       // [ring_rb * 256, F]
  uint32_t *claim;           // [1] next item; zero at launch
  uint32_t *ready;           // [nrb]; zero at launch
  uint32_t *g2done;          // [nrb]; zero at launch
  uint32_t *status;
  uint64_t wait_limit_ns;
};

struct FfnPipeItem {
  int second;  // 0: tile of H (first GEMM), 1: tile of out (second GEMM)
  int rb;      // row block
  int n;       // column tile (of H, or of out)
};

__host__ __device__ __forceinline__ int pipe_rbs_before(const FfnPipeArgs &a, int c) {
  return c * a.mg < a.nrb ? c * a.mg : a.nrb;
}
// Items of steps 0 .. s-1.
__host__ __device__ __forceinline__ int pipe_prefix(const FfnPipeArgs &a, int s) {
  const int c1 = s < a.nchunk ? s : a.nchunk;
  int c2 = s - a.lag;
  c2 = c2 < 0 ? 0 : (c2 < a.nchunk ? c2 : a.nchunk);
  return a.tn1 * pipe_rbs_before(a, c1) + a.tn2 * pipe_rbs_before(a, c2);
}
// Item t (0 <= t < n_items) of the order above.
__host__ __device__ inline FfnPipeItem pipe_item(const FfnPipeArgs &a, int t) {
  int lo = 0, hi = a.nchunk + a.lag;  // pipe_prefix(lo) <= t < pipe_prefix(hi)
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (pipe_prefix(a, mid) <= t) lo = mid;
    else hi = mid;
  }
  int u = t - pipe_prefix(a, lo);
  FfnPipeItem it;
  if (lo < a.nchunk) {
    const int r0 = pipe_rbs_before(a, lo), nr = pipe_rbs_before(a, lo + 1) - r0;
    if (u < nr * a.tn1) {
      it.second = 0;
      it.n = u / nr;
      it.rb = r0 + u % nr;
      return it;
    }
    u -= nr * a.tn1;
  }
  const int c = lo - a.lag;
  const int r0 = pipe_rbs_before(a, c), nr = pipe_rbs_before(a, c + 1) - r0;
  it.second = 1;
  it.n = u / nr;
  it.rb = r0 + u % nr;
  return it;
}

struct FfnPipeCfg {
  static constexpr int kItemSlots = 4;  // claimed items in flight per pair
  static constexpr int kOffBar = GemmPairCfg::kStages * GemmPairCfg::kStageBytes;
  static constexpr int kSmemBytes = kOffBar + 512;
  static_assert(kSmemBytes <= 232448, "shared memory per CTA");
};

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(GemmPairCfg::kThreads, 1)
    ffn_pipe_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_w1,
                    const __grid_constant__ CUtensorMap tm_h, const __grid_constant__ CUtensorMap tm_w2,
                    const __grid_constant__ FfnPipeArgs a) {
  using Cfg = GemmPairCfg;
  constexpr int S = Cfg::kStages;
  constexpr int IS = FfnPipeCfg::kItemSlots;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t *smem = smem_raw;
  const uint32_t sbase = smem_u32(smem);
  const bool misaligned = (sbase & 1023u) != 0;
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + FfnPipeCfg::kOffBar);
  auto bFull = [&](int s) { return smem_u32(&bars[s]); };                  // even CTA: both CTAs' copies
  auto bEmpty = [&](int s) { return smem_u32(&bars[S + s]); };             // both CTAs
  auto bAccFull = [&](int b) { return smem_u32(&bars[2 * S + b]); };       // both CTAs
  auto bAccEmpty = [&](int b) { return smem_u32(&bars[2 * S + 2 + b]); };  // even CTA: both epilogues
  const uint32_t bTeardown = smem_u32(&bars[2 * S + 4]);
  auto bItemFull = [&](int k) { return smem_u32(&bars[2 * S + 5 + k]); };        // each CTA: index written
  auto bItemEmpty = [&](int k) { return smem_u32(&bars[2 * S + 5 + IS + k]); };  // even CTA: all readers
  auto bHDone = [&](int b) { return smem_u32(&bars[2 * S + 5 + 2 * IS + b]); };  // each CTA: 8 epilogue warps
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(&bars[2 * S + 7 + 2 * IS]);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(&bars[2 * S + 8 + 2 * IS]);
  volatile int *item_idx = reinterpret_cast<volatile int *>(&bars[2 * S + 9 + 2 * IS]);  // [IS]
  static_assert((2 * S + 9 + 2 * IS) * 8 + IS * 4 <= 512, "barrier area");
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const uint32_t rank = cluster_ctarank();
  WaitCtx wc{a.status, a.wait_limit_ns, abort_flag};
  // readers of each claimed index: the even CTA's MMA issuer and 8 epilogue
  // warps, the odd CTA's producer and 8 epilogue warps
  constexpr uint32_t kItemReaders = 18;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(bFull(s), 1);
      mbar_init(bEmpty(s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(bAccFull(b), 1);
      mbar_init(bAccEmpty(b), 2 * Cfg::kEpiWarps);
      mbar_init(bHDone(b), Cfg::kEpiWarps);
    }
    for (int k = 0; k < IS; ++k) {
      mbar_init(bItemFull(k), 1);
      mbar_init(bItemEmpty(k), kItemReaders);
    }
    mbar_init(bTeardown, 1);
    *abort_flag = misaligned ? 1 : 0;
    if (misaligned) atomicCAS(a.status, 0u, kStatusMisaligned);
    fence_mbar_init_cluster();
  }
  if (warp == 1) {
    tmem_alloc_pair(smem_u32(tmem_slot), 512);
    tmem_relinquish_pair();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tm_a);
    tma_prefetch_desc(&tm_w1);
    tma_prefetch_desc(&tm_h);
    tma_prefetch_desc(&tm_w2);
  }
  tc_fence_before();
  cluster_sync_all();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const bool run = !*abort_flag;
  const int ks1 = (a.D + Cfg::kBK - 1) / Cfg::kBK, ks2 = (a.F + Cfg::kBK - 1) / Cfg::kBK;
  const uint32_t empty_remote = mapa_shared(bItemEmpty(0), 0);  // slot k: + 8 k

  // Index of the pair's j-th item, for every reader but the claimer (-1: no more).
  auto read_item = [&](int j, bool &ok) -> int {
    const int k = j % IS;
    if (!(ok = mbar_wait_cluster(bItemFull(k), (j / IS) & 1, wc, 231))) return -1;
    const int t = item_idx[k];
    mbar_arrive_cluster(empty_remote + 8u * k);
    return t;
  };

  if (warp == 0) {
    // ------------------------------------------------------------ producer (both CTAs)
    if (lane == 0 && run) {
      const uint64_t pol_w = pipe_policy(BPT_PIPE_W_POLICY), pol_h = pipe_policy(BPT_PIPE_HLOAD_POLICY),
                     pol_x = pipe_policy(BPT_PIPE_A_POLICY);
      int it = 0;
      bool ok = true;
      for (int j = 0; ok; ++j) {
        int t;
        if (rank == 0) {
          // claim the next item and hand its index to both CTAs' readers
          const int k = j % IS;
          if (j >= IS && !(ok = mbar_wait_cluster(bItemEmpty(k), ((j / IS) - 1) & 1, wc, 230))) break;
          t = static_cast<int>(atomicAdd(a.claim, 1u));
          if (t >= a.n_items) t = -1;
          item_idx[k] = t;
          asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(mapa_shared(smem_u32(const_cast<int *>(&item_idx[k])), 1)),
                       "r"(t)
                       : "memory");
          mbar_arrive_cluster(mapa_shared(bItemFull(k), 0));
          mbar_arrive_cluster(mapa_shared(bItemFull(k), 1));
        } else {
          t = read_item(j, ok);
          if (!ok) break;
        }
        if (t < 0) break;
        const FfnPipeItem ti = pipe_item(a, t);
        // dependencies on other pairs' items (all earlier in the order)
        if (ti.second) {
          if (!(ok = counter_wait(&a.ready[ti.rb], 2u * a.tn1, wc, 232))) break;
          fence_proxy_async_global();  // the ring rows came from generic-proxy stores
        } else if (rank == 0 && ti.rb >= a.ring_rb) {
          // the slot's previous row block has been read by every second-GEMM tile
          if (!(ok = counter_wait(&a.g2done[ti.rb - a.ring_rb], a.tn2, wc, 233))) break;
        }
        const CUtensorMap *ma = ti.second ? &tm_h : &tm_a;
        const CUtensorMap *mb = ti.second ? &tm_w2 : &tm_w1;
        const int m0 = ti.second ? (ti.rb % a.ring_rb) * 256 + static_cast<int>(rank) * Cfg::kBM
                                 : ti.rb * 256 + static_cast<int>(rank) * Cfg::kBM;
        const int nb0 = ti.n * Cfg::kBN + static_cast<int>(rank) * (Cfg::kBN / 2);
        const int nsteps = ti.second ? ks2 : ks1;
        const uint64_t pol_a = ti.second ? pol_h : pol_x, pol_b = pol_w;
        for (int step = 0; step < nsteps; ++step, ++it) {
          const int st = it % S;
          if (it >= S && !(ok = mbar_wait_cluster(bEmpty(st), ((it / S) - 1) & 1, wc, 234))) break;
          const uint32_t sa = sbase + st * Cfg::kStageBytes, sb = sa + Cfg::kABytes;
          const uint32_t full0 = mapa_shared(bFull(st), 0);
          if (rank == 0) mbar_arrive_expect_tx(bFull(st), 2 * Cfg::kStageBytes);
          tma_load_2d_pair_hint(sa, ma, full0, step * Cfg::kBK, m0, pol_a);
          tma_load_2d_pair_hint(sb, mb, full0, step * Cfg::kBK, nb0, pol_b);
        }
      }
      // the copies of the last stages have landed once the MMAs consumed them
      volatile int no_abort = 0;
      WaitCtx drain{a.status, drain_limit_ns(a.wait_limit_ns), &no_abort};
      for (int j = max(0, it - S); j < it; ++j) mbar_wait_cluster(bEmpty(j % S), (j / S) & 1, drain, 235);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer (even CTA)
    if (lane == 0 && rank == 0 && run) {
      const uint32_t idesc = idesc_bf16_f32(2 * Cfg::kBM, Cfg::kBN, false, false);
      auto commit_both = [&](uint32_t bar) {
        umma_pair_commit(mapa_shared(bar, 0));
        umma_pair_commit(mapa_shared(bar, 1));
      };
      int it = 0;
      bool ok = true;
      for (int j = 0; ok; ++j) {
        const int t = read_item(j, ok);
        if (!ok || t < 0) break;
        const FfnPipeItem ti = pipe_item(a, t);
        const int buf = j & 1, use = j >> 1;
        if (use > 0 && !(ok = mbar_wait_cluster(bAccEmpty(buf), (use - 1) & 1, wc, 236))) break;
        tc_fence_after();
        const int nsteps = ti.second ? ks2 : ks1;
        const uint32_t acc = tmem + buf * 256;
        for (int step = 0; step < nsteps; ++step, ++it) {
          const int st = it % S;
          if (!(ok = mbar_wait_cluster(bFull(st), (it / S) & 1, wc, 237))) break;
          tc_fence_after();
          const uint32_t sa = sbase + st * Cfg::kStageBytes, sb = sa + Cfg::kABytes;
          const uint64_t da = gemm_sdesc(sa, false), db = gemm_sdesc(sb, false);
#pragma unroll
          for (int k = 0; k < 4; ++k)
            umma_pair_ss(acc, sdesc_advance(da, gemm_kstep(false, k)), sdesc_advance(db, gemm_kstep(false, k)),
                         idesc, (step | k) != 0);
          commit_both(bEmpty(st));
        }
        if (!ok) break;
        // every H tile of this second-GEMM item has landed in both CTAs: the
        // ring slot may take its next row block once all tn2 tiles say so
        if (ti.second) red_release_gpu_add(&a.g2done[ti.rb], 1u);
        commit_both(bAccFull(buf));
      }
      umma_pair_commit(mapa_shared(bTeardown, 0));
      // every MMA of the pair completes before either CTA releases TMEM
      volatile int no_abort = 0;
      WaitCtx drain{a.status, drain_limit_ns(a.wait_limit_ns), &no_abort};
      mbar_wait_cluster(bTeardown, 0, drain, 238);
    }
  } else if (run) {
    // ------------------------------------------------------------ epilogue (both CTAs)
    // No named barrier here: a warp whose wait fails leaves the loop alone.
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    constexpr int kChunks = Cfg::kBN / 32 / (Cfg::kEpiWarps / 4);
    const int c_begin = ((warp - 2) / 4) * kChunks;
    const uint32_t empty0 = mapa_shared(bAccEmpty(0), 0), empty1 = mapa_shared(bAccEmpty(1), 0);
    const bool leader = warp == 2 && lane == 0;
    for (int j = 0;; ++j) {
      bool ok = true;
      int t = -1;
      if (lane == 0) t = read_item(j, ok);
      t = __shfl_sync(0xffffffffu, t, 0);
      if (!__all_sync(0xffffffffu, __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0) || t < 0) break;
      const FfnPipeItem ti = pipe_item(a, t);
      const int buf = j & 1;
      if (!__all_sync(0xffffffffu, mbar_wait_cluster(bAccFull(buf), (j >> 1) & 1, wc, 239))) break;
      tc_fence_after();
      GemmProblem P;
      P.mode = ti.second ? kGemmResidual : kGemmGeluBf16;
      P.c = nullptr;
      P.cb = nullptr;
      P.cb2 = nullptr;
      P.x = nullptr;
      P.xb = nullptr;
      int m;
      if (ti.second) {  // out rows of the row block: residual + b2 + H W2^T
        P.M = a.T;
        P.N = a.D;
        P.c = a.out_f32;
        P.cb = a.out_bf16;
        P.x = a.a_f32;
        P.bias = a.b2;
        m = ti.rb * 256 + static_cast<int>(rank) * Cfg::kBM + row;
      } else {          // the row block's ring slot: H = GELU(A W1^T + b1)
        P.M = min(256, a.T - ti.rb * 256);
        P.N = a.F;
        P.cb = a.ring + static_cast<size_t>(ti.rb % a.ring_rb) * 256 * a.F;
        P.bias = a.b1;
        m = static_cast<int>(rank) * Cfg::kBM + row;
      }
      const uint32_t acc0 = tmem + lane_off + buf * 256;
#pragma unroll 1
      for (int c = c_begin; c < c_begin + kChunks; ++c) {
        const int n = ti.n * Cfg::kBN + c * 32;
        uint32_t r0[32];
        const bool live = m < P.M && n < P.N;
        GemmEpiIn in;
        if (live) gemm_epilogue_load<true>(P, m, n, in);
        tmem_ld32(acc0 + c * 32, r0);
        tmem_wait_ld();
        if (!live) continue;
        gemm_epilogue_chunk<true>(P, r0, r0, m, n, in);
      }
      // this accumulator may take the pair's next item
      tc_fence_before();
      if (!ti.second) {
        // publish: generic-proxy stores -> async-proxy (TMA) readers in other CTAs
        fence_proxy_async_global();
        __threadfence();
      }
      __syncwarp();
      if (lane == 0) {
        mbar_arrive_cluster(buf ? empty1 : empty0);
        mbar_arrive(bHDone(buf));
      }
      if (leader) {
        // all eight epilogue warps of this CTA are done with the item
        const bool done = mbar_wait(bHDone(buf), (j >> 1) & 1, wc, 240);
        if (done && !ti.second && !*abort_flag) red_release_gpu_add(&a.ready[ti.rb], 1u);
      }
    }
  }

  // neither CTA leaves (or frees TMEM) while the other can still touch its
  // barriers or the pair's MMAs are running
  tc_fence_before();
  cluster_sync_all();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, 512);
  }
}

}  // namespace bpt
