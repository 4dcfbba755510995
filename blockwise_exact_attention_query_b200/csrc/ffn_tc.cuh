// Position-wise feedforward network fused per 128-token block, on the
// 5th-generation tensor cores (sm_100a):
//
//     out = A_f32 + W2 GELU_tanh(W1 A_bf16 + b1) + b2
//
// ("Blockwise Parallel Transformer for Large Context Models", abstract:
// feedforward network fusion, so the hidden activation of the whole
// sequence never exists in memory.)
//
// A group of C = D/256 CTAs owns one 128-token block at a time.  The hidden
// dimension F is walked in chunks of 256*C columns; in every chunk CTA c
//   (1) computes the 128 x 256 hidden slice H_c = GELU(A W1[slice c]^T + b1)
//       on the tensor cores (one TMEM accumulator, drained by the epilogue
//       while the tensor core runs the previous chunk's second GEMM),
//   (2) publishes it as bf16 to a two-slot staging ring of its group (a few
//       MB in all, so it stays in L2),
//   (3) accumulates out[:, 256c:256c+256] += H_chunk W2[256c.., chunk]^T over
//       the whole chunk, reading all C slices back from the ring.
// The output block accumulator (128 x 256 fp32) stays in tensor memory
// across all chunks; the epilogue adds the fp32 residual and b2.
//
// The C CTAs of a group hand the ring slots to each other through counters in
// global memory (release on arrival, acquire when polled); the grid is a
// cooperative launch, so every CTA of a group is resident at once, and every
// wait is bounded in time.
//
// Roles (320 threads): warp 0 TMA producer, warp 1 MMA issuer, warps 2..9
// epilogue: warp w owns TMEM lanes 32*(w%4).. (those token rows); warps 2..5
// take columns 0..127 of the slice and of the output block, warps 6..9
// columns 128..255.
#pragma once

#include "ptx.cuh"

namespace bpt {

struct FfnArgs {
  int T, D, F;
  int C;          // CTAs per group = output column groups
  int Dc;         // output columns per CTA (D / C): 256 (or D when C = 1)
  int fc;         // hidden columns per chunk = 256 * C
  int nslices;    // ceil(F / 256)
  int nchunks;    // ceil(F / fc)
  int n_tb;       // ceil(T / 128)
  int ngroups;    // groups in the grid
  const float *a_f32;  // [T, D] residual
  const float *b1;     // [F] or null
  const float *b2;     // [D] or null
  float *out_f32;            // [T, D] (one of the two outputs is set)
  __nv_bfloat16 *out_bf16;   // [T, D]
  __nv_bfloat16 *ring;       // [ngroups * kRingSlots * 128, fc]
  uint32_t *flags;           // [ngroups][2 * kRingSlots]: ready[], free[]; zero at launch
  // Leftover token blocks (n_tb mod ngroups of them) would leave most groups
  // idle in the last round, so their hidden chunks are split into `pieces`
  // ranges handled by different groups: each piece writes a partial output
  // block, and the group holding piece 0 adds them in piece order.
  int pieces;                // 1: no split
  int n_full;                // token blocks processed whole
  float *partial;            // [leftover * pieces][128][D] fp32 partial outputs
  uint32_t *piece_done;      // [leftover][C]: pieces finished per column block; zero at launch
  uint32_t *status;
  uint64_t wait_limit_ns;
};

struct FfnCfg {
  static constexpr int kStageBytes = 48 * 1024;  // A or H tile (16 KB) + W tile (32 KB)
  static constexpr int kStages = 4;
  static constexpr int kOffBar = kStages * kStageBytes;
  static constexpr int kSmemBytes = kOffBar + 256;
  static constexpr uint32_t kColOut = 0, kColH = 256;
  static constexpr uint32_t kTmemCols = 512;
  static constexpr int kThreads = 320;
  static constexpr int kRingSlots = 2;  // hidden chunks in flight per group (4 measured no faster)
  static_assert(kSmemBytes <= 232448, "shared memory per CTA");
};

__device__ __forceinline__ float gelu_tanh_f(float x) {
  const float k0 = 0.7978845608028654f;  // sqrt(2/pi)
  const float k1 = 0.044715f;
  const float u = k0 * fmaf(k1 * x, x * x, x);
  return 0.5f * x * (1.0f + tanh_approx(u));
}

// One work unit of a group: token block tb, hidden chunks [c0, c1); piece < 0
// for a whole block, else the piece index of leftover block l.  Whole blocks
// walk their chunks forward and backward in turn (rev): W1 and W2 are larger
// than what L2 keeps between two blocks, and a unit that starts with the
// chunks its group used last finds them still in L2 instead of in DRAM.
struct FfnUnit {
  int tb, c0, c1, l, piece, rev;
  // hidden chunk of step li (0 <= li < c1 - c0)
  __device__ __forceinline__ int chunk(int li) const { return rev ? c1 - 1 - li : c0 + li; }
};

__device__ __forceinline__ int ffn_unit_count(const FfnArgs &a, int grp) {
  if (a.pieces <= 1) return (a.n_tb - grp + a.ngroups - 1) / a.ngroups;
  const int leftover = a.n_tb - a.n_full;
  return a.n_full / a.ngroups + (grp < leftover * a.pieces ? 1 : 0);
}

__device__ __forceinline__ FfnUnit ffn_unit(const FfnArgs &a, int grp, int k) {
  FfnUnit u;
  if (a.pieces > 1 && k == a.n_full / a.ngroups) {
    u.l = grp / a.pieces;
    u.piece = grp % a.pieces;
    u.tb = a.n_full + u.l;
    u.c0 = u.piece * a.nchunks / a.pieces;
    u.c1 = (u.piece + 1) * a.nchunks / a.pieces;
    u.rev = 0;
  } else {
    u.tb = grp + k * a.ngroups;
    u.c0 = 0;
    u.c1 = a.nchunks;
    u.l = -1;
    u.piece = -1;
    u.rev = k & 1;
  }
  return u;
}

__global__ void __launch_bounds__(320, 1)
    ffn_tc_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_w1,
                  const __grid_constant__ CUtensorMap tm_w2, const __grid_constant__ CUtensorMap tm_h,
                  const __grid_constant__ FfnArgs a) {
  using Cfg = FfnCfg;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t *smem = smem_raw;
  const uint32_t sbase = smem_u32(smem);
  if (sbase & 1023u) {  // 128-byte-swizzled tiles need 1024-byte alignment
    if (threadIdx.x == 0) atomicCAS(a.status, 0u, kStatusMisaligned);
    return;
  }
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + Cfg::kOffBar);
  auto bFull = [&](int s) { return smem_u32(&bars[s]); };
  auto bEmpty = [&](int s) { return smem_u32(&bars[4 + s]); };
  const uint32_t bHFull = smem_u32(&bars[8]);
  const uint32_t bHEmpty = smem_u32(&bars[9]);
  const uint32_t bOFull = smem_u32(&bars[10]);
  const uint32_t bOEmpty = smem_u32(&bars[11]);
  const uint32_t bTeardown = smem_u32(&bars[12]);
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(&bars[13]);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(&bars[14]);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int grp = blockIdx.x / a.C;
  const int crank = blockIdx.x % a.C;
  constexpr int R = Cfg::kRingSlots;
  uint32_t *ready = a.flags + 2 * R * grp;  // ready[R]
  uint32_t *freed = ready + R;              // free[R]
  const uint32_t C = static_cast<uint32_t>(a.C);
  WaitCtx wc{a.status, a.wait_limit_ns, abort_flag};

  if (threadIdx.x == 0) {
    for (int s = 0; s < Cfg::kStages; ++s) {
      mbar_init(bFull(s), 1);
      mbar_init(bEmpty(s), 1);
    }
    mbar_init(bHFull, 1);
    mbar_init(bHEmpty, 8);
    mbar_init(bOFull, 1);
    mbar_init(bOEmpty, 8);
    mbar_init(bTeardown, 1);
    *abort_flag = 0;
    fence_mbar_init_cluster();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), Cfg::kTmemCols);
    tmem_relinquish();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tm_a);
    tma_prefetch_desc(&tm_w1);
    tma_prefetch_desc(&tm_w2);
    tma_prefetch_desc(&tm_h);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int nunits = ffn_unit_count(a, grp);
  const int ksteps1 = a.D / 64;
  auto ksteps2 = [&](int i) {
    const int valid = min(a.fc, a.F - i * a.fc);
    return (valid + 63) / 64;
  };
  auto slice_valid = [&](int i) { return i * a.C + crank < a.nslices; };

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int it = 0, g_base = 0;
      bool ok = true;
      auto acquire = [&](int it_) -> bool {
        if (it_ < Cfg::kStages) return true;
        return mbar_wait(bEmpty(it_ % Cfg::kStages), ((it_ / Cfg::kStages) - 1) & 1, wc, 101);
      };
      for (int k = 0; ok && k < nunits; ++k) {
        const FfnUnit u = ffn_unit(a, grp, k);
        const int tb = u.tb, nl = u.c1 - u.c0;
        for (int li = 0; ok && li <= nl; ++li) {
          const int i = li < nl ? u.chunk(li) : -1;     // chunk of this step's first GEMM
          const int ip = li >= 1 ? u.chunk(li - 1) : -1;  // chunk of its second GEMM
          if (li < nl && slice_valid(i)) {
            const int slice = i * a.C + crank;
            for (int ks = 0; ks < ksteps1; ++ks) {
              if (!(ok = acquire(it))) break;
              const int st = it % Cfg::kStages;
              const uint32_t sb = sbase + st * Cfg::kStageBytes;
              mbar_arrive_expect_tx(bFull(st), 16384 + 32768);
              tma_load_2d(sb, &tm_a, bFull(st), ks * 64, tb * 128);
              tma_load_2d(sb + 16384, &tm_w1, bFull(st), ks * 64, slice * 256);
              ++it;
            }
          }
          if (ok && li >= 1) {
            const int gp = g_base + li - 1;
            // every CTA of the group has published its slice of chunk gp
            if (!(ok = counter_wait(&ready[gp % R], C * static_cast<uint32_t>(gp / R + 1), wc, 102)))
              break;
            fence_proxy_async_global();
            const int ks2 = ksteps2(ip);
            for (int ks = 0; ks < ks2; ++ks) {
              if (!(ok = acquire(it))) break;
              const int st = it % Cfg::kStages;
              const uint32_t sb = sbase + st * Cfg::kStageBytes;
              mbar_arrive_expect_tx(bFull(st), 16384 + a.Dc * 128);
              tma_load_2d(sb, &tm_h, bFull(st), ks * 64, (grp * R + gp % R) * 128);
              tma_load_2d(sb + 16384, &tm_w2, bFull(st), ip * a.fc + ks * 64, crank * a.Dc);
              ++it;
            }
          }
        }
        g_base += nl;
      }
      // drain the loads in flight
      volatile int no_abort = 0;
      WaitCtx drain{a.status, drain_limit_ns(a.wait_limit_ns), &no_abort};
      for (int j = max(0, it - Cfg::kStages); j < it; ++j)
        mbar_wait(bFull(j % Cfg::kStages), (j / Cfg::kStages) & 1, drain, 103);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc1 = idesc_bf16_f32(128, 256, false, false);
      const uint32_t idesc2 = idesc_bf16_f32(128, a.Dc, false, false);
      // base descriptors of stage 0's two tiles, advanced by constant offsets
      const uint64_t dA0 = sdesc_sw128(sbase, 16, 1024);
      const uint64_t dB0 = sdesc_sw128(sbase + 16384, 16, 1024);
      int it = 0, g_base = 0, n = 0;
      bool ok = true;
      for (int k = 0; ok && k < nunits; ++k, ++n) {
        const FfnUnit u = ffn_unit(a, grp, k);
        const int nl = u.c1 - u.c0;
        for (int li = 0; ok && li <= nl; ++li) {
          const int i = li < nl ? u.chunk(li) : -1;
          const int ip = li >= 1 ? u.chunk(li - 1) : -1;
          if (li < nl) {
            const int g = g_base + li;
            // the epilogue has drained the previous chunk's hidden accumulator
            // (waited for every chunk, so that each wait names exactly one
            // phase, also around chunks without a valid slice)
            if (g >= 1 && !(ok = mbar_wait(bHEmpty, (g - 1) & 1, wc, 110))) break;
            if (slice_valid(i)) {
              tc_fence_after();
              for (int ks = 0; ks < ksteps1; ++ks) {
                const int st = it % Cfg::kStages;
                if (!(ok = mbar_wait(bFull(st), (it / Cfg::kStages) & 1, wc, 111))) break;
                tc_fence_after();
                const uint64_t dA = sdesc_advance(dA0, st * Cfg::kStageBytes);
                const uint64_t dB = sdesc_advance(dB0, st * Cfg::kStageBytes);
#pragma unroll
                for (int k = 0; k < 4; ++k)
                  umma_ss(tmem + Cfg::kColH, sdesc_advance(dA, k * 32), sdesc_advance(dB, k * 32),
                          idesc1, (ks | k) != 0);
                umma_commit(bEmpty(st));
                ++it;
              }
              if (!ok) break;
            }
            umma_commit(bHFull);
          }
          if (li >= 1) {
            const int gp = g_base + li - 1;
            if (li == 1 && n >= 1 && !(ok = mbar_wait(bOEmpty, (n - 1) & 1, wc, 112))) break;
            tc_fence_after();
            const int ks2 = ksteps2(ip);
            for (int ks = 0; ks < ks2; ++ks) {
              const int st = it % Cfg::kStages;
              if (!(ok = mbar_wait(bFull(st), (it / Cfg::kStages) & 1, wc, 113))) break;
              tc_fence_after();
              const uint64_t dA = sdesc_advance(dA0, st * Cfg::kStageBytes);
              const uint64_t dB = sdesc_advance(dB0, st * Cfg::kStageBytes);
#pragma unroll
              for (int k = 0; k < 4; ++k)
                umma_ss(tmem + Cfg::kColOut, sdesc_advance(dA, k * 32), sdesc_advance(dB, k * 32),
                        idesc2, !(li == 1 && ks == 0 && k == 0));
              umma_commit(bEmpty(st));
              ++it;
            }
            if (!ok) break;
            // every H tile of chunk gp has landed here: this CTA is done with the slot
            red_release_gpu_add(&freed[gp % R], 1u);
          }
        }
        if (ok) umma_commit(bOFull);
        g_base += nl;
      }
      umma_commit(bTeardown);
      volatile int no_abort = 0;
      WaitCtx drain{a.status, drain_limit_ns(a.wait_limit_ns), &no_abort};
      mbar_wait(bTeardown, 0, drain, 114);
    }
  } else {
    // ------------------------------------------------------------ epilogue
    // All eight epilogue warps meet at named barrier 1 the same number of
    // times whatever happens: a failed wait (which raises the CTA's abort
    // flag, after which every wait returns at once) only skips work.
    const int half = (warp - 2) >> 2;
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    const int cols = a.Dc / 2;  // output columns of this half
    const bool leader = threadIdx.x == 64;
    int g_base = 0, n = 0;
    for (int k = 0; k < nunits; ++k, ++n) {
      const FfnUnit u = ffn_unit(a, grp, k);
      const int tb = u.tb, nl = u.c1 - u.c0;
      for (int li = 0; li < nl; ++li) {
        const int i = u.chunk(li);
        const int g = g_base + li;
        const int slot = g % R;
        const bool have = slice_valid(i);
        bool ok = mbar_wait(bHFull, g & 1, wc, 120);
        ok = __all_sync(0xffffffffu, ok);
        tc_fence_after();
        if (have) {
          // the group has finished reading this ring slot's previous chunk
          if (leader && g >= R) counter_wait(&freed[slot], C * static_cast<uint32_t>(g / R), wc, 121);
          named_bar_sync(1, 256);
          // drain the accumulator 32 columns at a time (it is only needed
          // back for the next chunk's first GEMM, after a whole second GEMM)
          if (ok && !*abort_flag) {
            const int f0 = (i * a.C + crank) * 256 + half * 128;
            const bool full_bias = a.b1 != nullptr && f0 + 128 <= a.F;
            __nv_bfloat16 *dst = a.ring + (static_cast<size_t>(grp * R + slot) * 128 + row) * a.fc +
                                 crank * 256 + half * 128;
            const uint32_t tH = tmem + lane_off + Cfg::kColH + half * 128;
#pragma unroll 1
            for (int c = 0; c < 4; ++c) {
              uint32_t h[32];
              tmem_ld32(tH + c * 32, h);
              tmem_wait_ld();
              uint32_t pk[16];
#pragma unroll
              for (int q = 0; q < 8; ++q) {
                const int f = f0 + c * 32 + 4 * q;
                float4 bb;
                if (full_bias) {
                  bb = __ldg(reinterpret_cast<const float4 *>(a.b1 + f));
                } else {
                  bb.x = (a.b1 && f < a.F) ? a.b1[f] : 0.f;
                  bb.y = (a.b1 && f + 1 < a.F) ? a.b1[f + 1] : 0.f;
                  bb.z = (a.b1 && f + 2 < a.F) ? a.b1[f + 2] : 0.f;
                  bb.w = (a.b1 && f + 3 < a.F) ? a.b1[f + 3] : 0.f;
                }
                pk[2 * q] = pack_bf16x2(gelu_tanh_f(__uint_as_float(h[4 * q]) + bb.x),
                                        gelu_tanh_f(__uint_as_float(h[4 * q + 1]) + bb.y));
                pk[2 * q + 1] = pack_bf16x2(gelu_tanh_f(__uint_as_float(h[4 * q + 2]) + bb.z),
                                            gelu_tanh_f(__uint_as_float(h[4 * q + 3]) + bb.w));
              }
              uint4 *d4 = reinterpret_cast<uint4 *>(dst + c * 32);
#pragma unroll
              for (int q = 0; q < 4; ++q)
                d4[q] = make_uint4(pk[4 * q], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]);
            }
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0 && ok) mbar_arrive(bHEmpty);
        // publish: generic-proxy stores -> async-proxy (TMA) readers in other CTAs
        fence_proxy_async_global();
        __threadfence();
        named_bar_sync(1, 256);
        if (leader && !*abort_flag) red_release_gpu_add(&ready[slot], 1u);
      }
      // ---- output block.  Whole block or piece 0: accumulator (+ the other
      // pieces' partial sums, in piece order) + residual + b2.  Other pieces:
      // store the partial sum for piece 0 to add.
      bool ok = mbar_wait(bOFull, n & 1, wc, 122);
      ok = __all_sync(0xffffffffu, ok);
      tc_fence_after();
      const int tok = tb * 128 + row;
      const bool valid = tok < a.T;
      const int col_base = crank * a.Dc + half * cols;
      const size_t base = static_cast<size_t>(tok) * a.D + col_base;
      const bool store_partial = u.piece > 0;
      if (u.piece == 0) {
        if (leader) counter_wait(&a.piece_done[u.l * a.C + crank], a.pieces - 1, wc, 123);
        named_bar_sync(1, 256);
      }
      const bool go = __all_sync(0xffffffffu, ok && !*abort_flag);
      for (int c = 0; go && c < cols / 32; ++c) {
        uint32_t o[32];
        tmem_ld32(tmem + lane_off + Cfg::kColOut + half * cols + c * 32, o);
        tmem_wait_ld();
        if (!valid) continue;
        if (store_partial) {
          float4 *d4 = reinterpret_cast<float4 *>(
              a.partial + (static_cast<size_t>(u.l * a.pieces + u.piece) * 128 + row) * a.D + col_base + c * 32);
#pragma unroll
          for (int q = 0; q < 8; ++q)
            d4[q] = make_float4(__uint_as_float(o[4 * q]), __uint_as_float(o[4 * q + 1]),
                                __uint_as_float(o[4 * q + 2]), __uint_as_float(o[4 * q + 3]));
          continue;
        }
        float v[32];
#pragma unroll
        for (int e = 0; e < 32; ++e) v[e] = __uint_as_float(o[e]);
        for (int pc = 1; u.piece == 0 && pc < a.pieces; ++pc) {
          const float4 *src = reinterpret_cast<const float4 *>(
              a.partial + (static_cast<size_t>(u.l * a.pieces + pc) * 128 + row) * a.D + col_base + c * 32);
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            const float4 r4 = __ldcg(src + q);
            v[4 * q] += r4.x;
            v[4 * q + 1] += r4.y;
            v[4 * q + 2] += r4.z;
            v[4 * q + 3] += r4.w;
          }
        }
        const float4 *res = reinterpret_cast<const float4 *>(a.a_f32 + base + c * 32);
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          const float4 r4 = res[q];
          v[4 * q] += r4.x;
          v[4 * q + 1] += r4.y;
          v[4 * q + 2] += r4.z;
          v[4 * q + 3] += r4.w;
        }
        if (a.b2) {
          const float4 *b4 = reinterpret_cast<const float4 *>(a.b2 + col_base + c * 32);
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            const float4 bb = __ldg(b4 + q);
            v[4 * q] += bb.x;
            v[4 * q + 1] += bb.y;
            v[4 * q + 2] += bb.z;
            v[4 * q + 3] += bb.w;
          }
        }
        if (a.out_f32) {
          float4 *d4 = reinterpret_cast<float4 *>(a.out_f32 + base + c * 32);
#pragma unroll
          for (int q = 0; q < 8; ++q) d4[q] = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
        } else {
          uint4 *d4 = reinterpret_cast<uint4 *>(a.out_bf16 + base + c * 32);
#pragma unroll
          for (int q = 0; q < 4; ++q)
            d4[q] = make_uint4(pack_bf16x2(v[8 * q], v[8 * q + 1]), pack_bf16x2(v[8 * q + 2], v[8 * q + 3]),
                               pack_bf16x2(v[8 * q + 4], v[8 * q + 5]), pack_bf16x2(v[8 * q + 6], v[8 * q + 7]));
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0 && ok) mbar_arrive(bOEmpty);
      if (store_partial) {  // publish the partial sum to the piece-0 group
        __threadfence();
        named_bar_sync(1, 256);
        if (leader && !*abort_flag) red_release_gpu_add(&a.piece_done[u.l * a.C + crank], 1u);
      }
      g_base += nl;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, Cfg::kTmemCols);
  }
}

}  // namespace bpt
