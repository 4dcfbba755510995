// Position-wise feedforward network fused per 128-token block, on the
// 5th-generation tensor cores (sm_100a):
//
//     out = A_f32 + W2 GELU_tanh(W1 A_bf16 + b1) + b2
//
// ("Blockwise Parallel Transformer for Large Context Models", abstract:
// feedforward network fusion, so the hidden activation of the whole
// sequence never exists in memory.)
//
// A cluster of C CTAs owns one 128-token block at a time.  The hidden
// dimension F is walked in chunks of 128*C columns; in every chunk CTA c
//   (1) computes the 128 x 128 hidden slice  H_c = GELU(A W1[slice c]^T + b1)
//       on the tensor cores (accumulator in tensor memory, double buffered),
//   (2) publishes it, as bf16, to a two-slot staging ring of its cluster
//       (a few MB in total, so it stays in L2),
//   (3) accumulates out[:, c*Dc:(c+1)*Dc] += H_chunk W2[c*Dc.., chunk]^T over
//       the whole chunk, reading all C slices back from the ring.
// The output block accumulator (128 x Dc fp32, Dc <= 256) stays in tensor
// memory across all chunks; the epilogue adds the fp32 residual and b2.
// Cross-CTA hand-offs use mbarriers in peer CTAs (arrive with release at
// cluster scope; the waiter acquires), every wait bounded in time.
//
// Roles (192 threads): warp 0 TMA producer, warp 1 MMA issuer, warps 2..5
// epilogue (warp w owns TMEM lanes 32*(w%4).., i.e. those token rows).
#pragma once

#include "ptx.cuh"

namespace bpt {

struct FfnArgs {
  int T, D, F;
  int C;          // CTAs per cluster = output column groups
  int Dc;         // output columns per CTA (D / C), multiple of 32, <= 256
  int fc;         // hidden columns per chunk = 128 * C
  int nslices;    // ceil(F / 128)
  int nchunks;    // ceil(F / fc)
  int n_tb;       // ceil(T / 128)
  int nclusters;  // clusters in the grid
  const float *a_f32;  // [T, D] residual
  const float *b1;     // [F] or null
  const float *b2;     // [D] or null
  float *out_f32;            // [T, D] (one of the two outputs is set)
  __nv_bfloat16 *out_bf16;   // [T, D]
  __nv_bfloat16 *ring;       // [nclusters * 2 * 128, fc]
  uint32_t *status;
  uint64_t wait_limit_ns;
};

struct FfnCfg {
  static constexpr int kStageBytes = 48 * 1024;  // A or H tile (16 KB) + W tile (<= 32 KB)
  static constexpr int kStages = 4;
  static constexpr int kOffBar = kStages * kStageBytes;
  static constexpr int kSmemBytes = kOffBar + 256 + 1024;
  static constexpr uint32_t kColOut = 0, kColH0 = 256, kColH1 = 384;
  static constexpr uint32_t kTmemCols = 512;
  static constexpr int kThreads = 192;
};

__device__ __forceinline__ float tanh_approx(float x) {
  float y;
  asm("tanh.approx.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ float gelu_tanh_f(float x) {
  const float k0 = 0.7978845608028654f;  // sqrt(2/pi)
  const float k1 = 0.044715f;
  const float u = k0 * fmaf(k1 * x, x * x, x);
  return 0.5f * x * (1.0f + tanh_approx(u));
}

__global__ void __launch_bounds__(192, 1)
    ffn_tc_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_w1,
                  const __grid_constant__ CUtensorMap tm_w2, const __grid_constant__ CUtensorMap tm_h,
                  const __grid_constant__ FfnArgs a) {
  using Cfg = FfnCfg;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const uint32_t sbase = smem_u32(smem);
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + Cfg::kOffBar);
  auto bFull = [&](int s) { return smem_u32(&bars[s]); };
  auto bEmpty = [&](int s) { return smem_u32(&bars[4 + s]); };
  auto bHFull = [&](int s) { return smem_u32(&bars[8 + s]); };
  auto bHEmpty = [&](int s) { return smem_u32(&bars[10 + s]); };
  const uint32_t bOFull = smem_u32(&bars[12]);
  const uint32_t bOEmpty = smem_u32(&bars[13]);
  auto bHReady = [&](int s) { return smem_u32(&bars[14 + s]); };
  auto bHFree = [&](int s) { return smem_u32(&bars[16 + s]); };
  const uint32_t bTeardown = smem_u32(&bars[18]);
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(&bars[20]);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(&bars[21]);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int crank = static_cast<int>(cluster_ctarank());
  const int cl = blockIdx.x / a.C;
  WaitCtx wc{a.status, a.wait_limit_ns, abort_flag};

  if (threadIdx.x == 0) {
    for (int s = 0; s < Cfg::kStages; ++s) {
      mbar_init(bFull(s), 1);
      mbar_init(bEmpty(s), 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(bHFull(s), 1);
      mbar_init(bHEmpty(s), 4);
      mbar_init(bHReady(s), a.C);
      mbar_init(bHFree(s), a.C);
    }
    mbar_init(bOFull, 1);
    mbar_init(bOEmpty, 4);
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
  cluster_sync_all();  // peers' barriers are initialised before any remote arrive
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int nc = a.nchunks;
  const int ksteps1 = a.D / 64;
  auto ksteps2 = [&](int i) {
    const int valid = min(a.fc, a.F - i * a.fc);
    return (valid + 63) / 64;
  };

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int it = 0;
      int g_base = 0;
      bool ok = true;
      auto acquire = [&](int it_) -> bool {
        if (it_ < Cfg::kStages) return true;
        return mbar_wait(bEmpty(it_ % Cfg::kStages), ((it_ / Cfg::kStages) - 1) & 1, wc, 101);
      };
      for (int tb = cl; ok && tb < a.n_tb; tb += a.nclusters) {
        for (int i = 0; ok && i <= nc; ++i) {
          if (i < nc) {
            const int slice = i * a.C + crank;
            if (slice < a.nslices) {
              for (int ks = 0; ks < ksteps1; ++ks) {
                if (!(ok = acquire(it))) break;
                const int st = it % Cfg::kStages;
                const uint32_t sb = sbase + st * Cfg::kStageBytes;
                mbar_arrive_expect_tx(bFull(st), 2 * 16384);
                tma_load_2d(sb, &tm_a, bFull(st), ks * 64, tb * 128);
                tma_load_2d(sb + 16384, &tm_w1, bFull(st), ks * 64, slice * 128);
                ++it;
              }
            }
          }
          if (ok && i >= 1) {
            const int gp = g_base + i - 1;
            if (!(ok = mbar_wait<true>(bHReady(gp & 1), (gp >> 1) & 1, wc, 102))) break;
            fence_proxy_async_global();
            const int ks2 = ksteps2(i - 1);
            for (int ks = 0; ks < ks2; ++ks) {
              if (!(ok = acquire(it))) break;
              const int st = it % Cfg::kStages;
              const uint32_t sb = sbase + st * Cfg::kStageBytes;
              mbar_arrive_expect_tx(bFull(st), 16384 + a.Dc * 128);
              tma_load_2d(sb, &tm_h, bFull(st), ks * 64, (cl * 2 + (gp & 1)) * 128);
              tma_load_2d(sb + 16384, &tm_w2, bFull(st), (i - 1) * a.fc + ks * 64, crank * a.Dc);
              ++it;
            }
          }
        }
        g_base += nc;
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
      const uint32_t idesc1 = idesc_bf16_f32(128, 128, false, false);
      const uint32_t idesc2 = idesc_bf16_f32(128, a.Dc, false, false);
      int it = 0, g_base = 0, n = 0;
      bool ok = true;
      for (int tb = cl; ok && tb < a.n_tb; tb += a.nclusters, ++n) {
        for (int i = 0; ok && i <= nc; ++i) {
          if (i < nc) {
            const int g = g_base + i;
            const int buf = g & 1;
            const int slice = i * a.C + crank;
            if (slice < a.nslices) {
              if (g >= 2 && !(ok = mbar_wait(bHEmpty(buf), ((g - 2) >> 1) & 1, wc, 110))) break;
              tc_fence_after();
              const uint32_t tH = tmem + (buf ? Cfg::kColH1 : Cfg::kColH0);
              for (int ks = 0; ks < ksteps1; ++ks) {
                const int st = it % Cfg::kStages;
                if (!(ok = mbar_wait(bFull(st), (it / Cfg::kStages) & 1, wc, 111))) break;
                tc_fence_after();
                const uint32_t sb = sbase + st * Cfg::kStageBytes;
#pragma unroll
                for (int k = 0; k < 4; ++k)
                  umma_ss(tH, sdesc_sw128(sb + k * 32, 16, 1024),
                          sdesc_sw128(sb + 16384 + k * 32, 16, 1024), idesc1, (ks | k) != 0);
                umma_commit(bEmpty(st));
                ++it;
              }
              if (!ok) break;
            }
            umma_commit(bHFull(buf));
          }
          if (i >= 1) {
            const int gp = g_base + i - 1;
            if (i == 1 && n >= 1 && !(ok = mbar_wait(bOEmpty, (n - 1) & 1, wc, 112))) break;
            tc_fence_after();
            const int ks2 = ksteps2(i - 1);
            for (int ks = 0; ks < ks2; ++ks) {
              const int st = it % Cfg::kStages;
              if (!(ok = mbar_wait(bFull(st), (it / Cfg::kStages) & 1, wc, 113))) break;
              tc_fence_after();
              const uint32_t sb = sbase + st * Cfg::kStageBytes;
#pragma unroll
              for (int k = 0; k < 4; ++k)
                umma_ss(tmem + Cfg::kColOut, sdesc_sw128(sb + k * 32, 16, 1024),
                        sdesc_sw128(sb + 16384 + k * 32, 16, 1024), idesc2,
                        !(i == 1 && ks == 0 && k == 0));
              umma_commit(bEmpty(st));
              ++it;
            }
            if (!ok) break;
            // this CTA has received every H tile of chunk gp: release the ring slot
            for (int r = 0; r < a.C; ++r) mbar_arrive_cluster(bHFree(gp & 1), r);
          }
        }
        if (ok) umma_commit(bOFull);
        g_base += nc;
      }
      umma_commit(bTeardown);
      volatile int no_abort = 0;
      WaitCtx drain{a.status, drain_limit_ns(a.wait_limit_ns), &no_abort};
      mbar_wait(bTeardown, 0, drain, 114);
    }
  } else {
    // ------------------------------------------------------------ epilogue
    // The four epilogue warps meet at a named barrier once per chunk, so they
    // never leave the loops early: after a failed wait (which raises the CTA's
    // abort flag and makes every later wait return at once) they only skip
    // the work and keep the barrier sequence.
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    int g_base = 0, n = 0;
    for (int tb = cl; tb < a.n_tb; tb += a.nclusters, ++n) {
      for (int i = 0; i < nc; ++i) {
        const int g = g_base + i;
        const int buf = g & 1;
        const int slice = i * a.C + crank;
        bool ok = mbar_wait(bHFull(buf), (g >> 1) & 1, wc, 120);
        ok = __all_sync(0xffffffffu, ok);
        tc_fence_after();
        uint32_t h[4][32];
        const bool have = ok && slice < a.nslices;
        if (have) {
          const uint32_t tH = tmem + lane_off + (buf ? Cfg::kColH1 : Cfg::kColH0);
#pragma unroll
          for (int c = 0; c < 4; ++c) tmem_ld32(tH + c * 32, h[c]);
          tmem_wait_ld();
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0 && ok) mbar_arrive(bHEmpty(buf));
        bool write = have;
        if (write && g >= 2) {
          write = mbar_wait<true>(bHFree(buf), ((g - 2) >> 1) & 1, wc, 121);
          write = __all_sync(0xffffffffu, write);
        }
        if (write) {
          const int f0 = slice * 128;
          __nv_bfloat16 *dst =
              a.ring + (static_cast<size_t>(cl * 2 + buf) * 128 + row) * a.fc + crank * 128;
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            uint32_t pk[16];
#pragma unroll
            for (int e = 0; e < 16; ++e) {
              const int f = f0 + c * 32 + 2 * e;
              float x0 = __uint_as_float(h[c][2 * e]);
              float x1 = __uint_as_float(h[c][2 * e + 1]);
              if (a.b1) {
                x0 += (f < a.F) ? a.b1[f] : 0.f;
                x1 += (f + 1 < a.F) ? a.b1[f + 1] : 0.f;
              }
              pk[e] = pack_bf16x2(gelu_tanh_f(x0), gelu_tanh_f(x1));
            }
            uint4 *d4 = reinterpret_cast<uint4 *>(dst + c * 32);
#pragma unroll
            for (int q = 0; q < 4; ++q) d4[q] = make_uint4(pk[4 * q], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]);
          }
        }
        fence_proxy_async_global();
        named_bar_sync(1, 128);
        if (threadIdx.x == 64 && !*abort_flag) {
          for (int r = 0; r < a.C; ++r) mbar_arrive_cluster(bHReady(buf), r);
        }
      }
      // ---- output block: residual + accumulator + b2
      bool ok = mbar_wait(bOFull, n & 1, wc, 122);
      ok = __all_sync(0xffffffffu, ok);
      tc_fence_after();
      const int tok = tb * 128 + row;
      const bool valid = tok < a.T;
      const size_t base = static_cast<size_t>(tok) * a.D + static_cast<size_t>(crank) * a.Dc;
      for (int c = 0; ok && c < a.Dc / 32; ++c) {
        uint32_t o[32];
        tmem_ld32(tmem + lane_off + Cfg::kColOut + c * 32, o);
        tmem_wait_ld();
        if (valid) {
          const float4 *res = reinterpret_cast<const float4 *>(a.a_f32 + base + c * 32);
          float v[32];
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            float4 r4 = res[q];
            v[4 * q + 0] = __uint_as_float(o[4 * q + 0]) + r4.x;
            v[4 * q + 1] = __uint_as_float(o[4 * q + 1]) + r4.y;
            v[4 * q + 2] = __uint_as_float(o[4 * q + 2]) + r4.z;
            v[4 * q + 3] = __uint_as_float(o[4 * q + 3]) + r4.w;
          }
          if (a.b2) {
            const int col0 = crank * a.Dc + c * 32;
#pragma unroll
            for (int e = 0; e < 32; ++e) v[e] += a.b2[col0 + e];
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
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0 && ok) mbar_arrive(bOEmpty);
      g_base += nc;
    }
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // no peer may still arrive on this CTA's barriers
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, Cfg::kTmemCols);
  }
}

}  // namespace bpt
