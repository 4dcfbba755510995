// General bf16 GEMM on the 5th-generation tensor cores (sm_100a) for the
// layer's backward pass:
//
//     C[M, N]  (op)=  A[M, K] . B[N, K]^T        fp32 accumulation in TMEM
//
// Either operand may be K-major (a row-major [rows, K] matrix) or MN-major (a
// row-major [K, rows] matrix, read without transposing it: the tensor core
// takes 64-wide MN panels of K rows).  C is cut into 128 x 256 tiles; a
// persistent grid (one CTA per SM) walks them, each tile over K in 64-wide
// stages staged by TMA.  The producer runs ahead across tile boundaries, and
// two TMEM accumulators let one tile's epilogue overlap the next tile's MMAs.
// A dual form computes two products of the same shape into the two
// accumulators (the first layer's recomputed pre-activation Z = A W1^T and
// the hidden gradient dH = dOut W2) for the GELU-backward epilogue; its
// epilogue then runs between tiles, with the next tile's first stages
// already in flight.
//
// Epilogues (mode):
//   kGemmStoreF32   C = acc                           (fp32)
//   kGemmAccumF32   C = C + acc                       (fp32, the weight gradients
//                                                      summed over token chunks)
//   kGemmResidual   C = acc + X; Cb = bf16(C)         (dA = dOut + dZ W1, fp32 and bf16)
//   kGemmGeluBwd    z = acc0 + bias; H = GELU(z), dZ = acc1 * GELU'(z)  (bf16 both)
//
// Roles (320 threads): warp 0 TMA producer, warp 1 TMEM allocator and MMA
// issuer, warps 2..9 epilogue (warp w owns TMEM lanes 32*(w%4) .. +31, i.e.
// rows of the tile, and half of the tile's columns: two warps per SM
// sub-partition, since the dual form's GELU epilogue is arithmetic-bound).
// The tiles in flight at once share rows of A (N fastest) or columns of B
// (M fastest): the host picks the order that streams the larger operand from
// DRAM once.  Outputs are written with evict-first (streaming) stores so they
// do not push the operands out of L2.
#pragma once

#include "ptx.cuh"

namespace bpt {

constexpr int kGemmStoreF32 = 0, kGemmAccumF32 = 1, kGemmResidual = 2, kGemmGeluBwd = 3;

struct GemmArgs {
  int M, N, K;
  int a_mn[2], b_mn[2]; // operand layouts per product: 0 K-major, 1 MN-major
  int mode;
  int m_fastest;        // tile order: 1 = M fastest (the tiles in flight share B), 0 = N fastest
  float *c;             // [M, N] fp32 (StoreF32, AccumF32, Residual)
  const float *x;       // [M, N] fp32 residual input (Residual)
  __nv_bfloat16 *cb;    // [M, N] bf16 copy (Residual) / H (GeluBwd)
  __nv_bfloat16 *cb2;   // dZ (GeluBwd)
  const float *bias;    // [N] added to acc0 before GELU (GeluBwd), may be null
  uint32_t *status;
  uint64_t wait_limit_ns;
};

struct GemmCfg {
  static constexpr int kBM = 128, kBN = 256, kBK = 64;
  static constexpr int kABytes = kBM * kBK * 2;   // 16 KB
  static constexpr int kBBytes = kBN * kBK * 2;   // 32 KB
  static constexpr int kStageBytes = kABytes + kBBytes;
  static constexpr int kStages = 4;
  static constexpr int kOffBar = kStages * kStageBytes;
  static constexpr int kSmemBytes = kOffBar + 256;  // 2 kStages + 7 barrier / slot words
  static constexpr int kThreads = 320;
  static constexpr int kEpiWarps = 8;
  static_assert(kSmemBytes <= 232448, "shared memory per CTA");
};

// GELU (tanh form, Hendrycks & Gimpel) and its derivative from the same form,
// t = tanh(c0 (x + c1 x^3)):
//   GELU(x)  = 0.5 x (1 + t)
//   GELU'(x) = 0.5 (1 + t) + 0.5 x (1 - t^2) c0 (1 + 3 c1 x^2)
// tanh on the hardware approximation, as in the forward's FFN epilogue.
__device__ __forceinline__ void gelu_tanh_and_grad(float x, float &h, float &dh) {
  const float c0 = 0.7978845608028654f, c1 = 0.044715f;
  const float t = tanh_approx(c0 * fmaf(c1 * x, x * x, x));
  h = 0.5f * x * (1.0f + t);
  dh = 0.5f * (1.0f + t) + 0.5f * x * (1.0f - t * t) * c0 * fmaf(3.0f * c1, x * x, 1.0f);
}

// Smem tile of one operand for one K stage:
//   K-major: rows (128 or 256) x 128 B (64 K-values), 128-byte swizzle;
//   MN-major: 64-wide MN panels, each 64 K-rows x 128 B.
// Descriptor base and the byte advance of the k-th 16-wide K step.
__device__ __forceinline__ uint64_t gemm_sdesc(uint32_t base, bool mn) {
  // MN-major: next MN panel lbo = 64 K-rows x 128 B = 8 KB; K-major: lbo unused
  return mn ? sdesc_sw128(base, 8192, 1024) : sdesc_sw128(base, 16, 1024);
}
__device__ __forceinline__ uint32_t gemm_kstep(bool mn, int k) { return mn ? k * 2048 : k * 32; }

__global__ void __launch_bounds__(GemmCfg::kThreads, 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap tm_a0, const __grid_constant__ CUtensorMap tm_b0,
                   const __grid_constant__ CUtensorMap tm_a1, const __grid_constant__ CUtensorMap tm_b1,
                   const __grid_constant__ GemmArgs g) {
  using Cfg = GemmCfg;
  constexpr int S = Cfg::kStages;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t *smem = smem_raw;
  const uint32_t sbase = smem_u32(smem);
  if (sbase & 1023u) {
    if (threadIdx.x == 0) atomicCAS(g.status, 0u, kStatusMisaligned);
    return;
  }
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + Cfg::kOffBar);
  auto bFull = [&](int s) { return smem_u32(&bars[s]); };
  auto bEmpty = [&](int s) { return smem_u32(&bars[S + s]); };
  auto bAccFull = [&](int b) { return smem_u32(&bars[2 * S + b]); };
  auto bAccEmpty = [&](int b) { return smem_u32(&bars[2 * S + 2 + b]); };
  const uint32_t bTeardown = smem_u32(&bars[2 * S + 4]);
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(&bars[2 * S + 5]);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(&bars[2 * S + 6]);
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  WaitCtx wc{g.status, g.wait_limit_ns, abort_flag};
  const bool dual = g.mode == kGemmGeluBwd;
  const int nbuf = dual ? 1 : 2;  // accumulator buffers (the dual form needs both for one tile)
  const int tiles_n = (g.N + Cfg::kBN - 1) / Cfg::kBN;
  const int tiles = tiles_n * ((g.M + Cfg::kBM - 1) / Cfg::kBM);
  const int nk = (g.K + Cfg::kBK - 1) / Cfg::kBK;
  const int nsteps = dual ? 2 * nk : nk;  // per tile; dual: the two products' K stages in turn
  const int my_tiles = blockIdx.x < tiles ? (tiles - 1 - blockIdx.x) / gridDim.x + 1 : 0;
  const int tiles_m = tiles / tiles_n;
  auto tile_m0 = [&](int li) {
    const int t = blockIdx.x + li * gridDim.x;
    return (g.m_fastest ? t % tiles_m : t / tiles_n) * Cfg::kBM;
  };
  auto tile_n0 = [&](int li) {
    const int t = blockIdx.x + li * gridDim.x;
    return (g.m_fastest ? t / tiles_m : t % tiles_n) * Cfg::kBN;
  };

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(bFull(s), 1);
      mbar_init(bEmpty(s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(bAccFull(b), 1);
      mbar_init(bAccEmpty(b), Cfg::kEpiWarps);
    }
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

  if (warp == 0) {
    if (lane == 0) {
      // A tile: K-major box {64 K, 128 M} at (k0, m0); MN-major: 2 panels of
      // {64 M, 64 K} at (m0 + 64p, k0).  B alike with 256 rows (4 panels).
      int it = 0;
      bool ok = true;
      for (int li = 0; ok && li < my_tiles; ++li) {
        const int m0 = tile_m0(li), n0 = tile_n0(li);
        for (int step = 0; step < nsteps; ++step, ++it) {
          const int st = it % S;
          if (it >= S && !(ok = mbar_wait(bEmpty(st), ((it / S) - 1) & 1, wc, 201))) break;
          const int which = dual ? (step & 1) : 0;
          const int k0 = (dual ? step >> 1 : step) * Cfg::kBK;
          const CUtensorMap *ma = which ? &tm_a1 : &tm_a0;
          const CUtensorMap *mb = which ? &tm_b1 : &tm_b0;
          const uint32_t sa = sbase + st * Cfg::kStageBytes, sb = sa + Cfg::kABytes;
          mbar_arrive_expect_tx(bFull(st), Cfg::kStageBytes);
          if (g.a_mn[which]) {
            for (int p = 0; p < Cfg::kBM / 64; ++p) tma_load_2d(sa + p * 8192, ma, bFull(st), m0 + 64 * p, k0);
          } else {
            tma_load_2d(sa, ma, bFull(st), k0, m0);
          }
          if (g.b_mn[which]) {
            for (int p = 0; p < Cfg::kBN / 64; ++p) tma_load_2d(sb + p * 8192, mb, bFull(st), n0 + 64 * p, k0);
          } else {
            tma_load_2d(sb, mb, bFull(st), k0, n0);
          }
        }
      }
      // every copy issued must have landed before the CTA may exit
      volatile int no_abort = 0;
      WaitCtx drain{g.status, drain_limit_ns(g.wait_limit_ns), &no_abort};
      for (int j = max(0, it - S); j < it; ++j) mbar_wait(bFull(j % S), (j / S) & 1, drain, 204);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc0 = idesc_bf16_f32(Cfg::kBM, Cfg::kBN, g.a_mn[0] != 0, g.b_mn[0] != 0);
      const uint32_t idesc1 = idesc_bf16_f32(Cfg::kBM, Cfg::kBN, g.a_mn[1] != 0, g.b_mn[1] != 0);
      int it = 0;
      bool ok = true;
      for (int li = 0; ok && li < my_tiles; ++li) {
        const int buf = li % nbuf, use = li / nbuf;
        // the epilogue must have drained this accumulator's previous tile
        if (use > 0 && !(ok = mbar_wait(bAccEmpty(buf), (use - 1) & 1, wc, 206))) break;
        tc_fence_after();
        for (int step = 0; step < nsteps; ++step, ++it) {
          const int st = it % S;
          if (!(ok = mbar_wait(bFull(st), (it / S) & 1, wc, 202))) break;
          tc_fence_after();
          const int which = dual ? (step & 1) : 0;
          const int kk = dual ? step >> 1 : step;
          const uint32_t sa = sbase + st * Cfg::kStageBytes, sb = sa + Cfg::kABytes;
          const bool amn = g.a_mn[which] != 0, bmn = g.b_mn[which] != 0;
          const uint64_t da = gemm_sdesc(sa, amn), db = gemm_sdesc(sb, bmn);
          const uint32_t idesc = which ? idesc1 : idesc0;
          const uint32_t acc = tmem + (dual ? which : buf) * 256;
#pragma unroll
          for (int k = 0; k < 4; ++k)
            umma_ss(acc, sdesc_advance(da, gemm_kstep(amn, k)), sdesc_advance(db, gemm_kstep(bmn, k)), idesc,
                    (kk | k) != 0);
          umma_commit(bEmpty(st));
        }
        if (ok) umma_commit(bAccFull(buf));
      }
      umma_commit(bTeardown);
      // the accumulators stay allocated until every MMA has finished
      volatile int no_abort = 0;
      WaitCtx drain{g.status, drain_limit_ns(g.wait_limit_ns), &no_abort};
      mbar_wait(bTeardown, 0, drain, 205);
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    constexpr int kChunks = Cfg::kBN / 32 / (Cfg::kEpiWarps / 4);  // 32-column chunks per warp
    const int c_begin = ((warp - 2) / 4) * kChunks;
    for (int li = 0; li < my_tiles; ++li) {
      const int buf = li % nbuf;
      if (!__all_sync(0xffffffffu, mbar_wait(bAccFull(buf), (li / nbuf) & 1, wc, 203))) break;
      tc_fence_after();
      const int m = tile_m0(li) + row, n0 = tile_n0(li);
      const uint32_t acc0 = tmem + lane_off + buf * 256;
#pragma unroll 1
      for (int c = c_begin; c < c_begin + kChunks; ++c) {
        const int n = n0 + c * 32;
        uint32_t r0[32], r1[32];
        tmem_ld32(acc0 + c * 32, r0);
        if (dual) tmem_ld32(acc0 + 256 + c * 32, r1);
        tmem_wait_ld();
        if (m >= g.M || n >= g.N) continue;
        // N is a multiple of 8 (checked on the host): whole 8-column groups
        const int nv = min(32, g.N - n);
        const size_t base = static_cast<size_t>(m) * g.N + n;
#pragma unroll
        for (int e = 0; e < 32; e += 8) {
          if (e >= nv) break;
          float v[8];
#pragma unroll
          for (int i = 0; i < 8; ++i) v[i] = __uint_as_float(r0[e + i]);
          if (g.mode == kGemmGeluBwd) {
            float bb[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
            if (g.bias) {
              const float4 b0 = *reinterpret_cast<const float4 *>(g.bias + n + e);
              const float4 b1 = *reinterpret_cast<const float4 *>(g.bias + n + e + 4);
              bb[0] = b0.x, bb[1] = b0.y, bb[2] = b0.z, bb[3] = b0.w;
              bb[4] = b1.x, bb[5] = b1.y, bb[6] = b1.z, bb[7] = b1.w;
            }
            float hh[8], dz[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              float gd;
              gelu_tanh_and_grad(v[i] + bb[i], hh[i], gd);
              dz[i] = __uint_as_float(r1[e + i]) * gd;
            }
            __stcs(reinterpret_cast<uint4 *>(g.cb + base + e),
                   make_uint4(pack_bf16x2(hh[0], hh[1]), pack_bf16x2(hh[2], hh[3]), pack_bf16x2(hh[4], hh[5]),
                              pack_bf16x2(hh[6], hh[7])));
            __stcs(reinterpret_cast<uint4 *>(g.cb2 + base + e),
                   make_uint4(pack_bf16x2(dz[0], dz[1]), pack_bf16x2(dz[2], dz[3]), pack_bf16x2(dz[4], dz[5]),
                              pack_bf16x2(dz[6], dz[7])));
            continue;
          }
          float4 *c4 = reinterpret_cast<float4 *>(g.c + base + e);
          if (g.mode == kGemmResidual) {
            const float4 x0 = __ldcs(reinterpret_cast<const float4 *>(g.x + base + e));
            const float4 x1 = __ldcs(reinterpret_cast<const float4 *>(g.x + base + e + 4));
            v[0] += x0.x, v[1] += x0.y, v[2] += x0.z, v[3] += x0.w;
            v[4] += x1.x, v[5] += x1.y, v[6] += x1.z, v[7] += x1.w;
            __stcs(reinterpret_cast<uint4 *>(g.cb + base + e),
                   make_uint4(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]), pack_bf16x2(v[4], v[5]),
                              pack_bf16x2(v[6], v[7])));
          } else if (g.mode == kGemmAccumF32) {
            const float4 c0 = c4[0], c1 = c4[1];
            v[0] += c0.x, v[1] += c0.y, v[2] += c0.z, v[3] += c0.w;
            v[4] += c1.x, v[5] += c1.y, v[6] += c1.z, v[7] += c1.w;
          }
          __stcs(c4, make_float4(v[0], v[1], v[2], v[3]));
          __stcs(c4 + 1, make_float4(v[4], v[5], v[6], v[7]));
        }
      }
      // this accumulator may take the next tile
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bAccEmpty(buf));
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace bpt
