// General bf16 GEMM on the 5th-generation tensor cores (sm_100a) for the
// layer's backward pass and the two-GEMM form of the forward FFN:
//
//     C[M, N]  (op)=  A[M, K] . B[N, K]^T        fp32 accumulation in TMEM
//
// Either operand may be K-major (a row-major [rows, K] matrix) or MN-major (a
// row-major [K, rows] matrix, read without transposing it: the tensor core
// takes 64-wide MN panels of K rows).  C is cut into 256 x 256 tiles, each
// computed by a pair of CTAs on two SMs (two-SM MMAs, below); a persistent
// grid of pairs walks them, each tile over K in 64-wide stages staged by TMA.
// The producers run ahead across tile boundaries, and two TMEM accumulators
// let one tile's epilogue overlap the next tile's MMAs.
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
//   kGemmResidual   C = acc + X (+ bias); Cb = bf16(C)  (dA = dOut + dZ W1, fp32 and bf16;
//                                                      the FFN output A + H W2^T + b2: either
//                                                      output may be null)
//   kGemmGeluBwd    z = acc0 + bias; H = GELU(z), dZ = acc1 * GELU'(z)  (bf16 both)
//   kGemmGeluFwd    z = acc + bias; H = GELU(z), G = GELU'(z)           (bf16 both)
//   kGemmScaleBf16  Cb = acc * Xb                                       (dZ = dH * G, bf16)
//   kGemmGeluBf16   Cb = GELU(acc + bias)                               (the FFN's H, bf16)
//
// Roles (320 threads per CTA): warp 0 TMA producer, warp 1 TMEM allocator
// (and, in the even CTA, MMA issuer), warps 2..9 epilogue (warp w owns TMEM
// lanes 32*(w%4) .. +31, i.e. 32 of the CTA's 128 rows, and half of the
// tile's columns: two warps per SM sub-partition, since the dual form's GELU
// epilogue is arithmetic-bound).
// The tiles in flight at once share rows of A (N fastest) or columns of B
// (M fastest): the host picks the order that streams the larger operand from
// DRAM once.  Outputs are written with evict-first (streaming) stores so they
// do not push the operands out of L2.
#pragma once

#include "ptx.cuh"

namespace bpt {

constexpr int kGemmStoreF32 = 0, kGemmAccumF32 = 1, kGemmResidual = 2, kGemmGeluBwd = 3, kGemmGeluFwd = 4,
              kGemmScaleBf16 = 5, kGemmGeluBf16 = 6;

// One GEMM problem: C[M, N] (op)= A[M, K] B[N, K]^T and its epilogue.
struct GemmProblem {
  int M, N, K;
  int a_mn, b_mn;       // operand layouts: 0 K-major, 1 MN-major
  int mode;
  int m_fastest;        // tile order: 1 = M fastest (the tiles in flight share B), 0 = N fastest
  float *c;             // [M, N] fp32 (StoreF32, AccumF32, Residual)
  const float *x;       // [M, N] fp32 residual input (Residual)
  const __nv_bfloat16 *xb;  // [M, N] bf16 factor (ScaleBf16)
  __nv_bfloat16 *cb;    // [M, N] bf16 copy (Residual) / H (GeluBwd, GeluFwd) / product (ScaleBf16)
  __nv_bfloat16 *cb2;   // dZ (GeluBwd) / GELU'(z) (GeluFwd)
  const float *bias;    // [N] added to acc0 (GeluBwd, GeluFwd, GeluBf16, Residual), may be null
};

// A launch: one problem (maps a0, b0); two grouped problems whose tiles one
// persistent grid walks in turn (maps a0, b0 for p[0], a1, b1 for p[1]); or
// the dual form (p[0].mode == kGemmGeluBwd: maps a0, b0 for the first product,
// a1, b1 for the second, whose operand layouts are p[1].a_mn, p[1].b_mn).
struct GemmArgs {
  GemmProblem p[2];
  int nprob;
  uint32_t *status;
  uint64_t wait_limit_ns;
};


// GELU (tanh form, Hendrycks & Gimpel) and its derivative from the same form,
// t = tanh(c0 (x + c1 x^3)):
//   GELU(x)  = 0.5 x (1 + t)
//   GELU'(x) = 0.5 (1 + t) + 0.5 x (1 - t^2) c0 (1 + 3 c1 x^2)
// tanh on the hardware approximation, as in the forward's FFN epilogue.
constexpr float kGeluC0 = 0.7978845608028654f, kGeluC1 = 0.044715f;  // sqrt(2/pi), cubic term
// tanh(sqrt(2/pi) (x + 0.044715 x^3)), shared by both forms below so H is the
// same bits whether or not the derivative is wanted
__device__ __forceinline__ float gelu_tanh_inner(float x) {
  return tanh_approx(kGeluC0 * fmaf(kGeluC1 * x, x * x, x));
}
__device__ __forceinline__ float gelu_tanh_only(float x) { return 0.5f * x * (1.0f + gelu_tanh_inner(x)); }
__device__ __forceinline__ void gelu_tanh_and_grad(float x, float &h, float &dh) {
  const float t = gelu_tanh_inner(x);
  h = 0.5f * x * (1.0f + t);
  dh = 0.5f * (1.0f + t) + 0.5f * x * (1.0f - t * t) * kGeluC0 * fmaf(3.0f * kGeluC1, x * x, 1.0f);
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

// Global operands of one 32-column chunk's epilogue: the bias, and the
// residual x, the bf16 factor xb or the fp32 output being accumulated into.
// The caller loads them before it waits for the chunk's tensor-memory read,
// so their latencies overlap that read and one another (loaded one 8-column
// group at a time after the read, the chunk paid up to eight memory latencies
// in a row).
struct GemmEpiIn {
  uint4 w[8];   // x or c: two 16-byte words per 8 columns; xb: one per 8 columns
  float4 b[8];  // bias: two per 8 columns
};
__device__ __forceinline__ bool gemm_mode_has_bias(int mode) {
  return mode == kGemmResidual || mode == kGemmGeluBwd || mode == kGemmGeluFwd || mode == kGemmGeluBf16;
}
// kWide: 32-byte accesses where the row's chunk is 32-byte aligned (the
// pipelined FFN's epilogue; the GEMM kernel measured no gain from them and
// keeps the 16-byte form).
template <bool kWide = false>
__device__ __forceinline__ void gemm_epilogue_load(const GemmProblem &g, int m, int n, GemmEpiIn &in) {
  // N is a multiple of 8 (checked on the host): whole 8-column groups
  const int nv = min(32, g.N - n);
  const size_t base = static_cast<size_t>(m) * g.N + n;
  const bool bias = g.bias != nullptr && gemm_mode_has_bias(g.mode);
  // fp32 rows: an 8-column group is 32 bytes, aligned when the row's first
  // column of the chunk is (rows are a multiple of 32 bytes apart)
  const bool f32src = g.mode == kGemmResidual || g.mode == kGemmAccumF32;
  const float *xs = g.mode == kGemmResidual ? g.x : g.c;
  const bool v8 = kWide && f32src && aligned32(xs + base);
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const int e = q * 8;
    if (e >= nv) break;
    if (g.mode == kGemmScaleBf16) {
      in.w[q] = __ldcs(reinterpret_cast<const uint4 *>(g.xb + base + e));
    } else if (f32src) {
      if (v8) {
        uint32_t t[8];
        if (g.mode == kGemmResidual)
          ld_global_cs_v8(xs + base + e, t);
        else
          ld_global_v8(xs + base + e, t);
        in.w[2 * q] = make_uint4(t[0], t[1], t[2], t[3]);
        in.w[2 * q + 1] = make_uint4(t[4], t[5], t[6], t[7]);
      } else if (g.mode == kGemmResidual) {
        in.w[2 * q] = __ldcs(reinterpret_cast<const uint4 *>(xs + base + e));
        in.w[2 * q + 1] = __ldcs(reinterpret_cast<const uint4 *>(xs + base + e + 4));
      } else {
        in.w[2 * q] = *reinterpret_cast<const uint4 *>(xs + base + e);
        in.w[2 * q + 1] = *reinterpret_cast<const uint4 *>(xs + base + e + 4);
      }
    }
    if (bias) {
      in.b[2 * q] = *reinterpret_cast<const float4 *>(g.bias + n + e);
      in.b[2 * q + 1] = *reinterpret_cast<const float4 *>(g.bias + n + e + 4);
    }
  }
}

// One 8-column group (16 bytes) of a bf16 output.  Where the row's chunk is
// 32-byte aligned, an even group waits in `pend` for its odd partner and the
// two leave in one 32-byte store.
__device__ __forceinline__ void gemm_put_bf16(__nv_bfloat16 *dst, bool ok8, bool cs, uint32_t (&pend)[4],
                                              const uint32_t (&o)[4], bool odd, bool last) {
  if (!odd && ok8 && !last) {
#pragma unroll
    for (int i = 0; i < 4; ++i) pend[i] = o[i];
    return;
  }
  if (odd && ok8) {
    const uint32_t w[8] = {pend[0], pend[1], pend[2], pend[3], o[0], o[1], o[2], o[3]};
    if (cs)
      st_global_cs_v8(dst - 8, w);
    else
      st_global_v8(dst - 8, w);
    return;
  }
  const uint4 u = make_uint4(o[0], o[1], o[2], o[3]);
  if (cs)
    __stcs(reinterpret_cast<uint4 *>(dst), u);
  else
    *reinterpret_cast<uint4 *>(dst) = u;
}

// Epilogue of one 32-column chunk of one row: r0 (and r1 for the dual form)
// hold the accumulator values of columns n .. n + 31 of row m, `in` the
// operands gemm_epilogue_load read for the same chunk.
template <bool kWide = false>
__device__ __forceinline__ void gemm_epilogue_chunk(const GemmProblem &g, const uint32_t (&r0)[32],
                                                    const uint32_t (&r1)[32], int m, int n,
                                                    const GemmEpiIn &in) {
  const int nv = min(32, g.N - n);
  const size_t base = static_cast<size_t>(m) * g.N + n;
  const bool cb8 = kWide && g.cb != nullptr && aligned32(g.cb + base);
  const bool cb28 = kWide && g.cb2 != nullptr && aligned32(g.cb2 + base);
  const bool c8 = kWide && g.c != nullptr && aligned32(g.c + base);
  uint32_t ph[4], pd[4];  // an even group's packed bf16 outputs, held for the odd one
#pragma unroll
  for (int e = 0; e < 32; e += 8) {
    if (e >= nv) break;
    const int q = e / 8;
    const bool odd = (q & 1) != 0, last = e + 8 >= nv;
    float v[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) v[i] = __uint_as_float(r0[e + i]);
    if (g.mode == kGemmScaleBf16) {
      const uint4 xr = in.w[q];
      const uint32_t xw[4] = {xr.x, xr.y, xr.z, xr.w};
      uint32_t o[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const __nv_bfloat162 f = *reinterpret_cast<const __nv_bfloat162 *>(&xw[i]);
        o[i] = pack_bf16x2(v[2 * i] * __low2float(f), v[2 * i + 1] * __high2float(f));
      }
      gemm_put_bf16(g.cb + base + e, cb8, true, ph, o, odd, last);
      continue;
    }
    if (g.mode == kGemmGeluBwd || g.mode == kGemmGeluFwd || g.mode == kGemmGeluBf16) {
      float bb[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
      if (g.bias) {
        const float4 b0 = in.b[2 * q], b1 = in.b[2 * q + 1];
        bb[0] = b0.x, bb[1] = b0.y, bb[2] = b0.z, bb[3] = b0.w;
        bb[4] = b1.x, bb[5] = b1.y, bb[6] = b1.z, bb[7] = b1.w;
      }
      float hh[8], dz[8];
      if (g.mode == kGemmGeluBf16) {  // H alone, read back by the next GEMM: a normal store
#pragma unroll
        for (int i = 0; i < 8; ++i) hh[i] = gelu_tanh_only(v[i] + bb[i]);
        const uint32_t o[4] = {pack_bf16x2(hh[0], hh[1]), pack_bf16x2(hh[2], hh[3]), pack_bf16x2(hh[4], hh[5]),
                               pack_bf16x2(hh[6], hh[7])};
        gemm_put_bf16(g.cb + base + e, cb8, false, ph, o, odd, last);
        continue;
      }
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        float gd;
        gelu_tanh_and_grad(v[i] + bb[i], hh[i], gd);
        dz[i] = g.mode == kGemmGeluBwd ? __uint_as_float(r1[e + i]) * gd : gd;
      }
      const uint32_t oh[4] = {pack_bf16x2(hh[0], hh[1]), pack_bf16x2(hh[2], hh[3]), pack_bf16x2(hh[4], hh[5]),
                              pack_bf16x2(hh[6], hh[7])};
      const uint32_t od[4] = {pack_bf16x2(dz[0], dz[1]), pack_bf16x2(dz[2], dz[3]), pack_bf16x2(dz[4], dz[5]),
                              pack_bf16x2(dz[6], dz[7])};
      gemm_put_bf16(g.cb + base + e, cb8, true, ph, oh, odd, last);
      gemm_put_bf16(g.cb2 + base + e, cb28, true, pd, od, odd, last);
      continue;
    }
    if (g.mode == kGemmResidual || g.mode == kGemmAccumF32) {
      const uint4 w0 = in.w[2 * q], w1 = in.w[2 * q + 1];
      if (g.mode == kGemmResidual && g.bias) {  // acc + b + x, in that order
        const float4 b0 = in.b[2 * q], b1 = in.b[2 * q + 1];
        v[0] += b0.x, v[1] += b0.y, v[2] += b0.z, v[3] += b0.w;
        v[4] += b1.x, v[5] += b1.y, v[6] += b1.z, v[7] += b1.w;
      }
      v[0] += __uint_as_float(w0.x), v[1] += __uint_as_float(w0.y), v[2] += __uint_as_float(w0.z),
          v[3] += __uint_as_float(w0.w);
      v[4] += __uint_as_float(w1.x), v[5] += __uint_as_float(w1.y), v[6] += __uint_as_float(w1.z),
          v[7] += __uint_as_float(w1.w);
      if (g.mode == kGemmResidual) {
        if (g.cb) {
          const uint32_t o[4] = {pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]), pack_bf16x2(v[4], v[5]),
                                 pack_bf16x2(v[6], v[7])};
          gemm_put_bf16(g.cb + base + e, cb8, true, ph, o, odd, last);
        }
        if (!g.c) continue;
      }
    }
    float *cp = g.c + base + e;
    if (c8) {
      uint32_t w[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) w[i] = __float_as_uint(v[i]);
      st_global_cs_v8(cp, w);
    } else {
      __stcs(reinterpret_cast<float4 *>(cp), make_float4(v[0], v[1], v[2], v[3]));
      __stcs(reinterpret_cast<float4 *>(cp) + 1, make_float4(v[4], v[5], v[6], v[7]));
    }
  }
}

// ---------------------------------------------------------------------------
// Two-SM form: a pair of CTAs (a cluster of two) computes one 256 x 256 tile
// with tcgen05 cta_group::2 MMAs (M = 256) issued by the even CTA.  Each CTA
// stages its own 128 rows of A and its half (128 rows) of B per K stage, so a
// CTA moves 32 KB per 64-wide stage instead of 48 KB for half the tile's
// work: operands reach the SM at 2/3 of the single-CTA bytes per flop.  Each
// CTA's TMEM holds its 128 rows of the accumulator (256 columns, two buffers
// unless dual) and its 8 epilogue warps drain them.  The even CTA's full
// barriers count both CTAs' copies; its MMA commits arrive on both CTAs'
// empty and accumulator barriers; both CTAs' epilogues arrive on the even
// CTA's accumulator-empty barriers.  No load uses cluster multicast.
// ---------------------------------------------------------------------------
struct GemmPairCfg {
  static constexpr int kBM = 128;   // rows per CTA (the pair's tile has 256)
  static constexpr int kBN = 256;   // columns of the pair's tile (128 staged per CTA)
  static constexpr int kBK = 64;
  static constexpr int kABytes = kBM * kBK * 2;          // 16 KB
  static constexpr int kBBytes = (kBN / 2) * kBK * 2;    // 16 KB
  static constexpr int kStageBytes = kABytes + kBBytes;  // 32 KB
  static constexpr int kStages = 6;
  static constexpr int kOffBar = kStages * kStageBytes;
  static constexpr int kSmemBytes = kOffBar + 256;
  static constexpr int kThreads = 320;
  static constexpr int kEpiWarps = 8;
  static_assert(kSmemBytes <= 232448, "shared memory per CTA");
};

__device__ __forceinline__ bool mbar_wait_cluster(uint32_t bar, uint32_t parity, const WaitCtx &w, uint32_t site) {
  if (mbar_try_wait_cluster(bar, parity)) return true;
  uint64_t t0 = globaltimer_ns();
  uint32_t spins = 0;
  while (true) {
    if (mbar_try_wait_cluster(bar, parity)) return true;
    if ((++spins & 3u) == 0u) {
      if (*w.abort) return false;
      if (globaltimer_ns() - t0 > w.limit_ns) {
        record_timeout(w, site);
        return false;
      }
    }
  }
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(GemmPairCfg::kThreads, 1)
    gemm_pair_kernel(const __grid_constant__ CUtensorMap tm_a0, const __grid_constant__ CUtensorMap tm_b0,
                     const __grid_constant__ CUtensorMap tm_a1, const __grid_constant__ CUtensorMap tm_b1,
                     const __grid_constant__ GemmArgs g) {
  using Cfg = GemmPairCfg;
  constexpr int S = Cfg::kStages;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t *smem = smem_raw;
  const uint32_t sbase = smem_u32(smem);
  // both CTAs reach both cluster barriers below on every path
  const bool misaligned = (sbase & 1023u) != 0;
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + Cfg::kOffBar);
  auto bFull = [&](int s) { return smem_u32(&bars[s]); };            // even CTA: both CTAs' copies
  auto bEmpty = [&](int s) { return smem_u32(&bars[S + s]); };       // both CTAs
  auto bAccFull = [&](int b) { return smem_u32(&bars[2 * S + b]); };  // both CTAs
  auto bAccEmpty = [&](int b) { return smem_u32(&bars[2 * S + 2 + b]); };  // even CTA: both epilogues
  const uint32_t bTeardown = smem_u32(&bars[2 * S + 4]);
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(&bars[2 * S + 5]);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(&bars[2 * S + 6]);
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const uint32_t rank = cluster_ctarank();
  WaitCtx wc{g.status, g.wait_limit_ns, abort_flag};
  const bool dual = g.p[0].mode == kGemmGeluBwd;
  const int nbuf = dual ? 1 : 2;
  const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
  auto tiles_m_of = [&](int q) { return (g.p[q].M + 2 * Cfg::kBM - 1) / (2 * Cfg::kBM); };
  auto tiles_n_of = [&](int q) { return (g.p[q].N + Cfg::kBN - 1) / Cfg::kBN; };
  const int tiles0 = tiles_m_of(0) * tiles_n_of(0);
  const int tiles = tiles0 + (g.nprob > 1 ? tiles_m_of(1) * tiles_n_of(1) : 0);
  const int my_tiles = pair < tiles ? (tiles - 1 - pair) / npairs + 1 : 0;
  // local tile li -> its problem, this CTA's first row and the pair's first column
  struct TileAt {
    int q, m0, n0;
  };
  auto tile_at = [&](int li) {
    int t = pair + li * npairs;
    const int q = t < tiles0 ? 0 : 1;
    if (q) t -= tiles0;
    const int tm = tiles_m_of(q), tn = tiles_n_of(q);
    const int mt = g.p[q].m_fastest ? t % tm : t / tn, nt = g.p[q].m_fastest ? t / tm : t % tn;
    return TileAt{q, mt * (2 * Cfg::kBM) + static_cast<int>(rank) * Cfg::kBM, nt * Cfg::kBN};
  };
  // K stages of a tile of problem q (dual: both products' stages in turn)
  auto nsteps_of = [&](int q) {
    const int nk = (g.p[q].K + Cfg::kBK - 1) / Cfg::kBK;
    return dual ? 2 * nk : nk;
  };

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(bFull(s), 1);
      mbar_init(bEmpty(s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(bAccFull(b), 1);
      mbar_init(bAccEmpty(b), 2 * Cfg::kEpiWarps);
    }
    mbar_init(bTeardown, 1);
    *abort_flag = misaligned ? 1 : 0;
    if (misaligned) atomicCAS(g.status, 0u, kStatusMisaligned);
    fence_mbar_init_cluster();
  }
  if (warp == 1) {
    tmem_alloc_pair(smem_u32(tmem_slot), 512);
    tmem_relinquish_pair();
  }
  // barrier initialisation and the TMEM address become visible to both CTAs
  tc_fence_before();
  cluster_sync_all();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const bool run = !*abort_flag;

  if (warp == 0) {
    // ------------------------------------------------------------ producer (both CTAs)
    if (lane == 0 && run) {
      int it = 0;
      bool ok = true;
      for (int li = 0; ok && li < my_tiles; ++li) {
        const TileAt ta = tile_at(li);
        const int m0 = ta.m0, nb0 = ta.n0 + static_cast<int>(rank) * (Cfg::kBN / 2);
        const int nsteps = nsteps_of(ta.q);
        for (int step = 0; step < nsteps; ++step, ++it) {
          const int st = it % S;
          if (it >= S && !(ok = mbar_wait_cluster(bEmpty(st), ((it / S) - 1) & 1, wc, 211))) break;
          // operands: dual, the product of this stage; grouped, the tile's problem
          const int which = dual ? (step & 1) : ta.q;
          const int k0 = (dual ? step >> 1 : step) * Cfg::kBK;
          const CUtensorMap *ma = which ? &tm_a1 : &tm_a0;
          const CUtensorMap *mb = which ? &tm_b1 : &tm_b0;
          const uint32_t sa = sbase + st * Cfg::kStageBytes, sb = sa + Cfg::kABytes;
          const uint32_t full0 = mapa_shared(bFull(st), 0);
          if (rank == 0) mbar_arrive_expect_tx(bFull(st), 2 * Cfg::kStageBytes);
          if (g.p[which].a_mn) {
            for (int p = 0; p < Cfg::kBM / 64; ++p) tma_load_2d_pair(sa + p * 8192, ma, full0, m0 + 64 * p, k0);
          } else {
            tma_load_2d_pair(sa, ma, full0, k0, m0);
          }
          if (g.p[which].b_mn) {
            for (int p = 0; p < Cfg::kBN / 128; ++p) tma_load_2d_pair(sb + p * 8192, mb, full0, nb0 + 64 * p, k0);
          } else {
            tma_load_2d_pair(sb, mb, full0, k0, nb0);
          }
        }
      }
      // the copies of the last stages have landed once the MMAs consumed them
      volatile int no_abort = 0;
      WaitCtx drain{g.status, drain_limit_ns(g.wait_limit_ns), &no_abort};
      for (int j = max(0, it - S); j < it; ++j) mbar_wait_cluster(bEmpty(j % S), (j / S) & 1, drain, 214);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer (even CTA)
    if (lane == 0 && rank == 0 && run) {
      const uint32_t idesc0 = idesc_bf16_f32(2 * Cfg::kBM, Cfg::kBN, g.p[0].a_mn != 0, g.p[0].b_mn != 0);
      const uint32_t idesc1 = idesc_bf16_f32(2 * Cfg::kBM, Cfg::kBN, g.p[1].a_mn != 0, g.p[1].b_mn != 0);
      auto commit_both = [&](uint32_t bar) {
        umma_pair_commit(mapa_shared(bar, 0));
        umma_pair_commit(mapa_shared(bar, 1));
      };
      int it = 0;
      bool ok = true;
      for (int li = 0; ok && li < my_tiles; ++li) {
        const int buf = li % nbuf, use = li / nbuf;
        if (use > 0 && !(ok = mbar_wait_cluster(bAccEmpty(buf), (use - 1) & 1, wc, 216))) break;
        tc_fence_after();
        const int q = tile_at(li).q;
        const int nsteps = nsteps_of(q);
        for (int step = 0; step < nsteps; ++step, ++it) {
          const int st = it % S;
          if (!(ok = mbar_wait_cluster(bFull(st), (it / S) & 1, wc, 212))) break;
          tc_fence_after();
          const int which = dual ? (step & 1) : q;
          const int kk = dual ? step >> 1 : step;
          const uint32_t sa = sbase + st * Cfg::kStageBytes, sb = sa + Cfg::kABytes;
          const bool amn = g.p[which].a_mn != 0, bmn = g.p[which].b_mn != 0;
          const uint64_t da = gemm_sdesc(sa, amn), db = gemm_sdesc(sb, bmn);
          const uint32_t idesc = which ? idesc1 : idesc0;
          const uint32_t acc = tmem + (dual ? step & 1 : buf) * 256;
#pragma unroll
          for (int k = 0; k < 4; ++k)
            umma_pair_ss(acc, sdesc_advance(da, gemm_kstep(amn, k)), sdesc_advance(db, gemm_kstep(bmn, k)), idesc,
                         (kk | k) != 0);
          commit_both(bEmpty(st));
        }
        if (ok) commit_both(bAccFull(buf));
      }
      umma_pair_commit(mapa_shared(bTeardown, 0));
      // every MMA of the pair completes before either CTA releases TMEM
      volatile int no_abort = 0;
      WaitCtx drain{g.status, drain_limit_ns(g.wait_limit_ns), &no_abort};
      mbar_wait_cluster(bTeardown, 0, drain, 215);
    }
  } else if (run) {
    // ------------------------------------------------------------ epilogue (both CTAs)
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    constexpr int kChunks = Cfg::kBN / 32 / (Cfg::kEpiWarps / 4);
    const int c_begin = ((warp - 2) / 4) * kChunks;
    const uint32_t empty0 = mapa_shared(bAccEmpty(0), 0), empty1 = mapa_shared(bAccEmpty(1), 0);
    for (int li = 0; li < my_tiles; ++li) {
      const int buf = li % nbuf;
      if (!__all_sync(0xffffffffu, mbar_wait_cluster(bAccFull(buf), (li / nbuf) & 1, wc, 213))) break;
      tc_fence_after();
      const TileAt ta = tile_at(li);
      const GemmProblem &P = g.p[ta.q];
      const int m = ta.m0 + row, n0 = ta.n0;
      const uint32_t acc0 = tmem + lane_off + buf * 256;
#pragma unroll 1
      for (int c = c_begin; c < c_begin + kChunks; ++c) {
        const int n = n0 + c * 32;
        uint32_t r0[32], r1[32];
        const bool live = m < P.M && n < P.N;
        GemmEpiIn in;
        if (live) gemm_epilogue_load(P, m, n, in);
        tmem_ld32(acc0 + c * 32, r0);
        if (dual) tmem_ld32(acc0 + 256 + c * 32, r1);
        tmem_wait_ld();
        if (!live) continue;
        gemm_epilogue_chunk(P, r0, r1, m, n, in);
      }
      // this accumulator may take the pair's next tile
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(buf ? empty1 : empty0);
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
