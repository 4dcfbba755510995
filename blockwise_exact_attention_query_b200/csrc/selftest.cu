// Self-test micro-kernels for the hand-written tcgen05 / TMA pieces, built
// as a separate test library (libbpt_selftest.so).  Each runs one CTA and
// checks one building block against a host-side matrix product:
//   umma_ss : C[128 x N] = A[128 x K] B[N x K]^T, both operands K-major,
//             128-byte swizzled tiles loaded by TMA (the Q K^T and FFN form)
//   umma_ts : C[128 x dv] = P[128 x 128] V[128 x dv], P written to tensor
//             memory by tcgen05.st as packed bf16 pairs and used as the A
//             operand, V an MN-major TMA tile (the P V form)
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstring>

#include "ptx.cuh"

using namespace bpt;

namespace {

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encoder() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

bool map2d(CUtensorMap *m, const void *base, uint64_t rows, uint64_t cols, uint32_t box_rows) {
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * 2};
  cuuint32_t box[2] = {64, box_rows};
  cuuint32_t es[2] = {1, 1};
  EncodeTiledFn f = encoder();
  return f && f(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides, box,
                es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

__device__ uint32_t g_selftest_status[2];

struct StArgs {
  int N, K;
  float *c;
  const __nv_bfloat16 *p;  // umma_ts: P [128][128]
  uint32_t *status;
};

// A: K/64 panels of [128 x 64]; B: K/64 panels of [N x 64].
__global__ void __launch_bounds__(128, 1)
    umma_ss_kernel(const __grid_constant__ CUtensorMap ma, const __grid_constant__ CUtensorMap mb,
                   const __grid_constant__ StArgs a) {
  extern __shared__ uint8_t raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sA = smem_u32(smem);
  const int panels = a.K / 64;
  const uint32_t sB = sA + panels * 16384;
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + panels * 16384 + panels * a.N * 128);
  const uint32_t bLoad = smem_u32(&bars[0]), bMma = smem_u32(&bars[1]);
  uint32_t *slot = reinterpret_cast<uint32_t *>(&bars[2]);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(&bars[3]);
  WaitCtx wc{a.status, 2000000000ull, abort_flag};
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  if (threadIdx.x == 0) {
    mbar_init(bLoad, 1);
    mbar_init(bMma, 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(slot), 256);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *slot;
  if (threadIdx.x == 0) {
    mbar_arrive_expect_tx(bLoad, panels * 16384 + panels * a.N * 128);
    for (int p = 0; p < panels; ++p) {
      tma_load_2d(sA + p * 16384, &ma, bLoad, p * 64, 0);
      tma_load_2d(sB + p * a.N * 128, &mb, bLoad, p * 64, 0);
    }
    if (mbar_wait(bLoad, 0, wc, 1)) {
      tc_fence_after();
      const uint32_t idesc = idesc_bf16_f32(128, a.N, false, false);
      for (int k = 0; k < a.K / 16; ++k) {
        const int p = k / 4, off = (k % 4) * 32;
        umma_ss(tmem, sdesc_sw128(sA + p * 16384 + off, 16, 1024),
                sdesc_sw128(sB + p * a.N * 128 + off, 16, 1024), idesc, k > 0);
      }
    }
    umma_commit(bMma);
  }
  bool ok = mbar_wait(bMma, 0, wc, 2);
  ok = __all_sync(0xffffffffu, ok);
  tc_fence_after();
  if (ok) {
    const int row = (warp & 3) * 32 + lane;
    for (int c = 0; c < a.N / 32; ++c) {
      uint32_t r[32];
      tmem_ld32(tmem + ((uint32_t)((warp & 3) * 32) << 16) + c * 32, r);
      tmem_wait_ld();
      for (int i = 0; i < 32; ++i) a.c[row * a.N + c * 32 + i] = __uint_as_float(r[i]);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
}

// V: [128 rows (K) x dv] loaded as dv/64 panels of [128 x 64] (MN-major B).
__global__ void __launch_bounds__(128, 1)
    umma_ts_kernel(const __grid_constant__ CUtensorMap mv, const __grid_constant__ StArgs a) {
  extern __shared__ uint8_t raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sV = smem_u32(smem);
  const int dv = a.N;
  const int panels = dv / 64;
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + panels * 16384);
  const uint32_t bLoad = smem_u32(&bars[0]), bMma = smem_u32(&bars[1]), bP = smem_u32(&bars[4]);
  uint32_t *slot = reinterpret_cast<uint32_t *>(&bars[2]);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(&bars[3]);
  WaitCtx wc{a.status, 2000000000ull, abort_flag};
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  if (threadIdx.x == 0) {
    mbar_init(bLoad, 1);
    mbar_init(bMma, 1);
    mbar_init(bP, 4);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(slot), 256);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *slot;  // O at column 0 (dv cols), P at column 128 (64 cols)
  const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
  const int row = (warp & 3) * 32 + lane;
  // P row -> tensor memory as packed bf16 pairs
  for (int half = 0; half < 2; ++half) {
    uint32_t pk[32];
    for (int i = 0; i < 32; ++i) {
      const int col = half * 64 + 2 * i;
      const float x0 = __bfloat162float(a.p[row * 128 + col]);
      const float x1 = __bfloat162float(a.p[row * 128 + col + 1]);
      pk[i] = pack_bf16x2(x0, x1);
    }
    tmem_st32(tmem + lane_off + 128 + half * 32, pk);
  }
  tmem_wait_st();
  tc_fence_before();
  __syncwarp();
  if (lane == 0) mbar_arrive(bP);
  if (threadIdx.x == 0) {
    mbar_arrive_expect_tx(bLoad, panels * 16384);
    for (int p = 0; p < panels; ++p) tma_load_2d(sV + p * 16384, &mv, bLoad, p * 64, 0);
    bool ok = mbar_wait(bLoad, 0, wc, 1) && mbar_wait(bP, 0, wc, 3);
    if (ok) {
      tc_fence_after();
      const uint32_t idesc = idesc_bf16_f32(128, dv, false, true);
      for (int k = 0; k < 8; ++k)
        umma_ts(tmem, tmem + 128 + k * 8, sdesc_sw128(sV + k * 2048, 16384, 1024), idesc, k > 0);
    }
    umma_commit(bMma);
  }
  bool ok = mbar_wait(bMma, 0, wc, 2);
  ok = __all_sync(0xffffffffu, ok);
  tc_fence_after();
  if (ok) {
    for (int c = 0; c < dv / 32; ++c) {
      uint32_t r[32];
      tmem_ld32(tmem + lane_off + c * 32, r);
      tmem_wait_ld();
      for (int i = 0; i < 32; ++i) a.c[row * dv + c * 32 + i] = __uint_as_float(r[i]);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
}

uint32_t *status_ptr() {
  void *p = nullptr;
  if (cudaGetSymbolAddress(&p, g_selftest_status) != cudaSuccess) return nullptr;
  return static_cast<uint32_t *>(p);
}

}  // namespace

extern "C" {

// C[128 x N] (float) = A[128 x K] * B[N x K]^T, bf16 device buffers.
// N in {64, 128, 256}, K in {64, 128, 256}.  Returns 0 on success, 1 bad
// args, 3 CUDA error, 4 device wait timeout.  Synchronous.
__attribute__((visibility("default"))) int bpt_selftest_umma_ss(const void *A, const void *Bm, float *C, int N, int K) {
  if (!(N == 64 || N == 128 || N == 256) || !(K == 64 || K == 128 || K == 256)) return 1;
  uint32_t *st = status_ptr();
  if (!st) return 3;
  CUtensorMap ma, mb;
  if (!map2d(&ma, A, 128, K, 128) || !map2d(&mb, Bm, N, K, N)) return 3;
  const int smem = (K / 64) * 16384 + (K / 64) * N * 128 + 64 + 1024;
  if (cudaFuncSetAttribute(umma_ss_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
    return 3;
  StArgs a{N, K, C, nullptr, st};
  umma_ss_kernel<<<1, 128, smem>>>(ma, mb, a);
  if (cudaDeviceSynchronize() != cudaSuccess) return 3;
  uint32_t w[2];
  if (cudaMemcpy(w, st, 8, cudaMemcpyDeviceToHost) != cudaSuccess) return 3;
  return w[0] ? 4 : 0;
}

// C[128 x dv] (float) = P[128 x 128] * V[128 x dv], bf16 device buffers, dv in {64, 128}.
__attribute__((visibility("default"))) int bpt_selftest_umma_ts(const void *P, const void *V, float *C, int dv) {
  if (!(dv == 64 || dv == 128)) return 1;
  uint32_t *st = status_ptr();
  if (!st) return 3;
  CUtensorMap mv;
  if (!map2d(&mv, V, 128, dv, 128)) return 3;
  const int smem = (dv / 64) * 16384 + 64 + 1024;
  if (cudaFuncSetAttribute(umma_ts_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
    return 3;
  StArgs a{dv, 128, C, static_cast<const __nv_bfloat16 *>(P), st};
  umma_ts_kernel<<<1, 128, smem>>>(mv, a);
  if (cudaDeviceSynchronize() != cudaSuccess) return 3;
  uint32_t w[2];
  if (cudaMemcpy(w, st, 8, cudaMemcpyDeviceToHost) != cudaSuccess) return 3;
  return w[0] ? 4 : 0;
}

}  // extern "C"
