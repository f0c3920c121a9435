// gemm_sm100.cu -- tensor-core GEMM (tcgen05 + TMA) for the HSTU layer's two
// projections, with the epilogue fused:
//   f1: C = SiLU(A B^T + bias)            ([U|V|Q|K] = SiLU(x W1^T + b1))
//   f2: C = A B^T + bias + R              (y = x + G W2^T + b2)
// (DLRMv4 article, section "Model architecture: HSTU replaces the
// feature-interaction stack": one projection makes the layer's internal
// representations; the gated output replaces the cross network and FFN.)
//
// A [M,K] and B [N,K] are bf16 with K contiguous (B in the nn.Linear [out,in]
// layout), C [M,N] bf16, fp32 accumulation in tensor memory.  One CTA per
// 128 x 256 output tile; K in 64-element blocks through a 4-stage TMA ring
// (128-byte swizzle); warp 0 loads, warp 1 issues the MMAs (one thread),
// warps 4-7 run the epilogue (thread = output row) straight from tensor
// memory to global memory.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "internal.h"
#include "tile_common.cuh"

namespace hstu {
namespace gemm_tc {

constexpr int kBM = 128, kBN = 256, kBK = 64, kStages = 4, kThreads = 256;

struct Smem {
  alignas(1024) uint8_t a[kStages][kBM * kBK * 2];   // 16 KB per stage
  alignas(1024) uint8_t b[kStages][kBN * kBK * 2];   // 32 KB per stage
  uint64_t full[kStages], empty[kStages], acc_full, drain;
  uint32_t tmem_base;
};

struct Params {
  int64_t M, N, K;
  const float *bias;
  const __nv_bfloat16 *res;
  int64_t ldr;
  __nv_bfloat16 *c;
  int64_t ldc;
  int epi;
  WaitCtl wait;
  uint64_t drain_ns;
};

__global__ void __launch_bounds__(kThreads, 1)
    gemm_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
                const Params p) {
  extern __shared__ uint8_t smem_raw[];
  Smem &sm = *reinterpret_cast<Smem *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                       ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t m0 = int64_t(blockIdx.y) * kBM, n0 = int64_t(blockIdx.x) * kBN;
  const int nk = int((p.K + kBK - 1) / kBK);
  if (warp == 0 && lane == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&sm.full[s], 1);
      mbar_init(&sm.empty[s], 1);
    }
    mbar_init(&sm.acc_full, 1);
    mbar_init(&sm.drain, 1);
    fence_mbar_init();
    tma_prefetch_desc(&tm_a);
    tma_prefetch_desc(&tm_b);
  }
  if (warp == 1) {
    tmem_alloc(&sm.tmem_base, 256);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;

  if (warp == 0) {
    if (elect_one()) {
      bool ok = true;
      int issued = 0;
      for (int kb = 0; kb < nk && ok; ++kb) {
        const int s = kb % kStages;
        if (kb >= kStages) ok = wait_bar(&sm.empty[s], ((kb / kStages) - 1) & 1, p.wait);
        if (!ok) break;
        mbar_arrive_expect_tx(&sm.full[s], (kBM + kBN) * kBK * 2);
        tma_load_2d(sm.a[s], &tm_a, &sm.full[s], kb * kBK, int32_t(m0));
        tma_load_2d(sm.b[s], &tm_b, &sm.full[s], kb * kBK, int32_t(n0));
        ++issued;
      }
      for (int kb = (issued > kStages ? issued - kStages : 0); kb < issued; ++kb)
        drain_bar(&sm.full[kb % kStages], (kb / kStages) & 1, p.wait.err, p.drain_ns);
    }
    __syncwarp();
  } else if (warp == 1) {
    if (elect_one()) {
      constexpr uint32_t idesc = idesc_bf16(kBM, kBN, false, false);
      bool ok = true;
      for (int kb = 0; kb < nk && ok; ++kb) {
        const int s = kb % kStages;
        ok = wait_bar(&sm.full[s], (kb / kStages) & 1, p.wait);
        if (!ok) break;
        tc_fence_after();
        const uint32_t a = smem_u32(sm.a[s]), b = smem_u32(sm.b[s]);
#pragma unroll
        for (int kk = 0; kk < kBK / 16; ++kk)
          umma_ss(tmem, sdesc_sw128(a + kk * 32, 16, 1024), sdesc_sw128(b + kk * 32, 16, 1024),
                  idesc, (kb > 0 || kk > 0) ? 1u : 0u);
        umma_commit(&sm.empty[s]);
      }
      umma_commit(&sm.acc_full);
      umma_commit(&sm.drain);
      drain_bar(&sm.drain, 0, p.wait.err, p.drain_ns);
    }
    __syncwarp();
  } else if (warp >= 4) {
    const int quad = warp & 3;
    const int64_t row = m0 + quad * 32 + lane;
    const uint32_t lane_base = tmem + (uint32_t(quad * 32) << 16);
    const bool ok = wait_bar(&sm.acc_full, 0, p.wait);
    tc_fence_after();
    if (ok) {
#pragma unroll 1
      for (int c0 = 0; c0 < kBN; c0 += 32) {
        uint32_t r[32];
        tmem_ld32(lane_base + c0, r);
        tmem_wait_ld(r);
        const int64_t col = n0 + c0;
        if (row >= p.M || col >= p.N) continue;
        float y[32];
#pragma unroll
        for (int e = 0; e < 32; ++e) y[e] = __uint_as_float(r[e]) + p.bias[col + e];
        if (p.epi == kEpiBiasSilu) {
#pragma unroll
          for (int e = 0; e < 32; ++e) y[e] = y[e] / (1.0f + __expf(-y[e]));
        } else if (p.epi == kEpiBiasResidual) {
          const uint4 *rr = reinterpret_cast<const uint4 *>(p.res + row * p.ldr + col);
#pragma unroll
          for (int v = 0; v < 4; ++v) {
            const uint4 u = rr[v];
            const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              y[v * 8 + 2 * e] += __uint_as_float(w[e] << 16);
              y[v * 8 + 2 * e + 1] += __uint_as_float(w[e] & 0xFFFF0000u);
            }
          }
        }
        uint4 *dst = reinterpret_cast<uint4 *>(p.c + row * p.ldc + col);
#pragma unroll
        for (int v = 0; v < 4; ++v)
          dst[v] = make_uint4(pack_bf16x2(y[8 * v], y[8 * v + 1]),
                              pack_bf16x2(y[8 * v + 2], y[8 * v + 3]),
                              pack_bf16x2(y[8 * v + 4], y[8 * v + 5]),
                              pack_bf16x2(y[8 * v + 6], y[8 * v + 7]));
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
}

}  // namespace gemm_tc

bool gemm_tc_supported(const void *a, int64_t lda, const void *b, int64_t ldb, const void *c,
                       int64_t ldc, int64_t M, int64_t N, int64_t K) {
  if (M <= 0 || N <= 0 || K <= 0) return false;
  if ((N % 32) || (K % 8) || (lda % 8) || (ldb % 8) || (ldc % 8)) return false;
  if ((reinterpret_cast<uintptr_t>(a) | reinterpret_cast<uintptr_t>(b) |
       reinterpret_cast<uintptr_t>(c)) & 15)
    return false;
  if (M >= (int64_t(1) << 31) || N >= (int64_t(1) << 31)) return false;
  return true;
}

cudaError_t launch_gemm_tc(const void *a, int64_t lda, const void *b, int64_t ldb,
                           const float *bias, const void *residual, int64_t ldr, void *c,
                           int64_t ldc, int64_t M, int64_t N, int64_t K, int epilogue,
                           const WaitCtl &w, cudaStream_t st) {
  using namespace gemm_tc;
  if (epilogue == kEpiBiasResidual &&
      ((reinterpret_cast<uintptr_t>(residual) & 15) || (ldr % 8)))
    return cudaErrorInvalidValue;
  CUtensorMap ta, tb;
  if (!encode_tmap_bf16_2d(&ta, a, uint64_t(K), uint64_t(M), uint64_t(lda) * 2, kBK, kBM) ||
      !encode_tmap_bf16_2d(&tb, b, uint64_t(K), uint64_t(N), uint64_t(ldb) * 2, kBK, kBN))
    return cudaErrorInvalidValue;
  Params prm;
  prm.M = M;
  prm.N = N;
  prm.K = K;
  prm.bias = bias;
  prm.res = static_cast<const __nv_bfloat16 *>(residual);
  prm.ldr = ldr;
  prm.c = static_cast<__nv_bfloat16 *>(c);
  prm.ldc = ldc;
  prm.epi = epilogue;
  prm.wait = w;
  prm.drain_ns = 4000000000ull;
  const size_t smem = sizeof(Smem) + 1024;
  static bool attr_done = false;
  if (!attr_done) {
    cudaError_t e =
        cudaFuncSetAttribute(gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
    if (e != cudaSuccess) return e;
    attr_done = true;
  }
  const dim3 grid(unsigned((N + kBN - 1) / kBN), unsigned((M + kBM - 1) / kBM));
  gemm_kernel<<<grid, kThreads, smem, st>>>(ta, tb, prm);
  count_launch();
  return cudaGetLastError();
}

}  // namespace hstu
