// gemm_sm100.cu -- tensor-core GEMM (tcgen05 + TMA) for the HSTU layer's two
// projections, with the epilogue fused:
//   f1: C = SiLU(A B^T + bias)            ([U|V|Q|K] = SiLU(x W1^T + b1))
//   f2: C = A B^T + bias + R              (y = x + G W2^T + b2)
// (DLRMv4 article, section "Model architecture: HSTU replaces the
// feature-interaction stack": one projection makes the layer's internal
// representations; the gated output replaces the cross network and FFN.)
//
// A [M,K] and B [N,K] are bf16 with K contiguous (B in the nn.Linear [out,in]
// layout), C [M,N] bf16, fp32 accumulation in tensor memory.
//
// Persistent: one CTA per SM walks the 128 x 256 output tiles (N fastest, so
// the CTAs in flight share A row blocks in L2).  K runs in 64-element blocks
// through a 4-stage TMA ring (128-byte swizzle).  Two tensor-memory
// accumulators of 256 columns let the epilogue of one tile overlap the MMAs
// of the next.
//   warp 0      TMA producer
//   warp 1      tcgen05 issuer (one thread)
//   warps 4-11  epilogue, two warpgroups (columns [0,128) and [128,256) of a
//               tile; thread = output row): tensor memory -> bias (+ SiLU or
//               + residual) -> bf16 -> global memory.
// SiLU(y) = h (1 + tanh h) with h = y / 2 (sigmoid(y) = (1 + tanh(y/2)) / 2):
// one transcendental per element.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>

#include "internal.h"
#include "tile_common.cuh"

namespace hstu {
namespace gemm_tc {

constexpr int kBM = 128, kBN = 256, kBK = 64, kStages = 4, kThreads = 384;

struct Smem {
  alignas(1024) uint8_t a[kStages][kBM * kBK * 2];   // 16 KB per stage
  alignas(1024) uint8_t b[kStages][kBN * kBK * 2];   // 32 KB per stage
  uint64_t full[kStages], empty[kStages], acc_full[2], acc_empty[2], drain;
  uint32_t tmem_base;
};

struct Params {
  int64_t M, N, K;
  int32_t tiles_n, tiles;
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
  const int nk = int((p.K + kBK - 1) / kBK);
  // this CTA's tiles: blockIdx.x, blockIdx.x + gridDim.x, ...
  const int n_my = p.tiles > int(blockIdx.x) ? (p.tiles - 1 - int(blockIdx.x)) / int(gridDim.x) + 1
                                             : 0;
  auto tile_m0 = [&](int i) {
    return int64_t((int(blockIdx.x) + i * int(gridDim.x)) / p.tiles_n) * kBM;
  };
  auto tile_n0 = [&](int i) {
    return int64_t((int(blockIdx.x) + i * int(gridDim.x)) % p.tiles_n) * kBN;
  };
  if (warp == 0 && lane == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&sm.full[s], 1);
      mbar_init(&sm.empty[s], 1);
    }
    for (int x = 0; x < 2; ++x) {
      mbar_init(&sm.acc_full[x], 1);
      mbar_init(&sm.acc_empty[x], 256);
    }
    mbar_init(&sm.drain, 1);
    fence_mbar_init();
    tma_prefetch_desc(&tm_a);
    tma_prefetch_desc(&tm_b);
  }
  if (warp == 1) {
    tmem_alloc(&sm.tmem_base, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;

  if (warp == 0) {
    // ===================== TMA producer =====================
    if (elect_one()) {
      bool ok = true;
      int g = 0;   // k-blocks issued over all tiles (ring position)
      for (int i = 0; i < n_my && ok; ++i) {
        const int32_t m0 = int32_t(tile_m0(i)), n0 = int32_t(tile_n0(i));
        for (int kb = 0; kb < nk; ++kb, ++g) {
          const int s = g % kStages;
          if (g >= kStages) ok = wait_bar(&sm.empty[s], ((g / kStages) - 1) & 1, p.wait);
          if (!ok) break;
          mbar_arrive_expect_tx(&sm.full[s], (kBM + kBN) * kBK * 2);
          tma_load_2d(sm.a[s], &tm_a, &sm.full[s], kb * kBK, m0);
          tma_load_2d(sm.b[s], &tm_b, &sm.full[s], kb * kBK, n0);
        }
      }
      // every copy issued has landed before the CTA can exit
      for (int q = (g > kStages ? g - kStages : 0); q < g; ++q)
        drain_bar(&sm.full[q % kStages], (q / kStages) & 1, p.wait.err, p.drain_ns);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ===================== tcgen05 issuer =====================
    if (elect_one()) {
      constexpr uint32_t idesc = idesc_bf16(kBM, kBN, false, false);
      bool ok = true;
      int g = 0;
      for (int i = 0; i < n_my && ok; ++i) {
        const int acc = i & 1;
        // the epilogue has read this accumulator's previous tile out
        if (i >= 2) ok = wait_bar(&sm.acc_empty[acc], ((i >> 1) - 1) & 1, p.wait);
        if (!ok) break;
        tc_fence_after();
        const uint32_t d = tmem + uint32_t(acc) * kBN;
        for (int kb = 0; kb < nk && ok; ++kb, ++g) {
          const int s = g % kStages;
          ok = wait_bar(&sm.full[s], (g / kStages) & 1, p.wait);
          if (!ok) break;
          tc_fence_after();
          const uint64_t da = sdesc_sw128(smem_u32(sm.a[s]), 16, 1024);
          const uint64_t db = sdesc_sw128(smem_u32(sm.b[s]), 16, 1024);
#pragma unroll
          for (int kk = 0; kk < kBK / 16; ++kk)
            umma_ss(d, da + ((kk * 32) >> 4), db + ((kk * 32) >> 4), idesc,
                    (kb > 0 || kk > 0) ? 1u : 0u);
          umma_commit(&sm.empty[s]);
        }
        umma_commit(&sm.acc_full[acc]);
      }
      umma_commit(&sm.drain);
      drain_bar(&sm.drain, 0, p.wait.err, p.drain_ns);
    }
    __syncwarp();
  } else if (warp >= 4) {
    // ===================== epilogue =====================
    const int half = (warp - 4) >> 2;   // columns [128 half, 128 half + 128) of a tile
    const int quad = warp & 3;
    const uint32_t lane_base = tmem + (uint32_t(quad * 32) << 16);
    bool ok = true;
    for (int i = 0; i < n_my && ok; ++i) {
      const int acc = i & 1;
      ok = wait_bar_warp(&sm.acc_full[acc], (i >> 1) & 1, p.wait);
      if (!ok) break;
      tc_fence_after();
      const int64_t row = tile_m0(i) + quad * 32 + lane;
      const int64_t n0 = tile_n0(i) + half * 128;
#pragma unroll 1
      for (int c0 = 0; c0 < 128; c0 += 32) {
        uint32_t r[32];
        tmem_ld32(lane_base + uint32_t(acc) * kBN + half * 128 + c0, r);
        tmem_wait_ld(r);
        if (c0 + 32 == 128) {
          // this warpgroup's half of the accumulator is in registers
          tc_fence_before();
          mbar_arrive(&sm.acc_empty[acc]);
        }
        const int64_t col = n0 + c0;
        if (row >= p.M || col >= p.N) continue;
        float y[32];
        const float4 *bb = reinterpret_cast<const float4 *>(p.bias + col);
#pragma unroll
        for (int v = 0; v < 8; ++v) {
          const float4 b4 = __ldg(bb + v);
          y[4 * v] = __uint_as_float(r[4 * v]) + b4.x;
          y[4 * v + 1] = __uint_as_float(r[4 * v + 1]) + b4.y;
          y[4 * v + 2] = __uint_as_float(r[4 * v + 2]) + b4.z;
          y[4 * v + 3] = __uint_as_float(r[4 * v + 3]) + b4.w;
        }
        if (p.epi == kEpiBiasSilu) {
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            const float hh = 0.5f * y[e];
            y[e] = fmaf(hh, tanh_approx(hh), hh);
          }
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
    tmem_dealloc(tmem, 512);
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
  const int64_t tiles = ((M + 127) / 128) * ((N + 255) / 256);
  if (tiles >= (int64_t(1) << 30)) return false;
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
  if (reinterpret_cast<uintptr_t>(bias) & 15) return cudaErrorInvalidValue;
  CUtensorMap ta, tb;
  if (!encode_tmap_bf16_2d(&ta, a, uint64_t(K), uint64_t(M), uint64_t(lda) * 2, kBK, kBM) ||
      !encode_tmap_bf16_2d(&tb, b, uint64_t(K), uint64_t(N), uint64_t(ldb) * 2, kBK, kBN))
    return cudaErrorInvalidValue;
  Params prm;
  prm.M = M;
  prm.N = N;
  prm.K = K;
  prm.tiles_n = int32_t((N + kBN - 1) / kBN);
  prm.tiles = int32_t(((M + kBM - 1) / kBM) * prm.tiles_n);
  prm.bias = bias;
  prm.res = static_cast<const __nv_bfloat16 *>(residual);
  prm.ldr = ldr;
  prm.c = static_cast<__nv_bfloat16 *>(c);
  prm.ldc = ldc;
  prm.epi = epilogue;
  prm.wait = w;
  prm.drain_ns = 4000000000ull;
  const size_t smem = sizeof(Smem) + 1024;
  static PerDeviceOnce attr;
  static int n_sm_of[PerDeviceOnce::kMaxDevices];
  cudaError_t e = attr.run([&](int dev) {
    cudaError_t r =
        cudaFuncSetAttribute(gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
    if (r != cudaSuccess) return r;
    int n = 0;
    r = cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (r != cudaSuccess) return r;
    n_sm_of[dev] = n > 0 ? n : 1;
    return cudaSuccess;
  });
  if (e != cudaSuccess) return e;
  int dev = 0;
  e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const int n_sm = n_sm_of[dev];
  const unsigned grid = unsigned(std::min<int64_t>(prm.tiles, n_sm));
  gemm_kernel<<<grid, kThreads, smem, st>>>(ta, tb, prm);
  count_launch();
  return cudaGetLastError();
}

}  // namespace hstu
