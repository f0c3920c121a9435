// layer.cu -- the HSTU layer around the attention: LayerNorm gating and the
// CUDA-core GEMM used for shapes the tensor-core GEMM does not take.
//
// DLRMv4 article, section "Model architecture: HSTU replaces the
// feature-interaction stack": a single projection produces the layer's
// internal representations and a gated transformation combines the
// attention-aggregated features, replacing the cross network and FFN.
// Library reading: [U|V|Q|K] = SiLU(x W1^T + b1); G = LayerNorm(A) (.) U;
// y = x + G W2^T + b2.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "internal.h"

namespace hstu {

// ---------------------------------------------------------------------------
// C[M,N] = epilogue(A[M,K] B[N,K]^T), bf16 in/out, fp32 accumulation.
// 64x64 tile per block, 256 threads, 4x4 outputs per thread.
// ---------------------------------------------------------------------------
constexpr int kGT = 64;
constexpr int kGK = 32;

__global__ void __launch_bounds__(256) gemm_simt_kernel(
    const __nv_bfloat16 *__restrict__ A, int64_t lda, const __nv_bfloat16 *__restrict__ B,
    int64_t ldb, const float *__restrict__ bias, const __nv_bfloat16 *__restrict__ R,
    int64_t ldr, __nv_bfloat16 *__restrict__ C, int64_t ldc, int64_t M, int64_t N, int64_t K,
    int epi) {
  __shared__ float sa[kGK][kGT + 1];
  __shared__ float sb[kGK][kGT + 1];
  const int64_t m0 = int64_t(blockIdx.y) * kGT, n0 = int64_t(blockIdx.x) * kGT;
  const int tx = threadIdx.x % 16, ty = threadIdx.x / 16;
  float acc[4][4] = {};
  for (int64_t k0 = 0; k0 < K; k0 += kGK) {
    for (int x = threadIdx.x; x < kGT * kGK; x += 256) {
      const int r = x / kGK, c = x % kGK;
      const int64_t gm = m0 + r, gn = n0 + r, gk = k0 + c;
      sa[c][r] = (gm < M && gk < K) ? __bfloat162float(A[gm * lda + gk]) : 0.f;
      sb[c][r] = (gn < N && gk < K) ? __bfloat162float(B[gn * ldb + gk]) : 0.f;
    }
    __syncthreads();
#pragma unroll 8
    for (int c = 0; c < kGK; ++c) {
      float a[4], b[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        a[u] = sa[c][ty * 4 + u];
        b[u] = sb[c][tx * 4 + u];
      }
#pragma unroll
      for (int u = 0; u < 4; ++u)
#pragma unroll
        for (int w = 0; w < 4; ++w) acc[u][w] = fmaf(a[u], b[w], acc[u][w]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const int64_t gm = m0 + ty * 4 + u;
    if (gm >= M) continue;
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      const int64_t gn = n0 + tx * 4 + w;
      if (gn >= N) continue;
      float y = acc[u][w] + (bias ? bias[gn] : 0.f);
      if (epi == kEpiBiasSilu) y = y / (1.0f + __expf(-y));
      if (epi == kEpiBiasResidual) y += __bfloat162float(R[gm * ldr + gn]);
      C[gm * ldc + gn] = __float2bfloat16_rn(y);
    }
  }
}

cudaError_t launch_gemm_simt(const void *a, int64_t lda, const void *b, int64_t ldb,
                             const float *bias, const void *residual, int64_t ldr, void *c,
                             int64_t ldc, int64_t M, int64_t N, int64_t K, int epilogue,
                             cudaStream_t st) {
  if (M == 0 || N == 0) return cudaSuccess;
  const dim3 grid(unsigned((N + kGT - 1) / kGT), unsigned((M + kGT - 1) / kGT));
  gemm_simt_kernel<<<grid, 256, 0, st>>>(
      static_cast<const __nv_bfloat16 *>(a), lda, static_cast<const __nv_bfloat16 *>(b), ldb,
      bias, static_cast<const __nv_bfloat16 *>(residual), ldr, static_cast<__nv_bfloat16 *>(c),
      ldc, M, N, K, epilogue);
  count_launch();
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// G = LayerNorm(A) * gamma + beta, then (.) U.  One warp per token, F <= 1024
// features; float32 statistics (mean, biased variance), 16-byte loads.
// ---------------------------------------------------------------------------
template <int F, bool VEC_P>
__global__ void __launch_bounds__(256) ln_gate_kernel(
    const __nv_bfloat16 *__restrict__ A, int64_t lda, const __nv_bfloat16 *__restrict__ U,
    int64_t ldu, const float *__restrict__ gamma, const float *__restrict__ beta, float eps,
    __nv_bfloat16 *__restrict__ G, int64_t ldg, int64_t T) {
  constexpr int kPer = F / 32;          // features per lane
  constexpr int kVec = kPer >= 8 ? 8 : kPer;
  const int64_t t = int64_t(blockIdx.x) * 8 + threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  if (t >= T) return;
  float a[kPer], u[kPer];
  const __nv_bfloat16 *ar = A + t * lda;
  const __nv_bfloat16 *ur = U + t * ldu;
  // lane owns features [v*32*kVec + lane*kVec, +kVec) for v = 0 .. kPer/kVec-1
#pragma unroll
  for (int v = 0; v < kPer / kVec; ++v) {
    const int f0 = v * 32 * kVec + lane * kVec;
    if constexpr (kVec == 8) {
      const uint4 ra = *reinterpret_cast<const uint4 *>(ar + f0);
      const uint4 ru = *reinterpret_cast<const uint4 *>(ur + f0);
      const __nv_bfloat16 *pa = reinterpret_cast<const __nv_bfloat16 *>(&ra);
      const __nv_bfloat16 *pu = reinterpret_cast<const __nv_bfloat16 *>(&ru);
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        a[v * kVec + e] = __bfloat162float(pa[e]);
        u[v * kVec + e] = __bfloat162float(pu[e]);
      }
    } else {
#pragma unroll
      for (int e = 0; e < kVec; ++e) {
        a[v * kVec + e] = __bfloat162float(ar[f0 + e]);
        u[v * kVec + e] = __bfloat162float(ur[f0 + e]);
      }
    }
  }
  float s = 0.f;
#pragma unroll
  for (int e = 0; e < kPer; ++e) s += a[e];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  const float mean = s / F;
  float q = 0.f;
#pragma unroll
  for (int e = 0; e < kPer; ++e) {
    const float d = a[e] - mean;
    q = fmaf(d, d, q);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) q += __shfl_xor_sync(0xffffffffu, q, o);
  const float rstd = rsqrtf(q / F + eps);
  __nv_bfloat16 *gr = G + t * ldg;
#pragma unroll
  for (int v = 0; v < kPer / kVec; ++v) {
    const int f0 = v * 32 * kVec + lane * kVec;
    __align__(16) __nv_bfloat16 out[kVec];
    float gm[kVec], bt[kVec];
    if constexpr (VEC_P && kVec == 8) {
      // 16-byte aligned gamma / beta: two float4 loads each for the lane's 8 features
      const float4 *g4 = reinterpret_cast<const float4 *>(gamma + f0);
      const float4 *b4 = reinterpret_cast<const float4 *>(beta + f0);
#pragma unroll
      for (int h2 = 0; h2 < 2; ++h2) {
        const float4 gv = __ldg(g4 + h2), bv = __ldg(b4 + h2);
        gm[4 * h2] = gv.x, gm[4 * h2 + 1] = gv.y, gm[4 * h2 + 2] = gv.z, gm[4 * h2 + 3] = gv.w;
        bt[4 * h2] = bv.x, bt[4 * h2 + 1] = bv.y, bt[4 * h2 + 2] = bv.z, bt[4 * h2 + 3] = bv.w;
      }
    } else {
#pragma unroll
      for (int e = 0; e < kVec; ++e) {
        gm[e] = gamma[f0 + e];
        bt[e] = beta[f0 + e];
      }
    }
#pragma unroll
    for (int e = 0; e < kVec; ++e) {
      const float y = fmaf((a[v * kVec + e] - mean) * rstd, gm[e], bt[e]);
      out[e] = __float2bfloat16_rn(y * u[v * kVec + e]);
    }
    if constexpr (kVec == 8) {
      *reinterpret_cast<uint4 *>(gr + f0) = *reinterpret_cast<const uint4 *>(out);
    } else {
#pragma unroll
      for (int e = 0; e < kVec; ++e) gr[f0 + e] = out[e];
    }
  }
}

cudaError_t launch_ln_gate(const void *a, int64_t lda, const void *u, int64_t ldu,
                           const float *gamma, const float *beta, float eps, void *g,
                           int64_t ldg, int64_t T, int32_t F, cudaStream_t st) {
  if (T == 0) return cudaSuccess;
  const dim3 grid(unsigned((T + 7) / 8));
  const auto *A = static_cast<const __nv_bfloat16 *>(a);
  const auto *U = static_cast<const __nv_bfloat16 *>(u);
  auto *G = static_cast<__nv_bfloat16 *>(g);
  const bool vec = ((reinterpret_cast<uintptr_t>(gamma) | reinterpret_cast<uintptr_t>(beta)) & 15) == 0;
  switch (F) {
    case 32:
      if (vec)
        ln_gate_kernel<32, true><<<grid, 256, 0, st>>>(A, lda, U, ldu, gamma, beta, eps, G, ldg, T);
      else
        ln_gate_kernel<32, false><<<grid, 256, 0, st>>>(A, lda, U, ldu, gamma, beta, eps, G, ldg, T);
      break;
    case 64:
      if (vec)
        ln_gate_kernel<64, true><<<grid, 256, 0, st>>>(A, lda, U, ldu, gamma, beta, eps, G, ldg, T);
      else
        ln_gate_kernel<64, false><<<grid, 256, 0, st>>>(A, lda, U, ldu, gamma, beta, eps, G, ldg, T);
      break;
    case 128:
      if (vec)
        ln_gate_kernel<128, true><<<grid, 256, 0, st>>>(A, lda, U, ldu, gamma, beta, eps, G, ldg, T);
      else
        ln_gate_kernel<128, false><<<grid, 256, 0, st>>>(A, lda, U, ldu, gamma, beta, eps, G, ldg, T);
      break;
    case 256:
      if (vec)
        ln_gate_kernel<256, true><<<grid, 256, 0, st>>>(A, lda, U, ldu, gamma, beta, eps, G, ldg, T);
      else
        ln_gate_kernel<256, false><<<grid, 256, 0, st>>>(A, lda, U, ldu, gamma, beta, eps, G, ldg, T);
      break;
    case 512:
      if (vec)
        ln_gate_kernel<512, true><<<grid, 256, 0, st>>>(A, lda, U, ldu, gamma, beta, eps, G, ldg, T);
      else
        ln_gate_kernel<512, false><<<grid, 256, 0, st>>>(A, lda, U, ldu, gamma, beta, eps, G, ldg, T);
      break;
    case 1024:
      if (vec)
        ln_gate_kernel<1024, true><<<grid, 256, 0, st>>>(A, lda, U, ldu, gamma, beta, eps, G, ldg, T);
      else
        ln_gate_kernel<1024, false><<<grid, 256, 0, st>>>(A, lda, U, ldu, gamma, beta, eps, G, ldg, T);
      break;
    default: return cudaErrorInvalidValue;
  }
  count_launch();
  return cudaGetLastError();
}

}  // namespace hstu
