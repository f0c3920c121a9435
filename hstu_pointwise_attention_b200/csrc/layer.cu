// layer.cu -- the HSTU layer around the attention: LayerNorm gating and the
// CUDA-core GEMM used for shapes the tensor-core GEMM does not take.
//
// DLRMv4 article, section "Model architecture: HSTU replaces the
// feature-interaction stack": a single projection produces the layer's
// internal representations and a gated transformation combines the
// attention-aggregated features, replacing the cross network and FFN.
// Library reading: [U|V|Q|K] = SiLU(x W1^T + b1); G = LayerNorm(A) (.) U;
// y = x + G W2^T + b2.
#include <algorithm>

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

// ---------------------------------------------------------------------------
// Backward of G = LayerNorm(A) (.) U (one warp per token, F <= 1024 features),
// from dG:
//   xhat = (A - mean) rstd,  ln = xhat gamma + beta
//   G = ln (.) U (written: the output projection's weight gradient reads it)
//   dU = dG (.) ln,  dln = dG (.) U,  dxh = dln (.) gamma
//   dA = rstd (dxh - mean(dxh) - xhat mean(dxh (.) xhat))
//   dgamma += sum_t dln (.) xhat,  dbeta += sum_t dln   (float32, accumulated)
// Warps walk tokens with a grid stride; each lane keeps its features' dgamma /
// dbeta sums in registers, the block adds its warps' sums in shared memory
// and then into the float32 outputs.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void load_bf16x8(const __nv_bfloat16 *p, float (&x)[8]) {
  const uint4 r = *reinterpret_cast<const uint4 *>(p);
  const uint32_t w[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    x[2 * e] = __uint_as_float(w[e] << 16);
    x[2 * e + 1] = __uint_as_float(w[e] & 0xFFFF0000u);
  }
}
__device__ __forceinline__ void store_bf16x8(__nv_bfloat16 *p, const float (&x)[8]) {
  *reinterpret_cast<uint4 *>(p) = make_uint4(pack_bf16x2(x[0], x[1]), pack_bf16x2(x[2], x[3]),
                                             pack_bf16x2(x[4], x[5]), pack_bf16x2(x[6], x[7]));
}

template <int F>
__global__ void __launch_bounds__(256) ln_gate_bwd_kernel(
    const __nv_bfloat16 *__restrict__ A, int64_t lda, const __nv_bfloat16 *__restrict__ U,
    int64_t ldu, const __nv_bfloat16 *__restrict__ dG, int64_t lddg,
    const float *__restrict__ gamma, const float *__restrict__ beta, float eps,
    __nv_bfloat16 *__restrict__ G, int64_t ldg, __nv_bfloat16 *__restrict__ dU, int64_t lddu,
    __nv_bfloat16 *__restrict__ dA, int64_t ldda, float *__restrict__ dgamma,
    float *__restrict__ dbeta, int64_t T) {
  static_assert(F % 256 == 0 || F < 256, "lane layout");
  constexpr int kVec = F >= 256 ? 8 : F / 32;   // features per lane per vector
  constexpr int kPer = F / 32;                  // features per lane
  constexpr int kNv = kPer / kVec;
  __shared__ float s_dg[F], s_db[F];
  for (int f = threadIdx.x; f < F; f += blockDim.x) {
    s_dg[f] = 0.f;
    s_db[f] = 0.f;
  }
  __syncthreads();
  const int lane = threadIdx.x & 31;
  float acc_g[kPer], acc_b[kPer];
#pragma unroll
  for (int e = 0; e < kPer; ++e) {
    acc_g[e] = 0.f;
    acc_b[e] = 0.f;
  }
  // gamma / beta are re-read per token (L1 hits) to keep registers for the row
  // Three passes over a token's row keep few values live: the statistics
  // from A; then, a vector of features at a time, G, dU and the gradient
  // sums (U and dG are read once, G and dU written at once); then dA.
  for (int64_t t = int64_t(blockIdx.x) * 8 + (threadIdx.x >> 5); t < T;
       t += int64_t(gridDim.x) * 8) {
    float a[kPer], dxh[kPer];
#pragma unroll
    for (int v = 0; v < kNv; ++v) {
      const int f0 = v * 32 * kVec + lane * kVec;
      if constexpr (kVec == 8) {
        float x8[8];
        load_bf16x8(A + t * lda + f0, x8);
#pragma unroll
        for (int e = 0; e < 8; ++e) a[v * 8 + e] = x8[e];
      } else {
#pragma unroll
        for (int e = 0; e < kVec; ++e) a[v * kVec + e] = __bfloat162float(A[t * lda + f0 + e]);
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
    float m1 = 0.f, m2 = 0.f;
#pragma unroll
    for (int v = 0; v < kNv; ++v) {
      const int f0 = v * 32 * kVec + lane * kVec;
      float u[kVec], dg[kVec], o_g[kVec], o_u[kVec];
      if constexpr (kVec == 8) {
        load_bf16x8(U + t * ldu + f0, u);
        load_bf16x8(dG + t * lddg + f0, dg);
      } else {
#pragma unroll
        for (int e = 0; e < kVec; ++e) {
          u[e] = __bfloat162float(U[t * ldu + f0 + e]);
          dg[e] = __bfloat162float(dG[t * lddg + f0 + e]);
        }
      }
#pragma unroll
      for (int e = 0; e < kVec; ++e) {
        const int x = v * kVec + e;
        const float xh = (a[x] - mean) * rstd;
        const float gme = __ldg(gamma + f0 + e);
        const float ln = fmaf(xh, gme, __ldg(beta + f0 + e));
        o_g[e] = ln * u[e];
        o_u[e] = dg[e] * ln;
        const float dln = dg[e] * u[e];
        acc_g[x] = fmaf(dln, xh, acc_g[x]);
        acc_b[x] += dln;
        dxh[x] = dln * gme;
        m1 += dxh[x];
        m2 = fmaf(dxh[x], xh, m2);
      }
      if constexpr (kVec == 8) {
        store_bf16x8(G + t * ldg + f0, o_g);
        store_bf16x8(dU + t * lddu + f0, o_u);
      } else {
#pragma unroll
        for (int e = 0; e < kVec; ++e) {
          G[t * ldg + f0 + e] = __float2bfloat16_rn(o_g[e]);
          dU[t * lddu + f0 + e] = __float2bfloat16_rn(o_u[e]);
        }
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      m1 += __shfl_xor_sync(0xffffffffu, m1, o);
      m2 += __shfl_xor_sync(0xffffffffu, m2, o);
    }
    m1 /= F;
    m2 /= F;
#pragma unroll
    for (int v = 0; v < kNv; ++v) {
      const int f0 = v * 32 * kVec + lane * kVec;
      float o_a[kVec];
#pragma unroll
      for (int e = 0; e < kVec; ++e) {
        const int x = v * kVec + e;
        o_a[e] = rstd * (dxh[x] - m1 - (a[x] - mean) * rstd * m2);
      }
      if constexpr (kVec == 8) {
        store_bf16x8(dA + t * ldda + f0, o_a);
      } else {
#pragma unroll
        for (int e = 0; e < kVec; ++e) dA[t * ldda + f0 + e] = __float2bfloat16_rn(o_a[e]);
      }
    }
  }
#pragma unroll
  for (int v = 0; v < kNv; ++v) {
#pragma unroll
    for (int e = 0; e < kVec; ++e) {
      const int f = v * 32 * kVec + lane * kVec + e;
      atomicAdd(&s_dg[f], acc_g[v * kVec + e]);
      atomicAdd(&s_db[f], acc_b[v * kVec + e]);
    }
  }
  __syncthreads();
  for (int f = threadIdx.x; f < F; f += blockDim.x) {
    atomicAdd(dgamma + f, s_dg[f]);
    atomicAdd(dbeta + f, s_db[f]);
  }
}

cudaError_t launch_ln_gate_bwd(const LnGateBwdArgs &a, cudaStream_t st) {
  if (a.T == 0) return cudaSuccess;
  const int64_t blocks = std::min<int64_t>((a.T + 7) / 8, 4 * 148);
  const dim3 grid(static_cast<unsigned>(blocks));
  const auto *A = static_cast<const __nv_bfloat16 *>(a.a);
  const auto *U = static_cast<const __nv_bfloat16 *>(a.u);
  const auto *dG = static_cast<const __nv_bfloat16 *>(a.dg);
  auto *G = static_cast<__nv_bfloat16 *>(a.g);
  auto *dU = static_cast<__nv_bfloat16 *>(a.du);
  auto *dA = static_cast<__nv_bfloat16 *>(a.da);
#define HSTU_LNB(F_)                                                                           \
  ln_gate_bwd_kernel<F_><<<grid, 256, 0, st>>>(A, a.lda, U, a.ldu, dG, a.lddg, a.gamma, a.beta, \
                                               a.eps, G, a.ldg, dU, a.lddu, dA, a.ldda,        \
                                               a.dgamma, a.dbeta, a.T)
  switch (a.F) {
    case 32: HSTU_LNB(32); break;
    case 64: HSTU_LNB(64); break;
    case 128: HSTU_LNB(128); break;
    case 256: HSTU_LNB(256); break;
    case 512: HSTU_LNB(512); break;
    case 1024: HSTU_LNB(1024); break;
    default: return cudaErrorInvalidValue;
  }
#undef HSTU_LNB
  count_launch();
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// Column sums over tokens, with the SiLU backward fused in (SILU_BWD):
//   SILU_BWD: X <- X (.) SiLU'(Z) in place, then colsum += sum_t X
//   else:     colsum += sum_t X
// SiLU'(z) = sigma(z) (1 + z (1 - sigma(z))); with t = tanh(z / 2),
// sigma = (1 + t) / 2 and sigma (1 - sigma) = (1 - t^2) / 4.
// Block: 32 column groups of 8 features (one 16-byte load each, a warp reads
// 512 contiguous bytes of a row) x 8 row lanes; rows with a grid stride.
// ---------------------------------------------------------------------------
template <bool SILU_BWD>
__global__ void __launch_bounds__(256) colsum_kernel(__nv_bfloat16 *__restrict__ X, int64_t ldx,
                                                     const __nv_bfloat16 *__restrict__ Z,
                                                     int64_t ldz, float *__restrict__ colsum,
                                                     int64_t T, int64_t N) {
  __shared__ float red[8][32 * 8 + 1];
  const int cx = threadIdx.x & 31, ry = threadIdx.x >> 5;
  const int64_t c0 = (int64_t(blockIdx.x) * 32 + cx) * 8;
  const bool col_ok = c0 < N;
  float acc[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) acc[e] = 0.f;
  if (col_ok) {
    for (int64_t t = int64_t(blockIdx.y) * 8 + ry; t < T; t += int64_t(gridDim.y) * 8) {
      float x[8];
      load_bf16x8(X + t * ldx + c0, x);
      if constexpr (SILU_BWD) {
        float z[8];
        load_bf16x8(Z + t * ldz + c0, z);
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const float th = tanh_approx(0.5f * z[e]);
          const float sg = 0.5f + 0.5f * th;
          const float d = fmaf(0.25f * z[e], fmaf(-th, th, 1.0f), sg);
          x[e] *= d;
        }
        float xr[8];
        // the sums take the bf16-rounded values that are stored
#pragma unroll
        for (int e = 0; e < 8; ++e) xr[e] = __bfloat162float(__float2bfloat16_rn(x[e]));
        store_bf16x8(X + t * ldx + c0, x);
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[e] += xr[e];
      } else {
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[e] += x[e];
      }
    }
  }
#pragma unroll
  for (int e = 0; e < 8; ++e) red[ry][cx * 8 + e] = acc[e];
  __syncthreads();
  if (ry == 0 && col_ok) {
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      float sum = 0.f;
#pragma unroll
      for (int r = 0; r < 8; ++r) sum += red[r][cx * 8 + e];
      if (c0 + e < N) atomicAdd(colsum + c0 + e, sum);
    }
  }
}

cudaError_t launch_colsum(void *x, int64_t ldx, const void *z, int64_t ldz, float *colsum,
                          int64_t T, int64_t N, bool silu_bwd, cudaStream_t st) {
  if (T == 0 || N == 0) return cudaSuccess;
  if ((N % 8) || (ldx % 8) || (silu_bwd && (ldz % 8))) return cudaErrorInvalidValue;
  const int64_t slabs = (N / 8 + 31) / 32;
  const int64_t rows = std::max<int64_t>(1, std::min<int64_t>((T + 7) / 8, (4 * 148 + slabs - 1) / slabs));
  const dim3 grid(static_cast<unsigned>(slabs), static_cast<unsigned>(rows));
  auto *X = static_cast<__nv_bfloat16 *>(x);
  const auto *Z = static_cast<const __nv_bfloat16 *>(z);
  if (silu_bwd)
    colsum_kernel<true><<<grid, 256, 0, st>>>(X, ldx, Z, ldz, colsum, T, N);
  else
    colsum_kernel<false><<<grid, 256, 0, st>>>(X, ldx, Z, ldz, colsum, T, N);
  count_launch();
  return cudaGetLastError();
}

}  // namespace hstu
