// attn_simt.cu -- CUDA-core kernels of HSTU pointwise attention.
//
// These serve float32 problems, head sizes the tensor-core kernels do not
// take, and the bucket debug entry point.  One thread owns one query row
// (forward, dQ) or one key column (dK, dV, d rab); keys / queries are staged
// through shared memory in chunks.  Arithmetic per visible pair follows the
// definition in include/hstu.h (DLRMv4 article, section "Model architecture:
// HSTU replaces the feature-interaction stack"; readings of the library).
#include <algorithm>
#include <climits>

#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "internal.h"
#include "tile_common.cuh"

namespace hstu {

template <typename T>
__device__ __forceinline__ float ld_elem(const T *p);
template <>
__device__ __forceinline__ float ld_elem<float>(const float *p) { return *p; }
template <>
__device__ __forceinline__ float ld_elem<__nv_bfloat16>(const __nv_bfloat16 *p) {
  return __bfloat162float(*p);
}
template <typename T>
__device__ __forceinline__ void st_elem(T *p, float v);
template <>
__device__ __forceinline__ void st_elem<float>(float *p, float v) { *p = v; }
template <>
__device__ __forceinline__ void st_elem<__nv_bfloat16>(__nv_bfloat16 *p, float v) {
  *p = __float2bfloat16_rn(v);
}

__device__ __forceinline__ bool is_visible(int32_t i, int32_t j, int32_t nh) {
  return i < nh ? (j <= i) : (j < nh || j == i);
}
__device__ __forceinline__ int32_t position_of(int32_t i, int32_t nh) { return i < nh ? i : nh; }

// ---------------------------------------------------------------------------
// Prep: per-sequence timestamp span and float relative timestamps.
// ---------------------------------------------------------------------------
// One block per sequence (kPrepThreads threads): the span and order are
// found in one pass (each token is compared with its predecessor), then the
// float times written in a second; loops are unrolled so each thread keeps
// several loads in flight.
constexpr int kPrepThreads = 1024;

__device__ __forceinline__ void block_min_max_or(long long &lo, long long &hi, int &flag) {
  __shared__ long long smin[32], smax[32];
  __shared__ int sflag[32];
  for (int o = 16; o > 0; o >>= 1) {
    const long long a = __shfl_xor_sync(0xffffffffu, lo, o);
    const long long b = __shfl_xor_sync(0xffffffffu, hi, o);
    lo = a < lo ? a : lo;
    hi = b > hi ? b : hi;
    flag |= __shfl_xor_sync(0xffffffffu, flag, o);
  }
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
  if (l == 0) {
    smin[w] = lo;
    smax[w] = hi;
    sflag[w] = flag;
  }
  __syncthreads();
  if (w == 0) {
    const int nw = int(blockDim.x >> 5);
    lo = l < nw ? smin[l] : LLONG_MAX;
    hi = l < nw ? smax[l] : LLONG_MIN;
    flag = l < nw ? sflag[l] : 0;
    for (int o = 16; o > 0; o >>= 1) {
      const long long a = __shfl_xor_sync(0xffffffffu, lo, o);
      const long long b = __shfl_xor_sync(0xffffffffu, hi, o);
      lo = a < lo ? a : lo;
      hi = b > hi ? b : hi;
      flag |= __shfl_xor_sync(0xffffffffu, flag, o);
    }
    if (l == 0) {
      smin[0] = lo;
      smax[0] = hi;
      sflag[0] = flag;
    }
  }
  __syncthreads();
  lo = smin[0];
  hi = smax[0];
  flag = sflag[0];
}

__global__ void __launch_bounds__(kPrepThreads) prep_kernel(const int64_t *ts, const SeqInfo *seqs,
                                                             float *tf, int32_t *seq_fast) {
  const SeqInfo sq = seqs[blockIdx.x];
  const int64_t *t = ts + sq.start;
  long long lo = LLONG_MAX, hi = LLONG_MIN;
  int unsorted = 0;
#pragma unroll 4
  for (int32_t i = threadIdx.x; i < sq.len; i += blockDim.x) {
    const long long v = t[i];
    lo = v < lo ? v : lo;
    hi = v > hi ? v : hi;
    // Non-decreasing timestamps (flag kSeqSorted) let the backward bin its
    // time-bias gradient by runs, since buckets are then monotone along a row.
    if (i > 0) unsorted |= v < t[i - 1];
  }
  block_min_max_or(lo, hi, unsorted);
  // Differences computed in unsigned arithmetic so extreme timestamps cannot overflow.
  const bool fast = sq.len > 0 && (unsigned long long)(hi - lo) < (1ull << 24);
  if (threadIdx.x == 0)
    seq_fast[blockIdx.x] = (fast ? kSeqFastTime : 0) | (unsorted ? 0 : kSeqSorted);
#pragma unroll 4
  for (int32_t i = threadIdx.x; i < sq.len; i += blockDim.x)
    tf[sq.start + i] = fast ? float(t[i] - lo) : 0.0f;
}

cudaError_t launch_prep(const AttnProblem &p, const Scratch &s, cudaStream_t st) {
  if (p.batch == 0) return cudaSuccess;
  prep_kernel<<<p.batch, kPrepThreads, 0, st>>>(p.ts, s.seqs, s.tf, s.seq_fast);
  count_launch();
  return cudaGetLastError();
}

// Split work items add float32 partial sums; this turns the rows they cover
// into the scaled bf16 output.  Block y takes row range y; 4 features per
// thread (one 16-byte load, one 8-byte store).
__global__ void __launch_bounds__(256) rows_to_bf16_kernel(const float *src, __nv_bfloat16 *dst,
                                                           int64_t dst_rs, int32_t HD,
                                                           const int4 *rows, float scale) {
  const int4 rr = rows[blockIdx.y];
  const int32_t per_row = HD / 4;
  const int64_t n = int64_t(rr.y) * per_row;
  for (int64_t x = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; x < n;
       x += int64_t(gridDim.x) * blockDim.x) {
    const int64_t i = x / per_row;
    const int32_t c = int32_t(x % per_row) * 4;
    const float4 v = *reinterpret_cast<const float4 *>(src + (rr.z + i) * HD + c);
    *reinterpret_cast<uint2 *>(dst + (rr.x + i) * dst_rs + c) =
        make_uint2(pack_bf16x2(v.x * scale, v.y * scale), pack_bf16x2(v.z * scale, v.w * scale));
  }
}

cudaError_t launch_rows_to_bf16(const float *src, void *dst, int64_t dst_rs, int32_t H,
                                int32_t D, const int4 *rows, int32_t n, float scale,
                                cudaStream_t st) {
  if (n == 0) return cudaSuccess;
  const int32_t HD = H * D;
  if ((HD % 4) || (dst_rs % 4) || (reinterpret_cast<uintptr_t>(dst) & 7) ||
      (reinterpret_cast<uintptr_t>(src) & 15))
    return cudaErrorInvalidValue;
  const unsigned bx = unsigned(std::min<int64_t>(64, (int64_t(256) * HD / 4 + 255) / 256));
  rows_to_bf16_kernel<<<dim3(bx, unsigned(n)), 256, 0, st>>>(
      src, static_cast<__nv_bfloat16 *>(dst), dst_rs, HD, rows, scale);
  count_launch();
  return cudaGetLastError();
}

// Cached-history prep: sequence b's cached history (ts_h, tokens [start,
// start + n_h)) and its candidates in this call (ts_c, rows [cstart, cstart +
// n_c)); the span and float times cover both, the order flag the history
// (the keys; buckets are then monotone along every candidate's row).
__global__ void __launch_bounds__(kPrepThreads) prep_cached_kernel(
    const int64_t *ts_h, const int64_t *ts_c, const SeqInfo *seqs, const int64_t *cstart,
    float *tf, float *tfc, int32_t *seq_fast) {
  const SeqInfo sq = seqs[blockIdx.x];
  const int32_t n_h = sq.n_hist, n_c = sq.len - sq.n_hist;
  const int64_t cs = cstart[blockIdx.x];
  const int64_t *th = ts_h + sq.start;
  const int64_t *tc = ts_c + cs;
  long long lo = LLONG_MAX, hi = LLONG_MIN;
  int unsorted = 0;
#pragma unroll 4
  for (int32_t i = threadIdx.x; i < n_h + n_c; i += blockDim.x) {
    const long long v = i < n_h ? th[i] : tc[i - n_h];
    lo = v < lo ? v : lo;
    hi = v > hi ? v : hi;
    if (i > 0 && i < n_h) unsorted |= v < th[i - 1];
  }
  block_min_max_or(lo, hi, unsorted);
  const bool fast = n_h + n_c > 0 && (unsigned long long)(hi - lo) < (1ull << 24);
  if (threadIdx.x == 0)
    seq_fast[blockIdx.x] = (fast ? kSeqFastTime : 0) | (unsorted ? 0 : kSeqSorted);
#pragma unroll 4
  for (int32_t i = threadIdx.x; i < n_h; i += blockDim.x)
    tf[sq.start + i] = fast ? float(th[i] - lo) : 0.0f;
  for (int32_t i = threadIdx.x; i < n_c; i += blockDim.x)
    tfc[cs + i] = fast ? float(tc[i] - lo) : 0.0f;
}

cudaError_t launch_prep_cached(const AttnProblem &p, const Scratch &s, const CachedHist &ch,
                               float *tfc, cudaStream_t st) {
  if (p.batch == 0) return cudaSuccess;
  prep_cached_kernel<<<p.batch, kPrepThreads, 0, st>>>(p.ts, ch.ts_cand, s.seqs, ch.cstart, s.tf, tfc,
                                              s.seq_fast);
  count_launch();
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// Forward: one thread per query row, 64 rows per block, keys in chunks of 32.
// ---------------------------------------------------------------------------
constexpr int kSimtRows = 64;
constexpr int kSimtKeys = 32;

template <typename T, int DQ, int DV>
__global__ void __launch_bounds__(kSimtRows) fwd_simt_kernel(AttnProblem p, Scratch s, T *out) {
  extern __shared__ float sm[];
  float *sk = sm;                         // [kSimtKeys][d_qk]
  float *sv = sk + kSimtKeys * p.d_qk;    // [kSimtKeys][d_v]
  const int2 item = s.simt_items[blockIdx.x];
  const int32_t h = blockIdx.y;
  const SeqInfo sq = s.seqs[item.x];
  const int32_t i = item.y * kSimtRows + threadIdx.x;
  const bool row_ok = i < sq.len;
  const T *q = static_cast<const T *>(p.q);
  const T *k = static_cast<const T *>(p.k);
  const T *v = static_cast<const T *>(p.v);
  const float *rp = p.rab_p + (p.rab_per_head ? h * p.nb_p : 0);
  const float *rt = p.rab_t + (p.rab_per_head ? h * p.nb_t : 0);
  float qr[DQ], acc[DV];
#pragma unroll
  for (int c = 0; c < DQ; ++c)
    qr[c] = (row_ok && c < p.d_qk) ? ld_elem(q + (sq.start + i) * p.q_rs + h * p.d_qk + c) : 0.f;
#pragma unroll
  for (int c = 0; c < DV; ++c) acc[c] = 0.f;
  const int64_t ti = row_ok ? p.ts[sq.start + i] : 0;
  const int32_t pi = position_of(i, sq.n_hist);
  const int32_t last_row = min(sq.len - 1, item.y * kSimtRows + kSimtRows - 1);
  for (int32_t k0 = 0; k0 <= last_row; k0 += kSimtKeys) {
    __syncthreads();
    for (int32_t x = threadIdx.x; x < kSimtKeys * p.d_qk; x += blockDim.x) {
      const int32_t j = k0 + x / p.d_qk, c = x % p.d_qk;
      sk[x] = j < sq.len ? ld_elem(k + (sq.start + j) * p.k_rs + h * p.d_qk + c) : 0.f;
    }
    for (int32_t x = threadIdx.x; x < kSimtKeys * p.d_v; x += blockDim.x) {
      const int32_t j = k0 + x / p.d_v, c = x % p.d_v;
      sv[x] = j < sq.len ? ld_elem(v + (sq.start + j) * p.v_rs + h * p.d_v + c) : 0.f;
    }
    __syncthreads();
    if (!row_ok) continue;
    for (int32_t jj = 0; jj < kSimtKeys; ++jj) {
      const int32_t j = k0 + jj;
      if (j >= sq.len || !is_visible(i, j, sq.n_hist)) continue;
      float dot = 0.f;
#pragma unroll
      for (int c = 0; c < DQ; ++c)
        if (c < p.d_qk) dot = fmaf(qr[c], sk[jj * p.d_qk + c], dot);
      const int32_t bp = pos_bucket(pi - position_of(j, sq.n_hist), p.nb_p);
      const int32_t bt = time_bucket_i64(ti - p.ts[sq.start + j], p.sub_bits, p.nb_t);
      const float sc = fmaf(p.alpha, dot, rp[bp] + rt[bt]);
      const float a = p.silu_scale * (sc / (1.0f + expf(-sc)));
#pragma unroll
      for (int c = 0; c < DV; ++c)
        if (c < p.d_v) acc[c] = fmaf(a, sv[jj * p.d_v + c], acc[c]);
    }
  }
  if (!row_ok) return;
  T *o = out + (sq.start + i) * p.o_rs + h * p.d_v;
#pragma unroll
  for (int c = 0; c < DV; ++c)
    if (c < p.d_v) st_elem(o + c, acc[c]);
}

template <typename T>
static cudaError_t fwd_simt_dispatch(const AttnProblem &p, const Scratch &s, void *out,
                                     cudaStream_t st) {
  const dim3 grid(s.n_simt_items, p.num_heads);
  const size_t smem = sizeof(float) * kSimtKeys * (p.d_qk + p.d_v);
  const int dmax = p.d_qk > p.d_v ? p.d_qk : p.d_v;
  T *o = static_cast<T *>(out);
  if (dmax <= 32)
    fwd_simt_kernel<T, 32, 32><<<grid, kSimtRows, smem, st>>>(p, s, o);
  else if (dmax <= 64)
    fwd_simt_kernel<T, 64, 64><<<grid, kSimtRows, smem, st>>>(p, s, o);
  else if (dmax <= 128)
    fwd_simt_kernel<T, 128, 128><<<grid, kSimtRows, smem, st>>>(p, s, o);
  else
    fwd_simt_kernel<T, 256, 256><<<grid, kSimtRows, smem, st>>>(p, s, o);
  count_launch();
  return cudaGetLastError();
}

cudaError_t launch_fwd_simt(const AttnProblem &p, const Scratch &s, void *out, cudaStream_t st) {
  if (s.n_simt_items == 0) return cudaSuccess;
  return p.dtype == 0 ? fwd_simt_dispatch<float>(p, s, out, st)
                      : fwd_simt_dispatch<__nv_bfloat16>(p, s, out, st);
}

// ---------------------------------------------------------------------------
// Backward, CUDA cores.
//   dq kernel:   one thread per query row i: dq_i = alpha sum_j dS_ij k_j.
//   dkdv kernel: one thread per key j: dk_j = alpha sum_i dS_ij q_i,
//                dv_j = silu_scale sum_i SiLU(s_ij) dout_i, d rab histograms.
// ---------------------------------------------------------------------------
template <typename T, int DQ, int DV>
__global__ void __launch_bounds__(kSimtRows) dq_simt_kernel(AttnProblem p, Scratch s,
                                                            const T *dout, T *dq) {
  extern __shared__ float sm[];
  float *sk = sm;
  float *sv = sk + kSimtKeys * p.d_qk;
  const int2 item = s.simt_items[blockIdx.x];
  const int32_t h = blockIdx.y;
  const SeqInfo sq = s.seqs[item.x];
  const int32_t i = item.y * kSimtRows + threadIdx.x;
  const bool row_ok = i < sq.len;
  const T *q = static_cast<const T *>(p.q);
  const T *k = static_cast<const T *>(p.k);
  const T *v = static_cast<const T *>(p.v);
  const float *rp = p.rab_p + (p.rab_per_head ? h * p.nb_p : 0);
  const float *rt = p.rab_t + (p.rab_per_head ? h * p.nb_t : 0);
  float qr[DQ], dor[DV], acc[DQ];
#pragma unroll
  for (int c = 0; c < DQ; ++c) {
    qr[c] = (row_ok && c < p.d_qk) ? ld_elem(q + (sq.start + i) * p.q_rs + h * p.d_qk + c) : 0.f;
    acc[c] = 0.f;
  }
#pragma unroll
  for (int c = 0; c < DV; ++c)
    dor[c] = (row_ok && c < p.d_v) ? ld_elem(dout + (sq.start + i) * p.do_rs + h * p.d_v + c)
                                   : 0.f;
  const int64_t ti = row_ok ? p.ts[sq.start + i] : 0;
  const int32_t pi = position_of(i, sq.n_hist);
  const int32_t last_row = min(sq.len - 1, item.y * kSimtRows + kSimtRows - 1);
  for (int32_t k0 = 0; k0 <= last_row; k0 += kSimtKeys) {
    __syncthreads();
    for (int32_t x = threadIdx.x; x < kSimtKeys * p.d_qk; x += blockDim.x) {
      const int32_t j = k0 + x / p.d_qk, c = x % p.d_qk;
      sk[x] = j < sq.len ? ld_elem(k + (sq.start + j) * p.k_rs + h * p.d_qk + c) : 0.f;
    }
    for (int32_t x = threadIdx.x; x < kSimtKeys * p.d_v; x += blockDim.x) {
      const int32_t j = k0 + x / p.d_v, c = x % p.d_v;
      sv[x] = j < sq.len ? ld_elem(v + (sq.start + j) * p.v_rs + h * p.d_v + c) : 0.f;
    }
    __syncthreads();
    if (!row_ok) continue;
    for (int32_t jj = 0; jj < kSimtKeys; ++jj) {
      const int32_t j = k0 + jj;
      if (j >= sq.len || !is_visible(i, j, sq.n_hist)) continue;
      float dot = 0.f, da = 0.f;
#pragma unroll
      for (int c = 0; c < DQ; ++c)
        if (c < p.d_qk) dot = fmaf(qr[c], sk[jj * p.d_qk + c], dot);
#pragma unroll
      for (int c = 0; c < DV; ++c)
        if (c < p.d_v) da = fmaf(dor[c], sv[jj * p.d_v + c], da);
      const int32_t bp = pos_bucket(pi - position_of(j, sq.n_hist), p.nb_p);
      const int32_t bt = time_bucket_i64(ti - p.ts[sq.start + j], p.sub_bits, p.nb_t);
      const float sc = fmaf(p.alpha, dot, rp[bp] + rt[bt]);
      const float sg = 1.0f / (1.0f + expf(-sc));
      const float ds = da * p.silu_scale * sg * (1.0f + sc * (1.0f - sg));
#pragma unroll
      for (int c = 0; c < DQ; ++c)
        if (c < p.d_qk) acc[c] = fmaf(p.alpha * ds, sk[jj * p.d_qk + c], acc[c]);
    }
  }
  if (!row_ok) return;
  T *o = dq + (sq.start + i) * p.dq_rs + h * p.d_qk;
#pragma unroll
  for (int c = 0; c < DQ; ++c)
    if (c < p.d_qk) st_elem(o + c, acc[c]);
}

template <typename T, int DQ, int DV>
__global__ void __launch_bounds__(kSimtRows) dkdv_simt_kernel(AttnProblem p, Scratch s,
                                                              const T *dout, T *dk, T *dv,
                                                              float *drab_p, float *drab_t) {
  extern __shared__ float sm[];
  float *sq_ = sm;                          // [kSimtKeys][d_qk] query chunk
  float *sdo = sq_ + kSimtKeys * p.d_qk;    // [kSimtKeys][d_v] dout chunk
  float *hp = sdo + kSimtKeys * p.d_v;      // [nb_p] d rab_p histogram
  float *ht = hp + p.nb_p;                  // [nb_t]
  const int2 item = s.simt_items[blockIdx.x];
  const int32_t h = blockIdx.y;
  const SeqInfo sq = s.seqs[item.x];
  const int32_t j = item.y * kSimtRows + threadIdx.x;
  const bool col_ok = j < sq.len;
  const T *q = static_cast<const T *>(p.q);
  const T *k = static_cast<const T *>(p.k);
  const T *v = static_cast<const T *>(p.v);
  const float *rp = p.rab_p + (p.rab_per_head ? h * p.nb_p : 0);
  const float *rt = p.rab_t + (p.rab_per_head ? h * p.nb_t : 0);
  for (int32_t x = threadIdx.x; x < p.nb_p; x += blockDim.x) hp[x] = 0.f;
  for (int32_t x = threadIdx.x; x < p.nb_t; x += blockDim.x) ht[x] = 0.f;
  float kr[DQ], vr[DV], adk[DQ], adv[DV];
#pragma unroll
  for (int c = 0; c < DQ; ++c) {
    kr[c] = (col_ok && c < p.d_qk) ? ld_elem(k + (sq.start + j) * p.k_rs + h * p.d_qk + c) : 0.f;
    adk[c] = 0.f;
  }
#pragma unroll
  for (int c = 0; c < DV; ++c) {
    vr[c] = (col_ok && c < p.d_v) ? ld_elem(v + (sq.start + j) * p.v_rs + h * p.d_v + c) : 0.f;
    adv[c] = 0.f;
  }
  const int64_t tj = col_ok ? p.ts[sq.start + j] : 0;
  const int32_t pj = position_of(j, sq.n_hist);
  const int32_t first = item.y * kSimtRows;
  for (int32_t i0 = first - first % kSimtKeys; i0 < sq.len; i0 += kSimtKeys) {
    __syncthreads();
    for (int32_t x = threadIdx.x; x < kSimtKeys * p.d_qk; x += blockDim.x) {
      const int32_t i = i0 + x / p.d_qk, c = x % p.d_qk;
      sq_[x] = i < sq.len ? ld_elem(q + (sq.start + i) * p.q_rs + h * p.d_qk + c) : 0.f;
    }
    for (int32_t x = threadIdx.x; x < kSimtKeys * p.d_v; x += blockDim.x) {
      const int32_t i = i0 + x / p.d_v, c = x % p.d_v;
      sdo[x] = i < sq.len ? ld_elem(dout + (sq.start + i) * p.do_rs + h * p.d_v + c) : 0.f;
    }
    __syncthreads();
    if (!col_ok) continue;
    for (int32_t ii = 0; ii < kSimtKeys; ++ii) {
      const int32_t i = i0 + ii;
      if (i >= sq.len || !is_visible(i, j, sq.n_hist)) continue;
      float dot = 0.f, da = 0.f;
#pragma unroll
      for (int c = 0; c < DQ; ++c)
        if (c < p.d_qk) dot = fmaf(sq_[ii * p.d_qk + c], kr[c], dot);
#pragma unroll
      for (int c = 0; c < DV; ++c)
        if (c < p.d_v) da = fmaf(sdo[ii * p.d_v + c], vr[c], da);
      const int32_t bp = pos_bucket(position_of(i, sq.n_hist) - pj, p.nb_p);
      const int32_t bt = time_bucket_i64(p.ts[sq.start + i] - tj, p.sub_bits, p.nb_t);
      const float sc = fmaf(p.alpha, dot, rp[bp] + rt[bt]);
      const float sg = 1.0f / (1.0f + expf(-sc));
      const float a = p.silu_scale * sc * sg;
      const float ds = da * p.silu_scale * sg * (1.0f + sc * (1.0f - sg));
#pragma unroll
      for (int c = 0; c < DQ; ++c)
        if (c < p.d_qk) adk[c] = fmaf(p.alpha * ds, sq_[ii * p.d_qk + c], adk[c]);
#pragma unroll
      for (int c = 0; c < DV; ++c)
        if (c < p.d_v) adv[c] = fmaf(a, sdo[ii * p.d_v + c], adv[c]);
      atomicAdd(hp + bp, ds);
      atomicAdd(ht + bt, ds);
    }
  }
  if (col_ok) {
    T *ok = dk + (sq.start + j) * p.dk_rs + h * p.d_qk;
    T *ov = dv + (sq.start + j) * p.dv_rs + h * p.d_v;
#pragma unroll
    for (int c = 0; c < DQ; ++c)
      if (c < p.d_qk) st_elem(ok + c, adk[c]);
#pragma unroll
    for (int c = 0; c < DV; ++c)
      if (c < p.d_v) st_elem(ov + c, adv[c]);
  }
  __syncthreads();
  float *gp = drab_p + (p.rab_per_head ? h * p.nb_p : 0);
  float *gt = drab_t + (p.rab_per_head ? h * p.nb_t : 0);
  for (int32_t x = threadIdx.x; x < p.nb_p; x += blockDim.x)
    if (hp[x] != 0.f) atomicAdd(gp + x, hp[x]);
  for (int32_t x = threadIdx.x; x < p.nb_t; x += blockDim.x)
    if (ht[x] != 0.f) atomicAdd(gt + x, ht[x]);
}

template <typename T>
static cudaError_t bwd_simt_dispatch(const AttnProblem &p, const Scratch &s, const void *dout,
                                     void *dq, void *dk, void *dv, float *drab_p, float *drab_t,
                                     cudaStream_t st) {
  const dim3 grid(s.n_simt_items, p.num_heads);
  const size_t smem_q = sizeof(float) * kSimtKeys * (p.d_qk + p.d_v);
  const size_t smem_k = smem_q + sizeof(float) * (p.nb_p + p.nb_t);
  const int dmax = p.d_qk > p.d_v ? p.d_qk : p.d_v;
  const T *g = static_cast<const T *>(dout);
  T *q_ = static_cast<T *>(dq);
  T *k_ = static_cast<T *>(dk);
  T *v_ = static_cast<T *>(dv);
#define HSTU_BWD_SIMT(DQ_, DV_)                                                              \
  do {                                                                                       \
    if (smem_k > 48 * 1024) {                                                                \
      cudaFuncSetAttribute(dkdv_simt_kernel<T, DQ_, DV_>,                                    \
                           cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem_k));        \
    }                                                                                        \
    dq_simt_kernel<T, DQ_, DV_><<<grid, kSimtRows, smem_q, st>>>(p, s, g, q_);               \
    dkdv_simt_kernel<T, DQ_, DV_><<<grid, kSimtRows, smem_k, st>>>(p, s, g, k_, v_, drab_p,  \
                                                                   drab_t);                  \
  } while (0)
  if (dmax <= 32)
    HSTU_BWD_SIMT(32, 32);
  else if (dmax <= 64)
    HSTU_BWD_SIMT(64, 64);
  else if (dmax <= 128)
    HSTU_BWD_SIMT(128, 128);
  else
    HSTU_BWD_SIMT(256, 256);
#undef HSTU_BWD_SIMT
  count_launch(2);
  return cudaGetLastError();
}

cudaError_t launch_bwd_simt(const AttnProblem &p, const Scratch &s, const void *dout, void *dq,
                            void *dk, void *dv, float *drab_p, float *drab_t, cudaStream_t st) {
  if (s.n_simt_items == 0) return cudaSuccess;
  return p.dtype == 0 ? bwd_simt_dispatch<float>(p, s, dout, dq, dk, dv, drab_p, drab_t, st)
                      : bwd_simt_dispatch<__nv_bfloat16>(p, s, dout, dq, dk, dv, drab_p,
                                                         drab_t, st);
}

// ---------------------------------------------------------------------------
// Debug: buckets of every pair through both time paths.
// ---------------------------------------------------------------------------
__global__ void debug_buckets_kernel(AttnProblem p, Scratch s, int32_t *bp, int32_t *bt,
                                     int32_t *bt_fast) {
  const int32_t b = blockIdx.y;
  const SeqInfo sq = s.seqs[b];
  int64_t base = 0;   // output offset of sequence b: sum of L_c^2, c < b
  for (int32_t c = 0; c < b; ++c) base += int64_t(s.seqs[c].len) * s.seqs[c].len;
  const int64_t L = sq.len;
  const int64_t n = L * L;
  const int fast = s.seq_fast[b] & kSeqFastTime;
  const int sh = 23 - p.sub_bits;
  const int32_t r0 = fast_r0(p.sub_bits);
  for (int64_t x = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; x < n;
       x += int64_t(gridDim.x) * blockDim.x) {
    const int32_t i = int32_t(x / L), j = int32_t(x % L);
    const int64_t o = base + x;
    if (!is_visible(i, j, sq.n_hist)) {
      bp[o] = -1;
      bt[o] = -1;
      bt_fast[o] = -1;
      continue;
    }
    bp[o] = pos_bucket(position_of(i, sq.n_hist) - position_of(j, sq.n_hist), p.nb_p);
    bt[o] = time_bucket_i64(p.ts[sq.start + i] - p.ts[sq.start + j], p.sub_bits, p.nb_t);
    if (fast && p.sub_bits <= 8) {
      const float dt = s.tf[sq.start + i] - s.tf[sq.start + j];
      const int32_t r = __float_as_int(dt) >> sh;
      const int32_t idx = (r > r0 ? r : r0) - r0;
      bt_fast[o] = idx < fast_table_size(p.sub_bits)
                       ? fast_table_bucket(idx, p.sub_bits, p.nb_t)
                       : -3;
    } else {
      bt_fast[o] = -2;
    }
  }
}

// Debug: one warp waits, bounded, on a shared-memory barrier that nothing
// arrives at, so the wait runs out, the timeout is recorded in the error word
// and the kernel returns (the path every tensor-core kernel takes when a
// wait runs out), without any fault.
__global__ void wait_probe_kernel(WaitCtl w) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
  }
  __syncwarp();
  wait_bar(&bar, 0, w);   // phase 0 never completes
}

cudaError_t launch_wait_probe(const WaitCtl &w, cudaStream_t st) {
  wait_probe_kernel<<<1, 32, 0, st>>>(w);
  count_launch();
  return cudaGetLastError();
}

cudaError_t launch_debug_buckets(const AttnProblem &p, const Scratch &s, int32_t *bp,
                                 int32_t *bt, int32_t *bt_fast, cudaStream_t st) {
  if (p.batch == 0) return cudaSuccess;
  const dim3 grid(64, p.batch);
  debug_buckets_kernel<<<grid, 256, 0, st>>>(p, s, bp, bt, bt_fast);
  count_launch();
  return cudaGetLastError();
}

}  // namespace hstu
