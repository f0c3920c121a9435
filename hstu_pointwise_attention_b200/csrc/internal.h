// internal.h -- structures shared by the API layer and the kernel launchers.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>
#include <mutex>

#include "common.cuh"

namespace hstu {

// One sequence of the jagged batch, as the kernels see it.
struct SeqInfo {
  int64_t start;   // first global token
  int32_t len;     // L
  int32_t n_hist;  // L - num_candidates (L in causal mode)
};

// Attention problem after validation (device pointers; strides in elements).
struct AttnProblem {
  int32_t batch, num_heads, d_qk, d_v, max_seq_len;
  int32_t nb_p, nb_t, sub_bits, rab_per_head, mask, dtype;
  int64_t total_tokens;
  int64_t q_rs, k_rs, v_rs, o_rs, do_rs, dq_rs, dk_rs, dv_rs;
  float alpha, silu_scale;
  const int64_t *ts;       // [T]
  const void *q, *k, *v;
  const float *rab_p, *rab_t;
};

// Backward d rab bins each tensor-core CTA may reduce into global memory:
// position bins [0, 512) then time bins [512, 1024).
constexpr int kBinAccPerCta = 1024;

// Per-sequence flags written by the prep kernel.
enum : int32_t {
  kSeqFastTime = 1,   // timestamp span < 2^24 s: float relative times are exact
  kSeqSorted = 2,     // timestamps non-decreasing
};

// Work items that cover only part of their range (short batches split long
// items so that no SM is left with most of the work): the range fields hold
// kUnsplit for an item that covers its whole range.
constexpr int32_t kUnsplit = 0x7fffffff;

// Device-side view of the per-call scratch carved out of the caller's
// workspace by the API layer.
struct Scratch {
  uint32_t *err;            // error word
  SeqInfo *seqs;            // [B]
  float *tf;                // [T] float(t - t_min(seq)) where the span allows
  int32_t *seq_fast;        // [B] 1 if the sequence's span < 2^24 s
  // tensor-core forward: {seq, tile pair, first key tile, end key tile}; a
  // pair split over key ranges adds its partial outputs into o_acc
  int4 *items;
  int32_t n_items;
  int2 *simt_items;         // SIMT work list: {seq, 64-row tile}
  int32_t n_simt_items;
  float *dq_acc;            // backward: float32 dQ accumulator [H][T][d_qk]
  float *bin_acc;           // backward: per-CTA d rab bins [kitems * H][kBinAccPerCta]
  // tensor-core backward: {seq, key tile, first query block, end query
  // block}; a key tile split over query runs adds its partial dK, dV into
  // dk_acc, dv_acc
  int4 *kitems;
  int32_t n_kitems;
  // Split items' float32 sums hold only the rows of split pairs / key tiles:
  // item_acc[i] (kitem_acc[i]) is the first accumulator row of item i's pair
  // (key tile), -1 for an unsplit item; a split row range {first global row,
  // rows, first accumulator row} lists what the conversion writes back.
  int32_t *item_acc;
  float *o_acc;             // [split rows][H][d_v] float32 (else null)
  int4 *split_rows;         // forward split ranges
  int32_t n_split_rows, n_split_acc_rows;
  int32_t *kitem_acc;
  float *dk_acc, *dv_acc;   // [split key rows][H][d] float32 (else null)
  int4 *ksplit_rows;        // backward split ranges
  int32_t n_ksplit_rows, n_ksplit_acc_rows;
};

// Counts kernel launches (hstu_kernel_launch_count); call once per launch.
void count_launch(int n = 1);

// Kernel attributes (the dynamic shared-memory limit) and device properties
// are per device.  A launcher keeps one PerDeviceOnce per kernel and does its
// set-up through it: the first launch on each device (the current one) runs
// the set-up, later launches on that device skip it.  Safe to call from
// several host threads; a set-up that fails is retried on the next call.
class PerDeviceOnce {
 public:
  static constexpr int kMaxDevices = 64;
  // fn(int device) -> cudaError_t
  template <class F>
  cudaError_t run(F &&fn) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    if (done_[dev].load(std::memory_order_acquire)) return cudaSuccess;
    std::lock_guard<std::mutex> lock(mu_);
    if (done_[dev].load(std::memory_order_relaxed)) return cudaSuccess;
    e = fn(dev);
    if (e == cudaSuccess) done_[dev].store(true, std::memory_order_release);
    return e;
  }
  // Whether the set-up has run on `dev` (for tests and diagnostics).
  bool done(int dev) const {
    return dev >= 0 && dev < kMaxDevices && done_[dev].load(std::memory_order_acquire);
  }

 private:
  std::atomic<bool> done_[kMaxDevices] = {};
  std::mutex mu_;
};

// Sets `kernel`'s dynamic shared-memory limit to `bytes` once per device.
template <class K>
cudaError_t set_smem_once(PerDeviceOnce &once, K kernel, size_t bytes) {
  return once.run([&](int) {
    return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, int(bytes));
  });
}

// Phase-trace buffers of a library built with -DHSTU_TRACE (copy out / zero);
// false when the build has no trace or the copy fails.
bool trace_bwd128_read(void *host, size_t bytes);
bool trace_bwd128_clear();
bool trace_fwd_read(void *host, size_t bytes);
bool trace_fwd_clear();
#ifdef HSTU_TRACE
constexpr bool kTraceBuild = true;
#else
constexpr bool kTraceBuild = false;
#endif

// --- launchers (return a cudaError_t of the launch) ---
// Copies `bytes` (a multiple of 16) from host memory at src to the 16-byte
// aligned device address dst through kernel parameters (no host wait); when
// err_clear is non-null the 16-byte device error word there is zeroed too.
cudaError_t launch_upload(void *dst, const void *src, size_t bytes, uint32_t *err_clear,
                          cudaStream_t st);
cudaError_t launch_prep(const AttnProblem &p, const Scratch &s, cudaStream_t st);
// For each range {first row r0, rows n, first accumulator row a0} of `rows`:
// dst[r0 + i][h d] = bf16(scale * src[a0 + i][h][d]); src float32 [*][H][D],
// dst bf16 with row stride dst_rs.
cudaError_t launch_rows_to_bf16(const float *src, void *dst, int64_t dst_rs, int32_t H,
                                int32_t D, const int4 *rows, int32_t n, float scale,
                                cudaStream_t st);

cudaError_t launch_fwd_simt(const AttnProblem &p, const Scratch &s, void *out,
                            cudaStream_t st);
cudaError_t launch_bwd_simt(const AttnProblem &p, const Scratch &s, const void *dout, void *dq,
                            void *dk, void *dv, float *drab_p, float *drab_t, cudaStream_t st);

// Tensor-core path (bf16, d_qk = d_v in {64, 128}).
bool fwd_tc_supported(const AttnProblem &p);
cudaError_t launch_fwd_tc(const AttnProblem &p, const Scratch &s, void *out, const WaitCtl &w,
                          cudaStream_t st);
// Cached-history forward (candidate micro-batches): in the AttnProblem, q is
// the candidates' query buffer; k, v, ts and total_tokens describe the cached
// history; the SeqInfo of sequence b is {history start, n_h + n_c, n_h}.
struct CachedHist {
  const int64_t *cstart;     // [B] device: first candidate row of each sequence
  const float *tfc;          // [Tc] device: candidate float times (prep)
  const int64_t *ts_cand;    // [Tc] device: candidate timestamps
  const void *k_cand, *v_cand;
  int64_t kc_rs, vc_rs;
  int64_t n_cand_tokens;     // Tc
};
cudaError_t launch_fwd_tc_cached(const AttnProblem &p, const Scratch &s, const CachedHist &ch,
                                 void *out, const WaitCtl &w, cudaStream_t st);
// Per-sequence times for the cached-history forward: span and order flags
// over history and candidates, float times relative to their minimum.
cudaError_t launch_prep_cached(const AttnProblem &p, const Scratch &s, const CachedHist &ch,
                               float *tfc, cudaStream_t st);
bool bwd_tc_supported(const AttnProblem &p);
cudaError_t launch_bwd_tc(const AttnProblem &p, const Scratch &s, const void *dout, void *dq,
                          void *dk, void *dv, float *drab_p, float *drab_t, const WaitCtl &w,
                          cudaStream_t st);

// d_qk = d_v = 128 backward (64-query blocks, dQ^T reduced from tensor memory).
cudaError_t launch_bwd128(const AttnProblem &p, const Scratch &s, const void *dout, void *dq,
                          void *dk, void *dv, float *drab_p, float *drab_t, const WaitCtl &w,
                          cudaStream_t st);
// dq = bf16(alpha silu_scale / 2 * accumulator) for the tensor-core backward.
cudaError_t launch_dq_convert(const AttnProblem &p, const Scratch &s, void *dq, cudaStream_t st);

// One warp waits, bounded by w.limit_ns, on a barrier nothing arrives at.
cudaError_t launch_wait_probe(const WaitCtl &w, cudaStream_t st);

cudaError_t launch_debug_buckets(const AttnProblem &p, const Scratch &s, int32_t *bp,
                                 int32_t *bt, int32_t *bt_fast, cudaStream_t st);

// Layer pieces (bf16).  The GEMM takes the tensor-core path when the shape
// and alignment allow it, the CUDA-core kernel otherwise.
cudaError_t launch_gemm(const void *a, int64_t lda, const void *b, int64_t ldb,
                        const float *bias, const void *residual, int64_t ldr, void *c,
                        int64_t ldc, int64_t M, int64_t N, int64_t K, int epilogue,
                        const WaitCtl &w, cudaStream_t st);
cudaError_t launch_gemm_simt(const void *a, int64_t lda, const void *b, int64_t ldb,
                             const float *bias, const void *residual, int64_t ldr, void *c,
                             int64_t ldc, int64_t M, int64_t N, int64_t K, int epilogue,
                             cudaStream_t st);
bool gemm_tc_supported(const void *a, int64_t lda, const void *b, int64_t ldb, const void *c,
                       int64_t ldc, int64_t M, int64_t N, int64_t K);
cudaError_t launch_gemm_tc(const void *a, int64_t lda, const void *b, int64_t ldb,
                           const float *bias, const void *residual, int64_t ldr, void *c,
                           int64_t ldc, int64_t M, int64_t N, int64_t K, int epilogue,
                           const WaitCtl &w, cudaStream_t st);
cudaError_t launch_ln_gate(const void *a, int64_t lda, const void *u, int64_t ldu,
                           const float *gamma, const float *beta, float eps, void *g,
                           int64_t ldg, int64_t T, int32_t F, cudaStream_t st);

// Backward of the LayerNorm gating (layer.cu): bf16 activations, float32
// gamma / beta and their gradients (accumulated).
struct LnGateBwdArgs {
  const void *a;  int64_t lda;     // attention output A
  const void *u;  int64_t ldu;     // gate U
  const void *dg; int64_t lddg;    // upstream dG
  const float *gamma, *beta;
  float eps;
  void *g;  int64_t ldg;           // out: G = LN(A) (.) U
  void *du; int64_t lddu;          // out: dU
  void *da; int64_t ldda;          // out: dA
  float *dgamma, *dbeta;           // accumulated
  int64_t T;
  int32_t F;
};
cudaError_t launch_ln_gate_bwd(const LnGateBwdArgs &a, cudaStream_t st);
// colsum[N] += sum over T rows of X (bf16 [T][ldx]); with silu_bwd, first
// X <- X (.) SiLU'(Z) in place.  N, ldx, ldz multiples of 8.
cudaError_t launch_colsum(void *x, int64_t ldx, const void *z, int64_t ldz, float *colsum,
                          int64_t T, int64_t N, bool silu_bwd, cudaStream_t st);

enum GemmEpilogue {
  kEpiBiasSilu = 0,       // C = SiLU(acc + bias)
  kEpiBiasResidual = 1,   // C = acc + bias + R
  kEpiBias = 2,           // C = acc + bias
  kEpiBiasSiluPre = 3,    // C = SiLU(acc + bias) and C2 = acc + bias
  kEpiF32Add = 4,         // float32 C += acc (K may be split over CTAs)
};

// One tensor-core GEMM C = A B^T (see gemm_sm100.cu).  bias may be null
// (no bias); the bias is float32 [N].
struct GemmDesc {
  const void *a;
  int64_t lda;
  bool a_mn;            // false: A is [M][lda] (K contiguous); true: stored [K][lda] (M contiguous)
  const void *b;
  int64_t ldb;
  bool b_mn;            // false: B is [N][ldb]; true: stored [K][ldb] (N contiguous)
  int64_t M, N, K;
  int epi;              // GemmEpilogue
  const float *bias;
  const void *res;      // kEpiBiasResidual: bf16 [M][ldr]
  int64_t ldr;
  void *c;              // bf16 [M][ldc] (float32 for kEpiF32Add)
  int64_t ldc;
  void *c2;             // kEpiBiasSiluPre: bf16 [M][ldc2]
  int64_t ldc2;
  int splits;           // K split over CTAs (kEpiF32Add only)
};
bool gemm_desc_supported(const GemmDesc &d);
cudaError_t launch_gemm_desc(const GemmDesc &d, const WaitCtl &w, cudaStream_t st);
// A split of K that gives about one work item per SM (kEpiF32Add GEMMs).
int gemm_split_for(int64_t M, int64_t N, int64_t K, int n_sm);

// Tensor-map encoding through the driver entry point (no libcuda link).
bool encode_tmap_bf16_3d(CUtensorMap *map, const void *base, uint64_t d0, uint64_t d1,
                         uint64_t d2, uint64_t stride1_bytes, uint64_t stride2_bytes,
                         uint32_t box0, uint32_t box1, uint32_t box2);
bool encode_tmap_bf16_2d(CUtensorMap *map, const void *base, uint64_t d0, uint64_t d1,
                         uint64_t stride1_bytes, uint32_t box0, uint32_t box1);
// The same with the 64-byte swizzle (a box of 32 bf16 columns: 16-byte unit
// u of row r sits at unit u ^ ((r >> 1) & 3) of the row in shared memory).
bool encode_tmap_bf16_2d_sw64(CUtensorMap *map, const void *base, uint64_t d0, uint64_t d1,
                              uint64_t stride1_bytes, uint32_t box0, uint32_t box1);
bool encode_tmap_f32_2d(CUtensorMap *map, const void *base, uint64_t d0, uint64_t d1,
                        uint64_t stride1_bytes, uint32_t box0, uint32_t box1,
                        bool swizzle = true);

}  // namespace hstu
