/*
 * hstu.h -- C ABI of libhstu.so: HSTU pointwise attention on B200 (sm_100a).
 *
 * What the library computes (sources: the DLRMv4 article "DLRMv4: MLPerf's
 * recommendation-training benchmark enters the sequence era", winzheng.jp,
 * section "Model architecture: HSTU replaces the feature-interaction stack",
 * which describes the HSTU layer in words -- one projection produces the
 * layer's internal representations, pointwise attention aggregates the
 * sequence with a bias from the positional and temporal distance of two
 * events, a gated transformation replaces the cross network and FFN -- and
 * section "How one training sample is processed by HSTU": per-user
 * time-ordered event tokens with timestamps, candidates appended at the end
 * and compared to the whole history in one causal forward pass; and "Actions
 * Speak Louder than Words", arXiv 2402.17152, abstract and contribution list:
 * HSTU, M-FALCON batched candidate inference):
 *
 *   sequence b = tokens [o_b, o_{b+1}); L = length; n_c candidates; n_h = L - n_c
 *   pos(i) = i (i < n_h) or n_h (candidates)
 *   visible(i, j) = j <= i (i < n_h);  j < n_h or j == i (i >= n_h)
 *   s_ij = alpha <q_i, k_j> + rab_pos[min(nb_p - 1, pos(i) - pos(j))]
 *                           + rab_time[min(nb_t - 1, tb(t_i - t_j))]
 *   out_i = silu_scale * sum_{visible j} SiLU(s_ij) v_j,   SiLU(x) = x sigmoid(x)
 *   tb(dt) = 0 (dt <= 0); dt (dt < 2^s); (e-s+1) 2^s + (dt >> (e-s)) - 2^s with
 *            e = floor(log2 dt), s = time_bucket_sub_bits.
 * The pages give no formula; this algebra and its constants are the library's
 * stated reading of them.
 *
 * Conventions for every entry point:
 *  - All device buffers are owned by the caller.  The library allocates no
 *    device memory; scratch lives in the caller's workspace, whose size the
 *    *_workspace_size functions return.  Keep a workspace per stream.
 *  - Calls are asynchronous on `stream` (a cudaStream_t passed as void*, NULL
 *    = legacy default stream) and never make the host wait for the device,
 *    except hstu_get_device_error.  The tile schedule is built on the host
 *    from seq_offsets_host and reaches the workspace as kernel parameters
 *    (no host-to-device memcpy), so a stream capture of a call records it
 *    whole and a replay reuses that schedule.
 *  - The host copies of seq_offsets / num_candidates are read during the call
 *    (validation and tile scheduling) and may be freed when it returns.
 *  - Argument errors are returned before any launch; outputs are untouched.
 *    HSTU_ERR_UNSUPPORTED means a valid request this build cannot serve.
 *    A device-side problem (a bounded wait that ran out) is recorded in the
 *    workspace and read with hstu_get_device_error.
 *  - Element types: dtype HSTU_F32 -> float; HSTU_BF16 -> bfloat16 (uint16
 *    storage).  rab tables and their gradients are always float32.
 *  - Layout: q, k, dq, dk are token-major [T][row_stride] with head h at
 *    columns [h*d_qk, (h+1)*d_qk); v, out, dout, dv likewise with d_v.  Row
 *    strides are in elements, so a fused projection output [T][U|V|Q|K] can
 *    be consumed in place.
 */
#ifndef HSTU_H
#define HSTU_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  HSTU_OK = 0,
  HSTU_ERR_INVALID_ARG = 1,    /* bad pointer, size, stride or offsets */
  HSTU_ERR_UNSUPPORTED = 2,    /* valid request this build does not serve */
  HSTU_ERR_WORKSPACE = 3,      /* workspace missing or too small */
  HSTU_ERR_CUDA = 4,           /* a CUDA runtime call or launch failed */
  HSTU_ERR_DEVICE_TIMEOUT = 5, /* a kernel's bounded wait ran out */
  HSTU_ERR_DEVICE = 6          /* a kernel recorded another device-side fault */
} hstu_status_t;

typedef enum { HSTU_F32 = 0, HSTU_BF16 = 1 } hstu_dtype_t;

typedef enum {
  HSTU_MASK_CAUSAL = 0,  /* every query sees the keys at or before it */
  HSTU_MASK_MFALCON = 1  /* last num_candidates[b] tokens: history + self only */
} hstu_mask_t;

/* Kernel family selection (for testing and measurement; AUTO is the fast path). */
typedef enum {
  HSTU_IMPL_AUTO = 0,    /* tensor-core (tcgen05) path when the shape allows it */
  HSTU_IMPL_SIMT = 1     /* CUDA-core path: any head size, float32 or bf16 */
} hstu_impl_t;

typedef struct {
  int32_t batch;                 /* B >= 0 sequences */
  int32_t num_heads;             /* H >= 1 */
  int32_t d_qk, d_v;             /* head sizes, 1..256 */
  int32_t max_seq_len;           /* every sequence length must be <= this */
  int32_t num_pos_buckets;       /* nb_p >= 1 */
  int32_t num_time_buckets;      /* nb_t >= 1 */
  int32_t time_bucket_sub_bits;  /* s in 0..8 */
  int32_t rab_per_head;          /* 0: tables [nb]; 1: tables [H][nb] */
  int32_t mask;                  /* hstu_mask_t */
  int32_t dtype;                 /* hstu_dtype_t of q, k, v, out, dout, dq, dk, dv */
  int32_t impl;                  /* hstu_impl_t */
  int64_t q_row_stride, k_row_stride, v_row_stride, o_row_stride;       /* elements */
  int64_t do_row_stride, dq_row_stride, dk_row_stride, dv_row_stride;   /* backward */
  float alpha;                   /* logit scale, typically 1/sqrt(d_qk) */
  float silu_scale;              /* post-SiLU scale, typically 1/max_seq_len */
} hstu_attn_params_t;

/* Human-readable name of a status code (static storage). */
const char *hstu_status_string(hstu_status_t status);

/* Library version string, e.g. "hstu-b200 0.1 sm_100a". */
const char *hstu_version(void);

/* Bytes of workspace hstu_attn_fwd (is_bwd = 0) or hstu_attn_bwd (is_bwd = 1)
 * needs for this problem.  seq_offsets_host[B+1] as for the compute calls.
 * Returns HSTU_ERR_INVALID_ARG for the same argument errors the compute call
 * would reject. */
hstu_status_t hstu_attn_workspace_size(const hstu_attn_params_t *params,
                                       const int64_t *seq_offsets_host, int32_t is_bwd,
                                       size_t *bytes);

/* Forward attention: out = the formula at the top of this file.
 *  seq_offsets_host  [B+1] host; 0 = o_0 <= o_1 <= ... <= o_B = T, and every
 *                    length <= max_seq_len.
 *  num_candidates_host [B] host, required iff mask == HSTU_MASK_MFALCON,
 *                    0 <= n_c <= length.
 *  timestamps_dev    [T] int64 seconds, device.
 *  q, k, v           device, dtype, layout above.
 *  rab_pos, rab_time device float32 tables (see rab_per_head).
 *  out               device [T][o_row_stride], dtype; every row is written.
 *  workspace         device, >= hstu_attn_workspace_size(.., 0, ..) bytes,
 *                    256-byte aligned. */
hstu_status_t hstu_attn_fwd(const hstu_attn_params_t *params, const int64_t *seq_offsets_host,
                            const int32_t *num_candidates_host, const int64_t *timestamps_dev,
                            const void *q, const void *k, const void *v, const float *rab_pos,
                            const float *rab_time, void *out, void *workspace,
                            size_t workspace_bytes, void *stream);

/* Backward attention.  Inputs as hstu_attn_fwd plus dout (the gradient of
 * out).  Writes dq, dk, dv (dtype, strides dq/dk/dv_row_stride; every row is
 * written) and ACCUMULATES into drab_pos / drab_time (float32, same shape as
 * the tables; the caller zeroes them first).  With SiLU'(x) = sigmoid(x)
 * (1 + x (1 - sigmoid(x))) and dS_ij = <dout_i, v_j> silu_scale SiLU'(s_ij):
 *   dv_j = silu_scale sum_i SiLU(s_ij) dout_i;  dq_i = alpha sum_j dS_ij k_j;
 *   dk_j = alpha sum_i dS_ij q_i;  drab_*[bucket_ij] += dS_ij. */
hstu_status_t hstu_attn_bwd(const hstu_attn_params_t *params, const int64_t *seq_offsets_host,
                            const int32_t *num_candidates_host, const int64_t *timestamps_dev,
                            const void *q, const void *k, const void *v, const float *rab_pos,
                            const float *rab_time, const void *dout, void *dq, void *dk,
                            void *dv, float *drab_pos, float *drab_time, void *workspace,
                            size_t workspace_bytes, void *stream);

/* One HSTU layer forward, bf16 activations and weights, float32 accumulation:
 *   [U|V|Q|K] = SiLU(x W1^T + b1)        (one projection, column blocks of
 *                                          H*d_v, H*d_v, H*d_qk, H*d_qk)
 *   A = attention(Q, K, V)               (hstu_attn_fwd, strides into the
 *                                          projection output, no copies)
 *   G = LayerNorm(A; ln_eps, gamma, beta) (.) U   (over the H*d_v features)
 *   y = x + G W2^T + b2                  (residual != 0) or G W2^T + b2.
 *  x [T][d_model] bf16; w1 [2H(d_v+d_qk)][d_model] bf16; b1 float32;
 *  ln_gamma, ln_beta [H d_v] float32; w2 [d_model][H d_v] bf16; b2 float32;
 *  y [T][d_model] bf16 (may not alias x).  attn.dtype must be HSTU_BF16;
 *  the attn row strides are ignored (the layer sets them). */
typedef struct {
  hstu_attn_params_t attn;
  int32_t d_model;   /* 8..8192, multiple of 8 */
  int32_t residual;  /* nonzero: add x */
  float ln_eps;      /* > 0 */
  int32_t reserved;
} hstu_layer_params_t;

hstu_status_t hstu_layer_workspace_size(const hstu_layer_params_t *params,
                                        const int64_t *seq_offsets_host, size_t *bytes);

hstu_status_t hstu_layer_fwd(const hstu_layer_params_t *params, const int64_t *seq_offsets_host,
                             const int32_t *num_candidates_host, const int64_t *timestamps_dev,
                             const void *x, const void *w1, const float *b1,
                             const float *ln_gamma, const float *ln_beta, const void *w2,
                             const float *b2, const float *rab_pos, const float *rab_time,
                             void *y, void *workspace, size_t workspace_bytes, void *stream);

/* hstu_layer_fwd that also keeps the layer's projection: proj_out [T][N1]
 * bf16 (16-byte aligned; N1 = 2 H (d_v + d_qk)) receives [U|V|Q|K] =
 * SiLU(x W1^T + b1), written there instead of into the workspace.  Its V and
 * K column blocks are the history's keys and values that
 * hstu_layer_fwd_candidates reads (the M-FALCON history pass).  Workspace
 * and errors as hstu_layer_fwd (hstu_layer_workspace_size). */
hstu_status_t hstu_layer_fwd_keep_proj(const hstu_layer_params_t *params,
                                       const int64_t *seq_offsets_host,
                                       const int32_t *num_candidates_host,
                                       const int64_t *timestamps_dev, const void *x,
                                       const void *w1, const float *b1, const float *ln_gamma,
                                       const float *ln_beta, const void *w2, const float *b2,
                                       const float *rab_pos, const float *rab_time, void *y,
                                       void *proj_out, void *workspace, size_t workspace_bytes,
                                       void *stream);

/* M-FALCON candidate scoring against cached history keys and values.
 *
 * The "Actions Speak Louder than Words" abstract and contribution list name
 * M-FALCON, which serves candidates in mini-batches at a fixed inference
 * budget, and the DLRMv4 article ("How one training sample is processed by
 * HSTU") appends the candidates after the history and compares each with the
 * whole history.  Under the library's M-FALCON mask a candidate sees every
 * history token and itself, never another candidate, and sits at position
 * n_h; so a candidate's output depends only on the history and on itself,
 * and the history's keys and values can be computed once and kept while the
 * candidates arrive in any number of micro-batches of any size.  This call
 * scores one micro-batch: for sequence b its n_h(b) cached history tokens
 * and its n_c(b) candidates in this call, and gives every candidate exactly
 * the output the one-pass HSTU_MASK_MFALCON forward gives it.
 *  params            as hstu_attn_fwd; batch = B sequences; max_seq_len
 *                    bounds n_h + n_c; mask is ignored.  q/k/v_row_stride:
 *                    the candidates' q, k, v; o_row_stride: out.
 *  hist_offsets_host [B+1] host: history tokens of sequence b are rows
 *                    [hist_offsets[b], hist_offsets[b+1]) of k_hist / v_hist.
 *  cand_offsets_host [B+1] host: its candidates in this call are rows
 *                    [cand_offsets[b], cand_offsets[b+1]) of q, k, v, out.
 *  hist_timestamps_dev [Th], cand_timestamps_dev [Tc]: int64 seconds, device.
 *  k_hist, v_hist    device, the cached history [Th][row_stride] (e.g. the K
 *                    and V column blocks of hstu_layer_fwd_keep_proj's proj_out).
 *  out               [Tc][o_row_stride]; every candidate row is written.
 *  workspace         >= hstu_attn_candidates_workspace_size bytes, 256-aligned.
 * Tensor-core path only: bf16, d_qk = d_v in {64, 128}, 16-byte aligned
 * buffers and strides in multiples of 8 elements, <= 1024 buckets per table;
 * otherwise HSTU_ERR_UNSUPPORTED.  Other errors as hstu_attn_fwd. */
hstu_status_t hstu_attn_candidates_workspace_size(const hstu_attn_params_t *params,
                                                  const int64_t *hist_offsets_host,
                                                  const int64_t *cand_offsets_host,
                                                  size_t *bytes);

hstu_status_t hstu_attn_fwd_candidates(
    const hstu_attn_params_t *params, const int64_t *hist_offsets_host,
    const int64_t *cand_offsets_host, const int64_t *hist_timestamps_dev,
    const int64_t *cand_timestamps_dev, const void *q, const void *k, const void *v,
    const void *k_hist, const void *v_hist, int64_t k_hist_row_stride,
    int64_t v_hist_row_stride, const float *rab_pos, const float *rab_time, void *out,
    void *workspace, size_t workspace_bytes, void *stream);

/* One HSTU layer on a micro-batch of candidates only, against the history's
 * projection from hstu_layer_fwd_keep_proj (the candidate-only output path:
 * the projection, LayerNorm gating and output projection run on candidate
 * rows alone; only candidate positions feed the task head, DLRMv4 article,
 * "How one training sample is processed by HSTU"):
 *   [U|V|Q|K]_c = SiLU(x_cand W1^T + b1)
 *   A_c = hstu_attn_fwd_candidates(Q_c, K_c, V_c; cached K_h, V_h of hist_proj)
 *   y_cand = x_cand + (LayerNorm(A_c) (.) U_c) W2^T + b2   (residual as flagged)
 * Stacking: the history pass runs hstu_layer_fwd_keep_proj layer by layer on
 * the history alone (causal), keeping each layer's proj_out; each candidate
 * micro-batch then runs this call layer by layer, feeding y_cand forward.
 * The candidates' outputs equal the one-pass M-FALCON stack's.
 *  x_cand, y_cand [Tc][d_model] bf16 (y may not alias x); hist_proj [Th][N1].
 *  Weights, offsets and timestamps as hstu_layer_fwd / hstu_attn_fwd_candidates.
 *  workspace >= hstu_layer_candidates_workspace_size bytes, 256-aligned; its
 *  first 16 bytes are the device error word. */
hstu_status_t hstu_layer_candidates_workspace_size(const hstu_layer_params_t *params,
                                                   const int64_t *hist_offsets_host,
                                                   const int64_t *cand_offsets_host,
                                                   size_t *bytes);

hstu_status_t hstu_layer_fwd_candidates(
    const hstu_layer_params_t *params, const int64_t *hist_offsets_host,
    const int64_t *cand_offsets_host, const int64_t *hist_timestamps_dev,
    const int64_t *cand_timestamps_dev, const void *x_cand, const void *w1, const float *b1,
    const float *ln_gamma, const float *ln_beta, const void *w2, const float *b2,
    const float *rab_pos, const float *rab_time, const void *hist_proj, void *y_cand,
    void *workspace, size_t workspace_bytes, void *stream);

/* One HSTU layer backward (training): the gradients of hstu_layer_fwd's y
 * with respect to its input and every parameter, given dy = dL/dy.  By the
 * chain rule through the layer's steps in reverse:
 *   dG = dy W2;  dW2 += dy^T G;  db2 += sum_t dy
 *   dU = dG (.) LN(A);  dLN = dG (.) U;  dgamma += sum_t dLN (.) xhat;
 *   dbeta += sum_t dLN;  dA = (dxh - mean(dxh) - xhat mean(dxh (.) xhat)) / sigma
 *     with xhat = (A - mean) / sigma, sigma = sqrt(var + ln_eps), dxh = dLN (.) gamma
 *   dQ, dK, dV, drab_pos, drab_time = attention backward of dA (hstu_attn_bwd)
 *   dZ = [dU|dV|dQ|dK] (.) SiLU'(Z), Z = x W1^T + b1;  dW1 += dZ^T x;
 *   db1 += sum_t dZ;  dx = dZ W1 (+ dy when residual).
 * The forward's projection, attention and LayerNorm statistics are computed
 * again inside the call (no saved activations); the workspace holds them.
 *  x, w1, b1, ln_gamma, ln_beta, w2, b2, rab_pos, rab_time, params, offsets,
 *      candidates, timestamps: exactly as given to hstu_layer_fwd.
 *  dy  [T][d_model] bf16.   dx [T][d_model] bf16, written (may alias neither
 *      x nor dy).
 *  dw1 [N1][d_model], db1 [N1], dgamma, dbeta [H d_v], dw2 [d_model][H d_v],
 *      db2 [d_model], drab_pos, drab_time: float32, ACCUMULATED (+=), so
 *      gradients of several micro-batches add up; zero them first.
 *  workspace: >= hstu_layer_bwd_workspace_size bytes, 256-byte aligned; its
 *      first 16 bytes are the device error word (hstu_get_device_error).
 * Needs the tensor-core path: d_model and N1 = 2 H (d_v + d_qk) multiples of
 * 32, else HSTU_ERR_UNSUPPORTED.  Other errors as hstu_layer_fwd. */
hstu_status_t hstu_layer_bwd_workspace_size(const hstu_layer_params_t *params,
                                            const int64_t *seq_offsets_host, size_t *bytes);

hstu_status_t hstu_layer_bwd(const hstu_layer_params_t *params, const int64_t *seq_offsets_host,
                             const int32_t *num_candidates_host, const int64_t *timestamps_dev,
                             const void *x, const void *w1, const float *b1,
                             const float *ln_gamma, const float *ln_beta, const void *w2,
                             const float *b2, const float *rab_pos, const float *rab_time,
                             const void *dy, void *dx, float *dw1, float *db1, float *dgamma,
                             float *dbeta, float *dw2, float *db2, float *drab_pos,
                             float *drab_time, void *workspace, size_t workspace_bytes,
                             void *stream);

/* Debug (host only, no CUDA call): the work lists the attention calls build
 * for this batch, in launch order (longest first).  Each forward item is 4
 * int32 {sequence, pair of 128-row query tiles p (rows [256 p, 256 p + 256)),
 * first key tile, end key tile}: an unsplit item has first 0 and end
 * 0x7fffffff and walks key tiles 0 .. the pair's last tile; a split item
 * takes key tiles [first, end).  Each backward item is {sequence, 128-key
 * tile, first query block, end query block} for 64-query blocks, the same
 * way (0 / 0x7fffffff: the whole run of blocks that see the tile).  The
 * kernels skip tiles and blocks without a visible pair.  fwd_items and
 * bwd_items: host arrays of 4 * capacity int32; *n_fwd / *n_bwd receive the
 * counts even when they exceed capacity (then HSTU_ERR_INVALID_ARG).
 * Other errors as hstu_attn_workspace_size.  The pages have no counterpart:
 * this exists to check the schedule against a brute-force enumeration. */
hstu_status_t hstu_debug_plan(const hstu_attn_params_t *params, const int64_t *seq_offsets_host,
                              const int32_t *num_candidates_host, int32_t capacity,
                              int32_t *fwd_items, int32_t *n_fwd, int32_t *bwd_items,
                              int32_t *n_bwd);

/* Debug: the position and time buckets the kernels use, for every pair of
 * every sequence, dense per sequence like the attention masks: for sequence b
 * an L_b x L_b int32 block (row = query, column = key) at element offset
 * sum_{c<b} L_c^2; invisible pairs hold -1.  bt_fast receives the time bucket
 * through the tensor-core kernels' float-exponent table path (only valid
 * where a sequence's timestamp span is below 2^24 s; -2 elsewhere), bt the
 * general int64 path.  Output arrays are device buffers of sum L_b^2 int32.
 * Uses the attention workspace (is_bwd = 0 size). */
hstu_status_t hstu_debug_buckets(const hstu_attn_params_t *params,
                                 const int64_t *seq_offsets_host,
                                 const int32_t *num_candidates_host,
                                 const int64_t *timestamps_dev, int32_t *bp, int32_t *bt,
                                 int32_t *bt_fast, void *workspace, size_t workspace_bytes,
                                 void *stream);

/* Synchronises `stream` and reports the device-side status recorded in the
 * workspace by the most recent call that used it (HSTU_OK,
 * HSTU_ERR_DEVICE_TIMEOUT or HSTU_ERR_DEVICE); *detail (may be NULL)
 * receives the raw error word. */
hstu_status_t hstu_get_device_error(const void *workspace, void *stream, uint32_t *detail);

/* Test hook: bound, in microseconds, on every device-side wait of the
 * tensor-core kernels (default 4 s); 0 restores the default.  Process-wide
 * (an atomic store: calls that launch concurrently on other host threads see
 * either the old or the new bound). */
void hstu_set_wait_limit(uint32_t microseconds);

/* Test hook for the device-side failure path: launches one warp that waits,
 * bounded by limit_us microseconds (1 .. 60 s), on a shared-memory barrier
 * that nothing arrives at.  The wait runs out, the timeout bit is recorded in
 * the workspace's error word (cleared first) and the kernel returns, so a
 * following hstu_get_device_error on the same workspace reports
 * HSTU_ERR_DEVICE_TIMEOUT and the context stays usable.  workspace: device
 * buffer of at least 16 bytes, 256-byte aligned (any attention workspace).
 * Errors: HSTU_ERR_WORKSPACE, HSTU_ERR_INVALID_ARG, HSTU_ERR_CUDA.  The pages
 * have no counterpart; this exists to test the library's bounded waits. */
hstu_status_t hstu_debug_wait_probe(void *workspace, size_t workspace_bytes, uint32_t limit_us,
                                    void *stream);

/* Number of kernels this library has launched in this process (all devices,
 * all entry points).  For accounting in benchmarks and tests. */
uint64_t hstu_kernel_launch_count(void);

/* Phase traces of the tensor-core attention kernels, for performance work
 * only (the pages have no counterpart).  In a library built with
 * -DHSTU_TRACE (`python -m hstu_pointwise_attention_b200.build --trace`),
 * three CTAs of each launch (grid blocks 0, n/2, n-1) record the SM clock at
 * the phase boundaries of their work into a static device buffer per kernel
 * of 3 x 20 x 1024 uint64 entries: [CTA][warp][entry], entry = code << 56 |
 * ordinal << 40 | clock (40 bits).  Elementwise warps record from lane 0, the
 * MMA issuer (warp 1) per issued batch.
 *  kernel HSTU_TRACE_BWD128, the d = 128 backward, per 64-query block (ordinal
 *    the block's place in the CTA's run): 1 block start, 8/9/10 a 16-column
 *    chunk's tensor-memory load issued / landed / math done (ordinal 2 block
 *    + chunk), 11 P^T stored, 2 block handed to the issuer, 3 dQ^T ready, 4
 *    dQ^T reductions issued; issuer: 5 dQ^T, 6 S^T, 7 dP^T issued.
 *  kernel HSTU_TRACE_FWD, the forward (every head size and the cached-history
 *    variant), per key tile (ordinal the key-tile step n): 1 tile start,
 *    8/9/10 a 32-key chunk's load issued / landed / math done (ordinal 2 n +
 *    chunk), 11 P stored, 2 P handed to the issuer; issuer: 5 O += P V, 6 the
 *    next S issued (ordinal 2 n + query tile).
 * Later launches overwrite earlier entries slot by slot, so clear before the
 * launch to be read.  hstu_debug_trace_clear zeroes a kernel's buffer (current
 * device, waiting for the device); hstu_debug_trace_read copies min(bytes, the
 * buffer) to `host` (host memory, caller-owned).  Both return
 * HSTU_ERR_INVALID_ARG for an unknown kernel or a null `host`,
 * HSTU_ERR_UNSUPPORTED in a library built without the flag, HSTU_ERR_CUDA if
 * the copy fails. */
#define HSTU_TRACE_BWD128 0
#define HSTU_TRACE_FWD 1
hstu_status_t hstu_debug_trace_read(int32_t kernel, void *host, size_t bytes);
hstu_status_t hstu_debug_trace_clear(int32_t kernel);

/* Data-parallel split of a jagged batch over `world` ranks (host only, no
 * CUDA call).  Sequences are independent units of the attention, so a batch
 * shards by sequence with no exchange in the forward; the backward's only
 * exchange is the sum of the bias-table gradients.  The attention's cost
 * grows with the number of visible (query, key) pairs, n_h (n_h + 1) / 2 +
 * n_c (n_h + 1) for a sequence with n_h history tokens and n_c candidates,
 * so that is what the split balances: longest-processing-time first
 * (sequences by descending pair count, ties by index; each to the rank with
 * the least load so far, ties to the lower rank), which keeps the largest
 * rank load within 4/3 of the best possible.  The result is deterministic,
 * so every rank computes the same split from the same offsets.
 *  seq_offsets_host    [batch + 1], as for hstu_attn_fwd (o_0 = 0, non-decreasing).
 *  num_candidates_host [batch] or NULL (no candidates).
 *  rank_of_seq         [batch] out: the rank each sequence goes to.
 *  rank_pairs          [world] out, may be NULL: visible pairs per rank.
 * Errors: HSTU_ERR_INVALID_ARG (bad sizes, offsets or candidate counts). */
hstu_status_t hstu_partition_batch(const int64_t *seq_offsets_host,
                                   const int32_t *num_candidates_host, int32_t batch,
                                   int32_t world, int32_t *rank_of_seq, int64_t *rank_pairs);

/* Forward attention for callers that cannot allocate device memory.
 * (The pages have no counterpart; this is a deployment convenience.)
 *
 * Some callers may not call cudaMalloc or any allocating routine: code that
 * runs under a host framework's own memory manager, in a callback where
 * allocation is forbidden, or inside a tight latency budget where an
 * allocation could synchronise the device.  hstu_attn_fwd needs a workspace
 * from its caller; this entry point needs none.  Its scratch (the error
 * word, the tile schedule and the per-token float timestamps) lives in one
 * file-scope device array of HSTU_NOALLOC_SCRATCH_BYTES that every GPU which
 * loads the library holds until the process exits.
 *
 * Arguments, results and errors are those of hstu_attn_fwd minus the
 * workspace; the caller still passes every input and output buffer.
 *  - A problem whose scratch would exceed HSTU_NOALLOC_SCRATCH_BYTES (about
 *    T * 4 bytes + 8 bytes per sequence and per 64-row tile) is rejected with
 *    HSTU_ERR_WORKSPACE before any launch.
 *  - The first call on each device looks up the array's device address
 *    (cudaGetSymbolAddress) with that device current and caches it; make
 *    that first call before any stream capture.  If the device's context is
 *    torn down and re-created (cudaDeviceReset), the next call looks the
 *    address up again.
 *  - Every call on a device shares the one array and overwrites it; the
 *    call clears what must start at zero.  Calls that overlap on the GPU
 *    (different streams, or different host threads, without ordering) race
 *    on the array: serialise them.
 *  - Device-side wait timeouts are recorded in the array only; use
 *    hstu_attn_fwd with a workspace when they must be read back.
 *  - It allocates nothing: no cudaMalloc, cudaFree or allocating library
 *    routine is called. */
#define HSTU_NOALLOC_SCRATCH_BYTES (8u << 20)
hstu_status_t hstu_attn_fwd_noalloc(const hstu_attn_params_t *params,
                                    const int64_t *seq_offsets_host,
                                    const int32_t *num_candidates_host,
                                    const int64_t *timestamps_dev, const void *q, const void *k,
                                    const void *v, const float *rab_pos, const float *rab_time,
                                    void *out, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* HSTU_H */
