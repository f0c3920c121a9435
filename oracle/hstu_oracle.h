/*
 * hstu_oracle.h -- plain, slow, obviously correct CPU oracle of the HSTU
 * pointwise attention layer (float64 arithmetic, exact integer bucketing).
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the
 * benchmark's CPU-baseline leg may load this library.  It shares no code,
 * header, table or helper with the CUDA library; neither includes the other.
 *
 * What it computes follows these pages:
 *  [GR]     "Actions Speak Louder than Words: Trillion-Parameter Sequential
 *           Transducers for Generative Recommendations" (arXiv 2402.17152,
 *           hotpaper.ai summary), abstract and "technical approach" list:
 *           HSTU layer, M-FALCON candidate inference, length-8192 claim.
 *  [DLRMv4] "DLRMv4: MLPerf's recommendation-training benchmark enters the
 *           sequence era" (winzheng.jp), section "Model architecture: HSTU
 *           replaces the feature-interaction stack" (one projection makes the
 *           layer's internal representations; pointwise attention aggregates
 *           the sequence with a bias from the positional and temporal distance
 *           of two events; a gated transformation replaces cross network and
 *           FFN) and section "How one training sample is processed by HSTU"
 *           (per-user time-ordered event tokens carrying a timestamp,
 *           truncated to a fixed upper length; candidates appended at the end
 *           and compared to the full history in one causal forward pass).
 *
 * The pages give the layer in words only.  The algebra below is the plainest
 * reading consistent with them; every choice the pages leave open is a
 * documented convention (numbered R1..R14 in the design notes):
 *
 *   For sequence b (tokens [o_b, o_{b+1}), length L, n_c candidates,
 *   n_h = L - n_c) and head h, local query i, key j:
 *     pos(i) = i for i < n_h, n_h for candidates                      (R7)
 *     visible(i,j) = j <= i            if i < n_h                      (R6)
 *                  = j < n_h or j == i if i >= n_h (M-FALCON)
 *     bp = min(nb_p - 1, pos(i) - pos(j))                              (R3)
 *     bt = min(nb_t - 1, tb_s(t_i - t_j))                              (R4)
 *     s  = alpha * <q_i, k_j> + rab_p[bp] + rab_t[bt]                  (R1,R5)
 *     o_i = silu_scale * sum_{visible j} s*sigmoid(s) * v_j            (R2)
 *   tb_s(dt) = 0 (dt <= 0); dt (dt < 2^s);
 *              (e - s + 1) 2^s + (dt >> (e - s)) - 2^s, e = floor(log2 dt).
 * The layer around the attention (projection, LayerNorm gating, output
 * projection) is restated in numpy float64 in hstu_oracle.py, which calls
 * this library for the attention step.
 */
#ifndef HSTU_ORACLE_H
#define HSTU_ORACLE_H
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Shape and conventions of one jagged attention problem.  Every float array
 * handed to the oracle is float64 and contiguous:
 *   q, k   [T][H][d_qk]      v, out, dout [T][H][d_v]
 *   rab_p  [nb_p] (or [H][nb_p] when rab_per_head)   rab_t likewise [nb_t].
 * offsets[B+1] (offsets[0] = 0, offsets[B] = T); num_candidates[B] may be
 * NULL (causal mode, n_c = 0 for all sequences); timestamps[T] int64. */
typedef struct {
  int32_t batch, num_heads, d_qk, d_v;
  int32_t num_pos_buckets, num_time_buckets, time_bucket_sub_bits;
  int32_t rab_per_head;
  double alpha, silu_scale;
  const int64_t *offsets;
  const int32_t *num_candidates;
  const int64_t *timestamps;
} hstu_oracle_problem;

/* Integer bucket functions (R3, R4). */
int32_t hstu_oracle_time_bucket(int64_t dt, int32_t sub_bits, int32_t num_buckets);
int32_t hstu_oracle_pos_bucket(int64_t dp, int32_t num_buckets);

/* Visibility and position of local indices in a sequence of length L with
 * n_hist history tokens (n_hist = L in causal mode). */
int32_t hstu_oracle_visible(int64_t i, int64_t j, int64_t n_hist);
int64_t hstu_oracle_position(int64_t i, int64_t n_hist);

/* Per-pair buckets of every sequence, dense per sequence: for sequence b an
 * L_b x L_b int32 block (row i, column j) is appended to bp_out / bt_out;
 * invisible pairs hold -1.  Total size sum_b L_b^2. */
int hstu_oracle_buckets(const hstu_oracle_problem *p, int32_t *bp_out, int32_t *bt_out);

/* Forward attention.  rows == NULL: all T tokens, out is [T][H][d_v].
 * Otherwise only the n_rows listed global token indices, out is
 * [n_rows][H][d_v].  Returns 0 on success, nonzero on bad arguments. */
int hstu_oracle_attn_fwd(const hstu_oracle_problem *p, const double *q, const double *k,
                         const double *v, const double *rab_p, const double *rab_t,
                         const int64_t *rows, int64_t n_rows, double *out);

/* Backward attention (full).  dq, dk [T][H][d_qk]; dv [T][H][d_v] are
 * overwritten; drab_p, drab_t (same shape as rab_p / rab_t) are overwritten. */
int hstu_oracle_attn_bwd(const hstu_oracle_problem *p, const double *q, const double *k,
                         const double *v, const double *rab_p, const double *rab_t,
                         const double *dout, double *dq, double *dk, double *dv,
                         double *drab_p, double *drab_t);

/* Backward attention on samples, for sizes where the full pass is too slow.
 *  dq_rows[n_dq]  : global query tokens; dq_out [n_dq][H][d_qk]
 *  kv_cols[n_kv]  : global key tokens;   dk_out [n_kv][H][d_qk], dv_out [n_kv][H][d_v]
 *  drab_p_band    : if > 0, drab_p_out receives the sums of dS over the pairs whose
 *                   position bucket is < drab_p_band (entries >= band left 0);
 *                   drab_p_out may be NULL. */
int hstu_oracle_attn_bwd_sampled(const hstu_oracle_problem *p, const double *q, const double *k,
                                 const double *v, const double *rab_p, const double *rab_t,
                                 const double *dout, const int64_t *dq_rows, int64_t n_dq,
                                 double *dq_out, const int64_t *kv_cols, int64_t n_kv,
                                 double *dk_out, double *dv_out, int32_t drab_p_band,
                                 double *drab_p_out);

/* Both bias-table gradients in full, from the same per-pair definition as
 * hstu_oracle_attn_bwd (drab_p[bp] += dS, drab_t[bt] += dS over every visible
 * pair), without the dq / dk / dv sums: the work is split by (sequence, head,
 * 64 query rows) so that long single sequences use every thread.  Each piece
 * sums into its own partial table; the partials are added in a fixed order,
 * so the result does not depend on the thread count.  drab_p / drab_t are
 * written (not accumulated), shaped like rab_p / rab_t.  Returns 0, 1 on a
 * bad argument, 2 when out of memory. */
int hstu_oracle_attn_drab(const hstu_oracle_problem *p, const double *q, const double *k,
                          const double *v, const double *rab_p, const double *rab_t,
                          const double *dout, double *drab_p, double *drab_t);

/* Number of threads the oracle's parallel loops use (1 without OpenMP). */
int hstu_oracle_num_threads(void);

#ifdef __cplusplus
}
#endif
#endif
