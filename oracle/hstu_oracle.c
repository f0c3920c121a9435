/*
 * hstu_oracle.c -- plain CPU oracle of HSTU pointwise attention, float64.
 *
 * TEST INFRASTRUCTURE ONLY (tests, smoke check, benchmark CPU baseline).
 * Written straight from the definition stated in hstu_oracle.h: one loop
 * over (sequence, head, query i, key j), no tiling, no fusion, no reordering
 * beyond what the definition states.  Sources:
 *   [DLRMv4] "DLRMv4: MLPerf's recommendation-training benchmark enters the
 *            sequence era" (winzheng.jp), sections "Model architecture: HSTU
 *            replaces the feature-interaction stack" and "How one training
 *            sample is processed by HSTU".
 *   [GR]     "Actions Speak Louder than Words" (arXiv 2402.17152), abstract
 *            and the M-FALCON item of the contribution list.
 */
#include "hstu_oracle.h"

#include <math.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

int hstu_oracle_num_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

/* floor(log2(x)) for x >= 1, by counting halvings. */
static int floor_log2_i64(int64_t x) {
  int e = 0;
  while (x > 1) {
    x >>= 1;
    ++e;
  }
  return e;
}

/* [DLRMv4, "Model architecture"]: the bias depends on the temporal distance
 * of two events.  Reading R4: logarithmic buckets with sub_bits bits of
 * sub-octave resolution; non-positive distances fall in bucket 0, distances
 * below 2^s get a bucket each, and everything saturates in the last bucket. */
int32_t hstu_oracle_time_bucket(int64_t dt, int32_t sub_bits, int32_t num_buckets) {
  int64_t b;
  const int64_t s = sub_bits;
  if (dt <= 0) {
    b = 0;
  } else if (dt < ((int64_t)1 << s)) {
    b = dt;
  } else {
    const int64_t e = floor_log2_i64(dt);
    b = (e - s + 1) * ((int64_t)1 << s) + (dt >> (e - s)) - ((int64_t)1 << s);
  }
  if (b > num_buckets - 1) b = num_buckets - 1;
  return (int32_t)b;
}

/* [DLRMv4, "Model architecture"]: the bias depends on the positional distance
 * of two events.  Reading R3: clamped linear distance. */
int32_t hstu_oracle_pos_bucket(int64_t dp, int32_t num_buckets) {
  if (dp < 0) dp = 0;
  if (dp > num_buckets - 1) dp = num_buckets - 1;
  return (int32_t)dp;
}

/* [DLRMv4, "How one training sample is processed"]: the stack runs over one
 * causal sequence with the candidates appended at its end; [GR] M-FALCON
 * scores many candidates in one pass.  Reading R6: a history query sees every
 * earlier-or-equal event; a candidate sees the whole history and itself only. */
int32_t hstu_oracle_visible(int64_t i, int64_t j, int64_t n_hist) {
  if (i < n_hist) return j <= i;
  return j < n_hist || j == i;
}

/* Reading R7: every candidate sits at position n_hist (right after the history). */
int64_t hstu_oracle_position(int64_t i, int64_t n_hist) { return i < n_hist ? i : n_hist; }

static int check_problem(const hstu_oracle_problem *p) {
  if (!p || p->batch < 0 || p->num_heads <= 0 || p->d_qk <= 0 || p->d_v <= 0) return 1;
  if (p->num_pos_buckets <= 0 || p->num_time_buckets <= 0) return 1;
  if (p->time_bucket_sub_bits < 0 || p->time_bucket_sub_bits > 30) return 1;
  if (!p->offsets || !p->timestamps) return 1;
  if (p->offsets[0] != 0) return 1;
  for (int32_t b = 0; b < p->batch; ++b) {
    if (p->offsets[b + 1] < p->offsets[b]) return 1;
    if (p->num_candidates) {
      const int64_t L = p->offsets[b + 1] - p->offsets[b];
      if (p->num_candidates[b] < 0 || p->num_candidates[b] > L) return 1;
    }
  }
  return 0;
}

static int64_t n_hist_of(const hstu_oracle_problem *p, int32_t b) {
  const int64_t L = p->offsets[b + 1] - p->offsets[b];
  return L - (p->num_candidates ? p->num_candidates[b] : 0);
}

/* Index of global token t's sequence (linear search; the oracle is not fast). */
static int32_t seq_of_token(const hstu_oracle_problem *p, int64_t t) {
  for (int32_t b = 0; b < p->batch; ++b)
    if (t >= p->offsets[b] && t < p->offsets[b + 1]) return b;
  return -1;
}

/* The logit of one visible pair (global tokens gi, gj) for head h. */
static double pair_logit(const hstu_oracle_problem *p, int32_t b, int32_t h, int64_t gi,
                         int64_t gj, const double *q, const double *k, const double *rab_p,
                         const double *rab_t, int32_t *bp_out, int32_t *bt_out) {
  const int64_t o = p->offsets[b];
  const int64_t nh = n_hist_of(p, b);
  const int64_t H = p->num_heads, dqk = p->d_qk;
  const double *qi = q + (gi * H + h) * dqk;
  const double *kj = k + (gj * H + h) * dqk;
  double dot = 0.0;
  for (int64_t c = 0; c < dqk; ++c) dot += qi[c] * kj[c];
  const int64_t dp = hstu_oracle_position(gi - o, nh) - hstu_oracle_position(gj - o, nh);
  const int32_t bp = hstu_oracle_pos_bucket(dp, p->num_pos_buckets);
  const int32_t bt = hstu_oracle_time_bucket(p->timestamps[gi] - p->timestamps[gj],
                                             p->time_bucket_sub_bits, p->num_time_buckets);
  const double *tp = rab_p + (p->rab_per_head ? (int64_t)h * p->num_pos_buckets : 0);
  const double *tt = rab_t + (p->rab_per_head ? (int64_t)h * p->num_time_buckets : 0);
  if (bp_out) *bp_out = bp;
  if (bt_out) *bt_out = bt;
  return p->alpha * dot + tp[bp] + tt[bt];
}

static double sigmoid(double x) { return 1.0 / (1.0 + exp(-x)); }

int hstu_oracle_buckets(const hstu_oracle_problem *p, int32_t *bp_out, int32_t *bt_out) {
  if (check_problem(p) || !bp_out || !bt_out) return 1;
  int64_t base = 0;
  for (int32_t b = 0; b < p->batch; ++b) {
    const int64_t o = p->offsets[b], L = p->offsets[b + 1] - o, nh = n_hist_of(p, b);
    for (int64_t i = 0; i < L; ++i) {
      for (int64_t j = 0; j < L; ++j) {
        const int64_t idx = base + i * L + j;
        if (!hstu_oracle_visible(i, j, nh)) {
          bp_out[idx] = -1;
          bt_out[idx] = -1;
          continue;
        }
        const int64_t dp = hstu_oracle_position(i, nh) - hstu_oracle_position(j, nh);
        bp_out[idx] = hstu_oracle_pos_bucket(dp, p->num_pos_buckets);
        bt_out[idx] = hstu_oracle_time_bucket(p->timestamps[o + i] - p->timestamps[o + j],
                                              p->time_bucket_sub_bits, p->num_time_buckets);
      }
    }
    base += L * L;
  }
  return 0;
}

/* o_i for one query token gi and head h, written to out_row[d_v]. */
static void fwd_row(const hstu_oracle_problem *p, int32_t b, int32_t h, int64_t gi,
                    const double *q, const double *k, const double *v, const double *rab_p,
                    const double *rab_t, double *out_row) {
  const int64_t o = p->offsets[b], L = p->offsets[b + 1] - o, nh = n_hist_of(p, b);
  const int64_t H = p->num_heads, dv = p->d_v;
  for (int64_t c = 0; c < dv; ++c) out_row[c] = 0.0;
  const int64_t i = gi - o;
  for (int64_t j = 0; j < L; ++j) {
    if (!hstu_oracle_visible(i, j, nh)) continue;
    const double s = pair_logit(p, b, h, gi, o + j, q, k, rab_p, rab_t, NULL, NULL);
    const double a = p->silu_scale * s * sigmoid(s);
    const double *vj = v + ((o + j) * H + h) * dv;
    for (int64_t c = 0; c < dv; ++c) out_row[c] += a * vj[c];
  }
}

int hstu_oracle_attn_fwd(const hstu_oracle_problem *p, const double *q, const double *k,
                         const double *v, const double *rab_p, const double *rab_t,
                         const int64_t *rows, int64_t n_rows, double *out) {
  if (check_problem(p) || !q || !k || !v || !rab_p || !rab_t || !out) return 1;
  const int64_t T = p->offsets[p->batch];
  const int64_t H = p->num_heads, dv = p->d_v;
  const int64_t n = rows ? n_rows : T;
  for (int64_t r = 0; r < n; ++r) {
    const int64_t gi = rows ? rows[r] : r;
    if (gi < 0 || gi >= T) return 1;
  }
  int64_t r;
#pragma omp parallel for schedule(dynamic, 1)
  for (r = 0; r < n; ++r) {
    const int64_t gi = rows ? rows[r] : r;
    const int32_t b = seq_of_token(p, gi);
    for (int32_t h = 0; h < p->num_heads; ++h)
      fwd_row(p, b, h, gi, q, k, v, rab_p, rab_t, out + (r * H + h) * dv);
  }
  return 0;
}

/* Gradient of one visible pair, shared by the full and the sampled backward.
 * With a = silu_scale * SiLU(s) and SiLU'(s) = sigma(s) (1 + s (1 - sigma(s))):
 *   dA = <dO_i, v_j>;  dS = dA * silu_scale * SiLU'(s)
 *   dV_j += a dO_i;  dQ_i += alpha dS k_j;  dK_j += alpha dS q_i;
 *   drab_p[bp] += dS;  drab_t[bt] += dS. */
typedef struct {
  double a, dS;
  int32_t bp, bt;
} pair_grad;

static pair_grad pair_backward(const hstu_oracle_problem *p, int32_t b, int32_t h, int64_t gi,
                               int64_t gj, const double *q, const double *k, const double *v,
                               const double *rab_p, const double *rab_t, const double *dout) {
  const int64_t H = p->num_heads, dv = p->d_v;
  pair_grad g;
  const double s = pair_logit(p, b, h, gi, gj, q, k, rab_p, rab_t, &g.bp, &g.bt);
  const double sg = sigmoid(s);
  const double *doi = dout + (gi * H + h) * dv;
  const double *vj = v + (gj * H + h) * dv;
  double dA = 0.0;
  for (int64_t c = 0; c < dv; ++c) dA += doi[c] * vj[c];
  g.a = p->silu_scale * s * sg;
  g.dS = dA * p->silu_scale * sg * (1.0 + s * (1.0 - sg));
  return g;
}

int hstu_oracle_attn_bwd(const hstu_oracle_problem *p, const double *q, const double *k,
                         const double *v, const double *rab_p, const double *rab_t,
                         const double *dout, double *dq, double *dk, double *dv,
                         double *drab_p, double *drab_t) {
  if (check_problem(p) || !q || !k || !v || !rab_p || !rab_t || !dout || !dq || !dk || !dv ||
      !drab_p || !drab_t)
    return 1;
  const int64_t T = p->offsets[p->batch];
  const int64_t H = p->num_heads, dqk = p->d_qk, dvv = p->d_v;
  const int64_t nbp = p->num_pos_buckets, nbt = p->num_time_buckets;
  const int64_t tabs = p->rab_per_head ? H : 1;
  memset(dq, 0, sizeof(double) * T * H * dqk);
  memset(dk, 0, sizeof(double) * T * H * dqk);
  memset(dv, 0, sizeof(double) * T * H * dvv);
  memset(drab_p, 0, sizeof(double) * tabs * nbp);
  memset(drab_t, 0, sizeof(double) * tabs * nbt);
  /* One private drab pair per (sequence, head), summed in a fixed order
   * afterwards so the result does not depend on the thread count. */
  const int64_t units = (int64_t)p->batch * H;
  double *part_p = (double *)calloc((size_t)(units * nbp + 1), sizeof(double));
  double *part_t = (double *)calloc((size_t)(units * nbt + 1), sizeof(double));
  if (!part_p || !part_t) {
    free(part_p);
    free(part_t);
    return 2;
  }
  int64_t u;
#pragma omp parallel for schedule(dynamic, 1)
  for (u = 0; u < units; ++u) {
    const int32_t b = (int32_t)(u / H), h = (int32_t)(u % H);
    const int64_t o = p->offsets[b], L = p->offsets[b + 1] - o, nh = n_hist_of(p, b);
    for (int64_t i = 0; i < L; ++i) {
      for (int64_t j = 0; j < L; ++j) {
        if (!hstu_oracle_visible(i, j, nh)) continue;
        const int64_t gi = o + i, gj = o + j;
        const pair_grad g = pair_backward(p, b, h, gi, gj, q, k, v, rab_p, rab_t, dout);
        const double *doi = dout + (gi * H + h) * dvv;
        const double *qi = q + (gi * H + h) * dqk;
        const double *kj = k + (gj * H + h) * dqk;
        double *dvj = dv + (gj * H + h) * dvv;
        double *dqi = dq + (gi * H + h) * dqk;
        double *dkj = dk + (gj * H + h) * dqk;
        for (int64_t c = 0; c < dvv; ++c) dvj[c] += g.a * doi[c];
        for (int64_t c = 0; c < dqk; ++c) {
          dqi[c] += p->alpha * g.dS * kj[c];
          dkj[c] += p->alpha * g.dS * qi[c];
        }
        part_p[u * nbp + g.bp] += g.dS;
        part_t[u * nbt + g.bt] += g.dS;
      }
    }
  }
  for (u = 0; u < units; ++u) {
    const int64_t tab = p->rab_per_head ? (u % H) : 0;
    for (int64_t x = 0; x < nbp; ++x) drab_p[tab * nbp + x] += part_p[u * nbp + x];
    for (int64_t x = 0; x < nbt; ++x) drab_t[tab * nbt + x] += part_t[u * nbt + x];
  }
  free(part_p);
  free(part_t);
  return 0;
}

int hstu_oracle_attn_drab(const hstu_oracle_problem *p, const double *q, const double *k,
                          const double *v, const double *rab_p, const double *rab_t,
                          const double *dout, double *drab_p, double *drab_t) {
  if (check_problem(p) || !q || !k || !v || !rab_p || !rab_t || !dout || !drab_p || !drab_t)
    return 1;
  const int64_t H = p->num_heads;
  const int64_t nbp = p->num_pos_buckets, nbt = p->num_time_buckets;
  const int64_t tabs = p->rab_per_head ? H : 1;
  const int64_t rows = 64;
  /* pieces: (sequence b, head h, query rows [r0, r0 + 64)) in order */
  int64_t n_pieces = 0;
  for (int32_t b = 0; b < p->batch; ++b) {
    const int64_t L = p->offsets[b + 1] - p->offsets[b];
    n_pieces += H * ((L + rows - 1) / rows);
  }
  int64_t *piece_b = (int64_t *)calloc((size_t)(n_pieces + 1), sizeof(int64_t));
  double *part_p = (double *)calloc((size_t)(n_pieces * nbp + 1), sizeof(double));
  double *part_t = (double *)calloc((size_t)(n_pieces * nbt + 1), sizeof(double));
  if (!piece_b || !part_p || !part_t) {
    free(piece_b);
    free(part_p);
    free(part_t);
    return 2;
  }
  /* piece index -> (b, h, r0) packed as b * 2^40 + h * 2^20 + chunk */
  int64_t x = 0;
  for (int32_t b = 0; b < p->batch; ++b) {
    const int64_t L = p->offsets[b + 1] - p->offsets[b];
    for (int64_t h = 0; h < H; ++h)
      for (int64_t c = 0; c * rows < L; ++c) piece_b[x++] = ((int64_t)b << 40) | (h << 20) | c;
  }
  int64_t u;
#pragma omp parallel for schedule(dynamic, 1)
  for (u = 0; u < n_pieces; ++u) {
    const int32_t b = (int32_t)(piece_b[u] >> 40);
    const int32_t h = (int32_t)((piece_b[u] >> 20) & 0xFFFFF);
    const int64_t c = piece_b[u] & 0xFFFFF;
    const int64_t o = p->offsets[b], L = p->offsets[b + 1] - o, nh = n_hist_of(p, b);
    const int64_t i1 = (c + 1) * rows < L ? (c + 1) * rows : L;
    for (int64_t i = c * rows; i < i1; ++i) {
      for (int64_t j = 0; j < L; ++j) {
        if (!hstu_oracle_visible(i, j, nh)) continue;
        const pair_grad g = pair_backward(p, b, h, o + i, o + j, q, k, v, rab_p, rab_t, dout);
        part_p[u * nbp + g.bp] += g.dS;
        part_t[u * nbt + g.bt] += g.dS;
      }
    }
  }
  memset(drab_p, 0, sizeof(double) * tabs * nbp);
  memset(drab_t, 0, sizeof(double) * tabs * nbt);
  for (u = 0; u < n_pieces; ++u) {
    const int64_t tab = p->rab_per_head ? ((piece_b[u] >> 20) & 0xFFFFF) : 0;
    for (int64_t y = 0; y < nbp; ++y) drab_p[tab * nbp + y] += part_p[u * nbp + y];
    for (int64_t y = 0; y < nbt; ++y) drab_t[tab * nbt + y] += part_t[u * nbt + y];
  }
  free(piece_b);
  free(part_p);
  free(part_t);
  return 0;
}

int hstu_oracle_attn_bwd_sampled(const hstu_oracle_problem *p, const double *q, const double *k,
                                 const double *v, const double *rab_p, const double *rab_t,
                                 const double *dout, const int64_t *dq_rows, int64_t n_dq,
                                 double *dq_out, const int64_t *kv_cols, int64_t n_kv,
                                 double *dk_out, double *dv_out, int32_t drab_p_band,
                                 double *drab_p_out) {
  if (check_problem(p) || !q || !k || !v || !rab_p || !rab_t || !dout) return 1;
  const int64_t T = p->offsets[p->batch];
  const int64_t H = p->num_heads, dqk = p->d_qk, dvv = p->d_v;
  for (int64_t r = 0; r < n_dq; ++r)
    if (!dq_rows || !dq_out || dq_rows[r] < 0 || dq_rows[r] >= T) return 1;
  for (int64_t r = 0; r < n_kv; ++r)
    if (!kv_cols || !dk_out || !dv_out || kv_cols[r] < 0 || kv_cols[r] >= T) return 1;
  int64_t r;
  /* dQ_i needs row i only. */
#pragma omp parallel for schedule(dynamic, 1)
  for (r = 0; r < n_dq; ++r) {
    const int64_t gi = dq_rows[r];
    const int32_t b = seq_of_token(p, gi);
    const int64_t o = p->offsets[b], L = p->offsets[b + 1] - o, nh = n_hist_of(p, b);
    for (int32_t h = 0; h < H; ++h) {
      double *dqi = dq_out + (r * H + h) * dqk;
      for (int64_t c = 0; c < dqk; ++c) dqi[c] = 0.0;
      for (int64_t j = 0; j < L; ++j) {
        if (!hstu_oracle_visible(gi - o, j, nh)) continue;
        const pair_grad g = pair_backward(p, b, h, gi, o + j, q, k, v, rab_p, rab_t, dout);
        const double *kj = k + ((o + j) * H + h) * dqk;
        for (int64_t c = 0; c < dqk; ++c) dqi[c] += p->alpha * g.dS * kj[c];
      }
    }
  }
  /* dK_j, dV_j need column j only. */
#pragma omp parallel for schedule(dynamic, 1)
  for (r = 0; r < n_kv; ++r) {
    const int64_t gj = kv_cols[r];
    const int32_t b = seq_of_token(p, gj);
    const int64_t o = p->offsets[b], L = p->offsets[b + 1] - o, nh = n_hist_of(p, b);
    for (int32_t h = 0; h < H; ++h) {
      double *dkj = dk_out + (r * H + h) * dqk;
      double *dvj = dv_out + (r * H + h) * dvv;
      for (int64_t c = 0; c < dqk; ++c) dkj[c] = 0.0;
      for (int64_t c = 0; c < dvv; ++c) dvj[c] = 0.0;
      for (int64_t i = 0; i < L; ++i) {
        if (!hstu_oracle_visible(i, gj - o, nh)) continue;
        const pair_grad g = pair_backward(p, b, h, o + i, gj, q, k, v, rab_p, rab_t, dout);
        const double *qi = q + ((o + i) * H + h) * dqk;
        const double *doi = dout + ((o + i) * H + h) * dvv;
        for (int64_t c = 0; c < dqk; ++c) dkj[c] += p->alpha * g.dS * qi[c];
        for (int64_t c = 0; c < dvv; ++c) dvj[c] += g.a * doi[c];
      }
    }
  }
  /* drab_p over the pairs whose position bucket is below the band: these
   * pairs lie within drab_p_band - 1 positions of each other. */
  if (drab_p_band > 0 && drab_p_out) {
    const int64_t nbp = p->num_pos_buckets;
    const int64_t tabs = p->rab_per_head ? H : 1;
    const int64_t units = (int64_t)p->batch * H;
    double *part = (double *)calloc((size_t)(units * nbp + 1), sizeof(double));
    if (!part) return 2;
    int64_t u;
#pragma omp parallel for schedule(dynamic, 1)
    for (u = 0; u < units; ++u) {
      const int32_t b = (int32_t)(u / H), h = (int32_t)(u % H);
      const int64_t o = p->offsets[b], L = p->offsets[b + 1] - o, nh = n_hist_of(p, b);
      for (int64_t i = 0; i < L; ++i) {
        /* Keys before pos(i) - band + 1 are at least band positions away. */
        int64_t j0 = hstu_oracle_position(i, nh) - drab_p_band + 1;
        if (j0 < 0) j0 = 0;
        for (int64_t j = j0; j < L; ++j) {
          if (!hstu_oracle_visible(i, j, nh)) continue;
          const int64_t dp = hstu_oracle_position(i, nh) - hstu_oracle_position(j, nh);
          if (hstu_oracle_pos_bucket(dp, p->num_pos_buckets) >= drab_p_band) continue;
          const pair_grad g = pair_backward(p, b, h, o + i, o + j, q, k, v, rab_p, rab_t, dout);
          part[u * nbp + g.bp] += g.dS;
        }
      }
    }
    for (int64_t x = 0; x < tabs * nbp; ++x) drab_p_out[x] = 0.0;
    for (u = 0; u < units; ++u) {
      const int64_t tab = p->rab_per_head ? (u % H) : 0;
      for (int64_t x = 0; x < nbp; ++x) drab_p_out[tab * nbp + x] += part[u * nbp + x];
    }
    free(part);
  }
  return 0;
}
