// attn_bwd_common.cuh -- elementwise pieces shared by the tensor-core
// backward kernels: time-bucket index of a pair, d rab binning and the
// per-chunk SiLU backward (thread = key row, 32 query columns).
#pragma once

#include "internal.h"
#include "tile_common.cuh"

namespace hstu {
namespace bwd_ew {

// Kernel arguments of the tensor-core backward kernels.
struct BwdParams {
  const SeqInfo *seqs;
  const int4 *kitems;      // {seq, key tile, first query block, end query block (kUnsplit: all)}
  int32_t num_heads;
  const float *tf;
  const int64_t *ts;
  const int32_t *seq_fast;
  const float *rab_p, *rab_t;
  int32_t rab_per_head, nb_p, nb_t, sub_bits;
  float alpha;
  float dv_scale, dk_scale, drab_scale;
  __nv_bfloat16 *dk, *dv;
  int64_t dk_rs, dv_rs;
  int64_t total_tokens;
  float *dq_acc;           // [H][T][D]
  float *bin_acc;          // per-CTA d rab bins (position, then time), kBinAccPerCta each
  float *drab_p, *drab_t;
  WaitCtl wait;
  uint64_t drain_ns;
  float *dk_acc, *dv_acc;  // split key tiles: float32 partial dK, dV [split key rows][H][D]
  const int32_t *kitem_acc;  // first accumulator row of each item's key tile (split items)
};

// How a 32-column chunk bins its time-bias gradient (chosen warp-uniformly).
enum TMode : int {
  kTOne = 0,    // every lane's chunk lies in one bucket: plain chunk sum
  kTTwo = 1,    // at most two adjacent buckets per lane (fast, sorted times): split sum
  kTSlow = 2,   // anything else: per-element run-length with shared atomics
};

// Time-bucket table index of one pair (the same index the bias lookup uses).
template <bool FAST_T>
__device__ __forceinline__ int32_t time_index(const int64_t *tq, int c, float t_j_f, int64_t t_j,
                                              int sh, int32_t r0, int sub_bits, int nb_t) {
  if constexpr (FAST_T) {
    const float dt = reinterpret_cast<const float *>(tq)[c] - t_j_f;
    const int32_t rr = __float_as_int(dt) >> sh;
    return (rr > r0 ? rr : r0) - r0;
  } else {
    return time_bucket_i64(tq[c] - t_j, sub_bits, nb_t);
  }
}

__device__ __forceinline__ void flush_bin(float *hist, int b, float v) {
  if (v != 0.0f) atomicAdd(hist + b, v);
}

// Warp-collective flush (all 32 lanes call it, converged): the lanes that
// want to add v to bin b are grouped by bin, each group is summed with
// shuffles and one lane issues a single shared atomic.  Neighbouring keys
// usually share a bin, so this replaces up to 32 contended atomics on one
// address with one.
__device__ __forceinline__ void flush_warp(float *hist, int b, float v, bool want) {
  const int lane = threadIdx.x & 31;
  unsigned m = __ballot_sync(0xffffffffu, want && v != 0.0f);
  while (m) {
    const int leader = __ffs(m) - 1;
    const int lb = __shfl_sync(0xffffffffu, b, leader);
    const bool mine = ((m >> lane) & 1u) && b == lb;
    float s = mine ? v : 0.0f;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    if (lane == leader) atomicAdd(hist + lb, s);
    m &= ~__ballot_sync(0xffffffffu, mine);
  }
}

// Elementwise backward of one W-column chunk (W <= 32; thread = key row j):
//   h = s/2, t = tanh h, P = h (1 + t) = SiLU(s), g = (1 + t)(1 + h (1 - t)) = 2 SiLU'(s),
//   dS' = dA g; masked pairs give 0.  d rab sums: see TMode.  Position bins
// are per pair only near the diagonal (GATHER_P); elsewhere every pair is in
// the last bin and goes to a register sum.  Near the diagonal, with every
// query row a history row (DIAG_P), a pair's bin is the diagonal index
// i - j (clamped): lane l's element e lies on diagonal base + e - l, so one
// shuffle per element hands it to lane (e - l) mod 32, which keeps two
// register sums, p_hi for diagonal base + lane and p_lo for base + lane - 32.
// Otherwise (candidate rows) each pair goes to its bin, the clamp bin and
// zeros excepted.  With GRED the per-lane adds (run ends, per-pair position
// bins) are fire-and-forget float reductions into the CTA's own bins in
// global memory (gbin_p, gbin_t); shared-memory float atomics are a
// compare-and-swap loop, an order of magnitude slower under divergence.
template <int W, bool MASK, bool GATHER_P, bool FAST_T, int TMODE, bool DIAG_P, bool GRED,
          class SM>
__device__ __forceinline__ void bwd_chunk(const uint32_t (&rs)[W], const uint32_t (&rd)[W],
                                          uint32_t (&pk_p)[W / 2], uint32_t (&pk_d)[W / 2],
                                          SM &sm, const int64_t *tq, int cc, int32_t qs,
                                          int32_t j,
                                          int32_t pos_j, float t_j_f, int64_t t_j,
                                          float alpha_h, float row_c, const TileGeom &g,
                                          int nb_p_m1, int sub_bits, int nb_t, int32_t b_first, float uni_tb,
                                          float &s_all, float &s_lo, int &cur_b, float &acc_b,
                                          float &acc_far, float &p_hi, float &p_lo,
                                          float *gbin_p, float *gbin_t) {
  const int lane = threadIdx.x & 31;
  const int sh = 23 - sub_bits;
  const int32_t r0 = fast_r0(sub_bits);
  // kTTwo: the lane's pairs lie in bucket b_first or b_first + 1.  With the
  // exponent-table index max(bits(dt) >> sh, r0) - r0, "bucket >= b_first + 1"
  // is exactly dt >= the float whose bits are (b_first + 1 + r0) << sh (dt is
  // never negative here), so one compare picks the bias and the sum.
  static_assert(TMODE != kTTwo || FAST_T, "the two-bucket split needs float time deltas");
  float thr = 0.f, c_lo = 0.f, c_hi = 0.f;
  if constexpr (TMODE == kTTwo) {
    // t_q - t_j >= thr  <=>  t_q >= t_j + thr: both times and thr are
    // integers below 2^24 and the sum rounds monotonically, so the compare
    // is exact either way and the per-pair subtraction goes.
    thr = t_j_f + __int_as_float((b_first + 1 + r0) << sh);
    c_lo = sm.tbl_t[b_first];
    c_hi = sm.tbl_t[b_first + 1];
    if constexpr (!GATHER_P) {
      c_lo += row_c;
      c_hi += row_c;
    }
  }
  // the chunk's query times are the same for every lane: 16-byte loads,
  // four queries at a time, instead of one shared load per element
  float tq4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int e = 0; e < W; e += 2) {
    float pv[2], dv[2];
    if constexpr (FAST_T && TMODE != kTOne) {
      if ((e & 3) == 0) {
        const float4 t4 =
            *reinterpret_cast<const float4 *>(reinterpret_cast<const float *>(tq) + cc + e);
        tq4[0] = t4.x;
        tq4[1] = t4.y;
        tq4[2] = t4.z;
        tq4[3] = t4.w;
      }
    }
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int c = cc + e + u;             // query column within the tile
      const int32_t i = qs + c;             // local query index
      const float tqc = tq4[(e & 3) + u];   // the query's float time (float-time paths)
      float h;
      int32_t bp = nb_p_m1;
      bool hi = false;   // kTTwo: the pair is in bucket b_first + 1
      if constexpr (TMODE == kTTwo) hi = tqc >= thr;
      if constexpr (GATHER_P) {
        const int32_t dp = g.pos(i) - pos_j;
        bp = dp < nb_p_m1 ? (dp > 0 ? dp : 0) : nb_p_m1;
        const float cp = TMODE == kTOne   ? sm.tbl_p[bp] + uni_tb
                         : TMODE == kTTwo ? sm.tbl_p[bp] + (hi ? c_hi : c_lo)
                                          : sm.tbl_p[bp];
        h = fmaf(alpha_h, __uint_as_float(rs[e + u]), cp);
      } else {
        h = fmaf(alpha_h, __uint_as_float(rs[e + u]), TMODE == kTTwo ? (hi ? c_hi : c_lo) : row_c);
      }
      // one-bucket chunks carry their time bias in the row constant / uni_tb,
      // two-bucket chunks in c_lo / c_hi
      int32_t bt = 0;
      if constexpr (TMODE == kTSlow) {
        if constexpr (FAST_T) {
          const int32_t rr = __float_as_int(tqc - t_j_f) >> sh;
          bt = (rr > r0 ? rr : r0) - r0;
        } else {
          bt = time_index<FAST_T>(tq, c, t_j_f, t_j, sh, r0, sub_bits, nb_t);
        }
        h += sm.tbl_t[bt];
      }
      const float t = tanh_approx(h);
      const float t1 = 1.0f + t;
      float p = h * t1;                                // SiLU(s) = h (1 + t)
      const float gg = fmaf(t1, fmaf(-h, t, h), t1);   // 2 SiLU'(s) = (1 + t)(1 + h (1 - t))
      float ds = __uint_as_float(rd[e + u]) * gg;
      if constexpr (MASK) {
        const bool vis = g.visible(i, j);
        p = vis ? p : 0.0f;
        ds = vis ? ds : 0.0f;
      }
      pv[u] = p;
      dv[u] = ds;
      if constexpr (TMODE == kTOne) {
        s_all += ds;
      } else if constexpr (TMODE == kTTwo) {
        s_all += ds;
        s_lo += hi ? 0.0f : ds;
      } else {
        if (bt != cur_b) {
          if constexpr (GRED) {
            if (acc_b != 0.0f) red_add_f32(gbin_t + cur_b, acc_b);
          } else {
            flush_bin(sm.hist_t, cur_b, acc_b);
          }
          cur_b = bt;
          acc_b = 0.0f;
        }
        acc_b += ds;
      }
      if constexpr (GATHER_P && DIAG_P) {
        const float rr = __shfl_sync(0xffffffffu, ds, (e + u) - lane);
        if (lane <= e + u)
          p_hi += rr;
        else
          p_lo += rr;
      } else if constexpr (GATHER_P) {
        if (bp == nb_p_m1) {
          acc_far += ds;
        } else if (ds != 0.0f) {
          if constexpr (GRED)
            red_add_f32(gbin_p + bp, ds);
          else
            atomicAdd(&sm.hist_p[bp], ds);
        }
      } else if constexpr (TMODE == kTSlow) {
        acc_far += ds;
      }
    }
    pk_p[e / 2] = pack_bf16x2(pv[0], pv[1]);
    pk_d[e / 2] = pack_bf16x2(dv[0], dv[1]);
  }
}

}  // namespace bwd_ew
}  // namespace hstu
