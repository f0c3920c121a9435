// attn_bwd_sm100.cu -- backward HSTU pointwise attention on the 5th-generation
// tensor cores (tcgen05 + tensor memory + TMA), bf16 in, fp32 accumulate.
//
// Gradients of out_i = silu_scale sum_j SiLU(s_ij) v_j with
// s_ij = alpha <q_i,k_j> + rab_p[bp_ij] + rab_t[bt_ij] (include/hstu.h; the
// pointwise aggregation with positional and temporal bias of the DLRMv4
// article, section "Model architecture: HSTU replaces the feature-interaction
// stack"):
//   dA_ij = <dout_i, v_j>,  dS_ij = dA_ij silu_scale SiLU'(s_ij)
//   dv_j = silu_scale sum_i SiLU(s_ij) dout_i,  dk_j = alpha sum_i dS_ij q_i
//   dq_i = alpha sum_j dS_ij k_j,  drab_*[bucket_ij] += dS_ij.
//
// This file holds the d_qk = d_v = 64 kernel (d = 128 has its own,
// attn_bwd128_sm100.cu), the dQ conversion shared by both, and the dispatch.
//
// Design (one CTA = one (sequence, head, 128-key tile); loop over the
// 128-query tiles that can see the keys, each split into two 64-query halves,
// one per elementwise warpgroup):
//   warp 0      TMA producer: K and V once, then Q and dout per query tile;
//               stages the queries' timestamps.
//   warp 1      tcgen05 issuer: S^T_x = K Q_x^T and dP^T_x = V dout_x^T per
//               half x; dV += P^T_x dout_x and dK += dS^T_x Q_x with P^T and
//               dS^T read from tensor memory; dQ_part = dS K (M = queries)
//               with dS from shared memory.
//   warps 4-11  two elementwise warpgroups (thread = key row, 64 query columns
//               each): bias, SiLU, SiLU', mask, d rab partial sums; then
//               (thread = query row) group x stages the d-columns [x D/2,
//               (x+1) D/2) of the dQ partial, 32 at a time, in its half of the
//               freed dS tile and one thread adds it to the float32
//               accumulator with a TMA bulk tensor reduce-add; at the end dV
//               (group 0) and dK (group 1) leave tensor memory as bf16.
// Tensor memory (512 columns): half x owns [128x, 128x + 128): S^T at +0
// (P^T over its first 32 columns), dP^T at +64 (dS^T over its first 32);
// dQ_part [128, 128 + D) once the second half's S^T / dP^T are consumed;
// dV [256, 256 + D); dK [384, 384 + D).
// Scales: the kernel works with h = s/2, t = tanh h, p = h (1 + t) = SiLU(s)
// and g = (1 + t)(1 + h - h t) = 2 SiLU'(s); dV gets silu_scale, dK / dQ
// alpha silu_scale / 2, d rab silu_scale / 2.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>

#include "attn_bwd_common.cuh"
#include "internal.h"

namespace hstu {
namespace bwd_tc {
using namespace bwd_ew;

constexpr int kTile = kAttnTile;
constexpr int kThreads = 384;
constexpr int kMaxTbl = 512;
static_assert(2 * kMaxTbl <= kBinAccPerCta, "per-CTA bins hold both tables");

using Params = BwdParams;

template <int D>
struct Smem {
  static constexpr int kTileBytes = kTile * D * 2;
  alignas(1024) uint8_t k[kTileBytes];
  alignas(1024) uint8_t v[kTileBytes];
  alignas(1024) uint8_t q[2][kTileBytes];        // query tiles, 2-stage ring
  alignas(1024) uint8_t dout[kTileBytes];        // reloaded once dV is done with it
  alignas(1024) uint8_t ds[kTile * kTile * 2];   // dS, [key][query], 2 chunks of 64 queries
  alignas(16) int64_t tq[2][kTile];              // query timestamps per Q stage
  float tbl_p[kMaxTbl];
  float tbl_t[kMaxTbl];
  float hist_p[kMaxTbl];
  float hist_t[kMaxTbl];
  uint64_t kv_full, q_full[2], t_full[2], q_empty[2], do_full, do_empty;
  uint64_t s_full[2], p_full[2], dq_full, dq_empty, done, drain;
  uint32_t tmem_base;
};

// Tensor-memory columns.  Query half x (queries 64x .. 64x+63) owns
// [128x, 128x+128): S^T at +0 (P^T written over its first 32 columns) and
// dP^T at +64 (dS^T over its first 32).  dQ_part takes [128, 128+D) once the
// second half's S^T / dP^T are consumed; dV [256, 256+D); dK [384, 384+D).
__host__ __device__ constexpr uint32_t s_col(int x) { return uint32_t(128 * x); }
__host__ __device__ constexpr uint32_t dp_col(int x) { return uint32_t(128 * x + 64); }
constexpr uint32_t kDqCol = 128, kDvCol = 256, kDkCol = 384;

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    bwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
               const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
               const __grid_constant__ CUtensorMap tm_dq, const Params p) {
  extern __shared__ uint8_t smem_raw[];
  Smem<D> &sm = *reinterpret_cast<Smem<D> *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int32_t item_idx = blockIdx.x / p.num_heads;
  const int32_t h = blockIdx.x % p.num_heads;
  const int4 item = p.kitems[item_idx];   // never split for this kernel (.z, .w unused)
  const SeqInfo sq = p.seqs[item.x];
  const TileGeom g{sq.len, sq.n_hist};
  const int32_t kt = item.y;
  const int32_t n_qt = (g.L + kTile - 1) / kTile;
  const bool fast = (p.seq_fast[item.x] & kSeqFastTime) != 0 && p.sub_bits <= 4;
  const int tab = p.rab_per_head ? h : 0;

  // ---- tables and histograms ----
  {
    const float *rp = p.rab_p + tab * p.nb_p;
    const float *rt = p.rab_t + tab * p.nb_t;
    for (int x = tid; x < p.nb_p; x += kThreads) sm.tbl_p[x] = 0.5f * rp[x];
    const int nt = fast ? fast_table_size(p.sub_bits) : p.nb_t;
    for (int x = tid; x < nt; x += kThreads)
      sm.tbl_t[x] = 0.5f * rt[fast ? fast_table_bucket(x, p.sub_bits, p.nb_t) : x];
    for (int x = tid; x < kMaxTbl; x += kThreads) {
      sm.hist_p[x] = 0.f;
      sm.hist_t[x] = 0.f;
    }
  }
  if (warp == 0 && lane == 0) {
    mbar_init(&sm.kv_full, 1);
    for (int s2 = 0; s2 < 2; ++s2) {
      mbar_init(&sm.q_full[s2], 1);
      mbar_init(&sm.t_full[s2], 32);
      mbar_init(&sm.q_empty[s2], 1);
      mbar_init(&sm.s_full[s2], 1);
      mbar_init(&sm.p_full[s2], 128);
    }
    mbar_init(&sm.do_full, 1);
    mbar_init(&sm.do_empty, 1);
    mbar_init(&sm.dq_full, 1);
    mbar_init(&sm.dq_empty, 256);
    mbar_init(&sm.done, 1);
    mbar_init(&sm.drain, 1);
    fence_mbar_init();
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
    tma_prefetch_desc(&tm_do);
    tma_prefetch_desc(&tm_dq);
  }
  if (warp == 1) {
    tmem_alloc(&sm.tmem_base, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  constexpr uint32_t kHalfBytes = kTile * 64 * 2;   // one 128-row x 64-element box
  constexpr uint32_t kRows64 = 64 * 128;            // byte offset of row 64 in a box
  constexpr int kHalves = D / 64;

  if (warp < 4) {
  // warpgroup 0: loads and MMA issue need few registers
  regs_release_ctl();
  if (warp == 0) {
    // ===================== TMA producer =====================
    const bool leader = elect_one();
    const int32_t krow = int32_t(sq.start + kt * kTile);
    if (leader) {
      mbar_arrive_expect_tx(&sm.kv_full, 2 * kHalves * kHalfBytes);
      for (int hv = 0; hv < kHalves; ++hv) {
        tma_load_3d(sm.k + hv * kHalfBytes, &tm_k, &sm.kv_full, hv * 64, h, krow);
        tma_load_3d(sm.v + hv * kHalfBytes, &tm_v, &sm.kv_full, hv * 64, h, krow);
      }
    }
    __syncwarp();
    int n = 0;
    bool ok = true;
    for (int32_t qt = kt; qt < n_qt && ok; ++qt) {
      if (!g.active(qt, kt)) continue;
      const int st = n & 1;
      if (n >= 2) ok = wait_bar_warp(&sm.q_empty[st], ((n >> 1) - 1) & 1, p.wait);
      if (!ok) break;
      const int32_t qrow = int32_t(sq.start + qt * kTile);
      if (leader) {
        mbar_arrive_expect_tx(&sm.q_full[st], kHalves * kHalfBytes);
        for (int hv = 0; hv < kHalves; ++hv)
          tma_load_3d(sm.q[st] + hv * kHalfBytes, &tm_q, &sm.q_full[st], hv * 64, h, qrow);
      }
      for (int x = lane; x < kTile; x += 32) {
        const int32_t i = qt * kTile + x;
        if (fast)
          reinterpret_cast<float *>(&sm.tq[st][0])[x] = i < g.L ? p.tf[sq.start + i] : 0.f;
        else
          sm.tq[st][x] = i < g.L ? p.ts[sq.start + i] : 0;
      }
      mbar_arrive(&sm.t_full[st]);
      if (n >= 1) ok = wait_bar_warp(&sm.do_empty, (n - 1) & 1, p.wait);
      if (!ok) break;
      if (leader) {
        mbar_arrive_expect_tx(&sm.do_full, kHalves * kHalfBytes);
        for (int hv = 0; hv < kHalves; ++hv)
          tma_load_3d(sm.dout + hv * kHalfBytes, &tm_do, &sm.do_full, hv * 64, h, qrow);
      }
      ++n;
    }
    if (leader) {
      drain_bar(&sm.kv_full, 0, p.wait.err, p.drain_ns);
      for (int m = (n > 2 ? n - 2 : 0); m < n; ++m)
        drain_bar(&sm.q_full[m & 1], (m >> 1) & 1, p.wait.err, p.drain_ns);
      if (n > 0) drain_bar(&sm.do_full, (n - 1) & 1, p.wait.err, p.drain_ns);
    }
  } else if (warp == 1) {
    // ===================== tcgen05 issuer =====================
    if (elect_one()) {
      constexpr uint32_t idesc_s = idesc_bf16(kTile, 64, false, false);
      constexpr uint32_t idesc_kv = idesc_bf16(kTile, D, false, true);
      constexpr uint32_t idesc_q = idesc_bf16(kTile, D, true, true);
      const uint32_t k_addr = smem_u32(sm.k), v_addr = smem_u32(sm.v);
      const uint32_t q_addr[2] = {smem_u32(sm.q[0]), smem_u32(sm.q[1])};
      const uint32_t do_addr = smem_u32(sm.dout);
      const uint32_t ds_addr = smem_u32(sm.ds);
      // S^T_x = K Q_x^T (keys x queries of half x)
      auto issue_s = [&](int x, int st) {
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk / 4) * kHalfBytes + (kk % 4) * 32;
          umma_ss(tmem + s_col(x), sdesc_sw128(k_addr + off, 16, 1024),
                  sdesc_sw128(q_addr[st] + x * kRows64 + off, 16, 1024), idesc_s, kk > 0);
        }
      };
      // dP^T_x = V dout_x^T
      auto issue_dp = [&](int x) {
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk / 4) * kHalfBytes + (kk % 4) * 32;
          umma_ss(tmem + dp_col(x), sdesc_sw128(v_addr + off, 16, 1024),
                  sdesc_sw128(do_addr + x * kRows64 + off, 16, 1024), idesc_s, kk > 0);
        }
      };
      // dV += P_x^T dout_x and dK += dS_x^T Q_x over the half's 64 queries
      auto issue_dv = [&](int x, bool first) {
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          umma_ts(tmem + kDvCol, tmem + s_col(x) + kk * 8,
                  sdesc_sw128(do_addr + (64 * x + 16 * kk) * 128, kHalfBytes, 1024), idesc_kv,
                  (first && x == 0 && kk == 0) ? 0u : 1u);
      };
      auto issue_dk = [&](int x, int st, bool first) {
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          umma_ts(tmem + kDkCol, tmem + dp_col(x) + kk * 8,
                  sdesc_sw128(q_addr[st] + (64 * x + 16 * kk) * 128, kHalfBytes, 1024),
                  idesc_kv, (first && x == 0 && kk == 0) ? 0u : 1u);
      };
      // dQ_part = dS K  (queries x d, A = dS from shared memory, M-major)
      auto issue_dq = [&]() {
#pragma unroll
        for (int kk = 0; kk < kTile / 16; ++kk)
          umma_ss(tmem + kDqCol, sdesc_sw128(ds_addr + kk * 16 * 128, 64 * 128 * 2, 1024),
                  sdesc_sw128(k_addr + kk * 16 * 128, kHalfBytes, 1024), idesc_q, kk > 0);
      };
      bool ok = wait_bar(&sm.kv_full, 0, p.wait);
      // the active query tiles, in order
      auto next_qt = [&](int32_t qt) {
        for (++qt; qt < n_qt; ++qt)
          if (g.active(qt, kt)) return qt;
        return int32_t(-1);
      };
      int32_t qt = ok ? next_qt(kt - 1) : -1;
      if (qt >= 0) {
        ok = wait_bar(&sm.q_full[0], 0, p.wait);
        if (ok) ok = wait_bar(&sm.do_full, 0, p.wait);
        tc_fence_after();
        if (ok) {
          issue_s(0, 0);
          issue_dp(0);
          umma_commit(&sm.s_full[0]);
        }
      }
      int n = 0;
      while (ok && qt >= 0) {
        const int st = n & 1;
        if (n > 0) ok = wait_bar(&sm.dq_empty, (n - 1) & 1, p.wait);
        if (!ok) break;
        tc_fence_after();
        issue_s(1, st);
        issue_dp(1);
        umma_commit(&sm.s_full[1]);
        ok = wait_bar(&sm.p_full[0], n & 1, p.wait);
        if (!ok) break;
        tc_fence_after();
        issue_dv(0, n == 0);
        issue_dk(0, st, n == 0);
        ok = wait_bar(&sm.p_full[1], n & 1, p.wait);
        if (!ok) break;
        tc_fence_after();
        issue_dv(1, n == 0);
        umma_commit(&sm.do_empty);
        issue_dk(1, st, n == 0);
        issue_dq();
        umma_commit(&sm.dq_full);
        umma_commit(&sm.q_empty[st]);
        const int32_t qn = next_qt(qt);
        if (qn >= 0) {
          const int st1 = (n + 1) & 1;
          ok = wait_bar(&sm.q_full[st1], ((n + 1) >> 1) & 1, p.wait);
          if (!ok) break;
          tc_fence_after();
          issue_s(0, st1);
          ok = wait_bar(&sm.do_full, (n + 1) & 1, p.wait);
          if (!ok) break;
          tc_fence_after();
          issue_dp(0);
          umma_commit(&sm.s_full[0]);
        }
        qt = qn;
        ++n;
      }
      umma_commit(&sm.done);
      umma_commit(&sm.drain);
      drain_bar(&sm.drain, 0, p.wait.err, p.drain_ns);
    }
    __syncwarp();
  }
  } else {
    // ===================== elementwise warpgroups =====================
    regs_grow_ew();
    const int x = (warp - 4) >> 2;           // query half: columns [64x, 64x + 64)
    const int quad = warp & 3;
    const int32_t jl = quad * 32 + lane;     // key row within the tile (tensor-memory lane)
    const int32_t j = kt * kTile + jl;       // local key index
    const bool key_ok = j < g.L;
    const uint32_t lane_base = tmem + (uint32_t(quad * 32) << 16);
    const int32_t pos_j = g.pos(min(j, g.L - 1));
    const float t_j_f = (fast && key_ok) ? p.tf[sq.start + j] : 0.f;
    const int64_t t_j = (!fast && key_ok) ? p.ts[sq.start + j] : 0;
    const float alpha_h = 0.5f * p.alpha;
    const float row_c = sm.tbl_p[p.nb_p - 1];
    const int nb_p_m1 = p.nb_p - 1;
    const bool sorted = (p.seq_fast[item.x] & kSeqSorted) != 0;
    const int sh = 23 - p.sub_bits;
    const int32_t r0 = fast_r0(p.sub_bits);
    float *gbin_p = p.bin_acc + int64_t(blockIdx.x) * kBinAccPerCta;   // this CTA's own bins
    float *gbin_t = gbin_p + kMaxTbl;
    int cur_b = 0;
    float acc_b = 0.f, acc_far = 0.f;
    int n = 0;
    bool ok = true;
    for (int32_t qt = kt; qt < n_qt && ok; ++qt) {
      if (!g.active(qt, kt)) continue;
      const int st = n & 1;
      ok = wait_bar_warp(&sm.s_full[x], n & 1, p.wait);
      if (ok) ok = wait_bar_warp(&sm.t_full[st], (n >> 1) & 1, p.wait);
      if (!ok) break;
      tc_fence_after();
      const int64_t *tq = sm.tq[st];
      const int32_t qs = qt * kTile;
      const bool need_mask = !g.full_tile(qt, kt);
      const bool gather_p = g.min_pos_dist(qt, kt) < nb_p_m1;
      // One 32-query chunk of this half (S in rs, dP in rd, already loaded).
      auto do_chunk = [&](uint32_t (&rs)[32], uint32_t (&rd)[32], int c0) {
        const int cc = 64 * x + c0;          // query column within the tile
        uint32_t pk_p[16], pk_d[16];
        // Time-bucket range of this chunk (first and last in-range column).
        // With sorted timestamps buckets are monotone along the row, so equal
        // ends mean one bucket and ends one apart mean at most two.
        int tmode = kTSlow;
        int32_t b_first = 0, b_last = 0;
        if (fast && sorted && !need_mask) {
          const int last = max(cc, min(cc + 31, g.L - 1 - qs));
          b_first = time_index<true>(tq, cc, t_j_f, t_j, sh, r0, p.sub_bits, p.nb_t);
          b_last = time_index<true>(tq, last, t_j_f, t_j, sh, r0, p.sub_bits, p.nb_t);
          if (__all_sync(0xffffffffu, b_first == b_last))
            tmode = kTOne;
          else if (__all_sync(0xffffffffu, b_last >= b_first && b_last - b_first <= 1))
            tmode = kTTwo;
        }
        float s_all = 0.f, s_lo = 0.f, p_hi = 0.f, p_lo = 0.f;   // (position sums unused here)
        const float uni_tb = tmode == kTOne ? sm.tbl_t[b_first] : 0.f;
#define HSTU_BCHUNK(M_, G_, F_, T_, RC_)                                                     \
  bwd_chunk<32, M_, G_, F_, T_, false, true>(                                                   \
      rs, rd, pk_p, pk_d, sm, tq, cc, qs, j, pos_j, t_j_f, t_j, alpha_h, RC_, g, nb_p_m1,   \
      p.sub_bits, p.nb_t, b_first, uni_tb, s_all, s_lo, cur_b, acc_b, acc_far, p_hi, p_lo,  \
      gbin_p, gbin_t)
        if (fast) {
          if (need_mask) {
            HSTU_BCHUNK(true, true, true, kTSlow, row_c);
          } else if (gather_p) {
            if (tmode == kTOne)
              HSTU_BCHUNK(false, true, true, kTOne, row_c);
            else if (tmode == kTTwo)
              HSTU_BCHUNK(false, true, true, kTTwo, row_c);
            else
              HSTU_BCHUNK(false, true, true, kTSlow, row_c);
          } else {
            if (tmode == kTOne)
              HSTU_BCHUNK(false, false, true, kTOne, row_c + uni_tb);
            else if (tmode == kTTwo)
              HSTU_BCHUNK(false, false, true, kTTwo, row_c);
            else
              HSTU_BCHUNK(false, false, true, kTSlow, row_c);
          }
        } else {
          if (need_mask)
            HSTU_BCHUNK(true, true, false, kTSlow, row_c);
          else
            HSTU_BCHUNK(false, true, false, kTSlow, row_c);
        }
#undef HSTU_BCHUNK
        if (tmode != kTSlow) {
          // merge the chunk's one or two bucket sums into the running bin; a
          // finished run leaves as a fire-and-forget reduction into the CTA's
          // own bins, so no lane waits on another
          const float v_first = tmode == kTOne ? s_all : s_lo;
          if (b_first != cur_b) {
            if (acc_b != 0.f) red_add_f32(gbin_t + cur_b, acc_b);
            cur_b = b_first;
            acc_b = 0.f;
          }
          acc_b += v_first;
          if (tmode == kTTwo && b_last != b_first) {
            if (acc_b != 0.f) red_add_f32(gbin_t + cur_b, acc_b);
            cur_b = b_last;
            acc_b = s_all - s_lo;
          }
          if (!gather_p) acc_far += s_all;   // far tile: every pair is in the last position bin
        }
        tmem_st16(lane_base + s_col(x) + c0 / 2, pk_p);
        tmem_st16(lane_base + dp_col(x) + c0 / 2, pk_d);
        // dS row chunk -> shared memory, [key][query] with the 128-byte swizzle
        uint8_t *row = sm.ds + x * (64 * 128 * 2) + jl * 128;
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int unit = (c0 / 8) + u;
          *reinterpret_cast<uint4 *>(row + ((unit ^ (jl & 7)) << 4)) =
              make_uint4(pk_d[4 * u], pk_d[4 * u + 1], pk_d[4 * u + 2], pk_d[4 * u + 3]);
        }
      };
#pragma unroll 1
      for (int c0 = 0; c0 < 64; c0 += 32) {
        uint32_t rs[32], rd[32];
        tmem_ld32(lane_base + s_col(x) + c0, rs);
        tmem_ld32(lane_base + dp_col(x) + c0, rd);
        tmem_wait_ld(rs);
        tmem_wait_ld(rd);
        do_chunk(rs, rd, c0);
      }
      {
        float af = acc_far;   // warp sum, one shared atomic per warp and tile
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) af += __shfl_xor_sync(0xffffffffu, af, o);
        if (lane == 0 && af != 0.f) atomicAdd(&sm.hist_p[nb_p_m1], af);
        acc_far = 0.f;
      }
      tmem_wait_st();
      tc_fence_before();
      fence_proxy_async_smem();
      mbar_arrive(&sm.p_full[x]);
      // dQ partial (thread = query row) -> float32 workspace; group x takes
      // d-columns [x D/2, (x+1) D/2) in passes of 32: tensor memory ->
      // registers -> its 16 KB of the (now free) dS tile, 128-byte swizzled,
      // rows of other sequences zeroed -> one TMA reduce-add of the
      // 128 x 32 block into the accumulator.
      ok = wait_bar_warp(&sm.dq_full, n & 1, p.wait);
      if (!ok) break;
      tc_fence_after();
      {
        const int32_t i = qs + jl;            // tensor-memory lane = query row here
        const bool row_ok = i < g.L;
        const bool issuer = quad == 0 && lane == 0;
        uint8_t *stage = sm.ds + x * (64 * 128 * 2);
        uint8_t *srow = stage + jl * 128;
#pragma unroll 1
        for (int c = x * (D / 2); c < (x + 1) * (D / 2); c += 32) {
          uint32_t r[32];
          tmem_ld32(lane_base + kDqCol + c, r);
          tmem_wait_ld(r);
          if (c != x * (D / 2)) {   // the previous pass's reduce must have read the buffer
            if (issuer) bulk_wait_read_all();
            named_bar_sync(2 + x, 128);
          }
#pragma unroll
          for (int u = 0; u < 8; ++u)
            *reinterpret_cast<uint4 *>(srow + ((u ^ (jl & 7)) << 4)) =
                row_ok ? make_uint4(r[4 * u], r[4 * u + 1], r[4 * u + 2], r[4 * u + 3])
                       : make_uint4(0u, 0u, 0u, 0u);
          fence_proxy_async_smem();
          named_bar_sync(2 + x, 128);
          if (issuer) {
            tma_reduce_add_2d(&tm_dq, stage, c, int32_t(h * p.total_tokens + sq.start + qs));
            bulk_commit();
          }
        }
        // the staging area is this group's half of next step's dS tile
        if (issuer) bulk_wait_read_all();
        named_bar_sync(2 + x, 128);
      }
      tc_fence_before();
      mbar_arrive(&sm.dq_empty);
      ++n;
    }
    // ---- epilogue: dV (half 0's group) or dK (half 1's group), thread = key row ----
    if (ok) ok = wait_bar_warp(&sm.done, 0, p.wait);
    tc_fence_after();
    if (ok) {
      const uint32_t col = x == 0 ? kDvCol : kDkCol;
      const float scale = x == 0 ? p.dv_scale : p.dk_scale;
      __nv_bfloat16 *orow = x == 0 ? p.dv + (sq.start + j) * p.dv_rs + int64_t(h) * D
                                   : p.dk + (sq.start + j) * p.dk_rs + int64_t(h) * D;
#pragma unroll 1
      for (int c0 = 0; c0 < D; c0 += 32) {
        uint32_t r[32];
        tmem_ld32(lane_base + col + c0, r);
        tmem_wait_ld(r);
        if (key_ok) {
          uint32_t w[16];
#pragma unroll
          for (int e = 0; e < 16; ++e)
            w[e] = pack_bf16x2(__uint_as_float(r[2 * e]) * scale,
                               __uint_as_float(r[2 * e + 1]) * scale);
          uint4 *dst = reinterpret_cast<uint4 *>(orow + c0);
#pragma unroll
          for (int e = 0; e < 4; ++e)
            dst[e] = make_uint4(w[4 * e], w[4 * e + 1], w[4 * e + 2], w[4 * e + 3]);
        }
      }
    }
    // ---- d rab: flush this thread's sums, then the CTA's bins ----
    __syncwarp();
    flush_warp(sm.hist_t, cur_b, acc_b, true);
    // the dQ reduces this thread issued have landed
    if (quad == 0 && lane == 0) bulk_wait_all();
    __threadfence();   // this thread's reductions into the CTA's global bins are done
    named_bar_sync(1, 256);
    const int tid_ew = tid - 128;
    const int nt = fast ? fast_table_size(p.sub_bits) : p.nb_t;
    float *gp = p.drab_p + tab * p.nb_p;
    float *gt = p.drab_t + tab * p.nb_t;
    for (int xx = tid_ew; xx < p.nb_p; xx += 256) {
      const float v = sm.hist_p[xx] + __ldcg(gbin_p + xx);
      if (v != 0.f) atomicAdd(gp + xx, v * p.drab_scale);
    }
    for (int xx = tid_ew; xx < nt; xx += 256) {
      const float v = sm.hist_t[xx] + __ldcg(gbin_t + xx);
      if (v != 0.f) {
        const int b = fast ? fast_table_bucket(xx, p.sub_bits, p.nb_t) : xx;
        atomicAdd(gt + b, v * p.drab_scale);
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

// dq[t][h][:] = bf16(scale * dq_acc[h][t][:]), 8 features per thread.
__global__ void dq_convert_kernel(const float *__restrict__ acc, __nv_bfloat16 *__restrict__ dq,
                                  int64_t T, int32_t width, int64_t dq_rs, int64_t n, float scale) {
  const int32_t per_row = width / 8;
  for (int64_t x = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; x < n;
       x += int64_t(gridDim.x) * blockDim.x) {
    const int64_t row = x / per_row;              // h * T + t
    const int32_t c = int32_t(x - row * per_row) * 8;
    const int64_t hh = row / T, t = row - hh * T;
    const float4 a = *reinterpret_cast<const float4 *>(acc + row * width + c);
    const float4 b = *reinterpret_cast<const float4 *>(acc + row * width + c + 4);
    uint4 o;
    o.x = pack_bf16x2(a.x * scale, a.y * scale);
    o.y = pack_bf16x2(a.z * scale, a.w * scale);
    o.z = pack_bf16x2(b.x * scale, b.y * scale);
    o.w = pack_bf16x2(b.z * scale, b.w * scale);
    *reinterpret_cast<uint4 *>(dq + t * dq_rs + hh * width + c) = o;
  }
}

}  // namespace bwd_tc

cudaError_t launch_dq_convert(const AttnProblem &p, const Scratch &s, void *dq, cudaStream_t st) {
  const int64_t n = p.total_tokens * p.num_heads * (p.d_qk / 8);
  if (n == 0) return cudaSuccess;
  const unsigned blocks = unsigned(std::min<int64_t>((n + 255) / 256, 148 * 16));
  bwd_tc::dq_convert_kernel<<<blocks, 256, 0, st>>>(
      s.dq_acc, static_cast<__nv_bfloat16 *>(dq), p.total_tokens, p.d_qk, p.dq_rs, n,
      0.5f * p.alpha * p.silu_scale);
  count_launch();
  return cudaGetLastError();
}

bool bwd_tc_supported(const AttnProblem &p) {
  if (p.dtype != 1 || p.d_qk != p.d_v || (p.d_qk != 64 && p.d_qk != 128)) return false;
  if (p.nb_p > bwd_tc::kMaxTbl || p.nb_t > bwd_tc::kMaxTbl) return false;
  if (p.sub_bits <= 4 && fast_table_size(p.sub_bits) > bwd_tc::kMaxTbl) return false;
  if (p.total_tokens * p.num_heads >= (int64_t(1) << 31)) return false;
  const uintptr_t a = reinterpret_cast<uintptr_t>(p.q) | reinterpret_cast<uintptr_t>(p.k) |
                      reinterpret_cast<uintptr_t>(p.v);
  if (a & 15) return false;
  if ((p.q_rs | p.k_rs | p.v_rs) & 7) return false;
  return true;
}

template <int D>
static cudaError_t launch_bwd_tc_d(const AttnProblem &p, const Scratch &s, const void *dout,
                                   void *dq, void *dk, void *dv, float *drab_p, float *drab_t,
                                   const WaitCtl &w, cudaStream_t st) {
  using namespace bwd_tc;
  CUtensorMap tq, tk, tv, tdo, tdq;
  const uint64_t T = uint64_t(p.total_tokens);
  if (!encode_tmap_bf16_3d(&tq, p.q, D, p.num_heads, T, D * 2, uint64_t(p.q_rs) * 2, 64, 1,
                           kTile) ||
      !encode_tmap_bf16_3d(&tk, p.k, D, p.num_heads, T, D * 2, uint64_t(p.k_rs) * 2, 64, 1,
                           kTile) ||
      !encode_tmap_bf16_3d(&tv, p.v, D, p.num_heads, T, D * 2, uint64_t(p.v_rs) * 2, 64, 1,
                           kTile) ||
      !encode_tmap_bf16_3d(&tdo, dout, D, p.num_heads, T, D * 2, uint64_t(p.do_rs) * 2, 64, 1,
                           kTile) ||
      !encode_tmap_f32_2d(&tdq, s.dq_acc, D, T * p.num_heads, D * 4, 32, kTile))
    return cudaErrorInvalidValue;
  const size_t acc_bytes = sizeof(float) * size_t(T) * p.num_heads * D;
  cudaError_t e = cudaMemsetAsync(s.dq_acc, 0, acc_bytes, st);
  if (e != cudaSuccess) return e;
  const unsigned grid = unsigned(s.n_kitems) * unsigned(p.num_heads);
  e = cudaMemsetAsync(s.bin_acc, 0, sizeof(float) * kBinAccPerCta * size_t(grid), st);
  if (e != cudaSuccess) return e;
  Params prm;
  prm.seqs = s.seqs;
  prm.kitems = s.kitems;
  prm.num_heads = p.num_heads;
  prm.tf = s.tf;
  prm.ts = p.ts;
  prm.seq_fast = s.seq_fast;
  prm.rab_p = p.rab_p;
  prm.rab_t = p.rab_t;
  prm.rab_per_head = p.rab_per_head;
  prm.nb_p = p.nb_p;
  prm.nb_t = p.nb_t;
  prm.sub_bits = p.sub_bits;
  prm.alpha = p.alpha;
  prm.dv_scale = p.silu_scale;
  prm.dk_scale = 0.5f * p.alpha * p.silu_scale;
  prm.drab_scale = 0.5f * p.silu_scale;
  prm.dk = static_cast<__nv_bfloat16 *>(dk);
  prm.dv = static_cast<__nv_bfloat16 *>(dv);
  prm.dk_rs = p.dk_rs;
  prm.dv_rs = p.dv_rs;
  prm.total_tokens = p.total_tokens;
  prm.dq_acc = s.dq_acc;
  prm.bin_acc = s.bin_acc;
  prm.drab_p = drab_p;
  prm.drab_t = drab_t;
  prm.wait = w;
  prm.drain_ns = 4000000000ull;
  // At least 120 KB so a single CTA occupies an SM (it allocates all of TMEM).
  const size_t smem = std::max<size_t>(sizeof(Smem<D>) + 1024, 120 * 1024);
  static PerDeviceOnce attr;
  e = attr.run([&](int) {
    // The in-kernel register split assumes exactly kRegsLaunch registers per
    // thread at launch; refuse to launch otherwise (it would wait forever).
    cudaFuncAttributes fa;
    cudaError_t r = cudaFuncGetAttributes(&fa, bwd_kernel<D>);
    if (r != cudaSuccess) return r;
    if (fa.numRegs != kRegsLaunch) return cudaErrorInvalidConfiguration;
    return cudaFuncSetAttribute(bwd_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                int(smem));
  });
  if (e != cudaSuccess) return e;
  bwd_kernel<D><<<grid, kThreads, smem, st>>>(tq, tk, tv, tdo, tdq, prm);
  count_launch();
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  return launch_dq_convert(p, s, dq, st);
}

cudaError_t launch_bwd_tc(const AttnProblem &p, const Scratch &s, const void *dout, void *dq,
                          void *dk, void *dv, float *drab_p, float *drab_t, const WaitCtl &w,
                          cudaStream_t st) {
  if (s.n_kitems == 0) return cudaSuccess;
  return p.d_qk == 64 ? launch_bwd_tc_d<64>(p, s, dout, dq, dk, dv, drab_p, drab_t, w, st)
                      : launch_bwd128(p, s, dout, dq, dk, dv, drab_p, drab_t, w, st);
}

}  // namespace hstu
