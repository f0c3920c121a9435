// attn_bwd128_sm100.cu -- backward HSTU pointwise attention for d_qk = d_v =
// 128 on the 5th-generation tensor cores (tcgen05 + tensor memory + TMA),
// bf16 in, fp32 accumulate.  Same gradients as attn_bwd_sm100.cu (the
// pointwise aggregation with positional and temporal bias of the DLRMv4
// article, section "Model architecture: HSTU replaces the feature-interaction
// stack"):
//   dA_ij = <dout_i, v_j>,  dS_ij = dA_ij silu_scale SiLU'(s_ij)
//   dv_j = silu_scale sum_i SiLU(s_ij) dout_i,  dk_j = alpha sum_i dS_ij q_i
//   dq_i = alpha sum_j dS_ij k_j,  drab_*[bucket_ij] += dS_ij.
//
// One CTA = one (sequence, head, 128-key tile); it walks the 64-query blocks
// that can see its keys.  Consecutive blocks alternate between two groups of
// two elementwise warpgroups each, and group g owns tensor-memory slot g, so
// the two groups' blocks pipeline independently:
//   warp 0      TMA producer: K and V once; Q and dout blocks into a 3-deep
//               ring; the blocks' query timestamps.
//   warp 1      tcgen05 issuer, for block j of group g:
//                 S^T_j = K Q_j^T and dP^T_j = V dout_j^T into slot g;
//                 after the group's elementwise pass:
//                 dQ^T_j = K^T dS^T_j over dP^T_j's columns (dS^T in shared memory),
//                 dV += P^T_j dout_j (P^T in tensor memory), dK += dS^T_j Q_j;
//                 then block j+2's S^T (behind dV, which reads P^T) and, once
//                 the group has read dQ^T_j out, its dP^T.
//   warps 4-19  the two groups; the two warpgroups of a group take one half
//               of the block's 64 query columns each, so four warps per
//               sub-partition hide the latency of the elementwise chain.
//               Thread = key row: bias, SiLU, SiLU', mask, d rab sums, P^T
//               back to tensor memory, dS^T to shared memory.  Thread =
//               feature d: dQ^T_j leaves tensor memory as coalesced float32
//               reductions into the [H][T][D] accumulator, overlapping the
//               other group's pass.  At the end dV (group 0) and dK (group 1)
//               leave tensor memory as bf16, a column half per warpgroup.
// Tensor memory (512 columns): slot g = [128g, 128g + 128): S^T at +0, dP^T
// at +64 (then dQ^T); dV [256, 384); dK [384, 512).  P^T (bf16, two queries
// per column) of query columns [32h, 32h + 32) goes over S^T columns
// [32h, 32h + 16): inside the half's own S^T columns, after they are read.
// Scales: as in attn_bwd_sm100.cu (h = s/2 form; dV silu_scale, dK / dQ
// alpha silu_scale / 2, d rab silu_scale / 2).
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>

#include "attn_bwd_common.cuh"
#include "internal.h"

namespace hstu {
namespace bwd128 {
using namespace bwd_ew;

constexpr int D = 128;
constexpr int kKeys = kAttnTile;   // keys per CTA
constexpr int kBlk = 64;           // queries per block
constexpr int kSub = 16;           // query columns per elementwise chunk
constexpr int kRing = 3;           // Q / dout ring depth
constexpr int kThreads = 640;      // one control warpgroup + four elementwise (96 registers each)
constexpr int kMaxTbl = 512;
static_assert(2 * kMaxTbl <= kBinAccPerCta, "per-CTA bins hold both tables");
constexpr uint32_t kKChunk = kKeys * 64 * 2;   // 64-feature chunk of K or V (16 KB)
constexpr uint32_t kBChunk = kBlk * 64 * 2;    // 64-feature chunk of a Q / dout block (8 KB)

struct Smem {
  alignas(1024) uint8_t k[kKeys * D * 2];
  alignas(1024) uint8_t v[kKeys * D * 2];
  alignas(1024) uint8_t q[kRing][kBlk * D * 2];
  alignas(1024) uint8_t dout[kRing][kBlk * D * 2];
  alignas(1024) uint8_t ds[2][kKeys * kBlk * 2];   // dS^T per group, [key][query]
  alignas(16) int64_t tq[kRing][kBlk];             // query timestamps per ring slot
  float tbl_p[kMaxTbl];
  float tbl_t[kMaxTbl];
  float hist_p[kMaxTbl];
  float hist_t[kMaxTbl];
  uint64_t kv_full, q_full[kRing], do_full[kRing], t_full[kRing], qd_empty[kRing];
  uint64_t s_full[2], p_full[2], dq_full[2], dq_empty[2], done, drain;
  uint32_t tmem_base;
};

__host__ __device__ constexpr uint32_t s_col(int g) { return 128u * uint32_t(g); }
__host__ __device__ constexpr uint32_t dp_col(int g) { return 128u * uint32_t(g) + 64u; }
// Column (from the slot start) of P^T for query columns [c, c + 16), c a multiple of 16.
__host__ __device__ constexpr uint32_t p_col(int c) { return uint32_t((c & ~31) + (c & 31) / 2); }
constexpr uint32_t kDvCol = 256, kDkCol = 384;
static_assert(sizeof(Smem) + 1024 <= 227 * 1024, "shared memory budget");

// Next 64-query block after qb holding a pair visible to the key tile at ks (-1: none).
__device__ __forceinline__ int32_t next_block(const TileGeom &g, int32_t qb, int32_t n_qb,
                                              int32_t ks) {
  for (++qb; qb < n_qb; ++qb)
    if (g.active_rows(qb * kBlk, kBlk, ks)) return qb;
  return -1;
}

// ---- optional phase trace (library built with -DHSTU_TRACE; a no-op otherwise) ----
// Three CTAs (blocks 0, n/2 and n-1 of the grid) record the SM clock at each
// phase boundary: per warp (lane 0) for the elementwise warps, per issued
// batch for the MMA issuer.  Entry = code << 56 | block ordinal << 40 | clock.
// Codes: 1 block start (its S^T / dP^T and timestamps ready), 8 / 9 / 10 a
// 16-column chunk's tensor-memory load issued / landed / math done (ordinal
// 2 jb + chunk), 11 P^T stores done, 2 P^T / dS^T handed to the issuer, 3 dQ^T
// ready, 4 dQ^T reductions issued; issuer: 5 dQ^T issued, 6 S^T issued, 7
// dP^T issued.
#ifdef HSTU_TRACE
constexpr int kTraceCtas = 3, kTraceRecs = kThreads / 32, kTraceEntries = 1024;
__device__ unsigned long long g_trace[kTraceCtas][kTraceRecs][kTraceEntries];
__device__ __forceinline__ int trace_slot() {
  const unsigned n = gridDim.x;
  return blockIdx.x == 0 ? 0 : blockIdx.x == n / 2 ? 1 : blockIdx.x == n - 1 ? 2 : -1;
}
__device__ __forceinline__ void trace_put(int slot, int rec, int &n, unsigned code, int ord) {
  if (slot >= 0 && rec >= 0 && rec < kTraceRecs && n < kTraceEntries) {
    g_trace[slot][rec][n] = (static_cast<unsigned long long>(code) << 56) |
                            (static_cast<unsigned long long>(ord & 0xffff) << 40) |
                            (static_cast<unsigned long long>(clock64()) & ((1ull << 40) - 1));
    ++n;
  }
}
#else
__device__ __forceinline__ int trace_slot() { return -1; }
__device__ __forceinline__ void trace_put(int, int, int &, unsigned, int) {}
#endif

__global__ void __launch_bounds__(kThreads, 1)
    bwd128_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                  const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                  const BwdParams p) {
  extern __shared__ uint8_t smem_raw[];
  Smem &sm = *reinterpret_cast<Smem *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                       ~uintptr_t(1023));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int32_t item_idx = blockIdx.x / p.num_heads;
  const int32_t h = blockIdx.x % p.num_heads;
  const int4 item = p.kitems[item_idx];
  // A key tile split over its query run takes blocks [item.z, item.w) and
  // adds its partial dK, dV into dk_acc, dv_acc (they are sums over queries).
  const bool split = item.w != kUnsplit;
  const SeqInfo sq = p.seqs[item.x];
  const TileGeom g{sq.len, sq.n_hist};
  const int32_t kt = item.y;
  const int32_t ks = kt * kKeys;
  const int32_t n_qb = (g.L + kBlk - 1) / kBlk;
  // The query blocks that see this key tile form one contiguous run: from
  // the block at the tile's first key (earlier rows see none of its keys:
  // history rows are causal, a candidate before a candidate key tile sees
  // only itself) to the sequence end when the tile holds history keys
  // (every later history row and every candidate sees them), else to the
  // last block a candidate of the tile sits in.  A block of the run without
  // a visible pair would take the masked path and add nothing.
  int32_t qb_first = next_block(g, max(2 * kt, split ? item.z : 0) - 1, n_qb, ks);
  int32_t qb_end = qb_first < 0 ? 0 : min(n_qb, split ? item.w : n_qb);   // one past the last
  while (qb_end > qb_first + 1 && !g.active_rows((qb_end - 1) * kBlk, kBlk, ks)) --qb_end;
  if (qb_first >= qb_end) qb_first = -1;
  auto next_in_run = [&](int32_t qb) { return qb + 1 < qb_end ? qb + 1 : int32_t(-1); };
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
    for (int r = 0; r < kRing; ++r) {
      mbar_init(&sm.q_full[r], 1);
      mbar_init(&sm.do_full[r], 1);
      mbar_init(&sm.t_full[r], 32);
      mbar_init(&sm.qd_empty[r], 1);
    }
    for (int x = 0; x < 2; ++x) {
      mbar_init(&sm.s_full[x], 1);
      mbar_init(&sm.p_full[x], 256);
      mbar_init(&sm.dq_full[x], 1);
      mbar_init(&sm.dq_empty[x], 256);
    }
    mbar_init(&sm.done, 1);
    mbar_init(&sm.drain, 1);
    fence_mbar_init();
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
    tma_prefetch_desc(&tm_do);
  }
  if (warp == 1) {
    tmem_alloc(&sm.tmem_base, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  const int trs = trace_slot();
  int trn = 0;

  if (warp == 0) {
    // ===================== TMA producer =====================
    const bool leader = elect_one();
    if (leader) {
      const int32_t krow = int32_t(sq.start + ks);
      mbar_arrive_expect_tx(&sm.kv_full, 4 * kKChunk);
      for (int hv = 0; hv < 2; ++hv) {
        tma_load_3d(sm.k + hv * kKChunk, &tm_k, &sm.kv_full, hv * 64, h, krow);
        tma_load_3d(sm.v + hv * kKChunk, &tm_v, &sm.kv_full, hv * 64, h, krow);
      }
    }
    __syncwarp();
    int jb = 0;
    bool ok = true;
    for (int32_t qb = qb_first; qb >= 0; qb = next_in_run(qb), ++jb) {
      const int r = jb % kRing;
      const int32_t qrow = int32_t(sq.start + qb * kBlk);
      if (jb >= kRing) {
        // the slot is still in use: warm L2 with the block meanwhile
        if (leader) {
          for (int hv = 0; hv < 2; ++hv) {
            tma_prefetch_3d(&tm_q, hv * 64, h, qrow);
            tma_prefetch_3d(&tm_do, hv * 64, h, qrow);
          }
        }
        ok = wait_bar_warp(&sm.qd_empty[r], ((jb / kRing) - 1) & 1, p.wait);
      }
      if (!ok) break;
      if (leader) {
        mbar_arrive_expect_tx(&sm.q_full[r], 2 * kBChunk);
        for (int hv = 0; hv < 2; ++hv)
          tma_load_3d(sm.q[r] + hv * kBChunk, &tm_q, &sm.q_full[r], hv * 64, h, qrow);
        mbar_arrive_expect_tx(&sm.do_full[r], 2 * kBChunk);
        for (int hv = 0; hv < 2; ++hv)
          tma_load_3d(sm.dout[r] + hv * kBChunk, &tm_do, &sm.do_full[r], hv * 64, h, qrow);
      }
      // timestamps after both copies are in flight
      for (int x = lane; x < kBlk; x += 32) {
        const int32_t i = qb * kBlk + x;
        if (fast)
          reinterpret_cast<float *>(&sm.tq[r][0])[x] = i < g.L ? p.tf[sq.start + i] : 0.f;
        else
          sm.tq[r][x] = i < g.L ? p.ts[sq.start + i] : 0;
      }
      mbar_arrive(&sm.t_full[r]);
    }
    // every copy issued has landed before the CTA can exit
    if (leader) {
      drain_bar(&sm.kv_full, 0, p.wait.err, p.drain_ns);
      for (int m = (jb > kRing ? jb - kRing : 0); m < jb; ++m) {
        drain_bar(&sm.q_full[m % kRing], (m / kRing) & 1, p.wait.err, p.drain_ns);
        drain_bar(&sm.do_full[m % kRing], (m / kRing) & 1, p.wait.err, p.drain_ns);
      }
    }
  } else if (warp == 1) {
    // ===================== tcgen05 issuer =====================
    if (elect_one()) {
      constexpr uint32_t idesc_s = idesc_bf16(kKeys, kBlk, false, false);   // S^T, dP^T
      constexpr uint32_t idesc_acc = idesc_bf16(kKeys, D, false, true);     // dV, dK
      constexpr uint32_t idesc_dq = idesc_bf16(D, kBlk, true, true);        // dQ^T
      const uint32_t k_addr = smem_u32(sm.k), v_addr = smem_u32(sm.v);
      // Shared-memory descriptors are linear in the address (the start field
      // is address >> 4 and never carries inside shared memory), so each
      // operand's descriptor is built once per batch and advanced by
      // (offset >> 4): the issuing thread spends one add per operand per MMA.
      // S^T = K Q^T (or dP^T = V dout^T): M = keys, N = queries, both K-major over d
      auto issue_sd = [&](uint32_t col, uint32_t a_addr, uint32_t b_addr) {
        const uint64_t da = sdesc_sw128(a_addr, 16, 1024), db = sdesc_sw128(b_addr, 16, 1024);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          umma_ss(tmem + col, da + (((kk / 4) * kKChunk + (kk % 4) * 32) >> 4),
                  db + (((kk / 4) * kBChunk + (kk % 4) * 32) >> 4), idesc_s, kk > 0);
      };
      // dQ^T = K^T dS^T: M = d (K read feature-major), N = queries, K-dim = keys
      const uint64_t dk_mn = sdesc_sw128(k_addr, kKChunk, 1024);
      auto issue_dq = [&](int gg) {
        const uint64_t dd = sdesc_sw128(smem_u32(sm.ds[gg]), kKeys * 128, 1024);
#pragma unroll
        for (int kk = 0; kk < kKeys / 16; ++kk)
          umma_ss(tmem + dp_col(gg), dk_mn + ((kk * 16 * 128) >> 4), dd + ((kk * 16 * 128) >> 4),
                  idesc_dq, kk > 0);
      };
      // dV += P^T dout (P^T from tensor memory), dK += dS^T Q (dS^T from shared memory)
      auto issue_dvdk = [&](int gg, int r, bool first) {
        const uint64_t ddo = sdesc_sw128(smem_u32(sm.dout[r]), kBChunk, 1024);
        const uint64_t dq = sdesc_sw128(smem_u32(sm.q[r]), kBChunk, 1024);
        const uint64_t dds = sdesc_sw128(smem_u32(sm.ds[gg]), 16, 1024);
#pragma unroll
        for (int kk = 0; kk < kBlk / 16; ++kk)
          umma_ts(tmem + kDvCol, tmem + s_col(gg) + p_col(kk * 16), ddo + ((kk * 16 * 128) >> 4),
                  idesc_acc, (first && kk == 0) ? 0u : 1u);
#pragma unroll
        for (int kk = 0; kk < kBlk / 16; ++kk)
          umma_ss(tmem + kDkCol, dds + ((kk * 32) >> 4), dq + ((kk * 16 * 128) >> 4), idesc_acc,
                  (first && kk == 0) ? 0u : 1u);
      };
      int32_t nblk = 0;
      for (int32_t qb = qb_first; qb >= 0; qb = next_in_run(qb)) ++nblk;
      bool ok = wait_bar(&sm.kv_full, 0, p.wait);
      for (int jj = 0; jj < 2 && jj < nblk && ok; ++jj) {
        ok = wait_bar(&sm.q_full[jj], 0, p.wait);
        if (!ok) break;
        tc_fence_after();
        issue_sd(s_col(jj), k_addr, smem_u32(sm.q[jj]));
        ok = wait_bar(&sm.do_full[jj], 0, p.wait);
        if (!ok) break;
        tc_fence_after();
        issue_sd(dp_col(jj), v_addr, smem_u32(sm.dout[jj]));
        umma_commit(&sm.s_full[jj]);
      }
      // Event loop serving whichever group is ready, so one group's dQ^T
      // read-out never holds up the other's.  Per group g: jp[g] is the block
      // whose elementwise pass is awaited; sd[g] the block whose S^T / dP^T
      // are still to be issued (sd_st 0: needs its Q block; 1: needs the
      // group's previous dQ^T read out and its dout block).
      int jp[2] = {0, 1}, sd[2] = {-1, -1}, sd_st[2] = {0, 0};
      bool acc_started = false;
      uint64_t t_idle = 0;
      while (ok) {
        bool progress = false;
#pragma unroll
        for (int gg = 0; gg < 2; ++gg) {
          if (sd[gg] >= 0) {
            const int j2 = sd[gg], r2 = j2 % kRing;
            if (sd_st[gg] == 0 && mbar_test_wait(&sm.q_full[r2], (j2 / kRing) & 1)) {
              tc_fence_after();
              // in issue order behind dV, which reads P^T from these columns
              issue_sd(s_col(gg), k_addr, smem_u32(sm.q[r2]));
              trace_put(trs, 1, trn, 6u, j2);
              sd_st[gg] = 1;
              progress = true;
            }
            if (sd_st[gg] == 1 && mbar_test_wait(&sm.dq_empty[gg], ((j2 - 2) >> 1) & 1) &&
                mbar_test_wait(&sm.do_full[r2], (j2 / kRing) & 1)) {
              tc_fence_after();
              issue_sd(dp_col(gg), v_addr, smem_u32(sm.dout[r2]));
              umma_commit(&sm.s_full[gg]);
              trace_put(trs, 1, trn, 7u, j2);
              sd[gg] = -1;
              progress = true;
            }
          }
          const int jb = jp[gg];
          if (jb < nblk && sd[gg] != jb && mbar_test_wait(&sm.p_full[gg], (jb >> 1) & 1)) {
            tc_fence_after();
            const int r = jb % kRing;
            issue_dq(gg);
            trace_put(trs, 1, trn, 5u, jb);
            umma_commit(&sm.dq_full[gg]);
            issue_dvdk(gg, r, !acc_started);   // the first block served starts dV and dK
            acc_started = true;
            umma_commit(&sm.qd_empty[r]);
            if (jb + 2 < nblk) {
              sd[gg] = jb + 2;
              sd_st[gg] = 0;
            }
            jp[gg] = jb + 2;
            progress = true;
          }
        }
        if (jp[0] >= nblk && jp[1] >= nblk && sd[0] < 0 && sd[1] < 0) break;
        if (progress) {
          t_idle = 0;
          continue;
        }
        // Nothing ready: poll again (a sleep here measured slower: it delays
        // the next issue more than it frees issue slots); stop once another
        // role recorded an error or the limit passes.
        const uint64_t now = globaltimer_ns();
        if (t_idle == 0) {
          t_idle = now;
        } else if (*reinterpret_cast<volatile uint32_t *>(p.wait.err) != 0) {
          ok = false;
        } else if (now - t_idle > p.wait.limit_ns) {
          record_error(p.wait.err, kDevErrTimeout);
          ok = false;
        }
      }
      umma_commit(&sm.done);
      umma_commit(&sm.drain);
      drain_bar(&sm.drain, 0, p.wait.err, p.drain_ns);
    }
    __syncwarp();
  } else if (warp >= 4) {
    // ===================== elementwise warpgroups =====================
    const int x = ((warp - 4) >> 2) & 1;     // group: blocks with x = ordinal mod 2
    const int hx = (warp - 4) >> 3;          // query-column half of the group's blocks
    const int quad = warp & 3;
    const int32_t jl = quad * 32 + lane;     // tensor-memory lane: key row, then feature d
    const int32_t j = ks + jl;               // local key index
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
    uint8_t *ds_row = sm.ds[x] + jl * 128;
    int cur_b = 0;
    float acc_b = 0.f, acc_far = 0.f;
    int jb = 0;
    bool ok = true;
    for (int32_t qb = qb_first; qb >= 0 && ok; qb = next_in_run(qb), ++jb) {
      if ((jb & 1) != x) continue;
      const int r = jb % kRing;
      ok = wait_bar_warp(&sm.s_full[x], (jb >> 1) & 1, p.wait);
      if (ok) ok = wait_bar_warp(&sm.t_full[r], (jb / kRing) & 1, p.wait);
      if (!ok) break;
      tc_fence_after();
      if (lane == 0) trace_put(trs, warp, trn, 1u, jb);
      const int64_t *tq = sm.tq[r];
      const int32_t qs = qb * kBlk;
      const bool gather_p = g.min_pos_dist_rows(qs, ks) < nb_p_m1;
      // position bins by diagonal need history rows only; near-diagonal
      // blocks with candidate rows take the per-pair (masked) path
      const bool diag_p = qs + kBlk <= g.nh;
      const bool need_mask = !g.full_rows(qs, kBlk, ks) || (gather_p && !diag_p);
      // One kSub-query chunk (S^T in rs, dP^T in rd, already loaded); 16
      // columns keep the live registers and the code per variant small.
      auto do_chunk = [&](uint32_t (&rs)[kSub], uint32_t (&rd)[kSub], int cc) {
        uint32_t pk_p[kSub / 2], pk_d[kSub / 2];
        // Time-bucket range of this chunk (first and last in-range column).
        // With sorted timestamps buckets are monotone along the row, so equal
        // ends mean one bucket and ends one apart mean at most two.
        int tmode = kTSlow;
        int32_t b_first = 0, b_last = 0;
        if (fast && sorted && !need_mask && !gather_p) {   // only far blocks take the chunk modes
          const int last = max(cc, min(cc + kSub - 1, g.L - 1 - qs));
          b_first = time_index<true>(tq, cc, t_j_f, t_j, sh, r0, p.sub_bits, p.nb_t);
          b_last = time_index<true>(tq, last, t_j_f, t_j, sh, r0, p.sub_bits, p.nb_t);
          if (__all_sync(0xffffffffu, b_first == b_last))
            tmode = kTOne;
          else if (__all_sync(0xffffffffu, b_last >= b_first && b_last - b_first <= 1))
            tmode = kTTwo;
        }
        float s_all = 0.f, s_lo = 0.f, p_hi = 0.f, p_lo = 0.f;
        const float uni_tb = tmode == kTOne ? sm.tbl_t[b_first] : 0.f;
#define HSTU_BCHUNK(M_, G_, F_, T_, D_, RC_)                                                  \
  bwd_chunk<kSub, M_, G_, F_, T_, D_, true>(rs, rd, pk_p, pk_d, sm, tq, cc, qs, j, pos_j,    \
                                      t_j_f, t_j, alpha_h, RC_, g, nb_p_m1, p.sub_bits,     \
                                      p.nb_t, b_first, uni_tb, s_all, s_lo, cur_b, acc_b,   \
                                      acc_far, p_hi, p_lo, gbin_p, gbin_t)
        // Few variants keep the elementwise code small enough for the
        // instruction cache: the two common far-block time modes fully
        // specialised, the unmasked near-diagonal history blocks, and
        // everything else (the diagonal block, candidate rows, per-pair time
        // buckets, exact int64 times) through the general masked variants,
        // which are correct for any block.
        const bool far_fast = fast && !need_mask && !gather_p;
        if (far_fast && tmode == kTOne)
          HSTU_BCHUNK(false, false, true, kTOne, false, row_c + uni_tb);
        else if (far_fast && tmode == kTTwo)
          HSTU_BCHUNK(false, false, true, kTTwo, false, row_c);
        else if (fast) {
          // near-diagonal history blocks: past the diagonal block itself
          // every pair is visible, so only the position gather remains
          if (diag_p && !need_mask)
            HSTU_BCHUNK(false, true, true, kTSlow, true, row_c);
          else if (diag_p)
            HSTU_BCHUNK(true, true, true, kTSlow, true, row_c);
          else
            HSTU_BCHUNK(true, true, true, kTSlow, false, row_c);
        } else {
          // exact int64 times (spans of 2^24 s and more): one variant, position
          // sums per pair even for history rows
          HSTU_BCHUNK(true, true, false, kTSlow, false, row_c);
        }
#undef HSTU_BCHUNK
        // the chunk ran a general variant with diagonal position sums
        const bool general = tmode == kTSlow && fast;
        if (general && diag_p) {
          // the lane's two diagonals: (qs + cc + lane) - (first key of the warp), and 32 less
          const int32_t b_hi = qs + cc + lane - (ks + quad * 32);
          if (p_hi != 0.f) {
            if (b_hi >= nb_p_m1)
              acc_far += p_hi;
            else
              red_add_f32(gbin_p + b_hi, p_hi);
          }
          if (p_lo != 0.f) {
            if (b_hi - 32 >= nb_p_m1)
              acc_far += p_lo;
            else if (b_hi - 32 >= 0)
              red_add_f32(gbin_p + (b_hi - 32), p_lo);
          }
        }
        if (tmode != kTSlow) {
          // merge the chunk's one or two bucket sums into the running bin; a
          // finished run leaves as a fire-and-forget reduction into the CTA's
          // own bins, so no lane waits on another (a warp-collective shared
          // atomic here sat on every block's critical path)
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
          acc_far += s_all;   // far block: every pair is in the last position bin
        }
        tmem_st8(lane_base + s_col(x) + p_col(cc), pk_p);
        // dS^T row chunk -> shared memory, [key][query] with the 128-byte swizzle
#pragma unroll
        for (int u = 0; u < kSub / 8; ++u) {
          const int unit = (cc / 8) + u;
          *reinterpret_cast<uint4 *>(ds_row + ((unit ^ (jl & 7)) << 4)) =
              make_uint4(pk_d[4 * u], pk_d[4 * u + 1], pk_d[4 * u + 2], pk_d[4 * u + 3]);
        }
      };
#pragma unroll 1
      for (int c0 = hx * (kBlk / 2); c0 < (hx + 1) * (kBlk / 2); c0 += kSub) {
        uint32_t rs[kSub], rd[kSub];
        const int ci = 2 * jb + ((c0 / kSub) & 1);
        if (lane == 0) trace_put(trs, warp, trn, 8u, ci);
        tmem_ld16(lane_base + s_col(x) + c0, rs);
        tmem_ld16(lane_base + dp_col(x) + c0, rd);
        tmem_wait_ld(rs);
        tmem_wait_ld(rd);
        if (lane == 0) trace_put(trs, warp, trn, 9u, ci);
        do_chunk(rs, rd, c0);
        if (lane == 0) trace_put(trs, warp, trn, 10u, ci);
      }
      tmem_wait_st();
      if (lane == 0) trace_put(trs, warp, trn, 11u, jb);
      tc_fence_before();
      fence_proxy_async_smem();
      if (lane == 0) trace_put(trs, warp, trn, 2u, jb);
      mbar_arrive(&sm.p_full[x]);
      // dQ^T_j (thread = feature d, column = query) -> float32 accumulator;
      // a warp's 32 lanes cover 128 contiguous bytes of one query row.
      ok = wait_bar_warp(&sm.dq_full[x], (jb >> 1) & 1, p.wait);
      if (!ok) break;
      tc_fence_after();
      if (lane == 0) trace_put(trs, warp, trn, 3u, jb);
      {
        // the half's 32 columns to registers first: the columns go back to
        // the tensor cores (next dP^T) while the reductions drain
        uint32_t rq[32];
        tmem_ld32(lane_base + dp_col(x) + hx * 32, rq);
        tmem_wait_ld(rq);
        tc_fence_before();
        mbar_arrive(&sm.dq_empty[x]);
        const int32_t nq = min(kBlk, g.L - qs) - hx * 32;   // this half's queries in the sequence
        // a warp's 32 lanes (features) cover 128 contiguous bytes of one query row
        float *dst = p.dq_acc + (int64_t(h) * p.total_tokens + sq.start + qs + hx * 32) * D + jl;
#pragma unroll
        for (int c = 0; c < 32; ++c)
          if (c < nq) red_add_f32(dst + c * D, __uint_as_float(rq[c]));
      }
      if (lane == 0) trace_put(trs, warp, trn, 4u, jb);
    }
    // ---- epilogue: dV (group 0) or dK (group 1), thread = key row ----
    if (ok) ok = wait_bar_warp(&sm.done, 0, p.wait);
    tc_fence_after();
    if (ok) {
      const uint32_t col = x == 0 ? kDvCol : kDkCol;
      const float scale = x == 0 ? p.dv_scale : p.dk_scale;
      __nv_bfloat16 *orow = x == 0 ? p.dv + (sq.start + j) * p.dv_rs + int64_t(h) * D
                                   : p.dk + (sq.start + j) * p.dk_rs + int64_t(h) * D;
      // a split key tile whose part of the run held no block has nothing to add
      const bool any_block = qb_first >= 0;
#pragma unroll 1
      for (int c0 = hx * (D / 2); c0 < (hx + 1) * (D / 2); c0 += 32) {
        uint32_t r[32];
        tmem_ld32(lane_base + col + c0, r);
        tmem_wait_ld(r);
        if (split) {
          if (key_ok && any_block) {
            // the key tile's rows from its first accumulator row on
            const int64_t a_row = p.kitem_acc[item_idx] + jl;
            float *acc = (x == 0 ? p.dv_acc : p.dk_acc) + (a_row * p.num_heads + h) * int64_t(D) + c0;
#pragma unroll
            for (int e = 0; e < 32; e += 4)
              red_add_v4_f32(acc + e, __uint_as_float(r[e]), __uint_as_float(r[e + 1]),
                             __uint_as_float(r[e + 2]), __uint_as_float(r[e + 3]));
          }
        } else if (key_ok) {
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
    {
      float af = acc_far;   // the last position bin: one shared atomic per warp
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) af += __shfl_xor_sync(0xffffffffu, af, o);
      if (lane == 0 && af != 0.f) atomicAdd(&sm.hist_p[nb_p_m1], af);
    }
    __threadfence();   // this thread's reductions into the CTA's global bins are done
    named_bar_sync(1, 512);
    const int tid_ew = tid - 128;
    const int nt = fast ? fast_table_size(p.sub_bits) : p.nb_t;
    float *gp = p.drab_p + tab * p.nb_p;
    float *gt = p.drab_t + tab * p.nb_t;
    for (int xx = tid_ew; xx < p.nb_p; xx += 512) {
      const float v = sm.hist_p[xx] + __ldcg(gbin_p + xx);
      if (v != 0.f) atomicAdd(gp + xx, v * p.drab_scale);
    }
    for (int xx = tid_ew; xx < nt; xx += 512) {
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

}  // namespace bwd128

cudaError_t launch_bwd128(const AttnProblem &p, const Scratch &s, const void *dout, void *dq,
                          void *dk, void *dv, float *drab_p, float *drab_t, const WaitCtl &w,
                          cudaStream_t st) {
  using namespace bwd128;
  if (p.d_qk != D || p.d_v != D) return cudaErrorInvalidValue;
  CUtensorMap tq, tk, tv, tdo;
  const uint64_t T = uint64_t(p.total_tokens);
  if (!encode_tmap_bf16_3d(&tq, p.q, D, p.num_heads, T, D * 2, uint64_t(p.q_rs) * 2, 64, 1,
                           kBlk) ||
      !encode_tmap_bf16_3d(&tk, p.k, D, p.num_heads, T, D * 2, uint64_t(p.k_rs) * 2, 64, 1,
                           kKeys) ||
      !encode_tmap_bf16_3d(&tv, p.v, D, p.num_heads, T, D * 2, uint64_t(p.v_rs) * 2, 64, 1,
                           kKeys) ||
      !encode_tmap_bf16_3d(&tdo, dout, D, p.num_heads, T, D * 2, uint64_t(p.do_rs) * 2, 64, 1,
                           kBlk))
    return cudaErrorInvalidValue;
  const size_t acc_bytes = sizeof(float) * size_t(T) * p.num_heads * D;
  cudaError_t e = cudaMemsetAsync(s.dq_acc, 0, acc_bytes, st);
  if (e != cudaSuccess) return e;
  const unsigned grid = unsigned(s.n_kitems) * unsigned(p.num_heads);
  e = cudaMemsetAsync(s.bin_acc, 0, sizeof(float) * kBinAccPerCta * size_t(grid), st);
  if (e != cudaSuccess) return e;
  BwdParams prm;
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
  prm.dk_acc = s.dk_acc;
  prm.dv_acc = s.dv_acc;
  prm.kitem_acc = s.kitem_acc;
  const bool split = s.n_ksplit_rows > 0;
  if (split) {
    if (!s.dk_acc || !s.dv_acc) return cudaErrorInvalidValue;
    const size_t acc = sizeof(float) * size_t(s.n_ksplit_acc_rows) * p.num_heads * D;
    e = cudaMemsetAsync(s.dk_acc, 0, acc, st);
    if (e == cudaSuccess) e = cudaMemsetAsync(s.dv_acc, 0, acc, st);
    if (e != cudaSuccess) return e;
  }
  const size_t smem = sizeof(Smem) + 1024;
  static PerDeviceOnce attr;
  e = set_smem_once(attr, bwd128_kernel, smem);
  if (e != cudaSuccess) return e;
  bwd128_kernel<<<grid, kThreads, smem, st>>>(tq, tk, tv, tdo, prm);
  count_launch();
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  if (split) {
    e = launch_rows_to_bf16(s.dk_acc, dk, p.dk_rs, p.num_heads, D, s.ksplit_rows,
                            s.n_ksplit_rows, prm.dk_scale, st);
    if (e == cudaSuccess)
      e = launch_rows_to_bf16(s.dv_acc, dv, p.dv_rs, p.num_heads, D, s.ksplit_rows,
                              s.n_ksplit_rows, prm.dv_scale, st);
    if (e != cudaSuccess) return e;
  }
  return launch_dq_convert(p, s, dq, st);
}

}  // namespace hstu

namespace hstu {

// Phase trace buffer of the d = 128 backward (see g_trace): copy out / clear.
bool trace_bwd128_read(void *host, size_t bytes) {
#ifdef HSTU_TRACE
  const size_t n = bytes < sizeof(bwd128::g_trace) ? bytes : sizeof(bwd128::g_trace);
  return cudaMemcpyFromSymbol(host, bwd128::g_trace, n) == cudaSuccess;
#else
  (void)host;
  (void)bytes;
  return false;
#endif
}

bool trace_bwd128_clear() {
#ifdef HSTU_TRACE
  void *ptr = nullptr;
  if (cudaGetSymbolAddress(&ptr, bwd128::g_trace) != cudaSuccess) return false;
  return cudaMemset(ptr, 0, sizeof(bwd128::g_trace)) == cudaSuccess &&
         cudaDeviceSynchronize() == cudaSuccess;
#else
  return false;
#endif
}

}  // namespace hstu
