// attn_fwd_sm100.cu -- forward HSTU pointwise attention on the 5th-generation
// tensor cores (tcgen05 + tensor memory + TMA), bf16 in, fp32 accumulate.
//
// Computes, per sequence, head and query row i (include/hstu.h):
//   out_i = silu_scale * sum_{visible j} SiLU(alpha <q_i,k_j> + rab_p[bp] + rab_t[bt]) v_j
// (pointwise aggregation with a positional and temporal bias: DLRMv4 article,
// section "Model architecture: HSTU replaces the feature-interaction stack";
// candidates appended at the end of the causal sequence: section "How one
// training sample is processed by HSTU").
//
// Design (one CTA = one (sequence, head, pair of 128-row query tiles)):
//   warp 0      TMA producer: both Q tiles once, then K/V tiles through a
//               2-stage ring; also stages the keys' timestamps.
//   warp 1      tcgen05 issuer (one thread): S_X = Q_X K^T into tensor memory,
//               O_X += P_X V with P_X read from tensor memory.
//   warps 4-7   elementwise warpgroups for query tile A, key columns [0, 64)
//   warps 12-15 and [64, 128) (thread = query row); warps 8-11 and 16-19 the
//               same for tile B.  Four warps per sub-partition hide the
//               latency of the per-element chain.  Each loads its half of the
//               S row from tensor memory, adds the position / time bias,
//               applies SiLU and the mask, and writes P (bf16) back over the
//               half's own S columns; at the end it scales its half of O and
//               stores it.
// Tensor memory (512 columns): S_A [0,128) S_B [128,256) O_A [256,+D) O_B [384,+D).
// P of key columns [64h, 64h + 64) lies at S columns [64h, 64h + 32).
// Both query tiles share every K/V tile, halving K/V traffic.  Key tiles that
// no row of the pair can see (causal upper triangle, M-FALCON
// candidate-candidate blocks) are never loaded or multiplied.
//
// Per-element work is kept small: the logit is folded as h = s/2 so that
// SiLU(s) = s sigmoid(s) = h (1 + tanh h) needs one MUFU op (sigmoid(s) =
// (1 + tanh(s/2)) / 2).  Far from the diagonal the position bucket is constant and is
// folded into a per-row constant; the time bucket comes from the float
// exponent table (see common.cuh) when the sequence's time span allows it.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "internal.h"
#include "tile_common.cuh"

namespace hstu {
namespace fwd_tc {

constexpr int kTile = kAttnTile;  // rows per query tile and keys per key tile
constexpr int kStages = 2;        // K/V ring depth
constexpr int kThreads = 640;     // one control warpgroup + four elementwise (96 registers each)
// Column (from the tile's S start) of P for key columns [c, c + 16), c a multiple of 16.
__host__ __device__ constexpr uint32_t p_col(int c) { return uint32_t((c & ~63) + (c & 63) / 2); }
constexpr int kMaxTbl = 1024;     // max table entries (position, time) in shared memory

struct Params {
  const SeqInfo *seqs;
  const int4 *items;      // {seq, pair, first key tile, end key tile (kUnsplit: all)}
  int32_t num_heads;
  const float *tf;        // float(t - t_min) per token
  const int64_t *ts;      // raw timestamps
  const int32_t *seq_fast;
  const float *rab_p, *rab_t;
  int32_t rab_per_head, nb_p, nb_t, sub_bits;
  float alpha, out_scale;  // out_scale = silu_scale
  __nv_bfloat16 *out;
  int64_t o_rs;
  int64_t total_tokens;
  WaitCtl wait;
  uint64_t drain_ns;
  // Cached-history mode (candidate micro-batches, see launch_fwd_tc_cached):
  // queries are candidates in their own buffers, keys and values the cached
  // history.  Per sequence the first candidate row; the candidates' float /
  // int64 times; the candidates' own q, k, v rows for the self pair.
  const int64_t *cstart;
  const float *tfc;
  const int64_t *tsc;
  const __nv_bfloat16 *q_self, *k_self, *v_self;
  int64_t qs_rs, ks_rs, vs_rs;
  float *o_acc;           // split pairs: float32 partial outputs [split rows][H][D]
  const int32_t *item_acc;  // first accumulator row of each item's pair (split items)
};

template <int D>
struct Smem {
  static constexpr int kTileBytes = kTile * D * 2;   // one 128 x D bf16 tile
  alignas(1024) uint8_t q[2][kTileBytes];
  alignas(1024) uint8_t k[kStages][kTileBytes];
  alignas(1024) uint8_t v[kStages][kTileBytes];
  alignas(16) int64_t tk[kStages][kTile];            // key timestamps (float or int64)
  float tbl_p[kMaxTbl];                               // 0.5 * rab_p
  float tbl_t[kMaxTbl];                               // 0.5 * rab_t (or its exponent table)
  uint64_t q_full;
  uint64_t k_full[kStages], v_full[kStages], t_full[kStages], kv_empty[kStages];
  uint64_t s_full[2], p_full[2];
  uint64_t o_full;
  uint64_t drain;
  uint32_t tmem_base;
};

// Time-bucket table index of query i against key column c of stage st.
__device__ __forceinline__ int32_t fwd_time_index(const float *tkf, int c, float t_i_f, int sh,
                                                  int32_t r0) {
  const float dt = t_i_f - tkf[c];
  const int32_t rr = __float_as_int(dt) >> sh;
  return (rr > r0 ? rr : r0) - r0;
}

// How a 32-key chunk finds its time buckets (chosen warp-uniformly by the caller).
enum FwdT : int {
  kFwdUni = 0,   // one bucket for the whole chunk: bias folded into row_c / uni_tb
  kFwdTwo = 1,   // each row sees buckets b_lo and b_lo + 1 (fast, sorted times): one compare
  kFwdAny = 2,   // per-pair bucket and table lookup
};

// One 32-key chunk of one query row: P = SiLU(alpha s + bias) (masked), as
// bf16 pairs.  TM says how the time bias is found (FwdT).  For kFwdTwo,
// with T the float whose bits are (b_lo + 1 + R0) << (23 - sub_bits), on the
// exponent-table index bucket >= b_lo + 1 exactly when dt >= T (dt >= 0 in
// an unmasked chunk); thr = t_i - T, so that holds when t_j <= thr; c_lo /
// c_hi carry the two biases.
template <int D, bool MASK, bool GATHER_P, bool FAST_T, int TM, bool CACHED>
__device__ __forceinline__ void softmaxless_chunk(uint32_t (&r)[32], uint32_t (&pk)[16],
                                                  const Smem<D> &sm, int st, int c0, int32_t ks,
                                                  int32_t i, int32_t pos_i, float t_i_f,
                                                  int64_t t_i, float alpha_h, float row_c,
                                                  float uni_tb, float thr, float c_lo, float c_hi,
                                                  const TileGeom &g, int nb_p_m1,
                                                  int sub_bits, int nb_t) {
  static_assert(TM != kFwdTwo || FAST_T, "the two-bucket split needs float time deltas");
  const int sh = 23 - sub_bits;
  const int32_t r0 = fast_r0(sub_bits);
  const float *tkf = reinterpret_cast<const float *>(&sm.tk[st][0]);
  // the chunk's 32 key times are the same for every lane: 16-byte loads,
  // four keys at a time, instead of one shared load per element
  float tk4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int e = 0; e < 32; e += 2) {
    float pv[2];
    if constexpr (TM == kFwdTwo || (TM == kFwdAny && FAST_T)) {
      if ((e & 3) == 0) {
        const float4 t4 = *reinterpret_cast<const float4 *>(tkf + c0 + e);
        tk4[0] = t4.x;
        tk4[1] = t4.y;
        tk4[2] = t4.z;
        tk4[3] = t4.w;
      }
    }
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int c = c0 + e + u;
      const int32_t j = ks + c;
      const float tkc = tk4[(e & 3) + u];   // tkf[c] on the float-time paths
      float h;
      bool hi = false;
      if constexpr (TM == kFwdTwo) hi = tkc <= thr;
      if constexpr (GATHER_P) {
        const int32_t dp = pos_i - g.pos(j);
        const int32_t bp = dp < nb_p_m1 ? (dp > 0 ? dp : 0) : nb_p_m1;
        const float cp = TM == kFwdUni   ? sm.tbl_p[bp] + uni_tb
                         : TM == kFwdTwo ? sm.tbl_p[bp] + (hi ? c_hi : c_lo)
                                         : sm.tbl_p[bp];
        h = fmaf(alpha_h, __uint_as_float(r[e + u]), cp);
      } else {
        h = fmaf(alpha_h, __uint_as_float(r[e + u]), TM == kFwdTwo ? (hi ? c_hi : c_lo) : row_c);
      }
      if constexpr (TM != kFwdAny) {
      } else if constexpr (FAST_T) {
        const float dt = t_i_f - tkc;
        const int32_t rr = __float_as_int(dt) >> sh;
        h += sm.tbl_t[(rr > r0 ? rr : r0) - r0];
      } else {
        h += sm.tbl_t[time_bucket_i64(t_i - sm.tk[st][c], sub_bits, nb_t)];
      }
      float pval = fmaf(h, tanh_approx(h), h);
      if constexpr (MASK) {
        // cached history: a candidate sees every history key (its self pair
        // is added in the epilogue); the last key tile may reach past them
        const bool vis = CACHED ? (j < g.nh)
                                : ((j < g.L) && (i < g.nh ? (j <= i) : (j < g.nh || j == i)));
        pval = vis ? pval : 0.0f;
      }
      pv[u] = pval;
    }
    pk[e / 2] = pack_bf16x2(pv[0], pv[1]);
  }
}

// ---- optional phase trace (library built with -DHSTU_TRACE; a no-op otherwise) ----
// Three CTAs (grid blocks 0, n/2, n-1) record the SM clock at each phase
// boundary of every key tile: per warp (lane 0) for the elementwise warps,
// per issued batch for the MMA issuer.  Entry = code << 56 | ordinal << 40 |
// clock.  Codes: 1 key tile start (its S and key timestamps ready, ordinal
// the key-tile step n), 8 / 9 / 10 a 32-key chunk's tensor-memory load
// issued / landed / math done (ordinal 2 n + chunk), 11 P stores done, 2 P
// handed to the issuer; issuer: 5 O += P V issued, 6 the next S issued
// (ordinal 2 n + query tile, n the step the MMA serves).
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

template <int D, bool CACHED>
__global__ void __launch_bounds__(kThreads, 1)
    fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
               const __grid_constant__ CUtensorMap tm_v, const Params p) {
  extern __shared__ uint8_t smem_raw[];
  Smem<D> &sm = *reinterpret_cast<Smem<D> *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  const int32_t item_idx = blockIdx.x / p.num_heads;
  const int32_t h = blockIdx.x % p.num_heads;
  const int4 item = p.items[item_idx];
  const SeqInfo sq = p.seqs[item.x];
  // A pair split over key ranges takes key tiles [kt_lo, kt_hi) and adds its
  // partial output into o_acc (pointwise attention sums over keys, so the
  // pieces add up); an unsplit pair takes them all and stores bf16.
  const bool split = item.w != kUnsplit;
  const int32_t kt_lo = item.z;
  const TileGeom g{sq.len, sq.n_hist};
  const int32_t qtile[2] = {2 * item.y, 2 * item.y + 1};
  const bool fast = (p.seq_fast[item.x] & kSeqFastTime) != 0 && p.sub_bits <= 4;
  // Cached history: query tile qt holds candidates [128 qt, 128 qt + 128) of
  // the sequence's n_c = L - n_h, at virtual local index n_h + c (position
  // n_h); every key tile is a history tile.
  const int32_t n_cand = sq.len - sq.n_hist;
  const int64_t qrow_base = CACHED ? p.cstart[item.x] : sq.start;
  auto qvalid = [&](int32_t qt) { return CACHED ? qt * kTile < n_cand : g.valid(qt); };
  auto act = [&](int32_t qt, int32_t kt) {
    return CACHED ? (qt * kTile < n_cand && kt * kTile < g.nh) : g.active(qt, kt);
  };
  const int32_t last_kt = min(CACHED ? (g.nh > 0 ? (g.nh - 1) / kTile : -1)
                                     : max(g.valid(qtile[1]) ? qtile[1] : qtile[0], 0),
                              item.w - 1);

  // ---- tables (all threads) ----
  {
    const float *rp = p.rab_p + (p.rab_per_head ? h * p.nb_p : 0);
    const float *rt = p.rab_t + (p.rab_per_head ? h * p.nb_t : 0);
    for (int x = tid; x < p.nb_p; x += kThreads) sm.tbl_p[x] = 0.5f * rp[x];
    if (fast) {
      const int n = fast_table_size(p.sub_bits);
      for (int x = tid; x < n; x += kThreads)
        sm.tbl_t[x] = 0.5f * rt[fast_table_bucket(x, p.sub_bits, p.nb_t)];
    } else {
      for (int x = tid; x < p.nb_t; x += kThreads) sm.tbl_t[x] = 0.5f * rt[x];
    }
  }
  if (warp == 0 && lane == 0) {
    mbar_init(&sm.q_full, 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&sm.k_full[s], 1);
      mbar_init(&sm.v_full[s], 1);
      mbar_init(&sm.t_full[s], 32);
      mbar_init(&sm.kv_empty[s], 1);
    }
    for (int x = 0; x < 2; ++x) {
      mbar_init(&sm.s_full[x], 1);
      mbar_init(&sm.p_full[x], 2 * kTile);
    }
    mbar_init(&sm.o_full, 1);
    mbar_init(&sm.drain, 1);
    fence_mbar_init();
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
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
  constexpr uint32_t kHalfBytes = kTile * 64 * 2;   // one 128 x 64 bf16 box
  constexpr int kHalves = D / 64;

  if (warp == 0) {
    // ===================== TMA producer =====================
    const bool leader = elect_one();
    if (leader) {
      uint32_t bytes = kHalves * kHalfBytes;
      if (qvalid(qtile[1])) bytes *= 2;
      mbar_arrive_expect_tx(&sm.q_full, bytes);
      for (int x = 0; x < 2; ++x) {
        if (!qvalid(qtile[x])) continue;
        for (int hv = 0; hv < kHalves; ++hv)
          tma_load_3d(sm.q[x] + hv * kHalfBytes, &tm_q, &sm.q_full, hv * 64, h,
                      int32_t(qrow_base + qtile[x] * kTile));
      }
    }
    __syncwarp();
    int n = 0;
    bool ok = true;
    for (int32_t kt = kt_lo; kt <= last_kt && ok; ++kt) {
      if (!act(qtile[0], kt) && !act(qtile[1], kt)) continue;
      const int st = n % kStages;
      if (n >= kStages) ok = wait_bar_warp(&sm.kv_empty[st], ((n / kStages) - 1) & 1, p.wait);
      if (!ok) break;
      const int32_t row = int32_t(sq.start + kt * kTile);
      if (leader) {
        mbar_arrive_expect_tx(&sm.k_full[st], kHalves * kHalfBytes);
        for (int hv = 0; hv < kHalves; ++hv)
          tma_load_3d(sm.k[st] + hv * kHalfBytes, &tm_k, &sm.k_full[st], hv * 64, h, row);
        mbar_arrive_expect_tx(&sm.v_full[st], kHalves * kHalfBytes);
        for (int hv = 0; hv < kHalves; ++hv)
          tma_load_3d(sm.v[st] + hv * kHalfBytes, &tm_v, &sm.v_full[st], hv * 64, h, row);
      }
      for (int x = lane; x < kTile; x += 32) {
        const int32_t j = kt * kTile + x;
        int64_t val = 0;
        if (j < (CACHED ? g.nh : g.L)) {
          if (fast) {
            const float f = p.tf[sq.start + j];
            val = int64_t(__float_as_uint(f));
          } else {
            val = p.ts[sq.start + j];
          }
        }
        if (fast)
          reinterpret_cast<float *>(&sm.tk[st][0])[x] = __uint_as_float(uint32_t(val));
        else
          sm.tk[st][x] = val;
      }
      mbar_arrive(&sm.t_full[st]);
      ++n;
    }
    // Wait for this warp's own copies still in flight before leaving.
    if (leader) {
      drain_bar(&sm.q_full, 0, p.wait.err, p.drain_ns);
      for (int m = (n > kStages ? n - kStages : 0); m < n; ++m) {
        const int st = m % kStages;
        drain_bar(&sm.k_full[st], (m / kStages) & 1, p.wait.err, p.drain_ns);
        drain_bar(&sm.v_full[st], (m / kStages) & 1, p.wait.err, p.drain_ns);
      }
    }
  } else if (warp == 1) {
    // ===================== tcgen05 issuer =====================
    if (elect_one()) {
      constexpr uint32_t idesc_s = idesc_bf16(kTile, kTile, false, false);
      constexpr uint32_t idesc_o = idesc_bf16(kTile, D, false, true);
      const uint32_t q_addr[2] = {smem_u32(sm.q[0]), smem_u32(sm.q[1])};
      bool ok = wait_bar(&sm.q_full, 0, p.wait);
      tc_fence_after();
      // Step list: key tiles active for A or B, in order.
      auto next_kt = [&](int32_t kt) {
        for (++kt; kt <= last_kt; ++kt)
          if (act(qtile[0], kt) || act(qtile[1], kt)) return kt;
        return int32_t(-1);
      };
      // Descriptors are linear in the address (start field = address >> 4,
      // no carry inside shared memory): built once per batch, advanced by
      // (offset >> 4) per MMA.
      auto issue_s = [&](int x, int st) {
        const uint64_t dq = sdesc_sw128(q_addr[x], 16, 1024);
        const uint64_t dk = sdesc_sw128(smem_u32(sm.k[st]), 16, 1024);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = ((kk / 4) * kHalfBytes + (kk % 4) * 32) >> 4;
          umma_ss(tmem + x * 128, dq + off, dk + off, idesc_s, kk > 0);
        }
        umma_commit(&sm.s_full[x]);
      };
      bool first_o[2] = {true, true};
      uint32_t p_phase[2] = {0, 0};
      auto issue_o = [&](int x, int st) {
        const uint64_t dv = sdesc_sw128(smem_u32(sm.v[st]), kHalfBytes, 1024);
#pragma unroll
        for (int kk = 0; kk < kTile / 16; ++kk) {
          umma_ts(tmem + 256 + x * 128, tmem + x * 128 + p_col(kk * 16), dv + ((kk * 16 * 128) >> 4),
                  idesc_o, (first_o[x] && kk == 0) ? 0u : 1u);
        }
        first_o[x] = false;
      };
      int32_t kt = ok ? next_kt(kt_lo - 1) : -1;
      int n = 0;
      if (kt >= 0) {
        ok = wait_bar(&sm.k_full[0], 0, p.wait);
        tc_fence_after();
        if (ok) {
          for (int x = 0; x < 2; ++x)
            if (act(qtile[x], kt)) issue_s(x, 0);
        }
      }
      while (ok && kt >= 0) {
        const int st = n % kStages;
        const int32_t kt_next = next_kt(kt);
        const int st_next = (n + 1) % kStages;
        bool k_next_ready = false;
        ok = wait_bar(&sm.v_full[st], (n / kStages) & 1, p.wait);
        if (!ok) break;
        for (int x = 0; x < 2 && ok; ++x) {
          if (act(qtile[x], kt)) {
            ok = wait_bar(&sm.p_full[x], p_phase[x] & 1, p.wait);
            if (!ok) break;
            ++p_phase[x];
            tc_fence_after();
            issue_o(x, st);
            trace_put(trs, 1, trn, 5u, 2 * n + x);
          }
          if (kt_next >= 0 && act(qtile[x], kt_next)) {
            if (!k_next_ready) {
              ok = wait_bar(&sm.k_full[st_next], ((n + 1) / kStages) & 1, p.wait);
              if (!ok) break;
              tc_fence_after();
              k_next_ready = true;
            }
            issue_s(x, st_next);
            trace_put(trs, 1, trn, 6u, 2 * (n + 1) + x);
          }
        }
        if (!ok) break;
        umma_commit(&sm.kv_empty[st]);
        kt = kt_next;
        ++n;
      }
      umma_commit(&sm.o_full);
      // Drain: every MMA this thread issued has completed before teardown.
      umma_commit(&sm.drain);
      drain_bar(&sm.drain, 0, p.wait.err, p.drain_ns);
    }
    __syncwarp();
  } else if (warp >= 4) {
    // ===================== elementwise warpgroups =====================
    const int x = ((warp - 4) >> 2) & 1;    // 0: tile A, 1: tile B
    const int hx = (warp - 4) >> 3;         // key-column half
    const int quad = warp & 3;               // tensor-memory lane quadrant
    const int32_t qt = qtile[x];
    const int32_t r_loc = qt * kTile + quad * 32 + lane;   // row of the query tile pair
    // local query index (cached history: the candidate's virtual index n_h + c)
    const int32_t i = CACHED ? g.nh + r_loc : r_loc;
    const bool row_ok = CACHED ? r_loc < n_cand : i < g.L;
    const int64_t q_row = qrow_base + r_loc;               // row in the query / output buffers
    const uint32_t lane_base = tmem + (uint32_t(quad * 32) << 16);
    const uint32_t s_col = x * 128;
    if (qvalid(qt)) {
      const int32_t pos_i = CACHED ? g.nh : g.pos(min(i, g.L - 1));
      const float t_i_f = (fast && row_ok) ? (CACHED ? p.tfc[q_row] : p.tf[sq.start + i]) : 0.f;
      const int64_t t_i = (!fast && row_ok) ? (CACHED ? p.tsc[q_row] : p.ts[sq.start + i]) : 0;
      const float alpha_h = 0.5f * p.alpha;
      const float row_c = sm.tbl_p[p.nb_p - 1];
      const int32_t qs = qt * kTile;
      const int nb_p_m1 = p.nb_p - 1;
      const bool sorted = (p.seq_fast[item.x] & kSeqSorted) != 0;
      const int sh = 23 - p.sub_bits;
      const int32_t r0 = fast_r0(p.sub_bits);
      int n = 0, cnt = 0;
      bool ok = true;
      for (int32_t kt = kt_lo; kt <= last_kt && ok; ++kt) {
        const bool act_a = act(qtile[0], kt), act_b = act(qtile[1], kt);
        if (!act_a && !act_b) continue;
        const int st = n % kStages;
        if (act(qt, kt)) {
          ok = wait_bar_warp(&sm.s_full[x], cnt & 1, p.wait);
          if (ok) ok = wait_bar_warp(&sm.t_full[st], (n / kStages) & 1, p.wait);
          if (!ok) break;
          tc_fence_after();
          if (lane == 0) trace_put(trs, warp, trn, 1u, n);
          const int32_t ks = kt * kTile;
          const bool need_mask =
              CACHED ? (ks + kTile > g.nh)
                     : ((ks + kTile > g.L) || (ks + kTile - 1 > qs) || (ks + kTile > g.nh));
          const int32_t kmax = min(ks + kTile - 1, (CACHED ? g.nh : g.L) - 1);
          const bool gather_p = ((CACHED ? g.nh : g.pos(qs)) - g.pos(kmax)) < nb_p_m1;
#pragma unroll 1
          for (int c0 = hx * (kTile / 2); c0 < (hx + 1) * (kTile / 2); c0 += 32) {
            uint32_t r[32];
            uint32_t pk[16];
            const int ci = 2 * n + ((c0 >> 5) & 1);
            if (lane == 0) trace_put(trs, warp, trn, 8u, ci);
            tmem_ld32(lane_base + s_col + c0, r);
            // With sorted timestamps the time bucket is monotone along the
            // keys: equal buckets at the chunk's two ends mean one bucket.
            // Buckets fall along the keys (dt shrinks as j grows): with
            // sorted timestamps equal ends mean one bucket, ends one apart
            // mean two.
            int tm = kFwdAny;
            float uni_tb = 0.f, thr = 0.f, c_lo = 0.f, c_hi = 0.f;
            if (fast && sorted && !need_mask) {
              const float *tkf = reinterpret_cast<const float *>(&sm.tk[st][0]);
              const int32_t b0 = fwd_time_index(tkf, c0, t_i_f, sh, r0);
              const int32_t b1 = fwd_time_index(tkf, c0 + 31, t_i_f, sh, r0);
              if (__all_sync(0xffffffffu, b0 == b1)) {
                tm = kFwdUni;
                uni_tb = sm.tbl_t[b0];
              } else if (__all_sync(0xffffffffu, b0 >= b1 && b0 - b1 <= 1)) {
                tm = kFwdTwo;
                // t_i - t_j >= T  <=>  t_j <= t_i - T: integers below 2^24,
                // so the difference is exact and the per-pair subtraction goes
                thr = t_i_f - __int_as_float((b1 + 1 + r0) << sh);
                c_lo = sm.tbl_t[b1];
                c_hi = sm.tbl_t[b1 + 1];
                if (!gather_p) {
                  c_lo += row_c;
                  c_hi += row_c;
                }
              }
            }
            tmem_wait_ld(r);
            if (lane == 0) trace_put(trs, warp, trn, 9u, ci);
#define HSTU_CHUNK(M_, G_, F_, U_, RC_)                                                      \
  softmaxless_chunk<D, M_, G_, F_, U_, CACHED>(r, pk, sm, st, c0, ks, i, pos_i, t_i_f, t_i,   \
                                               alpha_h, \
                                       RC_, uni_tb, thr, c_lo, c_hi, g, nb_p_m1, p.sub_bits,  \
                                       p.nb_t)
            if (fast) {
              if (need_mask)
                HSTU_CHUNK(true, true, true, kFwdAny, row_c);
              else if (gather_p)
                if (tm == kFwdUni)
                  HSTU_CHUNK(false, true, true, kFwdUni, row_c);
                else if (tm == kFwdTwo)
                  HSTU_CHUNK(false, true, true, kFwdTwo, row_c);
                else
                  HSTU_CHUNK(false, true, true, kFwdAny, row_c);
              else if (tm == kFwdUni)
                HSTU_CHUNK(false, false, true, kFwdUni, row_c + uni_tb);
              else if (tm == kFwdTwo)
                HSTU_CHUNK(false, false, true, kFwdTwo, row_c);
              else
                HSTU_CHUNK(false, false, true, kFwdAny, row_c);
            } else {
              if (need_mask)
                HSTU_CHUNK(true, true, false, kFwdAny, row_c);
              else
                HSTU_CHUNK(false, true, false, kFwdAny, row_c);
            }
#undef HSTU_CHUNK
            if (lane == 0) trace_put(trs, warp, trn, 10u, ci);
            tmem_st16(lane_base + s_col + p_col(c0), pk);
          }
          tmem_wait_st();
          if (lane == 0) trace_put(trs, warp, trn, 11u, n);
          tc_fence_before();
          if (lane == 0) trace_put(trs, warp, trn, 2u, n);
          mbar_arrive(&sm.p_full[x]);
          ++cnt;
        }
        ++n;
      }
      // ---- epilogue: O (fp32, tensor memory) -> bf16 rows ----
      if (ok) ok = wait_bar_warp(&sm.o_full, 0, p.wait);
      tc_fence_after();
      // Cached history: the candidate's own pair (position and time distance
      // 0, buckets 0) on the CUDA cores: P_self = bf16(SiLU(alpha <q, k> +
      // rab_p[0] + rab_t[0])), then O += P_self v, as the tensor-core path
      // rounds P before its A.V product; of a split pair only the piece that
      // starts at key tile 0 adds it.  A candidate whose sequence has no
      // history has no key tile, so its accumulator was never written.
      float p_self = 0.f;
      const __nv_bfloat16 *v_self_row = nullptr;
      if constexpr (CACHED) {
        if (row_ok && (!split || item.z == 0)) {
          const __nv_bfloat16 *qr = p.q_self + q_row * p.qs_rs + int64_t(h) * D;
          const __nv_bfloat16 *kr = p.k_self + q_row * p.ks_rs + int64_t(h) * D;
          float dot = 0.f;
#pragma unroll 4
          for (int c = 0; c < D; c += 8) {
            const uint4 a4 = *reinterpret_cast<const uint4 *>(qr + c);
            const uint4 b4 = *reinterpret_cast<const uint4 *>(kr + c);
            const uint32_t wa[4] = {a4.x, a4.y, a4.z, a4.w}, wb[4] = {b4.x, b4.y, b4.z, b4.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              dot = fmaf(__uint_as_float(wa[e] << 16), __uint_as_float(wb[e] << 16), dot);
              dot = fmaf(__uint_as_float(wa[e] & 0xFFFF0000u), __uint_as_float(wb[e] & 0xFFFF0000u),
                         dot);
            }
          }
          const float hh = fmaf(0.5f * p.alpha, dot, sm.tbl_p[0] + sm.tbl_t[0]);
          p_self = __bfloat162float(__float2bfloat16_rn(fmaf(hh, tanh_approx(hh), hh)));
          v_self_row = p.v_self + q_row * p.vs_rs + int64_t(h) * D;
        }
      }
      const bool o_written = cnt > 0;
      if (ok) {
        __nv_bfloat16 *orow = p.out + (CACHED ? q_row : sq.start + i) * p.o_rs + int64_t(h) * D;
#pragma unroll 1
        for (int c0 = hx * (D / 2); c0 < (hx + 1) * (D / 2); c0 += 32) {
          uint32_t r[32];
          tmem_ld32(lane_base + 256 + x * 128 + c0, r);
          tmem_wait_ld(r);
          if (row_ok) {
            float o[32];
#pragma unroll
            for (int e = 0; e < 32; ++e) o[e] = o_written ? __uint_as_float(r[e]) : 0.f;
            if (CACHED && v_self_row) {
#pragma unroll
              for (int v8 = 0; v8 < 4; ++v8) {
                const uint4 u4 = *reinterpret_cast<const uint4 *>(v_self_row + c0 + 8 * v8);
                const uint32_t wv[4] = {u4.x, u4.y, u4.z, u4.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                  o[8 * v8 + 2 * e] = fmaf(p_self, __uint_as_float(wv[e] << 16), o[8 * v8 + 2 * e]);
                  o[8 * v8 + 2 * e + 1] =
                      fmaf(p_self, __uint_as_float(wv[e] & 0xFFFF0000u), o[8 * v8 + 2 * e + 1]);
                }
              }
            }
            if (split) {
              // partial output of a key range, unscaled, into the float32 sums
              if (o_written || v_self_row) {
                // the pair's rows from its first accumulator row on
                const int64_t a_row = p.item_acc[item_idx] + (r_loc - 2 * kTile * item.y);
                float *acc = p.o_acc + (a_row * p.num_heads + h) * D + c0;
#pragma unroll
                for (int e = 0; e < 32; e += 4)
                  red_add_v4_f32(acc + e, o[e], o[e + 1], o[e + 2], o[e + 3]);
              }
            } else {
              uint32_t w[16];
#pragma unroll
              for (int e = 0; e < 16; ++e)
                w[e] = pack_bf16x2(o[2 * e] * p.out_scale, o[2 * e + 1] * p.out_scale);
              uint4 *dst = reinterpret_cast<uint4 *>(orow + c0);
#pragma unroll
              for (int e = 0; e < 4; ++e)
                dst[e] = make_uint4(w[4 * e], w[4 * e + 1], w[4 * e + 2], w[4 * e + 3]);
            }
          }
        }
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

}  // namespace fwd_tc

bool fwd_tc_supported(const AttnProblem &p) {
  if (p.dtype != 1 || p.d_qk != p.d_v || (p.d_qk != 64 && p.d_qk != 128)) return false;
  if (p.nb_p > fwd_tc::kMaxTbl || p.nb_t > fwd_tc::kMaxTbl) return false;
  if (p.total_tokens >= (int64_t(1) << 31)) return false;
  // TMA: 16-byte aligned bases and row strides.
  const uintptr_t a = reinterpret_cast<uintptr_t>(p.q) | reinterpret_cast<uintptr_t>(p.k) |
                      reinterpret_cast<uintptr_t>(p.v);
  if (a & 15) return false;
  if ((p.q_rs | p.k_rs | p.v_rs) & 7) return false;
  if (p.o_rs & 7) return false;
  return true;
}

template <int D, bool CACHED>
static cudaError_t launch_fwd_tc_d(const AttnProblem &p, const Scratch &s, void *out,
                                   const WaitCtl &w, cudaStream_t st, const CachedHist *ch) {
  using namespace fwd_tc;
  CUtensorMap tq, tk, tv;
  // cached history: queries from the candidate buffers, keys / values from the cache
  const uint64_t Tq = uint64_t(CACHED ? ch->n_cand_tokens : p.total_tokens);
  // With no history at all nothing reads the key / value maps (no key tile
  // is active); they are then encoded over the candidates' own rows, since a
  // map needs a valid base and a non-empty extent.
  const bool no_keys = CACHED && p.total_tokens == 0;
  const void *kb = no_keys ? ch->k_cand : p.k, *vb = no_keys ? ch->v_cand : p.v;
  const uint64_t Tk = uint64_t(no_keys ? ch->n_cand_tokens : p.total_tokens);
  const int64_t k_rs = no_keys ? ch->kc_rs : p.k_rs, v_rs = no_keys ? ch->vc_rs : p.v_rs;
  if (!encode_tmap_bf16_3d(&tq, p.q, D, p.num_heads, Tq, D * 2, uint64_t(p.q_rs) * 2, 64, 1,
                           kTile) ||
      !encode_tmap_bf16_3d(&tk, kb, D, p.num_heads, Tk, D * 2, uint64_t(k_rs) * 2, 64, 1,
                           kTile) ||
      !encode_tmap_bf16_3d(&tv, vb, D, p.num_heads, Tk, D * 2, uint64_t(v_rs) * 2, 64, 1,
                           kTile))
    return cudaErrorInvalidValue;
  Params prm{};
  prm.seqs = s.seqs;
  prm.items = s.items;
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
  prm.out_scale = p.silu_scale;
  prm.out = static_cast<__nv_bfloat16 *>(out);
  prm.o_rs = p.o_rs;
  prm.total_tokens = p.total_tokens;
  prm.wait = w;
  prm.drain_ns = 4000000000ull;
  prm.o_acc = s.o_acc;
  prm.item_acc = s.item_acc;
  if (CACHED) {
    prm.cstart = ch->cstart;
    prm.tfc = ch->tfc;
    prm.tsc = ch->ts_cand;
    prm.q_self = static_cast<const __nv_bfloat16 *>(p.q);
    prm.k_self = static_cast<const __nv_bfloat16 *>(ch->k_cand);
    prm.v_self = static_cast<const __nv_bfloat16 *>(ch->v_cand);
    prm.qs_rs = p.q_rs;
    prm.ks_rs = ch->kc_rs;
    prm.vs_rs = ch->vc_rs;
  }
  // At least 120 KB so a single CTA occupies an SM (it allocates all of TMEM).
  const size_t smem = sizeof(Smem<D>) + 1024 > 120 * 1024 ? sizeof(Smem<D>) + 1024 : 120 * 1024;
  static PerDeviceOnce attr;
  cudaError_t e = set_smem_once(attr, fwd_kernel<D, CACHED>, smem);
  if (e != cudaSuccess) return e;
  const unsigned grid = unsigned(s.n_items) * unsigned(p.num_heads);
  fwd_kernel<D, CACHED><<<grid, kThreads, smem, st>>>(tq, tk, tv, prm);
  count_launch();
  return cudaGetLastError();
}

cudaError_t launch_fwd_tc(const AttnProblem &p, const Scratch &s, void *out, const WaitCtl &w,
                          cudaStream_t st) {
  if (s.n_items == 0) return cudaSuccess;
  const bool split = s.n_split_rows > 0;
  if (split && !s.o_acc) return cudaErrorInvalidValue;
  if (split) {
    const size_t bytes = sizeof(float) * size_t(s.n_split_acc_rows) * p.num_heads * p.d_v;
    cudaError_t e = cudaMemsetAsync(s.o_acc, 0, bytes, st);
    if (e != cudaSuccess) return e;
  }
  cudaError_t e = p.d_qk == 64 ? launch_fwd_tc_d<64, false>(p, s, out, w, st, nullptr)
                               : launch_fwd_tc_d<128, false>(p, s, out, w, st, nullptr);
  if (e != cudaSuccess || !split) return e;
  return launch_rows_to_bf16(s.o_acc, out, p.o_rs, p.num_heads, p.d_v, s.split_rows,
                             s.n_split_rows, p.silu_scale, st);
}

cudaError_t launch_fwd_tc_cached(const AttnProblem &p, const Scratch &s, const CachedHist &ch,
                                 void *out, const WaitCtl &w, cudaStream_t st) {
  if (s.n_items == 0) return cudaSuccess;
  const bool split = s.n_split_rows > 0;
  if (split && !s.o_acc) return cudaErrorInvalidValue;
  if (split) {
    const size_t bytes = sizeof(float) * size_t(s.n_split_acc_rows) * p.num_heads * p.d_v;
    cudaError_t e = cudaMemsetAsync(s.o_acc, 0, bytes, st);
    if (e != cudaSuccess) return e;
  }
  cudaError_t e = p.d_qk == 64 ? launch_fwd_tc_d<64, true>(p, s, out, w, st, &ch)
                               : launch_fwd_tc_d<128, true>(p, s, out, w, st, &ch);
  if (e != cudaSuccess || !split) return e;
  return launch_rows_to_bf16(s.o_acc, out, p.o_rs, p.num_heads, p.d_v, s.split_rows,
                             s.n_split_rows, p.silu_scale, st);
}

// Phase trace buffer of the forward (see g_trace): copy out / clear.
bool trace_fwd_read(void *host, size_t bytes) {
#ifdef HSTU_TRACE
  const size_t n = bytes < sizeof(fwd_tc::g_trace) ? bytes : sizeof(fwd_tc::g_trace);
  return cudaMemcpyFromSymbol(host, fwd_tc::g_trace, n) == cudaSuccess;
#else
  (void)host;
  (void)bytes;
  return false;
#endif
}

bool trace_fwd_clear() {
#ifdef HSTU_TRACE
  void *ptr = nullptr;
  if (cudaGetSymbolAddress(&ptr, fwd_tc::g_trace) != cudaSuccess) return false;
  return cudaMemset(ptr, 0, sizeof(fwd_tc::g_trace)) == cudaSuccess &&
         cudaDeviceSynchronize() == cudaSuccess;
#else
  return false;
#endif
}

}  // namespace hstu
