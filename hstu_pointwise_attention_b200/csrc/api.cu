// api.cu -- the extern "C" entry points of libhstu.so (include/hstu.h):
// argument validation, the jagged tile schedule, workspace carving and the
// launches.  Everything here is host code; every step of the computation runs
// in the kernels of attn_*.cu and layer.cu.
#include <cudaTypedefs.h>
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstring>
#include <mutex>
#include <vector>

#include "../../include/hstu.h"
#include "internal.h"

namespace hstu {

cudaError_t launch_gemm(const void *a, int64_t lda, const void *b, int64_t ldb,
                        const float *bias, const void *residual, int64_t ldr, void *c,
                        int64_t ldc, int64_t M, int64_t N, int64_t K, int epilogue,
                        const WaitCtl &w, cudaStream_t st) {
  const bool res_ok = epilogue != kEpiBiasResidual ||
                      ((reinterpret_cast<uintptr_t>(residual) & 15) == 0 && ldr % 8 == 0);
  const bool bias_ok = (reinterpret_cast<uintptr_t>(bias) & 15) == 0;   // float4 loads
  if (res_ok && bias_ok && gemm_tc_supported(a, lda, b, ldb, c, ldc, M, N, K))
    return launch_gemm_tc(a, lda, b, ldb, bias, residual, ldr, c, ldc, M, N, K, epilogue, w, st);
  return launch_gemm_simt(a, lda, b, ldb, bias, residual, ldr, c, ldc, M, N, K, epilogue, st);
}

// ---------------------------------------------------------------------------
// Tensor maps (driver entry point fetched through the runtime; no libcuda link)
// ---------------------------------------------------------------------------
static PFN_cuTensorMapEncodeTiled_v12000 tmap_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void *ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  }
  return fn;
}

bool encode_tmap_bf16_3d(CUtensorMap *map, const void *base, uint64_t d0, uint64_t d1,
                         uint64_t d2, uint64_t stride1_bytes, uint64_t stride2_bytes,
                         uint32_t box0, uint32_t box1, uint32_t box2) {
  auto enc = tmap_encoder();
  if (!enc) return false;
  const cuuint64_t dims[3] = {d0, d1, d2};
  const cuuint64_t strides[2] = {stride1_bytes, stride2_bytes};
  const cuuint32_t box[3] = {box0, box1, box2};
  const cuuint32_t estr[3] = {1, 1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides,
             box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
         CUDA_SUCCESS;
}

static bool encode_tmap_2d(CUtensorMapDataType dt, CUtensorMap *map, const void *base,
                           uint64_t d0, uint64_t d1, uint64_t stride1_bytes, uint32_t box0,
                           uint32_t box1, bool swizzle = true) {
  auto enc = tmap_encoder();
  if (!enc) return false;
  const cuuint64_t dims[2] = {d0, d1};
  const cuuint64_t strides[1] = {stride1_bytes};
  const cuuint32_t box[2] = {box0, box1};
  const cuuint32_t estr[2] = {1, 1};
  return enc(map, dt, 2, const_cast<void *>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE,
             swizzle ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
         CUDA_SUCCESS;
}

bool encode_tmap_bf16_2d(CUtensorMap *map, const void *base, uint64_t d0, uint64_t d1,
                         uint64_t stride1_bytes, uint32_t box0, uint32_t box1) {
  return encode_tmap_2d(CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, map, base, d0, d1, stride1_bytes, box0,
                        box1);
}

bool encode_tmap_bf16_2d_sw64(CUtensorMap *map, const void *base, uint64_t d0, uint64_t d1,
                              uint64_t stride1_bytes, uint32_t box0, uint32_t box1) {
  auto enc = tmap_encoder();
  if (!enc) return false;
  const cuuint64_t dims[2] = {d0, d1};
  const cuuint64_t strides[1] = {stride1_bytes};
  const cuuint32_t box[2] = {box0, box1};
  const cuuint32_t estr[2] = {1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides,
             box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
         CUDA_SUCCESS;
}

bool encode_tmap_f32_2d(CUtensorMap *map, const void *base, uint64_t d0, uint64_t d1,
                        uint64_t stride1_bytes, uint32_t box0, uint32_t box1, bool swizzle) {
  return encode_tmap_2d(CU_TENSOR_MAP_DATA_TYPE_FLOAT32, map, base, d0, d1, stride1_bytes, box0,
                        box1, swizzle);
}

// ---------------------------------------------------------------------------
// Validation, plan and workspace
// ---------------------------------------------------------------------------
static std::atomic<uint64_t> g_wait_limit_ns{0};   // 0: default
static std::atomic<uint64_t> g_launches{0};

void count_launch(int n) { g_launches.fetch_add(uint64_t(n), std::memory_order_relaxed); }
static constexpr uint64_t kDefaultWaitNs = 4000000000ull;

static size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

struct Plan {
  int64_t T = 0;
  std::vector<SeqInfo> seqs;
  std::vector<int4> items;        // tensor-core forward: {seq, tile pair, key tiles [z, w)}
  std::vector<int2> simt_items;   // CUDA-core: {seq, 64-row tile}
  std::vector<int4> kitems;       // tensor-core backward: {seq, key tile, query blocks [z, w)}
  std::vector<int32_t> item_acc, kitem_acc;   // first accumulator row of a split item, else -1
  std::vector<int4> split_rows;   // forward: {first row, rows, first accumulator row}
  std::vector<int4> ksplit_rows;  // backward: {first key row, rows, first accumulator row}
  int32_t split_acc_rows = 0, ksplit_acc_rows = 0;
};

struct WsLayout {
  size_t err, seqs, items, simt_items, kitems, split_rows, ksplit_rows, item_acc, kitem_acc, tf,
      seq_fast, dq_acc, bin_acc, o_acc, dk_acc, dv_acc, total;
};

// The tile schedule assumes a B200's SM count (a fixed number keeps plans,
// and so workspace sizes, independent of the device a call runs on).
constexpr int64_t kPlanSms = 148;

static hstu_status_t validate(const hstu_attn_params_t *p, const int64_t *off,
                              const int32_t *nc, bool bwd) {
  if (!p) return HSTU_ERR_INVALID_ARG;
  if (p->batch < 0 || p->num_heads < 1 || p->num_heads > 4096) return HSTU_ERR_INVALID_ARG;
  if (p->d_qk < 1 || p->d_qk > 256 || p->d_v < 1 || p->d_v > 256) return HSTU_ERR_INVALID_ARG;
  if (p->max_seq_len < 0) return HSTU_ERR_INVALID_ARG;
  if (p->num_pos_buckets < 1 || p->num_time_buckets < 1) return HSTU_ERR_INVALID_ARG;
  if (p->num_pos_buckets > (1 << 20) || p->num_time_buckets > (1 << 20))
    return HSTU_ERR_INVALID_ARG;
  if (p->time_bucket_sub_bits < 0 || p->time_bucket_sub_bits > 8) return HSTU_ERR_INVALID_ARG;
  if (p->rab_per_head != 0 && p->rab_per_head != 1) return HSTU_ERR_INVALID_ARG;
  if (p->mask != HSTU_MASK_CAUSAL && p->mask != HSTU_MASK_MFALCON) return HSTU_ERR_INVALID_ARG;
  if (p->dtype != HSTU_F32 && p->dtype != HSTU_BF16) return HSTU_ERR_INVALID_ARG;
  if (p->impl != HSTU_IMPL_AUTO && p->impl != HSTU_IMPL_SIMT) return HSTU_ERR_INVALID_ARG;
  if (!std::isfinite(p->alpha) || !std::isfinite(p->silu_scale)) return HSTU_ERR_INVALID_ARG;
  const int64_t wq = int64_t(p->num_heads) * p->d_qk, wv = int64_t(p->num_heads) * p->d_v;
  if (p->q_row_stride < wq || p->k_row_stride < wq || p->v_row_stride < wv ||
      p->o_row_stride < wv)
    return HSTU_ERR_INVALID_ARG;
  if (bwd && (p->do_row_stride < wv || p->dq_row_stride < wq || p->dk_row_stride < wq ||
              p->dv_row_stride < wv))
    return HSTU_ERR_INVALID_ARG;
  if (p->batch > 0 && !off) return HSTU_ERR_INVALID_ARG;
  if (p->mask == HSTU_MASK_MFALCON && p->batch > 0 && !nc) return HSTU_ERR_INVALID_ARG;
  if (p->batch > 0 && off[0] != 0) return HSTU_ERR_INVALID_ARG;
  for (int32_t b = 0; b < p->batch; ++b) {
    const int64_t L = off[b + 1] - off[b];
    if (L < 0 || L > p->max_seq_len) return HSTU_ERR_INVALID_ARG;
    if (p->mask == HSTU_MASK_MFALCON && (nc[b] < 0 || nc[b] > L)) return HSTU_ERR_INVALID_ARG;
  }
  const int64_t T = p->batch > 0 ? off[p->batch] : 0;
  if (T >= (int64_t(1) << 31)) return HSTU_ERR_UNSUPPORTED;
  return HSTU_OK;
}

// Work lists, longest first.  Forward: one item per (sequence, pair of
// 128-row query tiles); backward: one per (sequence, 128-key tile), which
// walks the run of 64-query blocks that see its keys.  When a batch is too
// small to give every SM several items (short jagged batches), an item
// longer than the average work per SM is split: a forward pair over
// ranges of key tiles, a backward key tile over parts of its query run.
// Pointwise attention has no normaliser, so the partial outputs of the
// pieces simply add up (in float32, converted once at the end).  Large
// batches (the 4 x 8192 workload) are never split.
static void build_plan(const hstu_attn_params_t *p, const int64_t *off, const int32_t *nc,
                       Plan &plan) {
  plan.T = p->batch > 0 ? off[p->batch] : 0;
  plan.seqs.resize(size_t(p->batch));
  struct Cost {
    int64_t cost;
    int4 item;
    int32_t acc;   // first accumulator row (split items), else -1
  };
  std::vector<Cost> pairs, ktiles;
  int64_t fwd_steps = 0, bwd_steps = 0;
  struct Pair {
    int32_t b, pr, nkt;
  };
  struct KTile {
    int32_t b, kt, qb0, qb1;
  };
  std::vector<Pair> all_pairs;
  std::vector<KTile> all_kt;
  for (int32_t b = 0; b < p->batch; ++b) {
    const int32_t L = int32_t(off[b + 1] - off[b]);
    const int32_t nh = L - (p->mask == HSTU_MASK_MFALCON ? nc[b] : 0);
    plan.seqs[b] = SeqInfo{off[b], L, nh};
    const int32_t n_qt = (L + 127) / 128, n_qb = (L + 63) / 64;
    for (int32_t pr = 0; 2 * pr < n_qt; ++pr) {
      // key tiles 0 .. the pair's last tile (history part and diagonal candidate tiles)
      const int32_t nkt = (2 * pr + 1 < n_qt ? 2 * pr + 1 : 2 * pr) + 1;
      all_pairs.push_back({b, pr, nkt});
      fwd_steps += nkt;
    }
    for (int32_t kt = 0; kt < n_qt; ++kt) {
      // the query blocks that see key tile kt: from its first key to the
      // sequence end (history keys) or to its last candidate (candidate tile)
      const int32_t ks = kt * 128;
      const int32_t end = ks < nh ? n_qb : (std::min(ks + 128, L) + 63) / 64;
      all_kt.push_back({b, kt, 2 * kt, end});
      bwd_steps += end - 2 * kt;
    }
    for (int32_t t = 0; t * 64 < L; ++t) plan.simt_items.push_back(make_int2(b, t));
  }
  // An item is split only when it is more than four times the average work
  // per SM (a lone long sequence among short ones, few heads): on the Zipf
  // workload (largest item about twice the average) splitting at the
  // average measured slower (the kernels did not shorten; the conversion
  // and the extra CTAs cost more), so such batches stay unsplit.
  const int64_t H = p->num_heads;
  const int64_t fwd_avg = std::max<int64_t>(1, (fwd_steps * H + kPlanSms - 1) / kPlanSms);
  const int64_t bwd_avg = std::max<int64_t>(1, (bwd_steps * H + kPlanSms - 1) / kPlanSms);
  const int64_t fwd_cut = std::max<int64_t>(2, fwd_avg);
  const bool bwd_splits = p->d_qk == 128 && p->d_v == 128;   // the d = 128 backward kernel
  const int64_t bwd_cut = std::max<int64_t>(4, bwd_avg);
  for (const Pair &q : all_pairs) {
    if (q.nkt <= 4 * fwd_avg || q.nkt <= fwd_cut) {
      pairs.push_back({q.nkt, make_int4(q.b, q.pr, 0, kUnsplit), -1});
      continue;
    }
    const SeqInfo &sq = plan.seqs[q.b];
    const int32_t r0 = q.pr * 256, rows = std::min(256, sq.len - r0);
    const int32_t acc = plan.split_acc_rows;
    plan.split_acc_rows += rows;
    plan.split_rows.push_back(make_int4(int32_t(sq.start + r0), rows, acc, 0));
    for (int32_t k0 = 0; k0 < q.nkt; k0 += int32_t(fwd_cut)) {
      const int32_t k1 = int32_t(std::min<int64_t>(q.nkt, k0 + fwd_cut));
      pairs.push_back({k1 - k0, make_int4(q.b, q.pr, k0, k1), acc});
    }
  }
  for (const KTile &k : all_kt) {
    const int32_t run = k.qb1 - k.qb0;
    if (!bwd_splits || run <= 4 * bwd_avg || run <= bwd_cut) {
      ktiles.push_back({run, make_int4(k.b, k.kt, 0, kUnsplit), -1});
      continue;
    }
    const SeqInfo &sq = plan.seqs[k.b];
    const int32_t r0 = k.kt * 128, rows = std::min(128, sq.len - r0);
    const int32_t acc = plan.ksplit_acc_rows;
    plan.ksplit_acc_rows += rows;
    plan.ksplit_rows.push_back(make_int4(int32_t(sq.start + r0), rows, acc, 0));
    for (int32_t q0 = k.qb0; q0 < k.qb1; q0 += int32_t(bwd_cut)) {
      const int32_t q1 = int32_t(std::min<int64_t>(k.qb1, q0 + bwd_cut));
      ktiles.push_back({q1 - q0, make_int4(k.b, k.kt, q0, q1), acc});
    }
  }
  auto by_cost = [](const Cost &a, const Cost &b) { return a.cost > b.cost; };
  std::stable_sort(pairs.begin(), pairs.end(), by_cost);
  std::stable_sort(ktiles.begin(), ktiles.end(), by_cost);
  for (auto &c : pairs) {
    plan.items.push_back(c.item);
    plan.item_acc.push_back(c.acc);
  }
  for (auto &c : ktiles) {
    plan.kitems.push_back(c.item);
    plan.kitem_acc.push_back(c.acc);
  }
}

static WsLayout layout_for(const hstu_attn_params_t *p, const Plan &plan, bool bwd) {
  WsLayout w{};
  size_t o = 0;
  w.err = o;
  o = align256(o + 16);
  // seqs .. ksplit_rows form one contiguous block, uploaded in one go
  w.seqs = o;
  o += sizeof(SeqInfo) * plan.seqs.size();
  w.items = o;   // the 16-byte items first: every array stays aligned to its element
  o += sizeof(int4) * plan.items.size();
  w.kitems = o;
  o += sizeof(int4) * plan.kitems.size();
  w.split_rows = o;
  o += sizeof(int4) * plan.split_rows.size();
  w.ksplit_rows = o;
  o += sizeof(int4) * plan.ksplit_rows.size();
  w.simt_items = o;
  o += sizeof(int2) * plan.simt_items.size();
  w.item_acc = o;
  o += sizeof(int32_t) * plan.item_acc.size();
  w.kitem_acc = o;
  o += sizeof(int32_t) * plan.kitem_acc.size();
  o = align256(o);
  w.tf = o;
  o = align256(o + sizeof(float) * size_t(plan.T));
  w.seq_fast = o;
  o = align256(o + sizeof(int32_t) * plan.seqs.size());
  w.dq_acc = o;
  if (bwd) o = align256(o + sizeof(float) * size_t(plan.T) * p->num_heads * p->d_qk);
  w.bin_acc = o;
  if (bwd) o = align256(o + sizeof(float) * kBinAccPerCta * plan.kitems.size() * p->num_heads);
  const size_t row_bytes = sizeof(float) * size_t(p->num_heads) * p->d_v;
  w.o_acc = o;
  if (!bwd && plan.split_acc_rows) o = align256(o + row_bytes * size_t(plan.split_acc_rows));
  w.dk_acc = o;
  if (bwd && plan.ksplit_acc_rows) o = align256(o + row_bytes * size_t(plan.ksplit_acc_rows));
  w.dv_acc = o;
  if (bwd && plan.ksplit_acc_rows) o = align256(o + row_bytes * size_t(plan.ksplit_acc_rows));
  w.total = o;
  return w;
}

static AttnProblem make_problem(const hstu_attn_params_t *p, int64_t T, const int64_t *ts,
                                const void *q, const void *k, const void *v, const float *rp,
                                const float *rt) {
  AttnProblem a{};
  a.batch = p->batch;
  a.num_heads = p->num_heads;
  a.d_qk = p->d_qk;
  a.d_v = p->d_v;
  a.max_seq_len = p->max_seq_len;
  a.nb_p = p->num_pos_buckets;
  a.nb_t = p->num_time_buckets;
  a.sub_bits = p->time_bucket_sub_bits;
  a.rab_per_head = p->rab_per_head;
  a.mask = p->mask;
  a.dtype = p->dtype;
  a.total_tokens = T;
  a.q_rs = p->q_row_stride;
  a.k_rs = p->k_row_stride;
  a.v_rs = p->v_row_stride;
  a.o_rs = p->o_row_stride;
  a.do_rs = p->do_row_stride;
  a.dq_rs = p->dq_row_stride;
  a.dk_rs = p->dk_row_stride;
  a.dv_rs = p->dv_row_stride;
  a.alpha = p->alpha;
  a.silu_scale = p->silu_scale;
  a.ts = ts;
  a.q = q;
  a.k = k;
  a.v = v;
  a.rab_p = rp;
  a.rab_t = rt;
  return a;
}

// Carves the scratch out of the workspace and uploads the plan (kernel
// parameters, no host wait).  The error word is cleared unless the caller
// (the layer) already did.
static cudaError_t stage_plan(const Plan &plan, const WsLayout &w, void *ws, Scratch &s,
                              cudaStream_t st, bool clear_err = true) {
  uint8_t *base = static_cast<uint8_t *>(ws);
  s.err = reinterpret_cast<uint32_t *>(base + w.err);
  s.seqs = reinterpret_cast<SeqInfo *>(base + w.seqs);
  s.items = reinterpret_cast<int4 *>(base + w.items);
  s.n_items = int32_t(plan.items.size());
  s.simt_items = reinterpret_cast<int2 *>(base + w.simt_items);
  s.n_simt_items = int32_t(plan.simt_items.size());
  s.kitems = reinterpret_cast<int4 *>(base + w.kitems);
  s.n_kitems = int32_t(plan.kitems.size());
  s.split_rows = reinterpret_cast<int4 *>(base + w.split_rows);
  s.n_split_rows = int32_t(plan.split_rows.size());
  s.n_split_acc_rows = plan.split_acc_rows;
  s.ksplit_rows = reinterpret_cast<int4 *>(base + w.ksplit_rows);
  s.n_ksplit_rows = int32_t(plan.ksplit_rows.size());
  s.n_ksplit_acc_rows = plan.ksplit_acc_rows;
  s.item_acc = reinterpret_cast<int32_t *>(base + w.item_acc);
  s.kitem_acc = reinterpret_cast<int32_t *>(base + w.kitem_acc);
  s.tf = reinterpret_cast<float *>(base + w.tf);
  s.seq_fast = reinterpret_cast<int32_t *>(base + w.seq_fast);
  s.dq_acc = reinterpret_cast<float *>(base + w.dq_acc);
  s.bin_acc = reinterpret_cast<float *>(base + w.bin_acc);
  s.o_acc = w.dk_acc > w.o_acc ? reinterpret_cast<float *>(base + w.o_acc) : nullptr;
  s.dk_acc = w.dv_acc > w.dk_acc ? reinterpret_cast<float *>(base + w.dk_acc) : nullptr;
  s.dv_acc = w.total > w.dv_acc ? reinterpret_cast<float *>(base + w.dv_acc) : nullptr;
  const size_t n = w.tf - w.seqs;   // a multiple of 256 (the layout aligns w.tf)
  std::vector<uint8_t> host(n, 0);
  auto put = [&](size_t at, const void *src, size_t bytes) {
    if (bytes) std::memcpy(host.data() + (at - w.seqs), src, bytes);
  };
  put(w.seqs, plan.seqs.data(), sizeof(SeqInfo) * plan.seqs.size());
  put(w.items, plan.items.data(), sizeof(int4) * plan.items.size());
  put(w.simt_items, plan.simt_items.data(), sizeof(int2) * plan.simt_items.size());
  put(w.kitems, plan.kitems.data(), sizeof(int4) * plan.kitems.size());
  put(w.split_rows, plan.split_rows.data(), sizeof(int4) * plan.split_rows.size());
  put(w.ksplit_rows, plan.ksplit_rows.data(), sizeof(int4) * plan.ksplit_rows.size());
  put(w.item_acc, plan.item_acc.data(), sizeof(int32_t) * plan.item_acc.size());
  put(w.kitem_acc, plan.kitem_acc.data(), sizeof(int32_t) * plan.kitem_acc.size());
  // Through kernel parameters: the host never waits for the device here.
  return launch_upload(base + w.seqs, host.data(), n, clear_err ? s.err : nullptr, st);
}

static hstu_status_t cuda_status(cudaError_t e) { return e == cudaSuccess ? HSTU_OK : HSTU_ERR_CUDA; }

static uint64_t wait_limit_ns() {
  const uint64_t v = g_wait_limit_ns.load(std::memory_order_relaxed);
  return v ? v : kDefaultWaitNs;
}

static WaitCtl wait_ctl(const Scratch &s) { return WaitCtl{s.err, wait_limit_ns()}; }

static bool aligned16(const void *ptr) { return (reinterpret_cast<uintptr_t>(ptr) & 15) == 0; }

static hstu_status_t attn_fwd_impl(const hstu_attn_params_t *params,
                                   const int64_t *seq_offsets_host,
                                   const int32_t *num_candidates_host,
                                   const int64_t *timestamps_dev, const void *q, const void *k,
                                   const void *v, const float *rab_pos, const float *rab_time,
                                   void *out, void *workspace, size_t workspace_bytes,
                                   void *stream, bool clear_err) {
  hstu_status_t st = validate(params, seq_offsets_host, num_candidates_host, false);
  if (st != HSTU_OK) return st;
  Plan plan;
  build_plan(params, seq_offsets_host, num_candidates_host, plan);
  if (plan.T > 0 && (!timestamps_dev || !q || !k || !v || !rab_pos || !rab_time || !out))
    return HSTU_ERR_INVALID_ARG;
  const WsLayout w = layout_for(params, plan, false);
  if (!workspace || workspace_bytes < w.total || (reinterpret_cast<uintptr_t>(workspace) & 255))
    return HSTU_ERR_WORKSPACE;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  Scratch s{};
  cudaError_t e = stage_plan(plan, w, workspace, s, cs, clear_err);
  if (e != cudaSuccess) return HSTU_ERR_CUDA;
  if (plan.T == 0) return HSTU_OK;
  AttnProblem prob = make_problem(params, plan.T, timestamps_dev, q, k, v, rab_pos, rab_time);
  e = launch_prep(prob, s, cs);
  if (e != cudaSuccess) return HSTU_ERR_CUDA;
  const bool tc = params->impl == HSTU_IMPL_AUTO && fwd_tc_supported(prob) && aligned16(out);
  e = tc ? launch_fwd_tc(prob, s, out, wait_ctl(s), cs) : launch_fwd_simt(prob, s, out, cs);
  return cuda_status(e);
}

static hstu_status_t attn_bwd_impl(const hstu_attn_params_t *params,
                                   const int64_t *seq_offsets_host,
                                   const int32_t *num_candidates_host,
                                   const int64_t *timestamps_dev, const void *q, const void *k,
                                   const void *v, const float *rab_pos, const float *rab_time,
                                   const void *dout, void *dq, void *dk, void *dv,
                                   float *drab_pos, float *drab_time, void *workspace,
                                   size_t workspace_bytes, void *stream, bool clear_err) {
  hstu_status_t st = validate(params, seq_offsets_host, num_candidates_host, true);
  if (st != HSTU_OK) return st;
  Plan plan;
  build_plan(params, seq_offsets_host, num_candidates_host, plan);
  if (plan.T > 0 && (!timestamps_dev || !q || !k || !v || !rab_pos || !rab_time || !dout ||
                     !dq || !dk || !dv || !drab_pos || !drab_time))
    return HSTU_ERR_INVALID_ARG;
  const WsLayout w = layout_for(params, plan, true);
  if (!workspace || workspace_bytes < w.total || (reinterpret_cast<uintptr_t>(workspace) & 255))
    return HSTU_ERR_WORKSPACE;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  Scratch s{};
  cudaError_t e = stage_plan(plan, w, workspace, s, cs, clear_err);
  if (e != cudaSuccess) return HSTU_ERR_CUDA;
  if (plan.T == 0) return HSTU_OK;
  AttnProblem prob = make_problem(params, plan.T, timestamps_dev, q, k, v, rab_pos, rab_time);
  e = launch_prep(prob, s, cs);
  if (e != cudaSuccess) return HSTU_ERR_CUDA;
  const bool tc = params->impl == HSTU_IMPL_AUTO && bwd_tc_supported(prob) && aligned16(dout) &&
                  aligned16(dq) && aligned16(dk) && aligned16(dv) &&
                  ((params->do_row_stride | params->dq_row_stride | params->dk_row_stride |
                    params->dv_row_stride) & 7) == 0;
  e = tc ? launch_bwd_tc(prob, s, dout, dq, dk, dv, drab_pos, drab_time, wait_ctl(s), cs)
         : launch_bwd_simt(prob, s, dout, dq, dk, dv, drab_pos, drab_time, cs);
  return cuda_status(e);
}

}  // namespace hstu

using namespace hstu;

extern "C" {

const char *hstu_status_string(hstu_status_t s) {
  switch (s) {
    case HSTU_OK: return "HSTU_OK";
    case HSTU_ERR_INVALID_ARG: return "HSTU_ERR_INVALID_ARG";
    case HSTU_ERR_UNSUPPORTED: return "HSTU_ERR_UNSUPPORTED";
    case HSTU_ERR_WORKSPACE: return "HSTU_ERR_WORKSPACE";
    case HSTU_ERR_CUDA: return "HSTU_ERR_CUDA";
    case HSTU_ERR_DEVICE_TIMEOUT: return "HSTU_ERR_DEVICE_TIMEOUT";
    case HSTU_ERR_DEVICE: return "HSTU_ERR_DEVICE";
  }
  return "HSTU_ERR_UNKNOWN";
}

const char *hstu_version(void) { return "hstu-b200 0.1 sm_100a"; }

uint64_t hstu_kernel_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

void hstu_set_wait_limit(uint32_t microseconds) {
  g_wait_limit_ns.store(uint64_t(microseconds) * 1000ull, std::memory_order_relaxed);
}

hstu_status_t hstu_attn_workspace_size(const hstu_attn_params_t *params,
                                       const int64_t *seq_offsets_host, int32_t is_bwd,
                                       size_t *bytes) {
  if (!bytes) return HSTU_ERR_INVALID_ARG;
  if (!params) return HSTU_ERR_INVALID_ARG;
  // Candidates only change the schedule's content, not its size.
  std::vector<int32_t> zeros(size_t(params->batch > 0 ? params->batch : 0), 0);
  hstu_attn_params_t p = *params;
  p.mask = HSTU_MASK_CAUSAL;
  hstu_status_t st = validate(&p, seq_offsets_host, nullptr, is_bwd != 0);
  if (st != HSTU_OK) return st;
  Plan plan;
  build_plan(&p, seq_offsets_host, zeros.data(), plan);
  *bytes = layout_for(&p, plan, is_bwd != 0).total;
  return HSTU_OK;
}

hstu_status_t hstu_attn_fwd(const hstu_attn_params_t *params, const int64_t *seq_offsets_host,
                            const int32_t *num_candidates_host, const int64_t *timestamps_dev,
                            const void *q, const void *k, const void *v, const float *rab_pos,
                            const float *rab_time, void *out, void *workspace,
                            size_t workspace_bytes, void *stream) {
  return attn_fwd_impl(params, seq_offsets_host, num_candidates_host, timestamps_dev, q, k, v,
                       rab_pos, rab_time, out, workspace, workspace_bytes, stream, true);
}

hstu_status_t hstu_attn_bwd(const hstu_attn_params_t *params, const int64_t *seq_offsets_host,
                            const int32_t *num_candidates_host, const int64_t *timestamps_dev,
                            const void *q, const void *k, const void *v, const float *rab_pos,
                            const float *rab_time, const void *dout, void *dq, void *dk,
                            void *dv, float *drab_pos, float *drab_time, void *workspace,
                            size_t workspace_bytes, void *stream) {
  return attn_bwd_impl(params, seq_offsets_host, num_candidates_host, timestamps_dev, q, k, v,
                       rab_pos, rab_time, dout, dq, dk, dv, drab_pos, drab_time, workspace,
                       workspace_bytes, stream, true);
}

hstu_status_t hstu_debug_buckets(const hstu_attn_params_t *params,
                                 const int64_t *seq_offsets_host,
                                 const int32_t *num_candidates_host,
                                 const int64_t *timestamps_dev, int32_t *bp, int32_t *bt,
                                 int32_t *bt_fast, void *workspace, size_t workspace_bytes,
                                 void *stream) {
  hstu_status_t st = validate(params, seq_offsets_host, num_candidates_host, false);
  if (st != HSTU_OK) return st;
  Plan plan;
  build_plan(params, seq_offsets_host, num_candidates_host, plan);
  if (plan.T > 0 && (!timestamps_dev || !bp || !bt || !bt_fast)) return HSTU_ERR_INVALID_ARG;
  const WsLayout w = layout_for(params, plan, false);
  if (!workspace || workspace_bytes < w.total || (reinterpret_cast<uintptr_t>(workspace) & 255))
    return HSTU_ERR_WORKSPACE;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  Scratch s{};
  cudaError_t e = stage_plan(plan, w, workspace, s, cs);
  if (e != cudaSuccess || plan.T == 0) return cuda_status(e);
  AttnProblem prob = make_problem(params, plan.T, timestamps_dev, nullptr, nullptr, nullptr,
                                  nullptr, nullptr);
  e = launch_prep(prob, s, cs);
  if (e != cudaSuccess) return HSTU_ERR_CUDA;
  return cuda_status(launch_debug_buckets(prob, s, bp, bt, bt_fast, cs));
}

hstu_status_t hstu_debug_plan(const hstu_attn_params_t *params, const int64_t *seq_offsets_host,
                              const int32_t *num_candidates_host, int32_t capacity,
                              int32_t *fwd_items, int32_t *n_fwd, int32_t *bwd_items,
                              int32_t *n_bwd) {
  if (!n_fwd || !n_bwd || capacity < 0) return HSTU_ERR_INVALID_ARG;
  hstu_status_t st = validate(params, seq_offsets_host, num_candidates_host, false);
  if (st != HSTU_OK) return st;
  Plan plan;
  build_plan(params, seq_offsets_host, num_candidates_host, plan);
  *n_fwd = int32_t(plan.items.size());
  *n_bwd = int32_t(plan.kitems.size());
  if (*n_fwd > capacity || *n_bwd > capacity) return HSTU_ERR_INVALID_ARG;
  if ((*n_fwd && !fwd_items) || (*n_bwd && !bwd_items)) return HSTU_ERR_INVALID_ARG;
  for (size_t i = 0; i < plan.items.size(); ++i) {
    const int4 &it = plan.items[i];
    int32_t *o = fwd_items + 4 * i;
    o[0] = it.x, o[1] = it.y, o[2] = it.z, o[3] = it.w;
  }
  for (size_t i = 0; i < plan.kitems.size(); ++i) {
    const int4 &it = plan.kitems[i];
    int32_t *o = bwd_items + 4 * i;
    o[0] = it.x, o[1] = it.y, o[2] = it.z, o[3] = it.w;
  }
  return HSTU_OK;
}

hstu_status_t hstu_debug_trace_read(int32_t kernel, void *host, size_t bytes) {
  if (kernel != HSTU_TRACE_BWD128 && kernel != HSTU_TRACE_FWD) return HSTU_ERR_INVALID_ARG;
  if (!kTraceBuild) return HSTU_ERR_UNSUPPORTED;
  if (!host) return HSTU_ERR_INVALID_ARG;
  const bool ok = kernel == HSTU_TRACE_FWD ? trace_fwd_read(host, bytes)
                                           : trace_bwd128_read(host, bytes);
  return ok ? HSTU_OK : HSTU_ERR_CUDA;
}

hstu_status_t hstu_debug_trace_clear(int32_t kernel) {
  if (kernel != HSTU_TRACE_BWD128 && kernel != HSTU_TRACE_FWD) return HSTU_ERR_INVALID_ARG;
  if (!kTraceBuild) return HSTU_ERR_UNSUPPORTED;
  const bool ok = kernel == HSTU_TRACE_FWD ? trace_fwd_clear() : trace_bwd128_clear();
  return ok ? HSTU_OK : HSTU_ERR_CUDA;
}

hstu_status_t hstu_debug_wait_probe(void *workspace, size_t workspace_bytes, uint32_t limit_us,
                                    void *stream) {
  if (!workspace || workspace_bytes < 16) return HSTU_ERR_WORKSPACE;
  if (reinterpret_cast<uintptr_t>(workspace) & 255) return HSTU_ERR_WORKSPACE;
  if (limit_us == 0 || limit_us > 60u * 1000u * 1000u) return HSTU_ERR_INVALID_ARG;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  uint32_t *err = static_cast<uint32_t *>(workspace);
  if (cudaMemsetAsync(err, 0, 16, cs) != cudaSuccess) return HSTU_ERR_CUDA;
  const WaitCtl w{err, uint64_t(limit_us) * 1000ull};
  return cuda_status(launch_wait_probe(w, cs));
}

hstu_status_t hstu_get_device_error(const void *workspace, void *stream, uint32_t *detail) {
  if (!workspace) return HSTU_ERR_INVALID_ARG;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  uint32_t word = 0;
  if (cudaStreamSynchronize(cs) != cudaSuccess) return HSTU_ERR_CUDA;
  if (cudaMemcpy(&word, workspace, sizeof(word), cudaMemcpyDeviceToHost) != cudaSuccess)
    return HSTU_ERR_CUDA;
  if (detail) *detail = word;
  if (word & kDevErrTimeout) return HSTU_ERR_DEVICE_TIMEOUT;
  if (word) return HSTU_ERR_DEVICE;
  return HSTU_OK;
}

// ---------------------------------------------------------------------------
// Layer
// ---------------------------------------------------------------------------
static hstu_status_t validate_layer(const hstu_layer_params_t *lp, const int64_t *off,
                                    const int32_t *nc, hstu_attn_params_t &ap) {
  if (!lp) return HSTU_ERR_INVALID_ARG;
  if (lp->d_model < 8 || lp->d_model > 8192 || (lp->d_model & 7)) return HSTU_ERR_INVALID_ARG;
  if (!(lp->ln_eps > 0.f) || !std::isfinite(lp->ln_eps)) return HSTU_ERR_INVALID_ARG;
  ap = lp->attn;
  const int64_t H = ap.num_heads;
  const int64_t n1 = 2 * H * (int64_t(ap.d_v) + ap.d_qk);
  ap.q_row_stride = ap.k_row_stride = ap.v_row_stride = n1;
  ap.o_row_stride = H * ap.d_v;
  hstu_status_t st = validate(&ap, off, nc, false);
  if (st != HSTU_OK) return st;
  if (ap.dtype != HSTU_BF16) return HSTU_ERR_UNSUPPORTED;
  const int64_t F = H * ap.d_v;
  if (F != 32 && F != 64 && F != 128 && F != 256 && F != 512 && F != 1024)
    return HSTU_ERR_UNSUPPORTED;
  if ((H * ap.d_qk) % 8) return HSTU_ERR_UNSUPPORTED;
  return HSTU_OK;
}

struct LayerWs {
  size_t proj, attn_out, gated, attn_ws, total;
};

static LayerWs layer_layout(const hstu_attn_params_t &ap, const Plan &plan, int64_t T) {
  LayerWs w{};
  const int64_t H = ap.num_heads;
  const int64_t n1 = 2 * H * (int64_t(ap.d_v) + ap.d_qk);
  size_t o = 0;
  // The attention workspace comes first so its device error word sits at
  // offset 0 of the layer workspace (hstu_get_device_error reads it there).
  w.attn_ws = o;
  o = align256(o + layout_for(&ap, plan, false).total);
  w.proj = o;
  o = align256(o + size_t(T) * n1 * 2);
  w.attn_out = o;
  o = align256(o + size_t(T) * H * ap.d_v * 2);
  w.gated = o;
  o = align256(o + size_t(T) * H * ap.d_v * 2);
  w.total = o;
  return w;
}

hstu_status_t hstu_layer_workspace_size(const hstu_layer_params_t *params,
                                        const int64_t *seq_offsets_host, size_t *bytes) {
  if (!bytes || !params) return HSTU_ERR_INVALID_ARG;
  hstu_layer_params_t lp = *params;
  lp.attn.mask = HSTU_MASK_CAUSAL;
  hstu_attn_params_t ap;
  hstu_status_t st = validate_layer(&lp, seq_offsets_host, nullptr, ap);
  if (st != HSTU_OK) return st;
  std::vector<int32_t> zeros(size_t(ap.batch > 0 ? ap.batch : 0), 0);
  Plan plan;
  build_plan(&ap, seq_offsets_host, zeros.data(), plan);
  *bytes = layer_layout(ap, plan, plan.T).total;
  return HSTU_OK;
}

static hstu_status_t layer_fwd_impl(const hstu_layer_params_t *params,
                                    const int64_t *seq_offsets_host,
                                    const int32_t *num_candidates_host,
                                    const int64_t *timestamps_dev, const void *x, const void *w1,
                                    const float *b1, const float *ln_gamma,
                                    const float *ln_beta, const void *w2, const float *b2,
                                    const float *rab_pos, const float *rab_time, void *y,
                                    void *proj_out, void *workspace, size_t workspace_bytes,
                                    void *stream) {
  hstu_attn_params_t ap;
  hstu_status_t st = validate_layer(params, seq_offsets_host, num_candidates_host, ap);
  if (st != HSTU_OK) return st;
  Plan plan;
  build_plan(&ap, seq_offsets_host, num_candidates_host, plan);
  const int64_t T = plan.T;
  if (T > 0 && (!timestamps_dev || !x || !w1 || !b1 || !ln_gamma || !ln_beta || !w2 || !b2 ||
                !rab_pos || !rab_time || !y))
    return HSTU_ERR_INVALID_ARG;
  if (T > 0 && x == y) return HSTU_ERR_INVALID_ARG;
  if (proj_out && (reinterpret_cast<uintptr_t>(proj_out) & 15)) return HSTU_ERR_INVALID_ARG;
  const LayerWs lw = layer_layout(ap, plan, T);
  if (!workspace || workspace_bytes < lw.total || (reinterpret_cast<uintptr_t>(workspace) & 255))
    return HSTU_ERR_WORKSPACE;
  if (T == 0) return HSTU_OK;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  uint8_t *ws = static_cast<uint8_t *>(workspace);
  const int64_t H = ap.num_heads, dqk = ap.d_qk, dv = ap.d_v, D = params->d_model;
  const int64_t n1 = 2 * H * (dv + dqk);
  // the projection goes to the caller's buffer when one is given (history K/V cache)
  uint8_t *proj = proj_out ? static_cast<uint8_t *>(proj_out) : ws + lw.proj;
  uint8_t *attn_out = ws + lw.attn_out;
  uint8_t *gated = ws + lw.gated;
  // One device error word (offset 0) serves the whole layer: cleared here,
  // set by any kernel whose bounded wait runs out.
  uint32_t *err = reinterpret_cast<uint32_t *>(ws + lw.attn_ws);
  cudaError_t e = cudaMemsetAsync(err, 0, 16, cs);
  if (e != cudaSuccess) return HSTU_ERR_CUDA;
  const WaitCtl wc{err, wait_limit_ns()};
  // f1 + SiLU: [U|V|Q|K] = SiLU(x W1^T + b1)
  e = launch_gemm(x, D, w1, D, b1, nullptr, 0, proj, n1, T, n1, D, kEpiBiasSilu, wc, cs);
  if (e != cudaSuccess) return HSTU_ERR_CUDA;
  // attention on strided views of the projection
  const void *u_ptr = proj;
  const void *v_ptr = proj + 2 * (H * dv);
  const void *q_ptr = proj + 2 * (2 * H * dv);
  const void *k_ptr = proj + 2 * (2 * H * dv + H * dqk);
  st = attn_fwd_impl(&ap, seq_offsets_host, num_candidates_host, timestamps_dev, q_ptr, k_ptr,
                     v_ptr, rab_pos, rab_time, attn_out, ws + lw.attn_ws, lw.proj - lw.attn_ws,
                     stream, false);
  if (st != HSTU_OK) return st;
  // G = LayerNorm(A) (.) U
  e = launch_ln_gate(attn_out, H * dv, u_ptr, n1, ln_gamma, ln_beta, params->ln_eps, gated,
                     H * dv, T, int32_t(H * dv), cs);
  if (e != cudaSuccess) return HSTU_ERR_CUDA;
  // y = x + G W2^T + b2
  e = launch_gemm(gated, H * dv, w2, H * dv, b2, params->residual ? x : nullptr, D, y, D, T, D,
                  H * dv, params->residual ? kEpiBiasResidual : kEpiBias, wc, cs);
  return cuda_status(e);
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Cached-history attention (M-FALCON candidate micro-batches)
// ---------------------------------------------------------------------------
namespace hstu {

struct CachedPlan {
  int64_t Th = 0, Tc = 0;
  std::vector<SeqInfo> seqs;
  std::vector<int4> items;        // {seq, candidate tile pair, first key tile, end (kUnsplit: all)}
  std::vector<int32_t> item_acc;  // first accumulator row of a split item, else -1
  std::vector<int4> split_rows;   // {first output row, rows, first accumulator row, 0}
  int32_t split_acc_rows = 0;
  std::vector<int64_t> cstart;
};

struct CachedWs {
  size_t err, seqs, items, split_rows, item_acc, cstart, tf, tfc, seq_fast, o_acc, total;
};

static hstu_status_t validate_cached(const hstu_attn_params_t *p, const int64_t *hoff,
                                     const int64_t *coff, int64_t kh_rs, int64_t vh_rs) {
  if (!p) return HSTU_ERR_INVALID_ARG;
  // the shared checks (dimensions, buckets, scales, strides) with an empty batch
  hstu_attn_params_t q = *p;
  q.batch = 0;
  q.mask = HSTU_MASK_CAUSAL;
  hstu_status_t st = validate(&q, nullptr, nullptr, false);
  if (st != HSTU_OK) return st;
  if (p->batch < 0) return HSTU_ERR_INVALID_ARG;
  if (kh_rs < int64_t(p->num_heads) * p->d_qk || vh_rs < int64_t(p->num_heads) * p->d_v)
    return HSTU_ERR_INVALID_ARG;
  if (p->batch > 0 && (!hoff || !coff || hoff[0] != 0 || coff[0] != 0))
    return HSTU_ERR_INVALID_ARG;
  for (int32_t b = 0; b < p->batch; ++b) {
    const int64_t nh = hoff[b + 1] - hoff[b], nc = coff[b + 1] - coff[b];
    if (nh < 0 || nc < 0 || nh + nc > p->max_seq_len) return HSTU_ERR_INVALID_ARG;
  }
  const int64_t Th = p->batch > 0 ? hoff[p->batch] : 0, Tc = p->batch > 0 ? coff[p->batch] : 0;
  if (Th >= (int64_t(1) << 31) || Tc >= (int64_t(1) << 31)) return HSTU_ERR_UNSUPPORTED;
  // the tensor-core path only (bf16, d_qk = d_v in {64, 128})
  if (p->dtype != HSTU_BF16 || p->d_qk != p->d_v || (p->d_qk != 64 && p->d_qk != 128) ||
      p->impl != HSTU_IMPL_AUTO)
    return HSTU_ERR_UNSUPPORTED;
  return HSTU_OK;
}

static void build_cached_plan(const hstu_attn_params_t *p, const int64_t *hoff,
                              const int64_t *coff, CachedPlan &plan) {
  plan.Th = p->batch > 0 ? hoff[p->batch] : 0;
  plan.Tc = p->batch > 0 ? coff[p->batch] : 0;
  plan.seqs.resize(size_t(p->batch));
  plan.cstart.resize(size_t(p->batch));
  struct Cost {
    int64_t cost;
    int4 item;
    int32_t acc;
  };
  std::vector<Cost> pairs;
  int64_t n_pairs = 0;
  for (int32_t b = 0; b < p->batch; ++b) {
    const int32_t nc = int32_t(coff[b + 1] - coff[b]);
    n_pairs += ((nc + 127) / 128 + 1) / 2;
  }
  // A micro-batch of few users gives few (pair, head) CTAs, each walking the
  // whole cached history: when they cannot fill the SMs, each pair's history
  // key tiles are split into up to kPlanSms / (pairs x heads) ranges whose
  // partial outputs add up in float32 (no normaliser), so about one wave of
  // CTAs shares the history.
  const int64_t ctas = n_pairs * p->num_heads;
  const int64_t pieces_max = ctas > 0 ? std::max<int64_t>(1, kPlanSms / ctas) : 1;
  for (int32_t b = 0; b < p->batch; ++b) {
    const int32_t nh = int32_t(hoff[b + 1] - hoff[b]), nc = int32_t(coff[b + 1] - coff[b]);
    plan.seqs[b] = SeqInfo{hoff[b], nh + nc, nh};
    plan.cstart[b] = coff[b];
    const int32_t n_qt = (nc + 127) / 128;
    const int32_t n_kt = (nh + 127) / 128;
    const int32_t pieces = int32_t(std::min<int64_t>(pieces_max, std::max(n_kt, 1)));
    for (int32_t pr = 0; 2 * pr < n_qt; ++pr) {
      if (pieces <= 1) {
        pairs.push_back({int64_t(n_kt) + 1, make_int4(b, pr, 0, kUnsplit), -1});
        continue;
      }
      const int32_t rows = std::min(256, nc - 256 * pr);
      const int32_t acc = plan.split_acc_rows;
      plan.split_acc_rows += rows;
      plan.split_rows.push_back(make_int4(int32_t(coff[b] + 256 * pr), rows, acc, 0));
      for (int32_t k = 0; k < pieces; ++k) {
        const int32_t k0 = int32_t(int64_t(n_kt) * k / pieces);
        const int32_t k1 = int32_t(int64_t(n_kt) * (k + 1) / pieces);
        pairs.push_back({int64_t(k1 - k0) + 1, make_int4(b, pr, k0, k1), acc});
      }
    }
  }
  std::stable_sort(pairs.begin(), pairs.end(),
                   [](const Cost &a, const Cost &b) { return a.cost > b.cost; });
  for (auto &c : pairs) {
    plan.items.push_back(c.item);
    plan.item_acc.push_back(c.acc);
  }
}

static CachedWs cached_layout(const CachedPlan &plan, const hstu_attn_params_t &ap) {
  CachedWs w{};
  size_t o = 0;
  w.err = o;
  o = align256(o + 16);
  w.seqs = o;   // seqs .. cstart: one upload
  o += sizeof(SeqInfo) * plan.seqs.size();
  o = (o + 15) & ~size_t(15);   // the 16-byte records stay aligned
  w.items = o;
  o += sizeof(int4) * plan.items.size();
  w.split_rows = o;
  o += sizeof(int4) * plan.split_rows.size();
  w.item_acc = o;
  o += sizeof(int32_t) * plan.item_acc.size();
  o = (o + 7) & ~size_t(7);
  w.cstart = o;
  o += sizeof(int64_t) * plan.cstart.size();
  o = align256(o);
  w.tf = o;
  o = align256(o + sizeof(float) * size_t(plan.Th));
  w.tfc = o;
  o = align256(o + sizeof(float) * size_t(plan.Tc));
  w.seq_fast = o;
  o = align256(o + sizeof(int32_t) * plan.seqs.size());
  w.o_acc = o;   // split pairs' float32 partial outputs [split rows][H][d_v]
  o = align256(o + sizeof(float) * size_t(plan.split_acc_rows) * size_t(ap.num_heads) *
                       size_t(ap.d_v));
  w.total = o;
  return w;
}

static hstu_status_t attn_cand_impl(const hstu_attn_params_t *params, const int64_t *hoff,
                                    const int64_t *coff, const int64_t *ts_hist,
                                    const int64_t *ts_cand, const void *q, const void *k,
                                    const void *v, const void *k_hist, const void *v_hist,
                                    int64_t kh_rs, int64_t vh_rs, const float *rab_pos,
                                    const float *rab_time, void *out, void *workspace,
                                    size_t workspace_bytes, void *stream, bool clear_err) {
  hstu_status_t st = validate_cached(params, hoff, coff, kh_rs, vh_rs);
  if (st != HSTU_OK) return st;
  CachedPlan plan;
  build_cached_plan(params, hoff, coff, plan);
  if (plan.Tc > 0 && (!ts_cand || !q || !k || !v || !rab_pos || !rab_time || !out))
    return HSTU_ERR_INVALID_ARG;
  if (plan.Th > 0 && (!ts_hist || !k_hist || !v_hist)) return HSTU_ERR_INVALID_ARG;
  const CachedWs w = cached_layout(plan, *params);
  if (!workspace || workspace_bytes < w.total || (reinterpret_cast<uintptr_t>(workspace) & 255))
    return HSTU_ERR_WORKSPACE;
  // TMA operands and 16-byte row loads: aligned bases, strides in 8-element steps
  const uintptr_t al = reinterpret_cast<uintptr_t>(q) | reinterpret_cast<uintptr_t>(k) |
                       reinterpret_cast<uintptr_t>(v) | reinterpret_cast<uintptr_t>(out) |
                       reinterpret_cast<uintptr_t>(k_hist) | reinterpret_cast<uintptr_t>(v_hist);
  if ((al & 15) || ((params->q_row_stride | params->k_row_stride | params->v_row_stride |
                     params->o_row_stride | kh_rs | vh_rs) & 7))
    return HSTU_ERR_UNSUPPORTED;
  if (params->num_pos_buckets > 1024 || params->num_time_buckets > 1024)
    return HSTU_ERR_UNSUPPORTED;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  uint8_t *base = static_cast<uint8_t *>(workspace);
  Scratch s{};
  s.err = reinterpret_cast<uint32_t *>(base + w.err);
  s.seqs = reinterpret_cast<SeqInfo *>(base + w.seqs);
  s.items = reinterpret_cast<int4 *>(base + w.items);
  s.n_items = int32_t(plan.items.size());
  s.tf = reinterpret_cast<float *>(base + w.tf);
  s.seq_fast = reinterpret_cast<int32_t *>(base + w.seq_fast);
  s.item_acc = reinterpret_cast<int32_t *>(base + w.item_acc);
  s.split_rows = reinterpret_cast<int4 *>(base + w.split_rows);
  s.n_split_rows = int32_t(plan.split_rows.size());
  s.n_split_acc_rows = plan.split_acc_rows;
  s.o_acc = plan.split_acc_rows > 0 ? reinterpret_cast<float *>(base + w.o_acc) : nullptr;
  const size_t n = w.tf - w.seqs;
  std::vector<uint8_t> host(n, 0);
  if (!plan.seqs.empty())
    std::memcpy(host.data(), plan.seqs.data(), sizeof(SeqInfo) * plan.seqs.size());
  if (!plan.items.empty())
    std::memcpy(host.data() + (w.items - w.seqs), plan.items.data(),
                sizeof(int4) * plan.items.size());
  if (!plan.split_rows.empty())
    std::memcpy(host.data() + (w.split_rows - w.seqs), plan.split_rows.data(),
                sizeof(int4) * plan.split_rows.size());
  if (!plan.item_acc.empty())
    std::memcpy(host.data() + (w.item_acc - w.seqs), plan.item_acc.data(),
                sizeof(int32_t) * plan.item_acc.size());
  if (!plan.cstart.empty())
    std::memcpy(host.data() + (w.cstart - w.seqs), plan.cstart.data(),
                sizeof(int64_t) * plan.cstart.size());
  cudaError_t e = launch_upload(base + w.seqs, host.data(), n, clear_err ? s.err : nullptr, cs);
  if (e != cudaSuccess) return HSTU_ERR_CUDA;
  if (plan.Tc == 0) return HSTU_OK;
  hstu_attn_params_t pk = *params;
  pk.k_row_stride = kh_rs;
  pk.v_row_stride = vh_rs;
  AttnProblem prob = make_problem(&pk, plan.Th, ts_hist, q, k_hist, v_hist, rab_pos, rab_time);
  CachedHist ch{};
  ch.cstart = reinterpret_cast<const int64_t *>(base + w.cstart);
  ch.tfc = reinterpret_cast<const float *>(base + w.tfc);
  ch.ts_cand = ts_cand;
  ch.k_cand = k;
  ch.v_cand = v;
  ch.kc_rs = params->k_row_stride;
  ch.vc_rs = params->v_row_stride;
  ch.n_cand_tokens = plan.Tc;
  e = launch_prep_cached(prob, s, ch, reinterpret_cast<float *>(base + w.tfc), cs);
  if (e != cudaSuccess) return HSTU_ERR_CUDA;
  return cuda_status(launch_fwd_tc_cached(prob, s, ch, out, wait_ctl(s), cs));
}

struct LayerCandWs {
  size_t attn_ws, proj, a, g, total;
};

static LayerCandWs layer_cand_layout(const hstu_attn_params_t &ap, const CachedPlan &plan) {
  LayerCandWs w{};
  const int64_t H = ap.num_heads, F = H * ap.d_v, n1 = 2 * H * (int64_t(ap.d_v) + ap.d_qk);
  size_t o = 0;
  w.attn_ws = o;   // its error word is the layer's (offset 0)
  o = align256(o + cached_layout(plan, ap).total);
  w.proj = o;
  o = align256(o + size_t(plan.Tc) * n1 * 2);
  w.a = o;
  o = align256(o + size_t(plan.Tc) * F * 2);
  w.g = o;
  o = align256(o + size_t(plan.Tc) * F * 2);
  w.total = o;
  return w;
}

static hstu_status_t validate_layer_cand(const hstu_layer_params_t *lp, const int64_t *hoff,
                                         const int64_t *coff, hstu_attn_params_t &ap) {
  if (!lp) return HSTU_ERR_INVALID_ARG;
  if (lp->d_model < 8 || lp->d_model > 8192 || (lp->d_model & 7)) return HSTU_ERR_INVALID_ARG;
  if (!(lp->ln_eps > 0.f) || !std::isfinite(lp->ln_eps)) return HSTU_ERR_INVALID_ARG;
  ap = lp->attn;
  const int64_t H = ap.num_heads;
  const int64_t n1 = 2 * H * (int64_t(ap.d_v) + ap.d_qk);
  ap.q_row_stride = ap.k_row_stride = ap.v_row_stride = n1;
  ap.o_row_stride = H * ap.d_v;
  hstu_status_t st = validate_cached(&ap, hoff, coff, n1, n1);
  if (st != HSTU_OK) return st;
  const int64_t F = H * ap.d_v;
  if (F != 32 && F != 64 && F != 128 && F != 256 && F != 512 && F != 1024)
    return HSTU_ERR_UNSUPPORTED;
  if ((H * ap.d_qk) % 8) return HSTU_ERR_UNSUPPORTED;
  return HSTU_OK;
}

}  // namespace hstu

extern "C" {

hstu_status_t hstu_layer_fwd(const hstu_layer_params_t *params, const int64_t *seq_offsets_host,
                             const int32_t *num_candidates_host, const int64_t *timestamps_dev,
                             const void *x, const void *w1, const float *b1,
                             const float *ln_gamma, const float *ln_beta, const void *w2,
                             const float *b2, const float *rab_pos, const float *rab_time,
                             void *y, void *workspace, size_t workspace_bytes, void *stream) {
  return layer_fwd_impl(params, seq_offsets_host, num_candidates_host, timestamps_dev, x, w1, b1,
                        ln_gamma, ln_beta, w2, b2, rab_pos, rab_time, y, nullptr, workspace,
                        workspace_bytes, stream);
}

hstu_status_t hstu_layer_fwd_keep_proj(const hstu_layer_params_t *params,
                                       const int64_t *seq_offsets_host,
                                       const int32_t *num_candidates_host,
                                       const int64_t *timestamps_dev, const void *x,
                                       const void *w1, const float *b1, const float *ln_gamma,
                                       const float *ln_beta, const void *w2, const float *b2,
                                       const float *rab_pos, const float *rab_time, void *y,
                                       void *proj_out, void *workspace, size_t workspace_bytes,
                                       void *stream) {
  if (!proj_out && params && params->attn.batch > 0) return HSTU_ERR_INVALID_ARG;
  return layer_fwd_impl(params, seq_offsets_host, num_candidates_host, timestamps_dev, x, w1, b1,
                        ln_gamma, ln_beta, w2, b2, rab_pos, rab_time, y, proj_out, workspace,
                        workspace_bytes, stream);
}

hstu_status_t hstu_attn_candidates_workspace_size(const hstu_attn_params_t *params,
                                                  const int64_t *hist_offsets_host,
                                                  const int64_t *cand_offsets_host,
                                                  size_t *bytes) {
  if (!bytes || !params) return HSTU_ERR_INVALID_ARG;
  const int64_t wq = int64_t(params->num_heads) * params->d_qk;
  const int64_t wv = int64_t(params->num_heads) * params->d_v;
  hstu_status_t st = validate_cached(params, hist_offsets_host, cand_offsets_host, wq, wv);
  if (st != HSTU_OK) return st;
  CachedPlan plan;
  build_cached_plan(params, hist_offsets_host, cand_offsets_host, plan);
  *bytes = cached_layout(plan, *params).total;
  return HSTU_OK;
}

hstu_status_t hstu_attn_fwd_candidates(
    const hstu_attn_params_t *params, const int64_t *hist_offsets_host,
    const int64_t *cand_offsets_host, const int64_t *hist_timestamps_dev,
    const int64_t *cand_timestamps_dev, const void *q, const void *k, const void *v,
    const void *k_hist, const void *v_hist, int64_t k_hist_row_stride,
    int64_t v_hist_row_stride, const float *rab_pos, const float *rab_time, void *out,
    void *workspace, size_t workspace_bytes, void *stream) {
  return attn_cand_impl(params, hist_offsets_host, cand_offsets_host, hist_timestamps_dev,
                        cand_timestamps_dev, q, k, v, k_hist, v_hist, k_hist_row_stride,
                        v_hist_row_stride, rab_pos, rab_time, out, workspace, workspace_bytes,
                        stream, true);
}

hstu_status_t hstu_layer_candidates_workspace_size(const hstu_layer_params_t *params,
                                                   const int64_t *hist_offsets_host,
                                                   const int64_t *cand_offsets_host,
                                                   size_t *bytes) {
  if (!bytes || !params) return HSTU_ERR_INVALID_ARG;
  hstu_attn_params_t ap;
  hstu_status_t st = validate_layer_cand(params, hist_offsets_host, cand_offsets_host, ap);
  if (st != HSTU_OK) return st;
  CachedPlan plan;
  build_cached_plan(&ap, hist_offsets_host, cand_offsets_host, plan);
  *bytes = layer_cand_layout(ap, plan).total;
  return HSTU_OK;
}

hstu_status_t hstu_layer_fwd_candidates(
    const hstu_layer_params_t *params, const int64_t *hist_offsets_host,
    const int64_t *cand_offsets_host, const int64_t *hist_timestamps_dev,
    const int64_t *cand_timestamps_dev, const void *x_cand, const void *w1, const float *b1,
    const float *ln_gamma, const float *ln_beta, const void *w2, const float *b2,
    const float *rab_pos, const float *rab_time, const void *hist_proj, void *y_cand,
    void *workspace, size_t workspace_bytes, void *stream) {
  hstu_attn_params_t ap;
  hstu_status_t st = validate_layer_cand(params, hist_offsets_host, cand_offsets_host, ap);
  if (st != HSTU_OK) return st;
  CachedPlan plan;
  build_cached_plan(&ap, hist_offsets_host, cand_offsets_host, plan);
  const int64_t Tc = plan.Tc;
  if (Tc > 0 && (!cand_timestamps_dev || !x_cand || !w1 || !b1 || !ln_gamma || !ln_beta ||
                 !w2 || !b2 || !rab_pos || !rab_time || !y_cand))
    return HSTU_ERR_INVALID_ARG;
  if (plan.Th > 0 && (!hist_timestamps_dev || !hist_proj)) return HSTU_ERR_INVALID_ARG;
  if (Tc > 0 && x_cand == y_cand) return HSTU_ERR_INVALID_ARG;
  const LayerCandWs lw = layer_cand_layout(ap, plan);
  if (!workspace || workspace_bytes < lw.total || (reinterpret_cast<uintptr_t>(workspace) & 255))
    return HSTU_ERR_WORKSPACE;
  if (Tc == 0) return HSTU_OK;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  uint8_t *ws = static_cast<uint8_t *>(workspace);
  const int64_t H = ap.num_heads, dqk = ap.d_qk, dv = ap.d_v, D = params->d_model;
  const int64_t F = H * dv, n1 = 2 * H * (dv + dqk);
  uint8_t *proj = ws + lw.proj, *a = ws + lw.a, *g = ws + lw.g;
  uint32_t *err = reinterpret_cast<uint32_t *>(ws + lw.attn_ws);
  cudaError_t e = cudaMemsetAsync(err, 0, 16, cs);
  if (e != cudaSuccess) return HSTU_ERR_CUDA;
  const WaitCtl wc{err, wait_limit_ns()};
  // the candidates' projection [U|V|Q|K] = SiLU(x W1^T + b1)
  e = launch_gemm(x_cand, D, w1, D, b1, nullptr, 0, proj, n1, Tc, n1, D, kEpiBiasSilu, wc, cs);
  if (e != cudaSuccess) return HSTU_ERR_CUDA;
  // attention against the cached history's V and K columns
  const uint8_t *hp = static_cast<const uint8_t *>(hist_proj);
  st = attn_cand_impl(&ap, hist_offsets_host, cand_offsets_host, hist_timestamps_dev,
                      cand_timestamps_dev, proj + 2 * (2 * F), proj + 2 * (2 * F + H * dqk),
                      proj + 2 * F, hp ? hp + 2 * (2 * F + H * dqk) : nullptr,
                      hp ? hp + 2 * F : nullptr, n1, n1, rab_pos, rab_time, a, ws + lw.attn_ws,
                      lw.proj - lw.attn_ws, stream, false);
  if (st != HSTU_OK) return st;
  // candidate rows only: G = LayerNorm(A) (.) U, y = x + G W2^T + b2
  e = launch_ln_gate(a, F, proj, n1, ln_gamma, ln_beta, params->ln_eps, g, F, Tc, int32_t(F), cs);
  if (e != cudaSuccess) return HSTU_ERR_CUDA;
  e = launch_gemm(g, F, w2, F, b2, params->residual ? x_cand : nullptr, D, y_cand, D, Tc, D, F,
                  params->residual ? kEpiBiasResidual : kEpiBias, wc, cs);
  return cuda_status(e);
}

// ---------------------------------------------------------------------------
// Layer backward
// ---------------------------------------------------------------------------
struct LayerBwdWs {
  size_t attn_ws, z, proj, a, dg, g, da, dproj, total;
};

static LayerBwdWs layer_bwd_layout(const hstu_attn_params_t &ap, const Plan &plan, int64_t T) {
  LayerBwdWs w{};
  const int64_t H = ap.num_heads, F = H * ap.d_v;
  const int64_t n1 = 2 * H * (int64_t(ap.d_v) + ap.d_qk);
  size_t o = 0;
  // attention workspace first: its error word is the layer's (offset 0)
  w.attn_ws = o;
  o = align256(o + std::max(layout_for(&ap, plan, false).total, layout_for(&ap, plan, true).total));
  w.z = o;
  o = align256(o + size_t(T) * n1 * 2);
  w.proj = o;
  o = align256(o + size_t(T) * n1 * 2);
  w.a = o;
  o = align256(o + size_t(T) * F * 2);
  w.dg = o;
  o = align256(o + size_t(T) * F * 2);
  w.g = o;
  o = align256(o + size_t(T) * F * 2);
  w.da = o;
  o = align256(o + size_t(T) * F * 2);
  w.dproj = o;
  o = align256(o + size_t(T) * n1 * 2);
  w.total = o;
  return w;
}

// The backward's GEMMs need the tensor-core path: N of every GEMM (N1, F,
// d_model) a multiple of 32.
static hstu_status_t validate_layer_bwd(const hstu_layer_params_t *lp, const int64_t *off,
                                        const int32_t *nc, hstu_attn_params_t &ap) {
  hstu_status_t st = validate_layer(lp, off, nc, ap);
  if (st != HSTU_OK) return st;
  const int64_t H = ap.num_heads;
  const int64_t n1 = 2 * H * (int64_t(ap.d_v) + ap.d_qk);
  if ((lp->d_model % 32) || (n1 % 32)) return HSTU_ERR_UNSUPPORTED;
  ap.do_row_stride = H * ap.d_v;
  ap.dq_row_stride = ap.dk_row_stride = ap.dv_row_stride = n1;
  return validate(&ap, off, nc, true);
}

hstu_status_t hstu_layer_bwd_workspace_size(const hstu_layer_params_t *params,
                                            const int64_t *seq_offsets_host, size_t *bytes) {
  if (!bytes || !params) return HSTU_ERR_INVALID_ARG;
  hstu_layer_params_t lp = *params;
  lp.attn.mask = HSTU_MASK_CAUSAL;
  hstu_attn_params_t ap;
  hstu_status_t st = validate_layer_bwd(&lp, seq_offsets_host, nullptr, ap);
  if (st != HSTU_OK) return st;
  std::vector<int32_t> zeros(size_t(ap.batch > 0 ? ap.batch : 0), 0);
  Plan plan;
  build_plan(&ap, seq_offsets_host, zeros.data(), plan);
  *bytes = layer_bwd_layout(ap, plan, plan.T).total;
  return HSTU_OK;
}

hstu_status_t hstu_layer_bwd(const hstu_layer_params_t *params, const int64_t *seq_offsets_host,
                             const int32_t *num_candidates_host, const int64_t *timestamps_dev,
                             const void *x, const void *w1, const float *b1,
                             const float *ln_gamma, const float *ln_beta, const void *w2,
                             const float *b2, const float *rab_pos, const float *rab_time,
                             const void *dy, void *dx, float *dw1, float *db1, float *dgamma,
                             float *dbeta, float *dw2, float *db2, float *drab_pos,
                             float *drab_time, void *workspace, size_t workspace_bytes,
                             void *stream) {
  hstu_attn_params_t ap;
  hstu_status_t st = validate_layer_bwd(params, seq_offsets_host, num_candidates_host, ap);
  if (st != HSTU_OK) return st;
  Plan plan;
  build_plan(&ap, seq_offsets_host, num_candidates_host, plan);
  const int64_t T = plan.T;
  if (T > 0 && (!timestamps_dev || !x || !w1 || !b1 || !ln_gamma || !ln_beta || !w2 || !b2 ||
                !rab_pos || !rab_time || !dy || !dx || !dw1 || !db1 || !dgamma || !dbeta ||
                !dw2 || !db2 || !drab_pos || !drab_time))
    return HSTU_ERR_INVALID_ARG;
  if (T > 0 && (dx == dy || dx == x)) return HSTU_ERR_INVALID_ARG;
  const LayerBwdWs lw = layer_bwd_layout(ap, plan, T);
  if (!workspace || workspace_bytes < lw.total || (reinterpret_cast<uintptr_t>(workspace) & 255))
    return HSTU_ERR_WORKSPACE;
  if (T == 0) return HSTU_OK;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  uint8_t *ws = static_cast<uint8_t *>(workspace);
  const int64_t H = ap.num_heads, dqk = ap.d_qk, dv = ap.d_v, D = params->d_model;
  const int64_t F = H * dv, n1 = 2 * H * (dv + dqk);
  uint8_t *z = ws + lw.z, *proj = ws + lw.proj, *a = ws + lw.a, *dg = ws + lw.dg;
  uint8_t *g = ws + lw.g, *da = ws + lw.da, *dproj = ws + lw.dproj;
  uint32_t *err = reinterpret_cast<uint32_t *>(ws + lw.attn_ws);
  cudaError_t e = cudaMemsetAsync(err, 0, 16, cs);
  if (e != cudaSuccess) return HSTU_ERR_CUDA;
  const WaitCtl wc{err, wait_limit_ns()};
  int dev = 0, n_sm = 148;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, dev);
  auto gemm = [&](const void *A, int64_t lda, bool a_mn, const void *B, int64_t ldb, bool b_mn,
                  int64_t M, int64_t N, int64_t K, int epi, const float *bias, const void *res,
                  int64_t ldr, void *C, int64_t ldc, void *C2, int64_t ldc2) {
    GemmDesc d{};
    d.a = A;
    d.lda = lda;
    d.a_mn = a_mn;
    d.b = B;
    d.ldb = ldb;
    d.b_mn = b_mn;
    d.M = M;
    d.N = N;
    d.K = K;
    d.epi = epi;
    d.bias = bias;
    d.res = res;
    d.ldr = ldr;
    d.c = C;
    d.ldc = ldc;
    d.c2 = C2;
    d.ldc2 = ldc2;
    d.splits = epi == kEpiF32Add ? gemm_split_for(M, N, K, n_sm) : 1;
    return launch_gemm_desc(d, wc, cs);
  };
  // 1. the forward again: Z = x W1^T + b1 and [U|V|Q|K] = SiLU(Z); A = attention
  e = gemm(x, D, false, w1, D, false, T, n1, D, kEpiBiasSiluPre, b1, nullptr, 0, proj, n1, z, n1);
  if (e != cudaSuccess) return HSTU_ERR_CUDA;
  const uint8_t *u_ptr = proj;
  const uint8_t *v_ptr = proj + 2 * F;
  const uint8_t *q_ptr = proj + 2 * (2 * F);
  const uint8_t *k_ptr = proj + 2 * (2 * F + H * dqk);
  const size_t attn_bytes = lw.z - lw.attn_ws;
  st = attn_fwd_impl(&ap, seq_offsets_host, num_candidates_host, timestamps_dev, q_ptr, k_ptr,
                     v_ptr, rab_pos, rab_time, a, ws + lw.attn_ws, attn_bytes, stream, false);
  if (st != HSTU_OK) return st;
  // 2. output projection: dG = dy W2 (W2 [d_model][F] read MN-major)
  e = gemm(dy, D, false, w2, F, true, T, F, D, kEpiBias, nullptr, nullptr, 0, dg, F, nullptr, 0);
  if (e != cudaSuccess) return HSTU_ERR_CUDA;
  // 3. gating and LayerNorm: G, dU (into the U columns of d[U|V|Q|K]), dA, dgamma, dbeta
  LnGateBwdArgs lg{};
  lg.a = a;
  lg.lda = F;
  lg.u = u_ptr;
  lg.ldu = n1;
  lg.dg = dg;
  lg.lddg = F;
  lg.gamma = ln_gamma;
  lg.beta = ln_beta;
  lg.eps = params->ln_eps;
  lg.g = g;
  lg.ldg = F;
  lg.du = dproj;
  lg.lddu = n1;
  lg.da = da;
  lg.ldda = F;
  lg.dgamma = dgamma;
  lg.dbeta = dbeta;
  lg.T = T;
  lg.F = int32_t(F);
  e = launch_ln_gate_bwd(lg, cs);
  if (e != cudaSuccess) return HSTU_ERR_CUDA;
  // 4. attention backward: dV, dQ, dK into their columns of d[U|V|Q|K]
  st = attn_bwd_impl(&ap, seq_offsets_host, num_candidates_host, timestamps_dev, q_ptr, k_ptr,
                     v_ptr, rab_pos, rab_time, da, dproj + 2 * (2 * F),
                     dproj + 2 * (2 * F + H * dqk), dproj + 2 * F, drab_pos, drab_time,
                     ws + lw.attn_ws, attn_bytes, stream, false);
  if (st != HSTU_OK) return st;
  // 5. dZ = d[U|V|Q|K] (.) SiLU'(Z) in place; db1 += sum_t dZ
  e = launch_colsum(dproj, n1, z, n1, db1, T, n1, true, cs);
  if (e != cudaSuccess) return HSTU_ERR_CUDA;
  // 6. weight gradients (K = tokens, split over CTAs, float32 accumulation)
  //    dW2 += dy^T G;  dW1 += dZ^T x
  e = gemm(dy, D, true, g, F, true, D, F, T, kEpiF32Add, nullptr, nullptr, 0, dw2, F, nullptr, 0);
  if (e != cudaSuccess) return HSTU_ERR_CUDA;
  e = gemm(dproj, n1, true, x, D, true, n1, D, T, kEpiF32Add, nullptr, nullptr, 0, dw1, D,
           nullptr, 0);
  if (e != cudaSuccess) return HSTU_ERR_CUDA;
  // 7. dx = dZ W1 (+ dy);  db2 += sum_t dy
  e = gemm(dproj, n1, false, w1, D, true, T, D, n1, params->residual ? kEpiBiasResidual : kEpiBias,
           nullptr, params->residual ? dy : nullptr, D, dx, D, nullptr, 0);
  if (e != cudaSuccess) return HSTU_ERR_CUDA;
  e = launch_colsum(const_cast<void *>(dy), D, nullptr, 0, db2, T, D, false, cs);
  return cuda_status(e);
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Allocation-free forward: the scratch is this file-scope device array.
// Host code must not pass `g_noalloc_scratch` itself to a kernel (in host
// code the name is only a stand-in); its device address is looked up once
// per device with cudaGetSymbolAddress, with that device current.
// ---------------------------------------------------------------------------
namespace hstu {

static __device__ __align__(256) uint8_t g_noalloc_scratch[HSTU_NOALLOC_SCRATCH_BYTES];

// Driver entry points used to tell contexts apart (no libcuda link).
typedef CUresult (*PfnCtxGetCurrent)(CUcontext *);
typedef CUresult (*PfnCtxGetId)(CUcontext, unsigned long long *);

static bool current_context_id(unsigned long long *id) {
  static PfnCtxGetCurrent get_cur = nullptr;
  static PfnCtxGetId get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *a = nullptr, *b = nullptr;
    cudaDriverEntryPointQueryResult qa, qb;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &a, cudaEnableDefault, &qa) == cudaSuccess &&
        qa == cudaDriverEntryPointSuccess)
      get_cur = reinterpret_cast<PfnCtxGetCurrent>(a);
    if (cudaGetDriverEntryPoint("cuCtxGetId", &b, cudaEnableDefault, &qb) == cudaSuccess &&
        qb == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<PfnCtxGetId>(b);
  });
  CUcontext ctx = nullptr;
  if (!get_cur || !get_id || get_cur(&ctx) != CUDA_SUCCESS || !ctx) return false;
  return get_id(ctx, id) == CUDA_SUCCESS;
}

// Device address of g_noalloc_scratch on the current device.  The address is
// looked up with cudaGetSymbolAddress (with that device current) the first
// time the entry point runs in a context and cached per device together with
// the context's id, so a context that was torn down and re-created (a device
// reset) gets a fresh lookup instead of a stale address.
constexpr int kMaxDevices = PerDeviceOnce::kMaxDevices;
struct NoallocSlot {
  unsigned long long ctx_id = 0;
  void *ptr = nullptr;
};
static NoallocSlot g_noalloc_slot[kMaxDevices];
static std::mutex g_noalloc_mu;

static hstu_status_t noalloc_scratch(void **out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return HSTU_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  unsigned long long id = 0;
  const bool have_id = current_context_id(&id);
  NoallocSlot &slot = g_noalloc_slot[dev];
  if (have_id && slot.ptr && slot.ctx_id == id) {
    *out = slot.ptr;
    return HSTU_OK;
  }
  void *ptr = nullptr;
  if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess || !ptr) return HSTU_ERR_CUDA;
  // The lookup creates the context if this thread had none yet.
  slot.ptr = ptr;
  slot.ctx_id = current_context_id(&id) ? id : 0;
  *out = ptr;
  return HSTU_OK;
}

// The scratch this forward needs, or HSTU_ERR_* for arguments the call would
// reject; no CUDA call.
static hstu_status_t noalloc_check(const hstu_attn_params_t *params, const int64_t *off,
                                   const int32_t *nc) {
  hstu_status_t st = validate(params, off, nc, false);
  if (st != HSTU_OK) return st;
  Plan plan;
  build_plan(params, off, nc, plan);
  if (layout_for(params, plan, false).total > HSTU_NOALLOC_SCRATCH_BYTES)
    return HSTU_ERR_WORKSPACE;
  return HSTU_OK;
}

}  // namespace hstu

extern "C" hstu_status_t hstu_attn_fwd_noalloc(const hstu_attn_params_t *params,
                                               const int64_t *seq_offsets_host,
                                               const int32_t *num_candidates_host,
                                               const int64_t *timestamps_dev, const void *q,
                                               const void *k, const void *v,
                                               const float *rab_pos, const float *rab_time,
                                               void *out, void *stream) {
  // Argument errors and oversize problems first, so a refused call never
  // touches the device.
  hstu_status_t st = noalloc_check(params, seq_offsets_host, num_candidates_host);
  if (st != HSTU_OK) return st;
  void *scratch = nullptr;
  st = noalloc_scratch(&scratch);
  if (st != HSTU_OK) return st;
  // The forward proper clears the error word and rewrites the schedule and
  // timestamps in the array.
  return attn_fwd_impl(params, seq_offsets_host, num_candidates_host, timestamps_dev, q, k, v,
                       rab_pos, rab_time, out, scratch, HSTU_NOALLOC_SCRATCH_BYTES, stream, true);
}
