// gemm_sm100.cu -- tensor-core GEMM (tcgen05 + TMA) for the HSTU layer's two
// projections, with the epilogue fused:
//   f1: C = SiLU(A B^T + bias)            ([U|V|Q|K] = SiLU(x W1^T + b1))
//   f2: C = A B^T + bias + R              (y = x + G W2^T + b2)
// (DLRMv4 article, section "Model architecture: HSTU replaces the
// feature-interaction stack": one projection makes the layer's internal
// representations; the gated output replaces the cross network and FFN.)
//
// A and B are bf16, each either K-major (A [M][K], B [N][K]: the nn.Linear
// [out][in] layout) or MN-major (stored [K][M] / [K][N]: the layouts the
// layer's backward meets, e.g. dW2 = dy^T G reads both operands token-major);
// fp32 accumulation in tensor memory.  C is bf16 [M][N], or float32 that the
// epilogue adds into (kEpiF32Add), which lets K be split over several CTAs
// (the weight gradients, whose K is the token count).
//
// Two persistent kernels.  Products with a K-major A, a bf16 epilogue and N
// a multiple of 256 (the layer's projections, and the backward's dG = dy W2
// and dx = dZ W1 with B read MN-major) run on CTA pairs (gemm_pair_kernel,
// below: 256 x 256 tiles, tcgen05 cta_group::2); the rest (the weight
// gradients: both operands MN-major, K split) on gemm_kernel: one CTA per
// SM walks the 128 x 256 output tiles (N fastest, so the CTAs in flight share
// A row blocks in L2).  K runs in 64-element blocks through a 4-stage TMA ring (128-byte
// swizzle).  Two tensor-memory accumulators of 256 columns let the epilogue
// of one tile overlap the MMAs of the next.
//   warp 0      TMA producer
//   warp 1      tcgen05 issuer (one thread)
//   warps 4-11  epilogue, two warpgroups (columns [0,128) and [128,256) of a
//               tile; thread = output row): tensor memory -> bias (+ SiLU, or
//               + residual) -> bf16 -> global memory; or float32 reductions.
// Operand staging: a K-major operand is one TMA box of 64 K-elements x rows
// (128-byte rows, 128-byte swizzle); an MN-major one is boxes of 64 M/N
// elements x 64 K-rows, 8 KB apart, which the MMA descriptor walks with a
// leading-byte offset of 8 KB between 64-element chunks.
// SiLU(y) = h (1 + tanh h) with h = y / 2 (sigmoid(y) = (1 + tanh(y/2)) / 2):
// one transcendental per element.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>

#include "internal.h"
#include "tile_common.cuh"

namespace hstu {
namespace gemm_tc {

constexpr int kBM = 128, kBN = 256, kBK = 64, kStages = 4, kThreads = 384;

struct Smem {
  alignas(1024) uint8_t a[kStages][kBM * kBK * 2];   // 16 KB per stage
  alignas(1024) uint8_t b[kStages][kBN * kBK * 2];   // 32 KB per stage
  uint64_t full[kStages], empty[kStages], acc_full[2], acc_empty[2], drain;
  uint32_t tmem_base;
};

struct Params {
  int64_t M, N, K;
  int32_t tiles_n, tiles, splits, items;
  int32_t a_mn, b_mn;
  const float *bias;   // [N] or null
  const __nv_bfloat16 *res;
  int64_t ldr;
  void *c;             // bf16 [M][ldc], or float32 for kEpiF32Add
  int64_t ldc;
  __nv_bfloat16 *c2;   // kEpiBiasSiluPre: pre-activation output
  int64_t ldc2;
  int epi;
  WaitCtl wait;
  uint64_t drain_ns;
};

constexpr uint32_t kChunkBytes = 64 * kBK * 2;   // one 64 x 64 MN-major box (8 KB)

__device__ __forceinline__ void red_add_v4(float *addr, float a, float b, float c, float d) {
  asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(addr), "f"(a), "f"(b),
               "f"(c), "f"(d)
               : "memory");
}

// Epilogue of 32 accumulator columns of one output row (thread = row):
// bias, then SiLU (also storing the pre-activation), residual, or plain, to
// bf16; or float32 reductions (kEpiF32Add).
__device__ __forceinline__ void epilogue_cols(const Params &p, int64_t row, int64_t col,
                                              const uint32_t (&r)[32]) {
  if (row >= p.M || col >= p.N) return;
  float y[32];
#pragma unroll
  for (int e = 0; e < 32; ++e) y[e] = __uint_as_float(r[e]);
  if (p.epi == kEpiF32Add) {
    float *dst = static_cast<float *>(p.c) + row * p.ldc + col;
#pragma unroll
    for (int v = 0; v < 8; ++v)
      red_add_v4(dst + 4 * v, y[4 * v], y[4 * v + 1], y[4 * v + 2], y[4 * v + 3]);
    return;
  }
  if (p.bias) {
    const float4 *bb = reinterpret_cast<const float4 *>(p.bias + col);
#pragma unroll
    for (int v = 0; v < 8; ++v) {
      const float4 b4 = __ldg(bb + v);
      y[4 * v] += b4.x;
      y[4 * v + 1] += b4.y;
      y[4 * v + 2] += b4.z;
      y[4 * v + 3] += b4.w;
    }
  }
  if (p.epi == kEpiBiasSiluPre) {
    uint4 *dz = reinterpret_cast<uint4 *>(p.c2 + row * p.ldc2 + col);
#pragma unroll
    for (int v = 0; v < 4; ++v)
      dz[v] = make_uint4(pack_bf16x2(y[8 * v], y[8 * v + 1]),
                         pack_bf16x2(y[8 * v + 2], y[8 * v + 3]),
                         pack_bf16x2(y[8 * v + 4], y[8 * v + 5]),
                         pack_bf16x2(y[8 * v + 6], y[8 * v + 7]));
  }
  if (p.epi == kEpiBiasSilu || p.epi == kEpiBiasSiluPre) {
#pragma unroll
    for (int e = 0; e < 32; ++e) {
      const float hh = 0.5f * y[e];
      y[e] = fmaf(hh, tanh_approx(hh), hh);
    }
  } else if (p.epi == kEpiBiasResidual) {
    const uint4 *rr = reinterpret_cast<const uint4 *>(p.res + row * p.ldr + col);
#pragma unroll
    for (int v = 0; v < 4; ++v) {
      const uint4 u = rr[v];
      const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        y[v * 8 + 2 * e] += __uint_as_float(w[e] << 16);
        y[v * 8 + 2 * e + 1] += __uint_as_float(w[e] & 0xFFFF0000u);
      }
    }
  }
  uint4 *dst = reinterpret_cast<uint4 *>(static_cast<__nv_bfloat16 *>(p.c) + row * p.ldc +
                                         col);
#pragma unroll
  for (int v = 0; v < 4; ++v)
    dst[v] = make_uint4(pack_bf16x2(y[8 * v], y[8 * v + 1]),
                        pack_bf16x2(y[8 * v + 2], y[8 * v + 3]),
                        pack_bf16x2(y[8 * v + 4], y[8 * v + 5]),
                        pack_bf16x2(y[8 * v + 6], y[8 * v + 7]));
}

__global__ void __launch_bounds__(kThreads, 1)
    gemm_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
                const Params p) {
  extern __shared__ uint8_t smem_raw[];
  Smem &sm = *reinterpret_cast<Smem *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                       ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nk = int((p.K + kBK - 1) / kBK);
  // this CTA's work items: blockIdx.x, blockIdx.x + gridDim.x, ...; item =
  // tile * splits + split, split s covering k-blocks [s nk / splits, (s+1) nk / splits)
  const int n_my = p.items > int(blockIdx.x) ? (p.items - 1 - int(blockIdx.x)) / int(gridDim.x) + 1
                                             : 0;
  auto item_of = [&](int i) { return int(blockIdx.x) + i * int(gridDim.x); };
  auto tile_m0 = [&](int i) { return int64_t((item_of(i) / p.splits) / p.tiles_n) * kBM; };
  auto tile_n0 = [&](int i) { return int64_t((item_of(i) / p.splits) % p.tiles_n) * kBN; };
  auto kb_begin = [&](int i) { return int((int64_t(item_of(i) % p.splits) * nk) / p.splits); };
  auto kb_end = [&](int i) { return int((int64_t(item_of(i) % p.splits + 1) * nk) / p.splits); };
  if (warp == 0 && lane == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&sm.full[s], 1);
      mbar_init(&sm.empty[s], 1);
    }
    for (int x = 0; x < 2; ++x) {
      mbar_init(&sm.acc_full[x], 1);
      mbar_init(&sm.acc_empty[x], 256);
    }
    mbar_init(&sm.drain, 1);
    fence_mbar_init();
    tma_prefetch_desc(&tm_a);
    tma_prefetch_desc(&tm_b);
  }
  if (warp == 1) {
    tmem_alloc(&sm.tmem_base, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;

  if (warp == 0) {
    // ===================== TMA producer =====================
    if (elect_one()) {
      bool ok = true;
      int g = 0;   // k-blocks issued over all tiles (ring position)
      for (int i = 0; i < n_my && ok; ++i) {
        const int32_t m0 = int32_t(tile_m0(i)), n0 = int32_t(tile_n0(i));
        const int kb1 = kb_end(i);
        for (int kb = kb_begin(i); kb < kb1; ++kb, ++g) {
          const int s = g % kStages;
          if (g >= kStages) ok = wait_bar(&sm.empty[s], ((g / kStages) - 1) & 1, p.wait);
          if (!ok) break;
          mbar_arrive_expect_tx(&sm.full[s], (kBM + kBN) * kBK * 2);
          if (p.a_mn) {
            for (int c = 0; c < kBM / 64; ++c)
              tma_load_2d(sm.a[s] + c * kChunkBytes, &tm_a, &sm.full[s], m0 + 64 * c, kb * kBK);
          } else {
            tma_load_2d(sm.a[s], &tm_a, &sm.full[s], kb * kBK, m0);
          }
          if (p.b_mn) {
            for (int c = 0; c < kBN / 64; ++c)
              tma_load_2d(sm.b[s] + c * kChunkBytes, &tm_b, &sm.full[s], n0 + 64 * c, kb * kBK);
          } else {
            tma_load_2d(sm.b[s], &tm_b, &sm.full[s], kb * kBK, n0);
          }
        }
      }
      // every copy issued has landed before the CTA can exit
      for (int q = (g > kStages ? g - kStages : 0); q < g; ++q)
        drain_bar(&sm.full[q % kStages], (q / kStages) & 1, p.wait.err, p.drain_ns);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ===================== tcgen05 issuer =====================
    if (elect_one()) {
      const uint32_t idesc = idesc_bf16(kBM, kBN, p.a_mn != 0, p.b_mn != 0);
      // K-major: 128-byte rows, a 16-element K step is 32 bytes along the row;
      // MN-major: 64-element chunks 8 KB apart, a K step is 16 rows of 128 bytes.
      const uint32_t a_lbo = p.a_mn ? kChunkBytes : 16u, b_lbo = p.b_mn ? kChunkBytes : 16u;
      const uint32_t a_step = p.a_mn ? (16 * 128) >> 4 : 32 >> 4;
      const uint32_t b_step = p.b_mn ? (16 * 128) >> 4 : 32 >> 4;
      bool ok = true;
      int g = 0;
      for (int i = 0; i < n_my && ok; ++i) {
        const int acc = i & 1;
        // the epilogue has read this accumulator's previous tile out
        if (i >= 2) ok = wait_bar(&sm.acc_empty[acc], ((i >> 1) - 1) & 1, p.wait);
        if (!ok) break;
        tc_fence_after();
        const uint32_t d = tmem + uint32_t(acc) * kBN;
        const int kb0 = kb_begin(i), kb1 = kb_end(i);
        for (int kb = kb0; kb < kb1 && ok; ++kb, ++g) {
          const int s = g % kStages;
          ok = wait_bar(&sm.full[s], (g / kStages) & 1, p.wait);
          if (!ok) break;
          tc_fence_after();
          const uint64_t da = sdesc_sw128(smem_u32(sm.a[s]), a_lbo, 1024);
          const uint64_t db = sdesc_sw128(smem_u32(sm.b[s]), b_lbo, 1024);
#pragma unroll
          for (int kk = 0; kk < kBK / 16; ++kk)
            umma_ss(d, da + kk * a_step, db + kk * b_step, idesc,
                    (kb > kb0 || kk > 0) ? 1u : 0u);
          umma_commit(&sm.empty[s]);
        }
        umma_commit(&sm.acc_full[acc]);
      }
      umma_commit(&sm.drain);
      drain_bar(&sm.drain, 0, p.wait.err, p.drain_ns);
    }
    __syncwarp();
  } else if (warp >= 4) {
    // ===================== epilogue =====================
    const int half = (warp - 4) >> 2;   // columns [128 half, 128 half + 128) of a tile
    const int quad = warp & 3;
    const uint32_t lane_base = tmem + (uint32_t(quad * 32) << 16);
    bool ok = true;
    for (int i = 0; i < n_my && ok; ++i) {
      const int acc = i & 1;
      ok = wait_bar_warp(&sm.acc_full[acc], (i >> 1) & 1, p.wait);
      if (!ok) break;
      tc_fence_after();
      const int64_t row = tile_m0(i) + quad * 32 + lane;
      const int64_t n0 = tile_n0(i) + half * 128;
#pragma unroll 1
      for (int c0 = 0; c0 < 128; c0 += 32) {
        uint32_t r[32];
        tmem_ld32(lane_base + uint32_t(acc) * kBN + half * 128 + c0, r);
        tmem_wait_ld(r);
        if (c0 + 32 == 128) {
          // this warpgroup's half of the accumulator is in registers
          tc_fence_before();
          mbar_arrive(&sm.acc_empty[acc]);
        }
        epilogue_cols(p, row, n0 + c0, r);
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


// ---------------------------------------------------------------------------
// CTA-pair GEMM (tcgen05 cta_group::2): a cluster of two CTAs on the two SMs
// of a pair computes a 256 x 256 tile.  Each CTA stages its own 128 rows of
// the A tile and its own 128 rows of the B tile; the even CTA's single thread
// issues M = 256, N = 256 MMAs that read both CTAs' shared memory and write
// each CTA's 128 rows of the accumulator into its own tensor memory.  Per SM
// and K step that is 32 KB of operands from L2 for 128 x 256 outputs, against
// 48 KB for the single-SM 128 x 256 tile, and a 6-stage ring in the same
// shared memory.
//   both CTAs: warp 0 TMA producer (copies complete on the even CTA's
//              full[s]), warps 4-19 epilogue of the CTA's own 128 rows, four
//              warpgroups of 64 columns each (twice the single-SM kernel's,
//              for more loads and stores in flight); each warp stages its
//              32 x 32 bf16 pieces in shared memory and writes them with bulk
//              tensor stores (row-contiguous, where a thread-per-row store
//              would touch 32 rows per instruction)
//   even CTA:  warp 1 issues the MMAs and commits to both CTAs' barriers
// An epilogue warp reports its accumulator columns read with a plain
// arrival on the even CTA's barrier: a cluster-scope release there would
// first wait for the warp's global stores.
// K-major A (B either way), one K split, bf16 epilogues only (the weight-gradient
// GEMMs keep the single-SM kernel).
constexpr int kPairStages = 6;
constexpr int kPairThreads = 640;   // control warpgroup + four epilogue warpgroups
constexpr uint32_t kHalfTileBytes = 128 * kBK * 2;   // 128 rows x 64 K, one operand, one CTA

constexpr int kPairEpiWarps = 16;
struct PairSmem {
  alignas(1024) uint8_t a[kPairStages][kHalfTileBytes];
  alignas(1024) uint8_t b[kPairStages][kHalfTileBytes];
  // per epilogue warp: its 32 rows x 32 columns of bf16 output, staged for a
  // bulk tensor store (64-byte rows, 64-byte swizzle)
  alignas(1024) uint8_t stage[kPairEpiWarps][32 * 64];
  uint64_t full[kPairStages], empty[kPairStages], acc_full[2], acc_empty[2], drain;
  uint32_t tmem_base;
};
// with the 1 KB the launcher adds for alignment: at most 227 KB per CTA
static_assert(sizeof(PairSmem) + 1024 <= 227 * 1024, "pair GEMM shared memory");

__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
// The shared::cluster address of the same shared variable in CTA `rank`.
__device__ __forceinline__ uint32_t map_to_rank(const void *p, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(smem_u32(p)), "r"(rank));
  return r;
}
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::
                   : "memory");
}
__device__ __forceinline__ void tmem_alloc_pair(uint32_t *dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                   smem_u32(dst_smem)),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish_pair() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void umma_pair_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                             uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// Arrive on the barrier `bar` of this CTA once every pair MMA this thread
// issued so far has completed.
__device__ __forceinline__ void umma_pair_commit(uint64_t *bar) {
  asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   smem_u32(bar))
               : "memory");
}
// The same on the barrier at this offset in both CTAs of the pair.
__device__ __forceinline__ void umma_pair_commit_both(uint64_t *bar) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64"
      " [%0], %1;" ::"r"(smem_u32(bar)),
      "h"(uint16_t(3))
      : "memory");
}
// Tiled 2-D copy into this CTA's shared memory whose completion is counted
// on `bar`, a barrier of either CTA of the pair (shared::cluster address).
__device__ __forceinline__ void tma_load_2d_pair(void *dst, const CUtensorMap *map, uint32_t bar,
                                                 int32_t c0, int32_t c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_u32(dst)),
      "l"(map), "r"(bar), "r"(c0), "r"(c1)
      : "memory");
}
// Software arrival on a barrier of either CTA of the pair.  It publishes
// no memory: the tensor-memory reads it reports are ordered by
// tcgen05.wait::ld and tcgen05.fence::before_thread_sync, so the arrival
// need not wait for the epilogue's global stores (a cluster-scope release
// would).
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cluster.b64 _, [%0];" ::"r"(bar) : "memory");
}

// Bulk tensor store of a staged box from shared memory, and its groups.
__device__ __forceinline__ void tma_store_2d(const CUtensorMap *map, const void *src, int32_t c0,
                                             int32_t c1) {
  asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%2, %3}], [%1];" ::"l"(
                   map),
               "r"(smem_u32(src)), "r"(c0), "r"(c1)
               : "memory");
}
__device__ __forceinline__ void bulk_commit() {
  asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}
// The staged source of every committed store has been read.
__device__ __forceinline__ void bulk_wait_read() {
  asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}
// Every committed store has completed.
__device__ __forceinline__ void bulk_wait_all() {
  asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}
__device__ __forceinline__ void fence_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
// Lane `row` of the warp writes its 32 bf16 values (16 packed pairs) into
// row `row` of the staged 32 x 32 box: 64-byte rows, 16-byte unit u at u ^
// ((row >> 1) & 3) (the 64-byte swizzle; conflict-free 16-byte stores).
__device__ __forceinline__ void stage_row(uint8_t *box, int row, const uint32_t (&w)[16]) {
#pragma unroll
  for (int u = 0; u < 4; ++u)
    *reinterpret_cast<uint4 *>(box + row * 64 + ((u ^ ((row >> 1) & 3)) << 4)) =
        make_uint4(w[4 * u], w[4 * u + 1], w[4 * u + 2], w[4 * u + 3]);
}

// Pair-kernel epilogue of 32 columns of the warp's 32 rows: bias, then SiLU
// (also staging the pre-activation), residual, or plain, to bf16, staged in
// shared memory and written by bulk tensor stores (rows past M are clipped
// by the store).
__device__ __forceinline__ void pair_epilogue_cols(const Params &p, const CUtensorMap *tm_c,
                                                   const CUtensorMap *tm_c2, uint8_t *box,
                                                   int64_t row0, int64_t col, int lane,
                                                   const uint32_t (&r)[32]) {
  const int64_t row = row0 + lane;
  float y[32];
#pragma unroll
  for (int e = 0; e < 32; ++e) y[e] = __uint_as_float(r[e]);
  if (p.bias) {
    const float4 *bb = reinterpret_cast<const float4 *>(p.bias + col);
#pragma unroll
    for (int v = 0; v < 8; ++v) {
      const float4 b4 = __ldg(bb + v);
      y[4 * v] += b4.x;
      y[4 * v + 1] += b4.y;
      y[4 * v + 2] += b4.z;
      y[4 * v + 3] += b4.w;
    }
  }
  uint32_t w[16];
  if (p.epi == kEpiBiasSiluPre) {
#pragma unroll
    for (int e = 0; e < 16; ++e) w[e] = pack_bf16x2(y[2 * e], y[2 * e + 1]);
    // the box is free once the previous store has read it
    if (lane == 0) bulk_wait_read();
    __syncwarp();
    stage_row(box, lane, w);
    fence_async_smem();
    __syncwarp();
    if (lane == 0) {
      tma_store_2d(tm_c2, box, int32_t(col), int32_t(row0));
      bulk_commit();
    }
  }
  if (p.epi == kEpiBiasSilu || p.epi == kEpiBiasSiluPre) {
#pragma unroll
    for (int e = 0; e < 32; ++e) {
      const float hh = 0.5f * y[e];
      y[e] = fmaf(hh, tanh_approx(hh), hh);
    }
  } else if (p.epi == kEpiBiasResidual && row < p.M) {
    const uint4 *rr = reinterpret_cast<const uint4 *>(p.res + row * p.ldr + col);
#pragma unroll
    for (int v = 0; v < 4; ++v) {
      const uint4 u = rr[v];
      const uint32_t wu[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        y[v * 8 + 2 * e] += __uint_as_float(wu[e] << 16);
        y[v * 8 + 2 * e + 1] += __uint_as_float(wu[e] & 0xFFFF0000u);
      }
    }
  }
#pragma unroll
  for (int e = 0; e < 16; ++e) w[e] = pack_bf16x2(y[2 * e], y[2 * e + 1]);
  if (lane == 0) bulk_wait_read();
  __syncwarp();
  stage_row(box, lane, w);
  fence_async_smem();
  __syncwarp();
  if (lane == 0) {
    tma_store_2d(tm_c, box, int32_t(col), int32_t(row0));
    bulk_commit();
  }
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kPairThreads, 1)
    gemm_pair_kernel(const __grid_constant__ CUtensorMap tm_a,
                     const __grid_constant__ CUtensorMap tm_b,
                     const __grid_constant__ CUtensorMap tm_c,
                     const __grid_constant__ CUtensorMap tm_c2, const Params p) {
  extern __shared__ uint8_t smem_raw[];
  PairSmem &sm = *reinterpret_cast<PairSmem *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();            // 0: the even CTA, which issues the MMAs
  const int pair = int(blockIdx.x >> 1), n_pairs = int(gridDim.x >> 1);
  const int nk = int((p.K + kBK - 1) / kBK);
  // this pair's 256 x 256 tiles: pair, pair + n_pairs, ... (N fastest)
  const int n_my = p.tiles > pair ? (p.tiles - 1 - pair) / n_pairs + 1 : 0;
  auto tile_of = [&](int i) { return pair + i * n_pairs; };
  auto tile_m0 = [&](int i) { return int64_t(tile_of(i) / p.tiles_n) * 256; };
  auto tile_n0 = [&](int i) { return int64_t(tile_of(i) % p.tiles_n) * 256; };
  if (warp == 0 && lane == 0) {
    for (int s = 0; s < kPairStages; ++s) {
      mbar_init(&sm.full[s], 1);    // the even CTA's producer (expecting both CTAs' bytes)
      mbar_init(&sm.empty[s], 1);   // the MMA commit
    }
    for (int x = 0; x < 2; ++x) {
      mbar_init(&sm.acc_full[x], 1);
      mbar_init(&sm.acc_empty[x], 32);   // one per epilogue warp, both CTAs
    }
    mbar_init(&sm.drain, 1);
    fence_mbar_init();
    tma_prefetch_desc(&tm_a);
    tma_prefetch_desc(&tm_b);
    tma_prefetch_desc(&tm_c);
  }
  if (warp == 1) {
    tmem_alloc_pair(&sm.tmem_base, 512);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  // both CTAs' barriers are initialised before either CTA signals the other's
  cluster_sync_all();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;

  if (warp == 0) {
    // ===================== TMA producer (both CTAs) =====================
    if (elect_one()) {
      bool ok = true;
      int g = 0;   // k-blocks issued over all tiles (ring position)
      const int32_t row_off = int32_t(rank) * 128;
      for (int i = 0; i < n_my && ok; ++i) {
        const int32_t m0 = int32_t(tile_m0(i)) + row_off, n0 = int32_t(tile_n0(i)) + row_off;
        for (int kb = 0; kb < nk; ++kb, ++g) {
          const int s = g % kPairStages;
          if (g >= kPairStages) ok = wait_bar(&sm.empty[s], ((g / kPairStages) - 1) & 1, p.wait);
          if (!ok) break;
          if (rank == 0) mbar_arrive_expect_tx(&sm.full[s], 4 * kHalfTileBytes);
          const uint32_t fb = map_to_rank(&sm.full[s], 0);
          tma_load_2d_pair(sm.a[s], &tm_a, fb, kb * kBK, m0);
          if (p.b_mn) {
            // two 64 x 64 boxes (N fastest), 8 KB apart
            for (int c = 0; c < 2; ++c)
              tma_load_2d_pair(sm.b[s] + c * kChunkBytes, &tm_b, fb, n0 + 64 * c, kb * kBK);
          } else {
            tma_load_2d_pair(sm.b[s], &tm_b, fb, kb * kBK, n0);
          }
        }
      }
      // every copy of the pair has landed before either CTA can exit (the
      // even CTA's full barriers count both CTAs' bytes)
      if (rank == 0)
        for (int q = (g > kPairStages ? g - kPairStages : 0); q < g; ++q)
          drain_bar(&sm.full[q % kPairStages], (q / kPairStages) & 1, p.wait.err, p.drain_ns);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ===================== tcgen05 issuer (even CTA) =====================
    if (rank == 0 && elect_one()) {
      const uint32_t idesc = idesc_bf16(256, 256, false, p.b_mn != 0);
      // K-major: a 16-element K step is 32 bytes along the 128-byte row;
      // MN-major: 64-element N chunks 8 KB apart, a K step is 16 rows of 128 bytes
      const uint32_t b_lbo = p.b_mn ? kChunkBytes : 16u;
      const uint32_t b_step = p.b_mn ? (16 * 128) >> 4 : 32 >> 4;
      bool ok = true;
      int g = 0;
      for (int i = 0; i < n_my && ok; ++i) {
        const int acc = i & 1;
        // both CTAs' epilogues have read this accumulator's previous tile out
        if (i >= 2) ok = wait_bar(&sm.acc_empty[acc], ((i >> 1) - 1) & 1, p.wait);
        if (!ok) break;
        tc_fence_after();
        const uint32_t d = tmem + uint32_t(acc) * 256;
        for (int kb = 0; kb < nk && ok; ++kb, ++g) {
          const int s = g % kPairStages;
          ok = wait_bar(&sm.full[s], (g / kPairStages) & 1, p.wait);
          if (!ok) break;
          tc_fence_after();
          const uint64_t da = sdesc_sw128(smem_u32(sm.a[s]), 16, 1024);
          const uint64_t db = sdesc_sw128(smem_u32(sm.b[s]), b_lbo, 1024);
#pragma unroll
          for (int kk = 0; kk < kBK / 16; ++kk)
            umma_pair_ss(d, da + kk * (32 >> 4), db + kk * b_step, idesc,
                         (kb > 0 || kk > 0) ? 1u : 0u);
          umma_pair_commit_both(&sm.empty[s]);
        }
        umma_pair_commit_both(&sm.acc_full[acc]);
      }
      umma_pair_commit(&sm.drain);
      drain_bar(&sm.drain, 0, p.wait.err, p.drain_ns);
    }
    __syncwarp();
  } else if (warp >= 4) {
    // ===================== epilogue (both CTAs, own 128 rows) =====================
    const int wg = (warp - 4) >> 2;   // columns [64 wg, 64 wg + 64) of a tile
    const int quad = warp & 3;
    const uint32_t lane_base = tmem + (uint32_t(quad * 32) << 16);
    const uint32_t acc_empty0 = map_to_rank(&sm.acc_empty[0], 0);
    const uint32_t acc_empty1 = map_to_rank(&sm.acc_empty[1], 0);
    bool ok = true;
    for (int i = 0; i < n_my && ok; ++i) {
      const int acc = i & 1;
      ok = wait_bar_warp(&sm.acc_full[acc], (i >> 1) & 1, p.wait);
      if (!ok) break;
      tc_fence_after();
      const int64_t row0 = tile_m0(i) + int64_t(rank) * 128 + quad * 32;
      const int64_t n0 = tile_n0(i) + wg * 64;
#pragma unroll 1
      for (int c0 = 0; c0 < 64; c0 += 32) {
        uint32_t r[32];
        tmem_ld32(lane_base + uint32_t(acc) * 256 + wg * 64 + c0, r);
        tmem_wait_ld(r);
        if (c0 + 32 == 64) {
          // this warp's part of the accumulator is in registers
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive_cluster(acc ? acc_empty1 : acc_empty0);
        }
        pair_epilogue_cols(p, &tm_c, &tm_c2, sm.stage[warp - 4], row0, n0 + c0, lane, r);
      }
    }
    // every store has completed before the CTA can exit
    if (lane == 0) bulk_wait_all();
    __syncwarp();
  }
  tc_fence_before();
  __syncthreads();
  // neither CTA leaves (or frees tensor memory) while the pair's MMAs,
  // copies or arrivals may still touch it
  cluster_sync_all();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, 512);
  }
}

}  // namespace gemm_tc

bool gemm_desc_supported(const GemmDesc &d) {
  if (d.M <= 0 || d.N <= 0 || d.K <= 0) return false;
  if ((d.N % 32) || (d.lda % 8) || (d.ldb % 8) || (d.ldc % (d.epi == kEpiF32Add ? 4 : 8)))
    return false;
  // K-major operands: K is the inner TMA dimension (16-byte multiple)
  if ((!d.a_mn || !d.b_mn) && (d.K % 8)) return false;
  if ((d.a_mn && (d.M % 8)) || (d.b_mn && (d.N % 8))) return false;
  if ((reinterpret_cast<uintptr_t>(d.a) | reinterpret_cast<uintptr_t>(d.b) |
       reinterpret_cast<uintptr_t>(d.c)) & 15)
    return false;
  if (d.bias && (reinterpret_cast<uintptr_t>(d.bias) & 15)) return false;
  if (d.epi == kEpiBiasResidual &&
      (!d.res || (reinterpret_cast<uintptr_t>(d.res) & 15) || (d.ldr % 8)))
    return false;
  if (d.epi == kEpiBiasSiluPre &&
      (!d.c2 || (reinterpret_cast<uintptr_t>(d.c2) & 15) || (d.ldc2 % 8)))
    return false;
  if (d.splits < 1 || (d.splits > 1 && d.epi != kEpiF32Add)) return false;
  if (d.M >= (int64_t(1) << 31) || d.N >= (int64_t(1) << 31) || d.K >= (int64_t(1) << 31))
    return false;
  const int64_t tiles = ((d.M + 127) / 128) * ((d.N + 255) / 256);
  if (tiles * d.splits >= (int64_t(1) << 30)) return false;
  return true;
}

bool gemm_tc_supported(const void *a, int64_t lda, const void *b, int64_t ldb, const void *c,
                       int64_t ldc, int64_t M, int64_t N, int64_t K) {
  GemmDesc d{};
  d.a = a;
  d.lda = lda;
  d.b = b;
  d.ldb = ldb;
  d.c = const_cast<void *>(c);
  d.ldc = ldc;
  d.M = M;
  d.N = N;
  d.K = K;
  d.epi = kEpiBias;
  d.splits = 1;
  return gemm_desc_supported(d);
}

// Shapes the CTA-pair kernel takes: K-major A, B either way, no K split, a bf16
// epilogue, N a multiple of 256 and at least one 256-row tile of M.
static bool gemm_pair_eligible(const GemmDesc &d) {
  return !d.a_mn && d.splits == 1 && d.epi != kEpiF32Add && d.N % 256 == 0 && d.M >= 256;
}

static cudaError_t launch_gemm_pair(const GemmDesc &d, const WaitCtl &w, cudaStream_t st) {
  using namespace gemm_tc;
  CUtensorMap ta, tb;
  if (!encode_tmap_bf16_2d(&ta, d.a, uint64_t(d.K), uint64_t(d.M), uint64_t(d.lda) * 2, kBK,
                           128) ||
      !(d.b_mn ? encode_tmap_bf16_2d(&tb, d.b, uint64_t(d.N), uint64_t(d.K),
                                     uint64_t(d.ldb) * 2, 64, kBK)
               : encode_tmap_bf16_2d(&tb, d.b, uint64_t(d.K), uint64_t(d.N),
                                     uint64_t(d.ldb) * 2, kBK, 128)))
    return cudaErrorInvalidValue;
  // output boxes of 32 columns x 32 rows (one epilogue warp's chunk)
  CUtensorMap tc, tc2;
  if (!encode_tmap_bf16_2d_sw64(&tc, d.c, uint64_t(d.N), uint64_t(d.M), uint64_t(d.ldc) * 2, 32,
                                32))
    return cudaErrorInvalidValue;
  tc2 = tc;
  if (d.epi == kEpiBiasSiluPre &&
      !encode_tmap_bf16_2d_sw64(&tc2, d.c2, uint64_t(d.N), uint64_t(d.M), uint64_t(d.ldc2) * 2,
                                32, 32))
    return cudaErrorInvalidValue;
  Params prm;
  prm.M = d.M;
  prm.N = d.N;
  prm.K = d.K;
  prm.tiles_n = int32_t(d.N / 256);
  prm.tiles = int32_t(((d.M + 255) / 256) * prm.tiles_n);
  prm.splits = 1;
  prm.items = prm.tiles;
  prm.a_mn = 0;
  prm.b_mn = d.b_mn ? 1 : 0;
  prm.bias = d.bias;
  prm.res = static_cast<const __nv_bfloat16 *>(d.res);
  prm.ldr = d.ldr;
  prm.c = d.c;
  prm.ldc = d.ldc;
  prm.c2 = static_cast<__nv_bfloat16 *>(d.c2);
  prm.ldc2 = d.ldc2;
  prm.epi = d.epi;
  prm.wait = w;
  prm.drain_ns = 4000000000ull;
  const size_t smem = sizeof(PairSmem) + 1024;
  static PerDeviceOnce attr;
  static int n_pairs_of[PerDeviceOnce::kMaxDevices];
  cudaError_t e = attr.run([&](int dev) {
    cudaError_t r = cudaFuncSetAttribute(gemm_pair_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
    if (r != cudaSuccess) return r;
    // pairs that can be resident at once (one per two SMs when nothing else runs)
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2, 1, 1);
    cfg.blockDim = dim3(kPairThreads, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeClusterDimension;
    at[0].val.clusterDim.x = 2;
    at[0].val.clusterDim.y = 1;
    at[0].val.clusterDim.z = 1;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    int n = 0;
    r = cudaOccupancyMaxActiveClusters(&n, gemm_pair_kernel, &cfg);
    if (r != cudaSuccess) return r;
    n_pairs_of[dev] = n > 0 ? n : 1;
    return cudaSuccess;
  });
  if (e != cudaSuccess) return e;
  int dev = 0;
  e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const unsigned grid = 2u * unsigned(std::min<int64_t>(prm.tiles, n_pairs_of[dev]));
  gemm_pair_kernel<<<grid, kPairThreads, smem, st>>>(ta, tb, tc, tc2, prm);
  count_launch();
  return cudaGetLastError();
}

cudaError_t launch_gemm_desc(const GemmDesc &d, const WaitCtl &w, cudaStream_t st) {
  using namespace gemm_tc;
  if (!gemm_desc_supported(d)) return cudaErrorInvalidValue;
  if (gemm_pair_eligible(d)) return launch_gemm_pair(d, w, st);
  CUtensorMap ta, tb;
  const bool ok_a =
      d.a_mn ? encode_tmap_bf16_2d(&ta, d.a, uint64_t(d.M), uint64_t(d.K), uint64_t(d.lda) * 2,
                                   64, kBK)
             : encode_tmap_bf16_2d(&ta, d.a, uint64_t(d.K), uint64_t(d.M), uint64_t(d.lda) * 2,
                                   kBK, kBM);
  const bool ok_b =
      d.b_mn ? encode_tmap_bf16_2d(&tb, d.b, uint64_t(d.N), uint64_t(d.K), uint64_t(d.ldb) * 2,
                                   64, kBK)
             : encode_tmap_bf16_2d(&tb, d.b, uint64_t(d.K), uint64_t(d.N), uint64_t(d.ldb) * 2,
                                   kBK, kBN);
  if (!ok_a || !ok_b) return cudaErrorInvalidValue;
  Params prm;
  prm.M = d.M;
  prm.N = d.N;
  prm.K = d.K;
  prm.tiles_n = int32_t((d.N + kBN - 1) / kBN);
  prm.tiles = int32_t(((d.M + kBM - 1) / kBM) * prm.tiles_n);
  const int nk = int((d.K + kBK - 1) / kBK);
  prm.splits = std::max(1, std::min(d.splits, nk));   // every split gets a k-block
  prm.items = prm.tiles * prm.splits;
  prm.a_mn = d.a_mn ? 1 : 0;
  prm.b_mn = d.b_mn ? 1 : 0;
  prm.bias = d.bias;
  prm.res = static_cast<const __nv_bfloat16 *>(d.res);
  prm.ldr = d.ldr;
  prm.c = d.c;
  prm.ldc = d.ldc;
  prm.c2 = static_cast<__nv_bfloat16 *>(d.c2);
  prm.ldc2 = d.ldc2;
  prm.epi = d.epi;
  prm.wait = w;
  prm.drain_ns = 4000000000ull;
  const size_t smem = sizeof(Smem) + 1024;
  static PerDeviceOnce attr;
  static int n_sm_of[PerDeviceOnce::kMaxDevices];
  cudaError_t e = attr.run([&](int dev) {
    cudaError_t r =
        cudaFuncSetAttribute(gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
    if (r != cudaSuccess) return r;
    int n = 0;
    r = cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (r != cudaSuccess) return r;
    n_sm_of[dev] = n > 0 ? n : 1;
    return cudaSuccess;
  });
  if (e != cudaSuccess) return e;
  int dev = 0;
  e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const int n_sm = n_sm_of[dev];
  const unsigned grid = unsigned(std::min<int64_t>(prm.items, n_sm));
  gemm_kernel<<<grid, kThreads, smem, st>>>(ta, tb, prm);
  count_launch();
  return cudaGetLastError();
}

int gemm_split_for(int64_t M, int64_t N, int64_t K, int n_sm) {
  const int64_t tiles = ((M + 127) / 128) * ((N + 255) / 256);
  const int64_t nk = (K + 63) / 64;
  // enough items to fill every SM once, at least 4 k-blocks per item
  int64_t s = (n_sm + tiles - 1) / tiles;
  s = std::min<int64_t>(s, std::max<int64_t>(1, nk / 4));
  return int(std::max<int64_t>(1, s));
}

cudaError_t launch_gemm_tc(const void *a, int64_t lda, const void *b, int64_t ldb,
                           const float *bias, const void *residual, int64_t ldr, void *c,
                           int64_t ldc, int64_t M, int64_t N, int64_t K, int epilogue,
                           const WaitCtl &w, cudaStream_t st) {
  GemmDesc d{};
  d.a = a;
  d.lda = lda;
  d.b = b;
  d.ldb = ldb;
  d.M = M;
  d.N = N;
  d.K = K;
  d.epi = epilogue;
  d.bias = bias;
  d.res = residual;
  d.ldr = ldr;
  d.c = c;
  d.ldc = ldc;
  d.splits = 1;
  return launch_gemm_desc(d, w, st);
}

}  // namespace hstu
