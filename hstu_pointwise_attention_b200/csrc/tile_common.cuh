// tile_common.cuh -- jagged tile geometry and bounded waits shared by the
// tensor-core attention kernels.
#pragma once

#include "common.cuh"

namespace hstu {

constexpr int kAttnTile = 128;   // query rows / keys per tile

// Which (query tile, key tile) pairs of one sequence hold a visible pair:
// a history query sees keys at or before it; a candidate (the last
// num_candidates tokens) sees the whole history and itself only.
struct TileGeom {
  int32_t L, nh;
  __device__ __forceinline__ int32_t pos(int32_t i) const { return i < nh ? i : nh; }
  // last key tile holding history keys some row of query tile qt can see
  __device__ __forceinline__ int32_t hist_end(int32_t qt) const {
    const int32_t qe = min((qt + 1) * kAttnTile, L);
    const int32_t m = min(qe, nh);
    return m > 0 ? (m - 1) / kAttnTile : -1;
  }
  __device__ __forceinline__ bool has_cand(int32_t qt) const {
    return min((qt + 1) * kAttnTile, L) > nh;
  }
  __device__ __forceinline__ bool valid(int32_t qt) const { return qt * kAttnTile < L; }
  __device__ __forceinline__ bool active(int32_t qt, int32_t kt) const {
    return valid(qt) && (kt <= hist_end(qt) || (has_cand(qt) && kt == qt));
  }
  __device__ __forceinline__ bool visible(int32_t i, int32_t j) const {
    return i < L && j < L && (i < nh ? (j <= i) : (j < nh || j == i));
  }
  // true when every (i, j) of the tile pair is visible and in range
  __device__ __forceinline__ bool full_tile(int32_t qt, int32_t kt) const {
    const int32_t qs = qt * kAttnTile, ks = kt * kAttnTile;
    return ks + kAttnTile <= nh && ks + kAttnTile - 1 <= qs && qs + kAttnTile <= L;
  }
  // smallest position distance of the tile pair (bounds the position bucket)
  __device__ __forceinline__ int32_t min_pos_dist(int32_t qt, int32_t kt) const {
    const int32_t kmax = min(kt * kAttnTile + kAttnTile - 1, L - 1);
    return pos(qt * kAttnTile) - pos(kmax);
  }

  // The same questions for query rows [qs, qs + qn) against the key tile
  // [ks, ks + kAttnTile).
  __device__ __forceinline__ bool active_rows(int32_t qs, int32_t qn, int32_t ks) const {
    if (qs >= L) return false;
    const int32_t qe = min(qs + qn, L);
    const int32_t hh = min(qe, nh) - 1;   // last history query among the rows
    if (hh >= qs && hh >= ks) return true;   // it sees key ks
    const int32_t c0 = max(qs, nh);          // first candidate among the rows
    if (c0 >= qe) return false;
    // candidates see every history key, and themselves
    return ks < nh || max(c0, ks) < min(qe, ks + kAttnTile);
  }
  __device__ __forceinline__ bool full_rows(int32_t qs, int32_t qn, int32_t ks) const {
    return ks + kAttnTile <= nh && ks + kAttnTile - 1 <= qs && qs + qn <= L;
  }
  __device__ __forceinline__ int32_t min_pos_dist_rows(int32_t qs, int32_t ks) const {
    return pos(qs) - pos(min(ks + kAttnTile - 1, L - 1));
  }
};

// Bounded wait that also gives up once another role has recorded an error.
__device__ __forceinline__ bool wait_bar(uint64_t *bar, uint32_t parity, const WaitCtl &w) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  while (true) {
#pragma unroll 1
    for (int i = 0; i < 64; ++i)
      if (mbar_try_wait(bar, parity)) return true;
    if (*reinterpret_cast<volatile uint32_t *>(w.err) != 0) return false;
    if (globaltimer_ns() - t0 > w.limit_ns) {
      record_error(w.err, kDevErrTimeout);
      return false;
    }
  }
}

// wait_bar for code a whole warp runs: every lane gets the same answer, so
// lanes leave a loop together and the warp-wide and named barriers after it
// stay matched even when a wait gives up.
__device__ __forceinline__ bool wait_bar_warp(uint64_t *bar, uint32_t parity, const WaitCtl &w) {
  return __all_sync(0xffffffffu, wait_bar(bar, parity, w));
}

// Drain wait used on the way out: long bound, ignores other roles' errors.
__device__ __forceinline__ void drain_bar(uint64_t *bar, uint32_t parity, uint32_t *err,
                                          uint64_t limit) {
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (globaltimer_ns() - t0 > limit) {
      record_error(err, kDevErrTimeout);
      return;
    }
  }
}

// Named barrier among `count` threads (id 1..15; id 0 is __syncthreads).
__device__ __forceinline__ void named_bar_sync(int id, int count) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}

// Warpgroup register re-allocation for the 384-thread attention kernels:
// the launch gives 168 registers to each of the 384 threads (64,512 total);
// warpgroup 0 (loads, MMA issue) drops to kRegsCtl and the two elementwise
// warpgroups rise to kRegsEw.  4*32*72 + 8*32*216 = 64,512: the split never
// asks for more than the launch holds.  The launchers check that the kernel
// was compiled to exactly kRegsLaunch registers before launching.
constexpr int kRegsLaunch = 168, kRegsCtl = 72, kRegsEw = 216;
static_assert(4 * 32 * kRegsCtl + 8 * 32 * kRegsEw <= 12 * 32 * kRegsLaunch,
              "register split exceeds the launch allocation");

template <int N = kRegsCtl>
__device__ __forceinline__ void regs_release_ctl() {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(N));
}
template <int N = kRegsEw>
__device__ __forceinline__ void regs_grow_ew() {
  asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(N));
}

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// Bulk tensor reduce-add (shared -> global, float32 add done at L2), tracked
// by the issuing thread's bulk-async group.
__device__ __forceinline__ void tma_reduce_add_2d(const CUtensorMap *map, const void *src,
                                                  int32_t c0, int32_t c1) {
  asm volatile(
      "cp.reduce.async.bulk.tensor.2d.global.shared::cta.add.bulk_group [%0, {%2, %3}], [%1];" ::
          "l"(map),
      "r"(smem_u32(src)), "r"(c0), "r"(c1)
      : "memory");
}
__device__ __forceinline__ void bulk_commit() {
  asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}
// The sources of this thread's bulk operations have been read (buffer reusable).
__device__ __forceinline__ void bulk_wait_read_all() {
  asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}
// This thread's bulk operations have fully completed.
__device__ __forceinline__ void bulk_wait_all() {
  asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}

__device__ __forceinline__ void red_add_f32(float *addr, float a) {
  asm volatile("red.global.add.f32 [%0], %1;" ::"l"(addr), "f"(a) : "memory");
}

// Four consecutive floats (16-byte aligned address) added in one reduction.
__device__ __forceinline__ void red_add_v4_f32(float *addr, float a, float b, float c, float d) {
  asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(addr), "f"(a), "f"(b),
               "f"(c), "f"(d)
               : "memory");
}

}  // namespace hstu
