// schedule.cu -- moves the host-built tile schedule (sequence table and work
// lists) into the caller's workspace without a host-to-device memcpy.
//
// A cudaMemcpyAsync from pageable host memory makes the calling thread wait
// for the stream, so every entry point would stall the host until the device
// caught up.  Here the bytes travel as the parameters of a small kernel: the
// launch copies them to the device itself, in stream order, without blocking
// the host, and a CUDA graph that captures the call keeps them.  A schedule
// larger than one launch's parameter space goes up in several launches.
#include <cuda_runtime.h>

#include <algorithm>
#include <cstring>

#include "internal.h"

namespace hstu {

// 32 KB of kernel parameters (CUDA 12.1+ on sm_70+) minus the header.
constexpr uint32_t kUploadBytes = 32704;

struct UploadArgs {
  uint4 *dst;         // 16-byte aligned destination
  uint32_t *err;      // when non-null: the 16-byte device error word to clear
  uint32_t n16;       // 16-byte words in data
  uint32_t pad;
  uint4 data[kUploadBytes / 16];
};
static_assert(sizeof(UploadArgs) <= 32764, "kernel parameter space");

__global__ void __launch_bounds__(256) upload_kernel(const __grid_constant__ UploadArgs a) {
  if (a.err && blockIdx.x == 0 && threadIdx.x < 4) a.err[threadIdx.x] = 0u;
  for (uint32_t i = blockIdx.x * blockDim.x + threadIdx.x; i < a.n16; i += gridDim.x * blockDim.x)
    a.dst[i] = a.data[i];
}

cudaError_t launch_upload(void *dst, const void *src, size_t bytes, uint32_t *err_clear,
                          cudaStream_t st) {
  if ((reinterpret_cast<uintptr_t>(dst) & 15) || (bytes & 15)) return cudaErrorInvalidValue;
  const uint8_t *s = static_cast<const uint8_t *>(src);
  uint8_t *d = static_cast<uint8_t *>(dst);
  size_t done = 0;
  bool first = true;
  while (first || done < bytes) {
    const size_t n = std::min<size_t>(bytes - done, kUploadBytes);
    UploadArgs a;
    a.dst = reinterpret_cast<uint4 *>(d + done);
    a.err = first ? err_clear : nullptr;
    a.n16 = uint32_t(n / 16);
    a.pad = 0;
    if (n) std::memcpy(a.data, s + done, n);
    const unsigned blocks = unsigned(std::max<size_t>(1, std::min<size_t>(8, (n / 16 + 255) / 256)));
    upload_kernel<<<blocks, 256, 0, st>>>(a);
    count_launch();
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    done += n;
    first = false;
  }
  return cudaSuccess;
}

}  // namespace hstu

// ---------------------------------------------------------------------------
// Data-parallel split of a jagged batch (hstu_partition_batch).
// ---------------------------------------------------------------------------
#include <numeric>
#include <vector>

#include "../../include/hstu.h"

extern "C" hstu_status_t hstu_partition_batch(const int64_t *seq_offsets_host,
                                              const int32_t *num_candidates_host, int32_t batch,
                                              int32_t world, int32_t *rank_of_seq,
                                              int64_t *rank_pairs) {
  if (batch < 0 || world < 1 || (batch > 0 && (!seq_offsets_host || !rank_of_seq)))
    return HSTU_ERR_INVALID_ARG;
  if (batch > 0 && seq_offsets_host[0] != 0) return HSTU_ERR_INVALID_ARG;
  std::vector<int64_t> cost(static_cast<size_t>(batch), 0);
  for (int32_t b = 0; b < batch; ++b) {
    const int64_t L = seq_offsets_host[b + 1] - seq_offsets_host[b];
    if (L < 0) return HSTU_ERR_INVALID_ARG;
    const int64_t nc = num_candidates_host ? num_candidates_host[b] : 0;
    if (nc < 0 || nc > L) return HSTU_ERR_INVALID_ARG;
    const int64_t nh = L - nc;
    // visible pairs: a history query i sees i + 1 keys, a candidate nh + 1
    cost[size_t(b)] = nh * (nh + 1) / 2 + nc * (nh + 1);
  }
  // Longest processing time first: sequences by descending pair count (ties
  // by index), each to the rank with the smallest load so far (ties to the
  // lower rank).  The result is deterministic.
  std::vector<int32_t> order(static_cast<size_t>(batch));
  std::iota(order.begin(), order.end(), 0);
  std::stable_sort(order.begin(), order.end(),
                   [&](int32_t a, int32_t b) { return cost[size_t(a)] > cost[size_t(b)]; });
  std::vector<int64_t> load(static_cast<size_t>(world), 0);
  for (int32_t b : order) {
    int32_t best = 0;
    for (int32_t r = 1; r < world; ++r)
      if (load[size_t(r)] < load[size_t(best)]) best = r;
    rank_of_seq[b] = best;
    load[size_t(best)] += cost[size_t(b)];
  }
  if (rank_pairs)
    for (int32_t r = 0; r < world; ++r) rank_pairs[r] = load[size_t(r)];
  return HSTU_OK;
}
