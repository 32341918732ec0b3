// Per-expert routing frequencies, accumulated across calls (CMF code specialist
// page, How it was made: the Calibrate step records per-layer expert routing
// frequencies over a representative corpus).  counts[e] += the number of
// (token, slot) entries of topk_idx equal to e; entries outside [0, E) are not
// counted.  Integer sums, so the result does not depend on scheduling.
#include "common.cuh"
#include "internal.h"

namespace moe {
namespace {

constexpr int kCountThreads = 512;

// block histogram in shared memory, then one 64-bit add per non-empty bin
__global__ void __launch_bounds__(kCountThreads) expert_counts_kernel(const int32_t* __restrict__ idx, int64_t n,
                                                                      int E, unsigned long long* __restrict__ counts) {
  pdl_wait();
  pdl_trigger();
  __shared__ uint32_t hist[1024];
  for (int e = threadIdx.x; e < E; e += blockDim.x) hist[e] = 0u;
  __syncthreads();
  const int64_t stride = (int64_t)gridDim.x * blockDim.x * 4;
  for (int64_t i0 = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) * 4; i0 < n; i0 += stride) {
    if (i0 + 4 <= n && (reinterpret_cast<uintptr_t>(idx + i0) & 15) == 0) {
      const int4 v = *reinterpret_cast<const int4*>(idx + i0);
      const int vals[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int j = 0; j < 4; ++j)
        if (vals[j] >= 0 && vals[j] < E) atomicAdd(&hist[vals[j]], 1u);
    } else {
      for (int64_t i = i0; i < n && i < i0 + 4; ++i) {
        const int v = idx[i];
        if (v >= 0 && v < E) atomicAdd(&hist[v], 1u);
      }
    }
  }
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x)
    if (hist[e]) atomicAdd(&counts[e], (unsigned long long)hist[e]);
}

}  // namespace

cudaError_t launch_expert_counts(const int32_t* idx, int64_t n, int E, uint64_t* counts, int num_sms,
                                 cudaStream_t s) {
  int64_t blocks = (n + kCountThreads * 16 - 1) / (kCountThreads * 16);
  if (blocks > 2 * num_sms) blocks = 2 * num_sms;
  if (blocks < 1) blocks = 1;
  return launch_k(expert_counts_kernel, dim3((unsigned)blocks), dim3(kCountThreads), 0, s, idx, n, E,
                  reinterpret_cast<unsigned long long*>(counts));
}

}  // namespace moe
