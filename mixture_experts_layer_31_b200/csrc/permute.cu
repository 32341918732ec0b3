// Expert-sorted order of the (token, slot) pairs: histogram, scan, stable
// counting-sort scatter.  A token runs only through its routed experts
// (Qwen3-30B-A3B LiteRT-LM card, Conversion Notes): grouping the pairs by
// expert lets each expert's weights be streamed once for all its tokens.
//
// Pair p = t * k + slot.  The pairs are cut into chunks of kPairChunk; every
// kernel walks a chunk in pair order, so the result is a deterministic, stable
// sort by expert (ties in pair order) with no order-dependent atomics.
#include "common.cuh"
#include "internal.h"
#include "route_dev.cuh"

namespace moe {
using route_dev::kSmallE;
using route_dev::kSortWarps;
namespace {

__global__ void __launch_bounds__(256) pair_histogram_kernel(const int32_t* __restrict__ idx, int P, int E,
                                                             int32_t* __restrict__ chunk_hist,
                                                             uint32_t* flags) {
  pdl_wait();
  pdl_trigger();
  extern __shared__ int32_t hist[];
  for (int e = threadIdx.x; e < E; e += blockDim.x) hist[e] = 0;
  __syncthreads();
  const int p0 = blockIdx.x * kPairChunk, p1 = min(P, p0 + kPairChunk);
  bool bad = false;
  for (int p = p0 + threadIdx.x; p < p1; p += blockDim.x) {
    const int e = idx[p];
    if (e >= 0 && e < E)
      atomicAdd(&hist[e], 1);
    else
      bad = true;
  }
  if (bad) raise_flag(flags, MOE_FLAG_BAD_EXPERT_INDEX);
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x) chunk_hist[(size_t)blockIdx.x * E + e] = hist[e];
}

// one block, one thread per expert: per-chunk bases, counts, offsets, touched list
__global__ void __launch_bounds__(1024) expert_scan_kernel(int NC, int E, int32_t* __restrict__ chunk_hist,
                                                           int32_t* __restrict__ counts,
                                                           int32_t* __restrict__ offsets,
                                                           int32_t* __restrict__ touched,
                                                           int32_t* __restrict__ group_base,
                                                           int32_t* __restrict__ tile_base, int chunk,
                                                           int32_t* __restrict__ meta) {
  pdl_wait();
  pdl_trigger();
  __shared__ int warp_sums[32];
  const int e = threadIdx.x;
  // two passes over the expert's column of chunk counts, each with kBatch loads in
  // flight: the total first, then (once the expert's offset is known) the
  // chunk bases, written in place
  constexpr int kBatch = 16;
  int running = 0;
  if (e < E) {
    for (int c0 = 0; c0 < NC; c0 += kBatch) {
      int v[kBatch];
#pragma unroll
      for (int j = 0; j < kBatch; ++j) v[j] = c0 + j < NC ? chunk_hist[(size_t)(c0 + j) * E + e] : 0;
#pragma unroll
      for (int j = 0; j < kBatch; ++j) running += v[j];
    }
    counts[e] = running;
  }
  int total;
  const int off = route_dev::block_exclusive_scan(e < E ? running : 0, warp_sums, &total);
  if (e < E) {
    offsets[e] = off;
    int base = off;
    for (int c0 = 0; c0 < NC; c0 += kBatch) {
      int v[kBatch];
#pragma unroll
      for (int j = 0; j < kBatch; ++j) v[j] = c0 + j < NC ? chunk_hist[(size_t)(c0 + j) * E + e] : 0;
#pragma unroll
      for (int j = 0; j < kBatch; ++j) {
        if (c0 + j < NC) chunk_hist[(size_t)(c0 + j) * E + e] = base;
        base += v[j];
      }
    }
  }
  if (e == 0) offsets[E] = total;
  int ntouched;
  const int tpos = route_dev::block_exclusive_scan((e < E && running > 0) ? 1 : 0, warp_sums, &ntouched);
  if (e < E && running > 0) touched[tpos] = e;
  // token groups per touched expert, prefixed in touched (= ascending expert) order
  const int groups = (e < E) ? (running + kGemvGroup - 1) / kGemvGroup : 0;
  int ngroups;
  const int gpos = route_dev::block_exclusive_scan(groups, warp_sums, &ngroups);
  if (e < E && running > 0) group_base[tpos] = gpos;
  // token chunks of the tensor-core path, same order
  const int chunks = (e < E) ? (running + chunk - 1) / chunk : 0;
  int nchunks;
  const int cpos = route_dev::block_exclusive_scan(chunks, warp_sums, &nchunks);
  if (e < E && running > 0) tile_base[tpos] = cpos;
  if (e == 0) {
    meta[0] = ntouched;
    meta[1] = total;
    meta[2] = ngroups;
    meta[3] = nchunks;
    meta[8] = 0;  // unit counters of the grouped GEMMs that follow
    meta[9] = 0;
    group_base[ntouched] = ngroups;
    tile_base[ntouched] = nchunks;
  }
}

// one warp per chunk: stable positions in pair order
__global__ void __launch_bounds__(128) pair_scatter_kernel(const int32_t* __restrict__ idx, int P, int E,
                                                           const int32_t* __restrict__ chunk_base,
                                                           int32_t* __restrict__ sorted_pair) {
  pdl_wait();
  pdl_trigger();
  extern __shared__ int32_t running_all[];
  const int w = warp_id(), lane = lane_id();
  const int c = blockIdx.x * (blockDim.x >> 5) + w;
  int32_t* running = running_all + w * E;
  const int nchunks = (P + kPairChunk - 1) / kPairChunk;
  if (c >= nchunks) return;
  for (int e = lane; e < E; e += 32) running[e] = chunk_base[(size_t)c * E + e];
  __syncwarp();
  const int p0 = c * kPairChunk, p1 = min(P, p0 + kPairChunk);
  const unsigned lt = (1u << lane) - 1u;
  for (int pb = p0; pb < p1; pb += 32) {
    const int p = pb + lane;
    int e = (p < p1) ? idx[p] : -1;
    if (e < 0 || e >= E) e = -1;
    const unsigned peers = __match_any_sync(0xFFFFFFFFu, e);
    int pos = 0;
    if (e >= 0) {
      pos = running[e] + __popc(peers & lt);
      sorted_pair[pos] = p;
    }
    __syncwarp();
    if (e >= 0 && lane == 31 - __clz(peers)) running[e] += __popc(peers);
    __syncwarp();
  }
}

__global__ void __launch_bounds__(1024) small_sort_kernel(const int32_t* __restrict__ idx, int P, int E,
                                                          int chunk, int32_t* __restrict__ counts,
                                                          int32_t* __restrict__ offsets,
                                                          int32_t* __restrict__ touched,
                                                          int32_t* __restrict__ group_base,
                                                          int32_t* __restrict__ tile_base,
                                                          int32_t* __restrict__ meta,
                                                          int32_t* __restrict__ sorted_pair, uint32_t* flags) {
  pdl_wait();
  pdl_trigger();
  __shared__ int32_t base[kSortWarps][kSmallE];
  __shared__ int4 warp_sums4[32];
  route_dev::block_small_sort(idx, P, E, chunk, counts, offsets, touched, group_base, tile_base, meta, sorted_pair,
                              flags, base, warp_sums4);
}

}  // namespace

bool small_sort_ok(int P, int E) { return P <= 8192 && E <= kSmallE; }

cudaError_t launch_small_sort(const int32_t* idx, int P, int E, int chunk, int32_t* counts, int32_t* offsets,
                              int32_t* touched, int32_t* group_base, int32_t* tile_base, int32_t* meta,
                              int32_t* sorted_pair, uint32_t* flags, cudaStream_t s) {
  return launch_k(small_sort_kernel, dim3(1), dim3(1024), 0, s, idx, P, E, chunk, counts, offsets, touched,
                    group_base, tile_base, meta, sorted_pair, flags);
}

cudaError_t launch_pair_histogram(const int32_t* idx, int P, int E, int32_t* chunk_hist, uint32_t* flags,
                                  cudaStream_t s) {
  const int NC = (P + kPairChunk - 1) / kPairChunk;
  return launch_k(pair_histogram_kernel, dim3(NC), dim3(256), E * sizeof(int32_t), s, idx, P, E, chunk_hist, flags);
}

cudaError_t launch_expert_scan(int NC, int E, int32_t* chunk_hist, int32_t* counts, int32_t* offsets,
                               int32_t* touched, int32_t* group_base, int32_t* tile_base, int chunk,
                               int32_t* meta, cudaStream_t s) {
  const int threads = ((E + 31) / 32) * 32;
  return launch_k(expert_scan_kernel, dim3(1), dim3(threads), 0, s, NC, E, chunk_hist, counts, offsets, touched,
                    group_base, tile_base, chunk, meta);
}

// The plan of a dense expert applied to every token (the shared expert): the
// sort's outputs for T pairs that all go to expert 0 in token order, and unit
// weights, written directly.
__global__ void __launch_bounds__(256) dense_plan_kernel(int T, int chunk, int32_t* __restrict__ counts,
                                                         int32_t* __restrict__ offsets, int32_t* __restrict__ touched,
                                                         int32_t* __restrict__ group_base,
                                                         int32_t* __restrict__ tile_base, int32_t* __restrict__ meta,
                                                         int32_t* __restrict__ sorted_pair, float* __restrict__ ones) {
  pdl_wait();
  pdl_trigger();
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < T; i += gridDim.x * blockDim.x) {
    sorted_pair[i] = i;
    ones[i] = 1.0f;
  }
  if (blockIdx.x == 0 && threadIdx.x == 0) {
    const int groups = (T + kGemvGroup - 1) / kGemvGroup, chunks = (T + chunk - 1) / chunk;
    counts[0] = T;
    offsets[0] = 0;
    offsets[1] = T;
    touched[0] = 0;
    group_base[0] = 0;
    group_base[1] = groups;
    tile_base[0] = 0;
    tile_base[1] = chunks;
    meta[0] = 1;
    meta[1] = T;
    meta[2] = groups;
    meta[3] = chunks;
    meta[8] = 0;  // unit counters of the expert GEMMs that follow
    meta[9] = 0;
  }
}

cudaError_t launch_dense_plan(int T, int chunk, int32_t* counts, int32_t* offsets, int32_t* touched,
                              int32_t* group_base, int32_t* tile_base, int32_t* meta, int32_t* sorted_pair,
                              float* ones, cudaStream_t s) {
  int blocks = (T + 255) / 256;
  if (blocks > 148) blocks = 148;
  if (blocks < 1) blocks = 1;
  return launch_k(dense_plan_kernel, dim3(blocks), dim3(256), 0, s, T, chunk, counts, offsets, touched, group_base,
                  tile_base, meta, sorted_pair, ones);
}

cudaError_t launch_pair_scatter(const int32_t* idx, int P, int E, const int32_t* chunk_base, int32_t* sorted_pair,
                                cudaStream_t s) {
  const int NC = (P + kPairChunk - 1) / kPairChunk;
  const int warps = 4;
  return launch_k(pair_scatter_kernel, dim3((NC + warps - 1) / warps), dim3(warps * 32), warps * E * sizeof(int32_t),
                    s, idx, P, E, chunk_base, sorted_pair);
}

}  // namespace moe
