// Device-side pieces of the routing shared by the kernels that route, sort,
// or do both in one launch: the warp-per-token top-k, the block prefix scan and
// the single-CTA stable counting sort by expert.  Header-only so that every
// kernel runs the same instructions.
#pragma once
#include <math.h>

#include "common.cuh"
#include "internal.h"

namespace moe {
namespace route_dev {

// exclusive prefix sum over the block (blockDim.x <= 1024); returns the block total in *total
__device__ __forceinline__ int block_exclusive_scan(int v, int* warp_sums, int* total) {
  const int lane = lane_id(), w = warp_id(), nw = blockDim.x >> 5;
  int incl = v;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int n = __shfl_up_sync(0xFFFFFFFFu, incl, off);
    if (lane >= off) incl += n;
  }
  if (lane == 31) warp_sums[w] = incl;
  __syncthreads();
  if (w == 0) {
    int s = lane < nw ? warp_sums[lane] : 0;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int n = __shfl_up_sync(0xFFFFFFFFu, s, off);
      if (lane >= off) s += n;
    }
    if (lane < nw) warp_sums[lane] = s;  // inclusive over warps
  }
  __syncthreads();
  const int before = (w > 0 ? warp_sums[w - 1] : 0) + incl - v;
  *total = warp_sums[nw - 1];
  __syncthreads();
  return before;
}


// (key, expert) ordering: larger key first, then smaller expert index
__device__ __forceinline__ bool better(float ka, int ea, float kb, int eb) {
  return ka > kb || (ka == kb && ea < eb);
}

// Top-k of token t by one warp: sums the S partial logits of every expert in a
// fixed order, forms the keys, selects k by repeated warp argmax (key
// descending, expert index ascending) and writes the renormalised weights.
// idx_copy (optional, e.g. shared memory) receives the selected experts too.
template <int PER_LANE, int S>
__device__ __forceinline__ void warp_topk(const float* __restrict__ partial, int T, int t, int E, int k, int router,
                                          const float* __restrict__ bias, const uint8_t* __restrict__ mask,
                                          float scale, int32_t* __restrict__ idx, float* __restrict__ wout,
                                          uint32_t* flags, int32_t* idx_copy = nullptr) {
  const int lane = lane_id();
  float logit[PER_LANE], key[PER_LANE];
  uint32_t avail = 0;
  bool bad = false;
  // the split sums in a fixed order (split 0 first); one split's loads in flight at a time
  float lsum[PER_LANE];
#pragma unroll
  for (int j = 0; j < PER_LANE; ++j) lsum[j] = 0.f;
#pragma unroll
  for (int s = 0; s < S; ++s) {
    float part[PER_LANE];
#pragma unroll
    for (int j = 0; j < PER_LANE; ++j)
      part[j] = (lane + 32 * j < E) ? partial[((size_t)s * T + t) * E + lane + 32 * j] : 0.f;
#pragma unroll
    for (int j = 0; j < PER_LANE; ++j) lsum[j] += part[j];
  }
#pragma unroll
  for (int j = 0; j < PER_LANE; ++j) {
    const int e = lane + 32 * j;
    logit[j] = 0.f;
    key[j] = -INFINITY;
    if (e < E) {
      const float l = lsum[j];
      logit[j] = l;
      const bool active = (mask == nullptr) || (mask[e] != 0);
      if (!isfinite(l)) {
        bad = true;
      } else if (active) {
        key[j] = (router == MOE_ROUTER_SIGMOID_BIAS) ? sigmoidf_acc(l) + (bias ? bias[e] : 0.f) : l;
        avail |= 1u << j;
      }
    }
  }
  if (__any_sync(0xFFFFFFFFu, bad) && lane == 0) raise_flag(flags, MOE_FLAG_NONFINITE_LOGIT);

  int my_e = -1;
  float my_r = 0.f;
  for (int slot = 0; slot < k; ++slot) {
    float bk = -INFINITY;
    int be = 0x7FFFFFFF;
#pragma unroll
    for (int j = 0; j < PER_LANE; ++j) {
      if ((avail >> j) & 1u) {
        const int e = lane + 32 * j;
        if (better(key[j], e, bk, be)) {
          bk = key[j];
          be = e;
        }
      }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      const float ok = __shfl_xor_sync(0xFFFFFFFFu, bk, off);
      const int oe = __shfl_xor_sync(0xFFFFFFFFu, be, off);
      if (better(ok, oe, bk, be)) {
        bk = ok;
        be = oe;
      }
    }
    const bool found = be != 0x7FFFFFFF;
    float r = 0.f;
    if (found && (be & 31) == lane) {
      const int jj = be >> 5;
#pragma unroll
      for (int j = 0; j < PER_LANE; ++j)
        if (j == jj) {
          r = (router == MOE_ROUTER_SIGMOID_BIAS) ? sigmoidf_acc(logit[j]) : logit[j];
          avail &= ~(1u << j);
        }
    }
    r = __shfl_sync(0xFFFFFFFFu, r, found ? (be & 31) : 0);
    if (lane == slot) {
      my_e = found ? be : -1;
      my_r = r;
    }
    if (!found && lane == 0) raise_flag(flags, MOE_FLAG_TOO_FEW_ACTIVE);
  }
  // renormalise over the chosen slots (softmax: exp relative to the best logit,
  // which the full softmax denominator cancels against)
  const float top = __shfl_sync(0xFFFFFFFFu, my_r, 0);
  float v = 0.f;
  if (lane < k && my_e >= 0) v = (router == MOE_ROUTER_SIGMOID_BIAS) ? my_r : expf(my_r - top);
  float total = v;
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) total += __shfl_xor_sync(0xFFFFFFFFu, total, off);
  if (lane < k) {
    idx[(size_t)t * k + lane] = my_e;
    if (idx_copy) idx_copy[t * k + lane] = my_e;
    wout[(size_t)t * k + lane] = (my_e >= 0 && total > 0.f) ? v / total * scale : 0.f;
  }
}

// Small batches: the whole sort in one CTA of 32 warps.  Warp w owns the
// contiguous pair segment [w*seg, (w+1)*seg): it counts its pairs per expert
// (no atomics: match_any groups equal experts, the last peer adds), the block
// turns (warp, expert) counts into exclusive bases, and each warp re-walks its
// segment in order to scatter.  Same stable order as the chunked kernels.
constexpr int kSmallE = 256;
constexpr int kSortWarps = 32;

// Called by all threads of a CTA of kSortWarps warps; base and warp_sums are
// shared memory of the caller ([kSortWarps][kSmallE] and [32] ints).
__device__ __forceinline__ void block_small_sort(const int32_t* idx, int P, int E, int chunk,
                                                 int32_t* __restrict__ counts, int32_t* __restrict__ offsets,
                                                 int32_t* __restrict__ touched, int32_t* __restrict__ group_base,
                                                 int32_t* __restrict__ tile_base, int32_t* __restrict__ meta,
                                                 int32_t* __restrict__ sorted_pair, uint32_t* flags,
                                                 int32_t (*base)[kSmallE], int* warp_sums) {
  const int w = warp_id(), lane = lane_id();
  for (int i = threadIdx.x; i < kSortWarps * kSmallE; i += blockDim.x) (&base[0][0])[i] = 0;
  __syncthreads();
  const int seg = (P + kSortWarps - 1) / kSortWarps;
  const int p0 = min(P, w * seg), p1 = min(P, p0 + seg);
  const unsigned lt = (1u << lane) - 1u;
  bool bad = false;
  for (int pb = p0; pb < p1; pb += 32) {
    const int p = pb + lane;
    int e = (p < p1) ? idx[p] : -1;
    if (p < p1 && (e < 0 || e >= E)) bad = true;
    if (e < 0 || e >= E) e = -1;
    const unsigned peers = __match_any_sync(0xFFFFFFFFu, e);
    if (e >= 0 && lane == 31 - __clz(peers)) base[w][e] += __popc(peers);
  }
  if (__any_sync(0xFFFFFFFFu, bad) && lane == 0) raise_flag(flags, MOE_FLAG_BAD_EXPERT_INDEX);
  __syncthreads();
  // per expert: exclusive prefix over warps, then over experts
  const int e = threadIdx.x;
  int running = 0;
  if (e < E) {
    for (int ww = 0; ww < kSortWarps; ++ww) {
      const int v = base[ww][e];
      base[ww][e] = running;
      running += v;
    }
    counts[e] = running;
  }
  int total;
  const int off = block_exclusive_scan(e < E ? running : 0, warp_sums, &total);
  if (e < E) {
    offsets[e] = off;
    for (int ww = 0; ww < kSortWarps; ++ww) base[ww][e] += off;
  }
  if (e == 0) offsets[E] = total;
  int ntouched;
  const int tpos = block_exclusive_scan((e < E && running > 0) ? 1 : 0, warp_sums, &ntouched);
  if (e < E && running > 0) touched[tpos] = e;
  const int groups = (e < E) ? (running + kGemvGroup - 1) / kGemvGroup : 0;
  int ngroups;
  const int gpos = block_exclusive_scan(groups, warp_sums, &ngroups);
  if (e < E && running > 0) group_base[tpos] = gpos;
  const int chunks = (e < E) ? (running + chunk - 1) / chunk : 0;
  int nchunks;
  const int cpos = block_exclusive_scan(chunks, warp_sums, &nchunks);
  if (e < E && running > 0) tile_base[tpos] = cpos;
  if (e == 0) {
    meta[0] = ntouched;
    meta[1] = total;
    meta[2] = ngroups;
    meta[3] = nchunks;
    group_base[ntouched] = ngroups;
    tile_base[ntouched] = nchunks;
  }
  __syncthreads();
  for (int pb = p0; pb < p1; pb += 32) {
    const int p = pb + lane;
    int ee = (p < p1) ? idx[p] : -1;
    if (ee < 0 || ee >= E) ee = -1;
    const unsigned peers = __match_any_sync(0xFFFFFFFFu, ee);
    if (ee >= 0) sorted_pair[base[w][ee] + __popc(peers & lt)] = p;
    __syncwarp();
    if (ee >= 0 && lane == 31 - __clz(peers)) base[w][ee] += __popc(peers);
    __syncwarp();
  }
}

}  // namespace route_dev
}  // namespace moe
