// Device-side pieces of the routing shared by the kernels that route, sort,
// or do both in one launch: the warp-per-token top-k, the block prefix scans and
// the one-CTA stable counting sort by expert.  Header-only so that every kernel
// runs the same instructions.
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
template <int PER_LANE, int S>
__device__ __forceinline__ void warp_topk(const float* __restrict__ partial, int T, int t, int E, int k, int router,
                                          const float* __restrict__ bias, const uint8_t* __restrict__ mask,
                                          float scale, int32_t* __restrict__ idx, float* __restrict__ wout,
                                          uint32_t* flags) {
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
    wout[(size_t)t * k + lane] = (my_e >= 0 && total > 0.f) ? v / total * scale : 0.f;
  }
}

// Exclusive prefix sums of four values at once over the block (blockDim.x <=
// 1024); the block totals go to *total.
__device__ __forceinline__ int4 block_exclusive_scan4(int4 v, int4* warp_sums4, int4* total) {
  const int lane = lane_id(), w = warp_id(), nw = blockDim.x >> 5;
  int4 incl = v;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int nx = __shfl_up_sync(0xFFFFFFFFu, incl.x, off);
    const int ny = __shfl_up_sync(0xFFFFFFFFu, incl.y, off);
    const int nz = __shfl_up_sync(0xFFFFFFFFu, incl.z, off);
    const int nw4 = __shfl_up_sync(0xFFFFFFFFu, incl.w, off);
    if (lane >= off) {
      incl.x += nx;
      incl.y += ny;
      incl.z += nz;
      incl.w += nw4;
    }
  }
  if (lane == 31) warp_sums4[w] = incl;
  __syncthreads();
  if (w == 0) {
    int4 s = lane < nw ? warp_sums4[lane] : make_int4(0, 0, 0, 0);
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int nx = __shfl_up_sync(0xFFFFFFFFu, s.x, off);
      const int ny = __shfl_up_sync(0xFFFFFFFFu, s.y, off);
      const int nz = __shfl_up_sync(0xFFFFFFFFu, s.z, off);
      const int nw4 = __shfl_up_sync(0xFFFFFFFFu, s.w, off);
      if (lane >= off) {
        s.x += nx;
        s.y += ny;
        s.z += nz;
        s.w += nw4;
      }
    }
    if (lane < nw) warp_sums4[lane] = s;  // inclusive over warps
  }
  __syncthreads();
  const int4 prev = w > 0 ? warp_sums4[w - 1] : make_int4(0, 0, 0, 0);
  *total = warp_sums4[nw - 1];
  __syncthreads();
  return make_int4(prev.x + incl.x - v.x, prev.y + incl.y - v.y, prev.z + incl.z - v.z, prev.w + incl.w - v.w);
}

// Small batches: the whole sort in one CTA of 32 warps.  The P pairs are cut
// into nseg <= 32 contiguous segments of whole 32-pair rounds; warp w < nseg
// owns segment w: it loads its pairs' experts into registers (all loads in
// flight at once), counts them per expert (no atomics: a ballot match groups equal
// experts, the last peer adds), the block turns (segment, expert) counts into
// exclusive bases with one four-way prefix scan, and each warp re-walks its
// segment in order to scatter.  Same stable order as the chunked kernels.
constexpr int kSmallE = 256;
constexpr int kSortWarps = 32;

// The lanes of the warp holding the same value as this lane, for values in
// [-1, kSmallE): nine ballots over the bits of value + 1 (what __match_any_sync
// returns, in a fixed handful of cheap instructions).
__device__ __forceinline__ unsigned match_small(int v) {
  static_assert(kSmallE <= 511, "nine bits");
  const unsigned key = (unsigned)(v + 1);
  unsigned peers = 0xFFFFFFFFu;
#pragma unroll
  for (int b = 0; b < 9; ++b) {
    const bool bit = (key >> b) & 1u;
    const unsigned m = __ballot_sync(0xFFFFFFFFu, bit);
    peers &= bit ? m : ~m;
  }
  return peers;
}
constexpr int kSortRounds = 8;  // 32-pair rounds per segment: P <= kSortWarps * 32 * kSortRounds = 8192

// Called by all threads of a CTA of kSortWarps warps; base and warp_sums are
// shared memory of the caller ([kSortWarps][kSmallE] ints and 4 x 32 ints,
// 16-byte aligned).  P <= 8192, E <= kSmallE.
__device__ __forceinline__ void block_small_sort(const int32_t* idx, int P, int E, int chunk,
                                                 int32_t* __restrict__ counts, int32_t* __restrict__ offsets,
                                                 int32_t* __restrict__ touched, int32_t* __restrict__ group_base,
                                                 int32_t* __restrict__ tile_base, int32_t* __restrict__ meta,
                                                 int32_t* __restrict__ sorted_pair, uint32_t* flags,
                                                 int32_t (*base)[kSmallE], int4* warp_sums4) {
  const int w = warp_id(), lane = lane_id();
  const int rounds = (P + 32 * kSortWarps - 1) / (32 * kSortWarps);  // per segment, <= kSortRounds
  const int seg = 32 * (rounds > 0 ? rounds : 1);
  const int nseg = (P + seg - 1) / seg;
  for (int i = threadIdx.x; i < nseg * kSmallE; i += blockDim.x) (&base[0][0])[i] = 0;
  const int p0 = min(P, w * seg), p1 = min(P, p0 + seg);
  int ev[kSortRounds];
  bool bad = false;
#pragma unroll
  for (int r = 0; r < kSortRounds; ++r) {
    const int p = p0 + 32 * r + lane;
    int e = (r < rounds && p < p1) ? idx[p] : -1;
    if (r < rounds && p < p1 && (e < 0 || e >= E)) bad = true;
    if (e < 0 || e >= E) e = -1;
    ev[r] = e;
  }
  __syncthreads();
  const unsigned lt = (1u << lane) - 1u;
  if (w < nseg) {
#pragma unroll
    for (int r = 0; r < kSortRounds; ++r) {
      if (r < rounds) {
        const int e = ev[r];
        const unsigned peers = match_small(e);
        if (e >= 0 && lane == 31 - __clz(peers)) base[w][e] += __popc(peers);
        __syncwarp();
      }
    }
  }
  if (__any_sync(0xFFFFFFFFu, bad) && lane == 0) raise_flag(flags, MOE_FLAG_BAD_EXPERT_INDEX);
  __syncthreads();
  // per expert: exclusive prefix over segments, then over experts
  const int e = threadIdx.x;
  int running = 0;
  if (e < E) {
    for (int ww = 0; ww < nseg; ++ww) {
      const int v = base[ww][e];
      base[ww][e] = running;
      running += v;
    }
    counts[e] = running;
  }
  const bool live = e < E && running > 0;
  const int4 mine = make_int4(e < E ? running : 0, live ? 1 : 0,
                              e < E ? (running + kGemvGroup - 1) / kGemvGroup : 0,
                              e < E ? (running + chunk - 1) / chunk : 0);
  int4 tot;
  const int4 pos = block_exclusive_scan4(mine, warp_sums4, &tot);
  // pos.x: offset, pos.y: position among touched experts, pos.z: first group, pos.w: first chunk
  if (e < E) {
    offsets[e] = pos.x;
    for (int ww = 0; ww < nseg; ++ww) base[ww][e] += pos.x;
  }
  if (live) {
    touched[pos.y] = e;
    group_base[pos.y] = pos.z;
    tile_base[pos.y] = pos.w;
  }
  if (e == 0) {
    offsets[E] = tot.x;
    meta[0] = tot.y;
    meta[1] = tot.x;
    meta[2] = tot.z;
    meta[3] = tot.w;
    group_base[tot.y] = tot.z;
    tile_base[tot.y] = tot.w;
  }
  __syncthreads();
  if (w < nseg) {
#pragma unroll
    for (int r = 0; r < kSortRounds; ++r) {
      if (r < rounds) {
        const int ee = ev[r];
        const unsigned peers = match_small(ee);
        if (ee >= 0) sorted_pair[base[w][ee] + __popc(peers & lt)] = p0 + 32 * r + lane;
        __syncwarp();
        if (ee >= 0 && lane == 31 - __clz(peers)) base[w][ee] += __popc(peers);
        __syncwarp();
      }
    }
  }
}

}  // namespace route_dev
}  // namespace moe
