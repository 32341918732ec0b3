// Router and expert sort for decode-sized batches, fused to two launches.
//
// The router is the Kimi-Linear one: sigmoid scores, top 8 on score plus
// correction bias, chosen scores renormalised and scaled by 2.446 (Kimi-Linear
// LiteRT-LM details page, Conversion notes).  The sort groups the (token, slot)
// pairs by expert so that each expert's weights stream once; a token runs only
// through its routed experts (Qwen3-30B-A3B LiteRT-LM card, Conversion Notes).
//
//   decode_logits_kernel  fp32 partial logits [S, T, E] straight from fp32
//                         W_r (S from 1 to 8: about 128 CTAs, and a slice of
//                         x and W_r that fits in shared memory): a CTA owns one S-th of H for
//                         8 experts, stages that slice in shared memory (all
//                         loads in flight at once), and its 8 warps split the
//                         slice's K range, each lane holding a 2-expert x
//                         4-token register tile; warps are added in a fixed
//                         order, and the top-k adds the S slices in a fixed
//                         order.  Every sum's order depends on H (and T) only,
//                         so a masked layer and its sliced twin get the same
//                         logits bit for bit.  T <= 32.
//   topk_sort_kernel      one CTA per token: its top-k (one warp); the CTA that
//                         finishes last then runs the stable counting sort by
//                         expert of all T*k pairs -- the same device code as the
//                         standalone kernels, without the launch in between.
#include "common.cuh"
#include "internal.h"
#include "route_dev.cuh"

namespace moe {
namespace {

// decode logits: CTA (slice sl of S along H, group of kGroupE experts); the
// slice of x (bf16 or fp32 as given, T rows) and of W_r (fp32, kGroupE rows)
// is bulk-copied into shared memory; 8 warps split the slice's K range, every
// lane owns a 2-expert x 4-token register tile (rows of experts past E hold
// stale shared memory: their sums are never stored).  S (1..8) spreads the
// work over about 128 CTAs and keeps the slice within shared memory.
constexpr int kGroupE = 8;       // experts per CTA
constexpr int kMaxDecodeT = 32;  // tokens
constexpr int kLogitWarps = 8;
constexpr int kLogitThreads = 32 * kLogitWarps;
constexpr int kRedFloats = kLogitWarps * kGroupE * kMaxDecodeT;
constexpr size_t kLogitSmemCap = 232448 - 64;  // 227 KB opt-in, less the static barrier

template <bool XBF16>
__host__ __device__ constexpr int x_elem_bytes() { return XBF16 ? 2 : 4; }

template <bool XBF16>
__global__ void __launch_bounds__(kLogitThreads) decode_logits_kernel(const void* __restrict__ x,
                                                                      const float* __restrict__ Wr, int T, int H,
                                                                      int E, int S, float* __restrict__ partial,
                                                                      int32_t* __restrict__ topk_done, uint32_t* flags) {
  pdl_wait();
  pdl_trigger();
  extern __shared__ __align__(16) uint8_t smb[];
  // the fused top-k launch that follows counts its finished CTAs from zero
  if (topk_done != nullptr && blockIdx.x == 0 && threadIdx.x == 0) *topk_done = 0;
  __shared__ __align__(8) uint64_t staged;
  const int len = H / S;                        // a multiple of 8
  const int sl = blockIdx.x % S, g = blockIdx.x / S;
  const int h0 = sl * len, e0 = g * kGroupE;
  const int ne = min(kGroupE, E - e0);          // experts of this CTA
  const int xpitch = len + 8;                   // elements; rows 16-byte aligned, banks staggered
  const int wpitch = len + 4;                   // floats
  float* red = reinterpret_cast<float*>(smb);   // [kLogitWarps][kGroupE][kMaxDecodeT]
  float* ws = red + kRedFloats;                 // [kGroupE][wpitch]; rows past ne unused
  uint8_t* xs = reinterpret_cast<uint8_t*>(ws + kGroupE * wpitch);  // [T][xpitch] of x's type
  constexpr int eb = x_elem_bytes<XBF16>();
  // stage the slice with one bulk copy per row, all in flight at once (rows are
  // contiguous; every address 16-byte aligned and every size a multiple of 16:
  // H % 64 == 0 and the pitches are multiples of 8 elements)
  if (threadIdx.x == 0) {
    mbar_init(&staged, 1);
    fence_mbar_init();
    mbar_arrive_expect_tx(&staged, (uint32_t)(T * len * eb + ne * len * 4));
    for (int t = 0; t < T; ++t)
      bulk_g2s(xs + (size_t)t * xpitch * eb, static_cast<const uint8_t*>(x) + ((size_t)t * H + h0) * eb,
               (uint32_t)(len * eb), &staged);
    for (int el = 0; el < ne; ++el)
      bulk_g2s(ws + (size_t)el * wpitch, Wr + (size_t)(e0 + el) * H + h0, (uint32_t)(len * 4), &staged);
  }
  __syncthreads();  // the barrier is initialised before anyone waits on it
  if (!mbar_wait(&staged, 0)) {
    if (threadIdx.x == 0) raise_flag(flags, MOE_FLAG_TIMEOUT);
    return;
  }
  __syncthreads();
  // lane tile: experts 2*(lane%4) .. +1, tokens 4*(lane/4) .. +3 (rows past T are
  // never read: their sums stay zero and are not stored); warp w takes the K
  // steps of 4 with index = w mod kLogitWarps, in ascending order
  const int w = warp_id(), lane = lane_id();
  const int ea = 2 * (lane % 4), ta = 4 * (lane / 4);
  float acc[2][4];
#pragma unroll
  for (int i = 0; i < 2; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;
  for (int c = 4 * w; c < len; c += 4 * kLogitWarps) {
    float4 wv[2];
#pragma unroll
    for (int i = 0; i < 2; ++i) wv[i] = *reinterpret_cast<const float4*>(ws + (ea + i) * wpitch + c);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      if (ta + j < T) {
        float xv[4];
        if (XBF16) {
          const uint2 u = *reinterpret_cast<const uint2*>(xs + ((size_t)(ta + j) * xpitch + c) * 2);
          xv[0] = bf16_to_f32(u.x & 0xFFFFu);
          xv[1] = bf16_to_f32(u.x >> 16);
          xv[2] = bf16_to_f32(u.y & 0xFFFFu);
          xv[3] = bf16_to_f32(u.y >> 16);
        } else {
          const float4 u = *reinterpret_cast<const float4*>(xs + ((size_t)(ta + j) * xpitch + c) * 4);
          xv[0] = u.x; xv[1] = u.y; xv[2] = u.z; xv[3] = u.w;
        }
#pragma unroll
        for (int i = 0; i < 2; ++i) {
          acc[i][j] = fmaf(wv[i].x, xv[0], acc[i][j]);
          acc[i][j] = fmaf(wv[i].y, xv[1], acc[i][j]);
          acc[i][j] = fmaf(wv[i].z, xv[2], acc[i][j]);
          acc[i][j] = fmaf(wv[i].w, xv[3], acc[i][j]);
        }
      }
    }
  }
#pragma unroll
  for (int i = 0; i < 2; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) red[w * (kGroupE * kMaxDecodeT) + (ea + i) * kMaxDecodeT + ta + j] = acc[i][j];
  __syncthreads();
  // warps in a fixed order -> partial[sl][t][e]
  for (int i = threadIdx.x; i < kGroupE * kMaxDecodeT; i += blockDim.x) {
    const int el = i / kMaxDecodeT, t = i % kMaxDecodeT, e = e0 + el;
    if (t < T && e < E) {
      float sum = 0.f;
#pragma unroll
      for (int ww = 0; ww < kLogitWarps; ++ww) sum += red[ww * (kGroupE * kMaxDecodeT) + i];
      partial[((size_t)sl * T + t) * E + e] = sum;
    }
  }
}

// One CTA of 1024 threads per token:
//   A  the CTA sums its token's S partial logits of every expert in the split
//      order (split 0 first, as the standalone top-k does) into shared memory
//      and forms the keys (the same expressions as the standalone top-k);
//   B  every selectable expert's rank among the selectable keys (key
//      descending, expert index ascending -- the order in which the standalone
//      top-k's repeated argmax picks them) is counted by four threads over a
//      quarter of the experts each; ranks below k are the slots.  Warp 0 then
//      renormalises exactly as the standalone top-k does (same values, same
//      lanes, same butterfly), so the routing is bit for bit the same;
//   C  the CTA that finishes last (a completion counter, zeroed by the logits
//      kernel before this launch) reads every token's routing back and runs the
//      stable counting sort, then re-arms the counter.
// No CTA waits for another: the last one to arrive does the sort.
// The logits and the sort's per-warp bases share one buffer (never live together).
constexpr int kFusedMaxT = 32, kFusedMaxE = 256, kFusedMaxK = 32;

template <int PER_LANE, int S>  // 32 * PER_LANE experts at most; S partial sums per logit
__global__ void __launch_bounds__(1024) topk_sort_kernel(const float* __restrict__ partial, int T, int E, int k,
                                                         int router, const float* __restrict__ bias,
                                                         const uint8_t* __restrict__ mask, float scale,
                                                         int32_t* __restrict__ idx, float* __restrict__ wout,
                                                         int chunk, int32_t* __restrict__ counts,
                                                         int32_t* __restrict__ offsets, int32_t* __restrict__ touched,
                                                         int32_t* __restrict__ group_base,
                                                         int32_t* __restrict__ tile_base, int32_t* __restrict__ meta,
                                                         int32_t* __restrict__ sorted_pair, int32_t* done,
                                                         uint32_t* flags) {
  pdl_wait();
  pdl_trigger();
  static_assert(kFusedMaxT * kFusedMaxE == route_dev::kSortWarps * route_dev::kSmallE, "shared buffer sizes");
  static_assert(32 * PER_LANE >= kFusedMaxE, "experts per launch");
  __shared__ __align__(16) int32_t buf[route_dev::kSortWarps][route_dev::kSmallE];  // logits, then sort bases
  __shared__ int32_t idx_s[kFusedMaxT * kFusedMaxK];
  __shared__ int4 warp_sums4[32];
  __shared__ int sel_e[kFusedMaxE];     // selectable flags, then nothing
  __shared__ int slot_e[kFusedMaxK];    // expert of each slot
  __shared__ float slot_r[kFusedMaxK];  // its router value (sigmoid or logit)
  __shared__ int last;
  float* logits = reinterpret_cast<float*>(&buf[0][0]);  // [E] of this CTA's token
  float* keys = logits + kFusedMaxE;                      // [E], -inf where not selectable
  int32_t* rank_part = &buf[2][0];                        // [4][E] partial ranks
  const int t = blockIdx.x;
  const int tid = threadIdx.x;
  // A
  bool bad = false;
  if (tid < E) {
    float p[S];
#pragma unroll
    for (int s = 0; s < S; ++s) p[s] = partial[((size_t)s * T + t) * E + tid];
    float sum = 0.f;
#pragma unroll
    for (int s = 0; s < S; ++s) sum += p[s];
    logits[tid] = sum;
    const bool active = (mask == nullptr) || (mask[tid] != 0);
    float key = -INFINITY;
    if (!isfinite(sum)) {
      bad = true;
    } else if (active) {
      key = (router == MOE_ROUTER_SIGMOID_BIAS) ? sigmoidf_acc(sum) + (bias ? bias[tid] : 0.f) : sum;
    }
    keys[tid] = key;
    // selectable: active, finite logit, and a key that compares (a NaN bias makes
    // a key the standalone top-k can never pick)
    sel_e[tid] = active && !bad && key == key ? 1 : 0;
  }
  const int nsel = __syncthreads_count(tid < E && sel_e[tid] != 0);
  if (__syncthreads_or(bad) && tid == 0) raise_flag(flags, MOE_FLAG_NONFINITE_LOGIT);
  // B: partial ranks, four threads per expert
  {
    const int e = tid & (kFusedMaxE - 1), q = tid / kFusedMaxE;  // q in 0..3
    if (e < E) {
      int r = 0;
      if (sel_e[e]) {
        const float ke = keys[e];
        const int lo = q * (kFusedMaxE / 4), hi = min(E, lo + kFusedMaxE / 4);
        for (int j = lo; j < hi; ++j) r += (sel_e[j] && route_dev::better(keys[j], j, ke, e)) ? 1 : 0;
      }
      rank_part[q * kFusedMaxE + e] = r;
    }
  }
  __syncthreads();
  int slot = -1;
  if (tid < E && sel_e[tid]) {
    const int r = rank_part[tid] + rank_part[kFusedMaxE + tid] + rank_part[2 * kFusedMaxE + tid] +
                  rank_part[3 * kFusedMaxE + tid];
    if (r < k) slot = r;
  }
  __syncthreads();  // every thread has read the selectable flags
  if (slot >= 0) {
    slot_e[slot] = tid;
    slot_r[slot] = (router == MOE_ROUTER_SIGMOID_BIAS) ? sigmoidf_acc(logits[tid]) : logits[tid];
  }
  __syncthreads();
  if (warp_id() == 0) {
    const int lane = lane_id();
    int my_e = -1;
    float my_r = 0.f;
    if (lane < k && lane < nsel) {
      my_e = slot_e[lane];
      my_r = slot_r[lane];
    }
    if (nsel < k && lane == 0) raise_flag(flags, MOE_FLAG_TOO_FEW_ACTIVE);
    // renormalise over the chosen slots (softmax: exp relative to the best logit)
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
    __threadfence();  // this token's routing is visible device-wide before the count below
  }
  __syncthreads();
  if (threadIdx.x == 0) last = atomicAdd(done, 1) == (int)gridDim.x - 1;
  __syncthreads();
  if (!last) return;
  // C (the last CTA): every other CTA's routing is visible once its count is
  __threadfence();
  for (int i = threadIdx.x; i < T * k; i += blockDim.x) idx_s[i] = __ldcg(idx + i);
  __syncthreads();
  route_dev::block_small_sort(idx_s, T * k, E, chunk, counts, offsets, touched, group_base, tile_base, meta,
                              sorted_pair, flags, buf, warp_sums4);
  if (threadIdx.x == 0) *done = 0;
}

}  // namespace

bool decode_route_ok(const moe_desc& d, int T) { return T >= 1 && T <= 32; }

bool fused_route_sort_ok(const moe_desc& d, int T) {
  return decode_route_ok(d, T) && T <= kFusedMaxT && d.E <= kFusedMaxE && d.k <= kFusedMaxK &&
         small_sort_ok(T * d.k, d.E);
}

static size_t decode_logits_smem(int H, int T, int S, bool xbf16) {
  const int len = H / S;
  return sizeof(float) * ((size_t)kRedFloats + (size_t)kGroupE * (len + 4)) + (size_t)T * (len + 8) * (xbf16 ? 2 : 4);
}

// power-of-two split of H: enough CTAs to spread the W_r stream and the FMAs
// over most of the SMs (S x E/8 >= 128), and a slice that fits in shared
// memory; at most 8 (the top-k templates stop there; 8 fits every H <= 8192
// at T <= 32)
int decode_logit_splits(const moe_desc& d, int T) {
  const int groups = (d.E + kGroupE - 1) / kGroupE;
  int S = 1;
  while (S < 8 && (S * groups < 128 || decode_logits_smem(d.H, T, S, d.xfmt == MOE_X_BF16) > kLogitSmemCap))
    S *= 2;
  return S;
}

cudaError_t launch_decode_logits(const moe_desc& d, const void* x, int T, float* partial, int S, uint32_t* flags,
                                 cudaStream_t s, int32_t* topk_done) {
  const dim3 grid(S * ((d.E + kGroupE - 1) / kGroupE));
  const bool xb = d.xfmt == MOE_X_BF16;
  const size_t smem = decode_logits_smem(d.H, T, S, xb);
  auto kern = xb ? decode_logits_kernel<true> : decode_logits_kernel<false>;
  cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (err != cudaSuccess) return err;
  return launch_k(kern, grid, dim3(kLogitThreads), smem, s, x, d.W_r, T, d.H, d.E, S, partial, topk_done, flags);
}

cudaError_t launch_topk_sort(const moe_desc& d, const float* partial, int S, int T, int32_t* idx, float* w,
                             int chunk, const Workspace& ws, uint32_t* flags, cudaStream_t s) {
#define MOE_TOPK_SORT(SS)                                                                                      \
  return launch_k(topk_sort_kernel<8, SS>, dim3(T), dim3(1024), 0, s, partial, T, d.E, d.k, d.router, d.b,     \
                  d.expert_mask, d.scale, idx, w, chunk, ws.counts, ws.offsets, ws.touched, ws.group_base,    \
                  ws.tile_base, ws.meta, ws.sorted_pair, ws.meta + kMetaTopkDone, flags)
  switch (S) {
    case 1: MOE_TOPK_SORT(1);
    case 2: MOE_TOPK_SORT(2);
    case 4: MOE_TOPK_SORT(4);
    default: MOE_TOPK_SORT(8);
  }
#undef MOE_TOPK_SORT
}

}  // namespace moe
