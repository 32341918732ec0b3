// Small-batch expert path: weight-streaming GEMV over the touched experts.
//
// With a few tokens per expert the layer is bound by reading the routed
// experts' weights once from HBM.  Work is (touched expert, block of output
// rows); every CTA of a persistent grid walks a contiguous range of those
// items.  Each warp streams whole weight rows with 16-byte non-allocating
// loads (several in flight per lane), dots them against the expert's tokens
// staged in shared memory as fp32, and finishes with a warp butterfly sum.
//
//   gate/up:  h[pos, i] = SiLU(s_g * <W_gate[e, i], x_t>) * (s_u * <W_up[e, i], x_t>)
//   down:     Yp[pair, r] = w_pair * s_d * <W_down[e, r], h[pos]>
// (SiLU-gated expert FFN of the routed experts only -- Qwen3-30B-A3B LiteRT-LM
// card, Conversion Notes; int8 per-row and int4 block-32 storage -- Kimi
// details page quantization bullet, Qwen3 card Available Artifacts table.)
#include "common.cuh"
#include "internal.h"

namespace moe {
namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kMaxG = 4;  // tokens per pass over a weight block

// elements per 16-byte chunk of a weight row
template <int WF>
struct Fmt;
template <>
struct Fmt<MOE_W_F32> { static constexpr int kVec = 4; };
template <>
struct Fmt<MOE_W_BF16> { static constexpr int kVec = 8; };
template <>
struct Fmt<MOE_W_INT8_ROW> { static constexpr int kVec = 16; };
template <>
struct Fmt<MOE_W_INT4_B32> { static constexpr int kVec = 32; };

template <int WF>
__device__ __forceinline__ void decode(const uint4& v, float* f) {
  const uint32_t u[4] = {v.x, v.y, v.z, v.w};
  if constexpr (WF == MOE_W_F32) {
#pragma unroll
    for (int j = 0; j < 4; ++j) f[j] = __uint_as_float(u[j]);
  } else if constexpr (WF == MOE_W_BF16) {
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      f[2 * j] = __uint_as_float(u[j] << 16);
      f[2 * j + 1] = __uint_as_float(u[j] & 0xFFFF0000u);
    }
  } else if constexpr (WF == MOE_W_INT8_ROW) {
#pragma unroll
    for (int j = 0; j < 4; ++j)
#pragma unroll
      for (int b = 0; b < 4; ++b) f[4 * j + b] = (float)((int32_t)(u[j] << (24 - 8 * b)) >> 24);
  } else {
#pragma unroll
    for (int j = 0; j < 4; ++j)
#pragma unroll
      for (int n = 0; n < 8; ++n) f[8 * j + n] = (float)((int32_t)(u[j] << (28 - 4 * n)) >> 28);
  }
}

// bytes of one weight row of length K
template <int WF>
__device__ __forceinline__ size_t row_bytes(int K) {
  if constexpr (WF == MOE_W_F32) return (size_t)K * 4;
  else if constexpr (WF == MOE_W_BF16) return (size_t)K * 2;
  else if constexpr (WF == MOE_W_INT8_ROW) return (size_t)K;
  else return (size_t)K / 2;
}

// acc[r][g] += <row r, xs[g]> over K, lanes striding 16-byte chunks.
// int4: the block-32 scale of chunk c (one chunk == one block) multiplies the
// chunk's partial sum.
template <int WF, int NR, int G>
__device__ __forceinline__ void dot_rows(const uint8_t* const (&rows)[NR], const float* const (&bscale)[NR],
                                         const float* __restrict__ xs, int K, float (&acc)[NR][kMaxG]) {
  constexpr int V = Fmt<WF>::kVec;
  const int nch = K / V;
  const int lane = lane_id();
  for (int c = lane; c < nch; c += 64) {
    uint4 wv[2][NR];
    const bool second = c + 32 < nch;
#pragma unroll
    for (int r = 0; r < NR; ++r) {
      wv[0][r] = ldg_stream(rows[r] + (size_t)c * 16);
      if (second) wv[1][r] = ldg_stream(rows[r] + (size_t)(c + 32) * 16);
    }
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      if (u == 1 && !second) break;
      const int cc = c + 32 * u;
      if constexpr (V <= 16) {
        // decode every row once, then read each token's x chunk once
        float wf[NR][V];
#pragma unroll
        for (int r = 0; r < NR; ++r) decode<WF>(wv[u][r], wf[r]);
#pragma unroll
        for (int g = 0; g < G; ++g) {
          const float4* xp = reinterpret_cast<const float4*>(xs + (size_t)g * K + (size_t)cc * V);
          float xv[V];
#pragma unroll
          for (int j = 0; j < V / 4; ++j) {
            const float4 q = xp[j];
            xv[4 * j] = q.x;
            xv[4 * j + 1] = q.y;
            xv[4 * j + 2] = q.z;
            xv[4 * j + 3] = q.w;
          }
#pragma unroll
          for (int r = 0; r < NR; ++r) {
            float part = 0.f;
#pragma unroll
            for (int j = 0; j < V; ++j) part = fmaf(wf[r][j], xv[j], part);
            acc[r][g] += part;
          }
        }
      } else {
#pragma unroll
        for (int r = 0; r < NR; ++r) {
          float wf[V];
          decode<WF>(wv[u][r], wf);
          const float s = bscale[r][cc];
#pragma unroll
          for (int g = 0; g < G; ++g) {
            const float4* xp = reinterpret_cast<const float4*>(xs + (size_t)g * K + (size_t)cc * V);
            float part = 0.f;
#pragma unroll
            for (int j = 0; j < V / 4; ++j) {
              const float4 xv = xp[j];
              part = fmaf(wf[4 * j], xv.x, part);
              part = fmaf(wf[4 * j + 1], xv.y, part);
              part = fmaf(wf[4 * j + 2], xv.z, part);
              part = fmaf(wf[4 * j + 3], xv.w, part);
            }
            acc[r][g] = fmaf(s, part, acc[r][g]);
          }
        }
      }
    }
  }
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, off);
  return v;
}

// stage g rows of the input into xs[g][0..K) as fp32
template <bool IN_BF16>
__device__ __forceinline__ void stage_rows(float* xs, const void* src, const int64_t* row_index, int g, int K) {
  const int per_row = K / 4;  // float4 / 4-element groups
  for (int i = threadIdx.x; i < g * per_row; i += blockDim.x) {
    const int r = i / per_row, c = (i - r * per_row) * 4;
    float4 v;
    if (IN_BF16) {
      const uint2 b = *reinterpret_cast<const uint2*>(static_cast<const uint16_t*>(src) + row_index[r] * K + c);
      v = make_float4(__uint_as_float(b.x << 16), __uint_as_float(b.x & 0xFFFF0000u), __uint_as_float(b.y << 16),
                      __uint_as_float(b.y & 0xFFFF0000u));
    } else {
      v = *reinterpret_cast<const float4*>(static_cast<const float*>(src) + row_index[r] * K + c);
    }
    *reinterpret_cast<float4*>(xs + (size_t)r * K + c) = v;
  }
}

struct GemvArgs {
  const void* in;        // gate/up: x [T, H]; down: hbuf [P, I]
  const void* W0;        // gate/up: W_gate; down: W_down
  const void* W1;        // gate/up: W_up
  const float* s0;
  const float* s1;
  const int32_t* offsets;
  const int32_t* touched;
  const int32_t* meta;
  const int32_t* sorted_pair;
  const float* topk_w;   // down only
  void* out;             // gate/up: hbuf [P, I]; down: yp [P, H]
  int R;                 // output rows per expert (I for gate/up, H for down)
  int K;                 // reduction length (H for gate/up, I for down)
  int k;                 // slots per token
};

// MODE 0: gate/up (2 rows of each matrix per warp); MODE 1: down (4 rows per warp)
template <int MODE, int WF, bool IN_BF16, bool OUT_F32>
__global__ void __launch_bounds__(kThreads) gemv_kernel(const GemvArgs a) {
  extern __shared__ __align__(16) float xs[];  // [kMaxG][K]
  __shared__ int64_t row_index[kMaxG];
  constexpr int NR = 4;
  constexpr int RPW = MODE == 0 ? 2 : 4;  // output rows per warp
  constexpr int RB = RPW * kWarps;         // output rows per item
  const int K = a.K, R = a.R;
  const int nblk = R / RB;
  const int n_items = a.meta[0] * nblk;
  const int per = (n_items + gridDim.x - 1) / gridDim.x;
  const int i0 = blockIdx.x * per, i1 = min(n_items, i0 + per);
  const int w = warp_id(), lane = lane_id();
  const size_t rbytes = row_bytes<WF>(K);
  int staged_e = -1, staged_g0 = -1;

  for (int it = i0; it < i1; ++it) {
    const int e = a.touched[it / nblk];
    const int rb = it - (it / nblk) * nblk;
    const int base = a.offsets[e], m = a.offsets[e + 1] - base;
    const int row0 = rb * RB + w * RPW;
    const uint8_t* rows[NR];
    const float* bsc[NR];
#pragma unroll
    for (int r = 0; r < NR; ++r) {
      const int row = MODE == 0 ? row0 + (r >> 1) : row0 + r;
      const void* W = (MODE == 0 && (r & 1)) ? a.W1 : a.W0;
      const float* S = (MODE == 0 && (r & 1)) ? a.s1 : a.s0;
      const size_t grow = (size_t)e * R + row;
      rows[r] = static_cast<const uint8_t*>(W) + grow * rbytes;
      bsc[r] = (WF == MOE_W_INT4_B32) ? S + grow * (K / 32) : nullptr;
    }
    for (int g0 = 0; g0 < m; g0 += kMaxG) {
      const int G = min(kMaxG, m - g0);
      if (staged_e != e || staged_g0 != g0) {
        __syncthreads();
        if (threadIdx.x < G) {
          const int pos = base + g0 + threadIdx.x;
          row_index[threadIdx.x] = MODE == 0 ? (int64_t)(a.sorted_pair[pos] / a.k) : (int64_t)pos;
        }
        __syncthreads();
        stage_rows<IN_BF16>(xs, a.in, row_index, G, K);
        __syncthreads();
        staged_e = e;
        staged_g0 = g0;
      }
      float acc[NR][kMaxG];
#pragma unroll
      for (int r = 0; r < NR; ++r)
#pragma unroll
        for (int g = 0; g < kMaxG; ++g) acc[r][g] = 0.f;
      if (G == 1)
        dot_rows<WF, NR, 1>(rows, bsc, xs, K, acc);
      else if (G == 2)
        dot_rows<WF, NR, 2>(rows, bsc, xs, K, acc);
      else
        dot_rows<WF, NR, kMaxG>(rows, bsc, xs, K, acc);
#pragma unroll
      for (int r = 0; r < NR; ++r)
#pragma unroll
        for (int g = 0; g < kMaxG; ++g)
          if (g < G) acc[r][g] = warp_sum(acc[r][g]);
      // lane (r', g) writes output row r' for token g
      if (lane < RPW * kMaxG) {
        const int rr = lane / kMaxG, g = lane % kMaxG;
        if (g < G) {
          const int pos = base + g0 + g;
          float v = 0.f;
#pragma unroll
          for (int q = 0; q < RPW; ++q)
#pragma unroll
            for (int gg = 0; gg < kMaxG; ++gg)
              if (q == rr && gg == g) {
                if (MODE == 0) {
                  float gv = acc[2 * q][gg], uv = acc[2 * q + 1][gg];
                  if (WF == MOE_W_INT8_ROW) {
                    gv *= a.s0[(size_t)e * R + row0 + q];
                    uv *= a.s1[(size_t)e * R + row0 + q];
                  }
                  v = silu_mul(gv, uv);
                } else {
                  v = acc[q][gg];
                  if (WF == MOE_W_INT8_ROW) v *= a.s0[(size_t)e * R + row0 + q];
                }
              }
          const int row = row0 + rr;
          if (MODE == 0) {
            if (OUT_F32)
              static_cast<float*>(a.out)[(size_t)pos * R + row] = v;
            else
              static_cast<uint16_t*>(a.out)[(size_t)pos * R + row] = f32_to_bf16(v);
          } else {
            const int pair = a.sorted_pair[pos];
            static_cast<float*>(a.out)[(size_t)pair * R + row] = a.topk_w[pair] * v;
          }
        }
      }
    }
  }
}

template <int MODE, int WF>
cudaError_t launch_wf(const GemvArgs& a, bool in_bf16, bool out_f32, int num_sms, cudaStream_t s) {
  const size_t smem = (size_t)kMaxG * a.K * sizeof(float);
  auto pick = [&]() {
    if (in_bf16) return out_f32 ? gemv_kernel<MODE, WF, true, true> : gemv_kernel<MODE, WF, true, false>;
    return out_f32 ? gemv_kernel<MODE, WF, false, true> : gemv_kernel<MODE, WF, false, false>;
  };
  auto kern = pick();
  cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (err != cudaSuccess) return err;
  int per_sm = 0;
  err = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kThreads, smem);
  if (err != cudaSuccess) return err;
  if (per_sm < 1) per_sm = 1;
  kern<<<num_sms * per_sm, kThreads, smem, s>>>(a);
  return cudaGetLastError();
}

template <int MODE>
cudaError_t launch_mode(const moe_desc& d, const GemvArgs& a, bool in_bf16, bool out_f32, int num_sms,
                        cudaStream_t s) {
  switch (d.wfmt) {
    case MOE_W_F32: return launch_wf<MODE, MOE_W_F32>(a, in_bf16, out_f32, num_sms, s);
    case MOE_W_BF16: return launch_wf<MODE, MOE_W_BF16>(a, in_bf16, out_f32, num_sms, s);
    case MOE_W_INT8_ROW: return launch_wf<MODE, MOE_W_INT8_ROW>(a, in_bf16, out_f32, num_sms, s);
    default: return launch_wf<MODE, MOE_W_INT4_B32>(a, in_bf16, out_f32, num_sms, s);
  }
}

}  // namespace

// h is fp32 when the weights are fp32 (the fp32 layer stays fp32 end to end), bf16 otherwise
static bool h_is_f32(const moe_desc& d) { return d.wfmt == MOE_W_F32; }

cudaError_t launch_gemv_gateup(const moe_desc& d, const void* x, int k, const Workspace& ws, int num_sms,
                               cudaStream_t s) {
  GemvArgs a{};
  a.in = x;
  a.W0 = d.W_gate;
  a.W1 = d.W_up;
  a.s0 = d.s_gate;
  a.s1 = d.s_up;
  a.offsets = ws.offsets;
  a.touched = ws.touched;
  a.meta = ws.meta;
  a.sorted_pair = ws.sorted_pair;
  a.out = ws.hbuf;
  a.R = d.I;
  a.K = d.H;
  a.k = k;
  return launch_mode<0>(d, a, d.xfmt == MOE_X_BF16, h_is_f32(d), num_sms, s);
}

cudaError_t launch_gemv_down(const moe_desc& d, const float* topk_w, int k, const Workspace& ws, int num_sms,
                             cudaStream_t s) {
  GemvArgs a{};
  a.in = ws.hbuf;
  a.W0 = d.W_down;
  a.s0 = d.s_down;
  a.offsets = ws.offsets;
  a.touched = ws.touched;
  a.meta = ws.meta;
  a.sorted_pair = ws.sorted_pair;
  a.topk_w = topk_w;
  a.out = ws.yp;
  a.R = d.H;
  a.K = d.I;
  a.k = k;
  return launch_mode<1>(d, a, !h_is_f32(d), true, num_sms, s);
}

}  // namespace moe
