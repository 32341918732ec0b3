// Router of the routed-MoE layer: fp32 logits, sigmoid+selection-bias or
// softmax keys, warp-shuffle top-k, renormalised weights times the scale.
//
// Kimi-Linear: sigmoid scores pick the top 8 after the correction bias is
// added; the chosen scores are renormalised and multiplied by 2.446
// (Kimi-Linear LiteRT-LM details page, Conversion notes).  Qwen3: softmax, top
// 8, renormalisation, all as plain graph ops (Qwen3-30B-A3B LiteRT-LM card,
// Conversion Notes).  Masked experts are never selectable (CMF page, Defrag
// step: runtime expert mask).
//
// Two kernels:
//   router_logits_kernel  tiled SIMT fp32 GEMM, partial[s][t][e] over S splits
//                         of the H reduction (S chosen from T so small batches
//                         still fill the GPU);
//   router_topk_kernel    one warp per token: sums the S partials in a fixed
//                         order, forms keys, selects k by repeated warp argmax
//                         (key descending, expert index ascending), and
//                         renormalises.
#include <math.h>

#include "common.cuh"
#include "internal.h"
#include "route_dev.cuh"

namespace moe {

int router_splits(int T) {
  if (T <= 64) return 8;
  if (T <= 256) return 4;
  if (T <= 2048) return 2;
  return 1;
}

namespace {

constexpr int kBT = 64, kBE = 64, kBK = 32;

template <bool XBF16>
__global__ void __launch_bounds__(256) router_logits_kernel(const void* __restrict__ x,
                                                            const float* __restrict__ Wr, int T, int H,
                                                            int E, int kc, float* __restrict__ partial) {
  pdl_wait();
  pdl_trigger();
  __shared__ __align__(16) float xs[kBK][kBT + 4];
  __shared__ __align__(16) float wsm[kBK][kBE + 4];
  const int t0 = blockIdx.x * kBT, e0 = blockIdx.y * kBE, s = blockIdx.z;
  const int kb = s * kc, ke = min(H, kb + kc);
  const int tid = threadIdx.x;
  const int tx = tid & 15, ty = tid >> 4;  // output micro-tile: experts 4*tx.., tokens 4*ty..
  const int lr = tid & 63, lq = (tid >> 6) * 8;  // loader: row lr, 8 columns from lq
  float acc[4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;

  // global -> registers for the K tile at k0 (zero outside the matrix)
  auto fetch = [&](int k0, float (&xv)[8], float (&wv)[8]) {
    const int t = t0 + lr;
    if (t < T && k0 < ke) {
      if (XBF16) {
        const uint4 v = *reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(x) + (size_t)t * H + k0 + lq);
        const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          xv[2 * j] = bf16_to_f32(u[j] & 0xFFFFu);
          xv[2 * j + 1] = bf16_to_f32(u[j] >> 16);
        }
      } else {
        const float4* p = reinterpret_cast<const float4*>(static_cast<const float*>(x) + (size_t)t * H + k0 + lq);
        const float4 a = p[0], b = p[1];
        xv[0] = a.x; xv[1] = a.y; xv[2] = a.z; xv[3] = a.w;
        xv[4] = b.x; xv[5] = b.y; xv[6] = b.z; xv[7] = b.w;
      }
    } else {
#pragma unroll
      for (int j = 0; j < 8; ++j) xv[j] = 0.f;
    }
    const int e = e0 + lr;
    if (e < E && k0 < ke) {
      const float4* p = reinterpret_cast<const float4*>(Wr + (size_t)e * H + k0 + lq);
      const float4 a = p[0], b = p[1];
      wv[0] = a.x; wv[1] = a.y; wv[2] = a.z; wv[3] = a.w;
      wv[4] = b.x; wv[5] = b.y; wv[6] = b.z; wv[7] = b.w;
    } else {
#pragma unroll
      for (int j = 0; j < 8; ++j) wv[j] = 0.f;
    }
  };
  float xv[8], wv[8];
  fetch(kb, xv, wv);
  for (int k0 = kb; k0 < ke; k0 += kBK) {
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      xs[lq + j][lr] = xv[j];
      wsm[lq + j][lr] = wv[j];
    }
    __syncthreads();
    fetch(k0 + kBK, xv, wv);  // next tile's loads overlap this tile's FMAs
#pragma unroll
    for (int kk = 0; kk < kBK; ++kk) {
      const float4 a = *reinterpret_cast<const float4*>(&xs[kk][ty * 4]);
      const float4 b = *reinterpret_cast<const float4*>(&wsm[kk][tx * 4]);
      const float av[4] = {a.x, a.y, a.z, a.w};
      const float bv[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int t = t0 + ty * 4 + i;
    if (t >= T) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int e = e0 + tx * 4 + j;
      if (e < E) partial[((size_t)s * T + t) * E + e] = acc[i][j];
    }
  }
}

template <int PER_LANE, int S>
__global__ void __launch_bounds__(256) router_topk_kernel(const float* __restrict__ partial, int T,
                                                          int E, int k, int router,
                                                          const float* __restrict__ bias,
                                                          const uint8_t* __restrict__ mask, float scale,
                                                          int32_t* __restrict__ idx, float* __restrict__ wout,
                                                          uint32_t* flags) {
  pdl_wait();
  pdl_trigger();
  const int t = blockIdx.x * (blockDim.x >> 5) + warp_id();
  if (t >= T) return;
  route_dev::warp_topk<PER_LANE, S>(partial, T, t, E, k, router, bias, mask, scale, idx, wout, flags);
}

// logits[t][e] = the S partial sums added in split order from 0.f: the same
// additions, in the same order, as the top-k kernels perform before ranking
__global__ void __launch_bounds__(256) logits_sum_kernel(const float* __restrict__ partial, int S, int T, int E,
                                                         float* __restrict__ logits) {
  pdl_wait();
  pdl_trigger();
  const size_t n = (size_t)T * E;
  for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x) {
    float sum = 0.f;
    for (int s = 0; s < S; ++s) sum += partial[(size_t)s * n + i];
    logits[i] = sum;
  }
}

}  // namespace

cudaError_t launch_logits_sum(const float* partial, int S, int T, int E, float* logits, int num_sms,
                              cudaStream_t s) {
  const size_t n = (size_t)T * E;
  int blocks = (int)((n + 255) / 256);
  if (blocks > num_sms * 8) blocks = num_sms * 8;
  if (blocks < 1) blocks = 1;
  return launch_k(logits_sum_kernel, dim3(blocks), dim3(256), 0, s, partial, S, T, E, logits);
}

cudaError_t launch_router_logits(const moe_desc& d, const void* x, int T, float* partial, int S,
                                 cudaStream_t s) {
  int kc = (d.H + S - 1) / S;
  kc = (kc + kBK - 1) / kBK * kBK;
  dim3 grid((T + kBT - 1) / kBT, (d.E + kBE - 1) / kBE, S);
  if (d.xfmt == MOE_X_BF16)
    return launch_k(router_logits_kernel<true>, grid, dim3(256), 0, s, x, d.W_r, T, d.H, d.E, kc, partial);
  return launch_k(router_logits_kernel<false>, grid, dim3(256), 0, s, x, d.W_r, T, d.H, d.E, kc, partial);
}

cudaError_t launch_router_topk(const moe_desc& d, const float* partial, int S, int T, int32_t* idx,
                               float* w, uint32_t* flags, cudaStream_t s) {
  const int warps = 8;
  dim3 grid((T + warps - 1) / warps);
#define MOE_TOPK(PL, SS)                                                                            \
  return launch_k(router_topk_kernel<PL, SS>, grid, dim3(warps * 32), 0, s, partial, T, d.E, d.k, d.router, \
                    d.b, d.expert_mask, d.scale, idx, w, flags)
  if (d.E <= 256) {
    switch (S) {
      case 1: MOE_TOPK(8, 1); break;
      case 2: MOE_TOPK(8, 2); break;
      case 4: MOE_TOPK(8, 4); break;
      default: MOE_TOPK(8, 8); break;
    }
  } else {
    switch (S) {
      case 1: MOE_TOPK(32, 1); break;
      case 2: MOE_TOPK(32, 2); break;
      case 4: MOE_TOPK(32, 4); break;
      default: MOE_TOPK(32, 8); break;
    }
  }
#undef MOE_TOPK
  return cudaGetLastError();
}

}  // namespace moe
