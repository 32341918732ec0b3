// Weighted combine back to token order: y[t] = sum over slots j (in slot order)
// of Yp[t*k + j], where Yp already holds w_j * FFN_{e_j}(x_t) (fp32, or bf16 for
// large bf16 batches).  fp32 sums in a fixed order, one rounding to y's dtype.
// The moe op itself adds no residual (the add stays outside the op --
// Qwen3-30B-A3B LiteRT-LM card, Conversion Notes, moe_fusion_guard bullet);
// the block entry point adds, after the
// routed slots, the shared expert's rows Ys[t] and then the residual stream,
// still before the one rounding.  Slots with an out-of-range expert index
// (only possible with caller-provided routing) contribute nothing.
#include "common.cuh"
#include "internal.h"

namespace moe {
namespace {

template <bool OUT_BF16, bool EXTRA>
__global__ void __launch_bounds__(256) combine_kernel(const int32_t* __restrict__ idx, int T, int H, int E,
                                                      int k, const float* __restrict__ yp,
                                                      const float* __restrict__ ys, const void* res, void* y) {
  pdl_wait();
  pdl_trigger();
  // res and y may alias (an in-place residual update): each element is read,
  // then written, by the same thread
  const int h4 = H / 4;
  const size_t n = (size_t)T * h4;
  for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x) {
    const int t = (int)(i / h4), c = (int)(i - (size_t)t * h4) * 4;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int j = 0; j < k; ++j) {
      const int e = idx[(size_t)t * k + j];
      if (e < 0 || e >= E) continue;
      const float4 v = *reinterpret_cast<const float4*>(yp + ((size_t)t * k + j) * H + c);
      acc.x += v.x;
      acc.y += v.y;
      acc.z += v.z;
      acc.w += v.w;
    }
    if (EXTRA) {
      // the block's remaining terms, in this order: shared expert, then residual
      if (ys) {
        const float4 v = *reinterpret_cast<const float4*>(ys + (size_t)t * H + c);
        acc.x += v.x;
        acc.y += v.y;
        acc.z += v.z;
        acc.w += v.w;
      }
      if (res) {
        float r[4];
        if (OUT_BF16) {
          const uint2 u = *reinterpret_cast<const uint2*>(static_cast<const uint16_t*>(res) + (size_t)t * H + c);
          r[0] = bf16_to_f32(u.x & 0xFFFFu);
          r[1] = bf16_to_f32(u.x >> 16);
          r[2] = bf16_to_f32(u.y & 0xFFFFu);
          r[3] = bf16_to_f32(u.y >> 16);
        } else {
          const float4 u = *reinterpret_cast<const float4*>(static_cast<const float*>(res) + (size_t)t * H + c);
          r[0] = u.x;
          r[1] = u.y;
          r[2] = u.z;
          r[3] = u.w;
        }
        acc.x += r[0];
        acc.y += r[1];
        acc.z += r[2];
        acc.w += r[3];
      }
    }
    if (OUT_BF16) {
      uint2 o;
      o.x = pack_bf16x2(acc.x, acc.y);
      o.y = pack_bf16x2(acc.z, acc.w);
      *reinterpret_cast<uint2*>(static_cast<uint16_t*>(y) + (size_t)t * H + c) = o;
    } else {
      *reinterpret_cast<float4*>(static_cast<float*>(y) + (size_t)t * H + c) = acc;
    }
  }
}

// bf16 per-pair outputs (and so bf16 x and y): eight columns per thread, 16-byte
// loads and stores; the same sums in the same order as above.
__device__ __forceinline__ void add_bf16x8(float (&acc)[8], const uint4 u) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    acc[2 * i] += bf16_to_f32(w[i] & 0xFFFFu);
    acc[2 * i + 1] += bf16_to_f32(w[i] >> 16);
  }
}

template <bool EXTRA>
__global__ void __launch_bounds__(256) combine_bf16_kernel(const int32_t* __restrict__ idx, int T, int H, int E,
                                                           int k, const uint16_t* __restrict__ yp,
                                                           const float* __restrict__ ys, const void* res, void* y) {
  pdl_wait();
  pdl_trigger();
  const int h8 = H / 8;
  const size_t n = (size_t)T * h8;
  for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x) {
    const int t = (int)(i / h8), c = (int)(i - (size_t)t * h8) * 8;
    float acc[8];
#pragma unroll
    for (int q = 0; q < 8; ++q) acc[q] = 0.f;
    for (int j = 0; j < k; ++j) {
      const int e = idx[(size_t)t * k + j];
      if (e < 0 || e >= E) continue;
      add_bf16x8(acc, *reinterpret_cast<const uint4*>(yp + ((size_t)t * k + j) * H + c));
    }
    if (EXTRA) {
      if (ys) {
        const float4 a = *reinterpret_cast<const float4*>(ys + (size_t)t * H + c);
        const float4 b = *reinterpret_cast<const float4*>(ys + (size_t)t * H + c + 4);
        acc[0] += a.x;
        acc[1] += a.y;
        acc[2] += a.z;
        acc[3] += a.w;
        acc[4] += b.x;
        acc[5] += b.y;
        acc[6] += b.z;
        acc[7] += b.w;
      }
      if (res) add_bf16x8(acc, *reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(res) + (size_t)t * H + c));
    }
    uint4 o;
    o.x = pack_bf16x2(acc[0], acc[1]);
    o.y = pack_bf16x2(acc[2], acc[3]);
    o.z = pack_bf16x2(acc[4], acc[5]);
    o.w = pack_bf16x2(acc[6], acc[7]);
    *reinterpret_cast<uint4*>(static_cast<uint16_t*>(y) + (size_t)t * H + c) = o;
  }
}

}  // namespace

template <bool OUT_BF16, bool EXTRA>
cudaError_t launch_combine_t(const moe_desc& d, const int32_t* idx, int T, const void* yp, bool yp_bf16, void* y,
                             int blocks, cudaStream_t s, const float* ys, const void* residual) {
  if (yp_bf16) {  // bf16 x, so y and the residual are bf16 too
    if (!OUT_BF16 || d.H % 8 != 0) return cudaErrorInvalidValue;
    const size_t n8 = (size_t)T * (d.H / 8);
    int b8 = (int)((n8 + 255) / 256);
    if (b8 > blocks) b8 = blocks;
    if (b8 < 1) b8 = 1;
    return launch_k(combine_bf16_kernel<EXTRA>, dim3(b8), dim3(256), 0, s, idx, T, d.H, d.E, d.k,
                    static_cast<const uint16_t*>(yp), ys, residual, y);
  }
  return launch_k(combine_kernel<OUT_BF16, EXTRA>, dim3(blocks), dim3(256), 0, s, idx, T, d.H, d.E, d.k,
                  static_cast<const float*>(yp), ys, residual, y);
}

cudaError_t launch_combine(const moe_desc& d, const int32_t* idx, int T, const void* yp, bool yp_bf16, void* y,
                           cudaStream_t s, const float* ys, const void* residual) {
  const size_t n = (size_t)T * (d.H / 4);
  int blocks = (int)((n + 255) / 256);
  if (blocks > 148 * 16) blocks = 148 * 16;
  if (blocks < 1) blocks = 1;
  const bool extra = ys != nullptr || residual != nullptr;
  if (d.xfmt == MOE_X_BF16)
    return extra ? launch_combine_t<true, true>(d, idx, T, yp, yp_bf16, y, blocks, s, ys, residual)
                 : launch_combine_t<true, false>(d, idx, T, yp, yp_bf16, y, blocks, s, ys, residual);
  return extra ? launch_combine_t<false, true>(d, idx, T, yp, yp_bf16, y, blocks, s, ys, residual)
               : launch_combine_t<false, false>(d, idx, T, yp, yp_bf16, y, blocks, s, ys, residual);
}

}  // namespace moe
