// Weighted combine back to token order: y[t] = sum over slots j (in slot order)
// of Yp[t*k + j], where Yp already holds w_j * FFN_{e_j}(x_t).  fp32 sums in a
// fixed order, one rounding to y's dtype.  The moe op itself adds no residual
// (the add stays outside the op -- Qwen3-30B-A3B LiteRT-LM card, Conversion
// Notes, moe_fusion_guard bullet); the block entry point adds, after the
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

}  // namespace

cudaError_t launch_combine(const moe_desc& d, const int32_t* idx, int T, const float* yp, void* y,
                           cudaStream_t s, const float* ys, const void* residual) {
  const size_t n = (size_t)T * (d.H / 4);
  int blocks = (int)((n + 255) / 256);
  if (blocks > 148 * 16) blocks = 148 * 16;
  if (blocks < 1) blocks = 1;
  const bool extra = ys != nullptr || residual != nullptr;
  if (d.xfmt == MOE_X_BF16) {
    if (extra)
      return launch_k(combine_kernel<true, true>, dim3(blocks), dim3(256), 0, s, idx, T, d.H, d.E, d.k, yp, ys,
                      residual, y);
    return launch_k(combine_kernel<true, false>, dim3(blocks), dim3(256), 0, s, idx, T, d.H, d.E, d.k, yp, ys,
                    residual, y);
  }
  if (extra)
    return launch_k(combine_kernel<false, true>, dim3(blocks), dim3(256), 0, s, idx, T, d.H, d.E, d.k, yp, ys,
                    residual, y);
  return launch_k(combine_kernel<false, false>, dim3(blocks), dim3(256), 0, s, idx, T, d.H, d.E, d.k, yp, ys,
                  residual, y);
}

}  // namespace moe
