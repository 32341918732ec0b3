// Weighted combine back to token order: y[t] = sum over slots j (in slot order)
// of Yp[t*k + j], where Yp already holds w_j * FFN_{e_j}(x_t).  fp32 sums in a
// fixed order, one rounding to y's dtype; no residual add (the add stays
// outside the moe op -- Qwen3-30B-A3B LiteRT-LM card, Conversion Notes,
// moe_fusion_guard bullet).  Slots with an out-of-range expert index (only
// possible with caller-provided routing) contribute nothing.
#include "common.cuh"
#include "internal.h"

namespace moe {
namespace {

template <bool OUT_BF16>
__global__ void __launch_bounds__(256) combine_kernel(const int32_t* __restrict__ idx, int T, int H, int E,
                                                      int k, const float* __restrict__ yp, void* __restrict__ y) {
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
                           cudaStream_t s) {
  const size_t n = (size_t)T * (d.H / 4);
  int blocks = (int)((n + 255) / 256);
  if (blocks > 148 * 16) blocks = 148 * 16;
  if (blocks < 1) blocks = 1;
  if (d.xfmt == MOE_X_BF16)
    return launch_k(combine_kernel<true>, dim3(blocks), dim3(256), 0, s, idx, T, d.H, d.E, d.k, yp, y);
  return launch_k(combine_kernel<false>, dim3(blocks), dim3(256), 0, s, idx, T, d.H, d.E, d.k, yp, y);
}

}  // namespace moe
