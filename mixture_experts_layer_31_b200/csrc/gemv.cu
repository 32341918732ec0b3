// Small-batch expert path: weight-streaming GEMV over the touched experts.
//
// With a few tokens per expert the layer is bound by reading the routed
// experts' weights once from HBM.  Each CTA (one per SM) runs a bulk-copy
// ring: one producer thread streams pieces of weight rows with
// cp.async.bulk into NS shared-memory stages (mbarrier completion, ~160 KB in
// flight per SM), and kCons consumer warps dot them against the expert's
// tokens, staged in shared memory as fp32.  Work items are (touched expert,
// block of RS output rows, group of kG tokens), group fastest so that a
// block's weights are re-read from L2 for an expert's later groups.
//
//   gate/up:  h[pos, i] = SiLU(s_g * <W_gate[e, i], x_t>) * (s_u * <W_up[e, i], x_t>)
//   down:     Yp[pair, r] = w_pair * s_d * <W_down[e, r], h[pos]>
// (SiLU-gated FFN of the routed experts only -- Qwen3-30B-A3B LiteRT-LM card,
// Conversion Notes; int8 per-row and int4 block-32 storage -- Kimi-Linear
// LiteRT-LM details page quantization bullet, Qwen3 card Available Artifacts.)
#include "common.cuh"
#include "internal.h"

namespace moe {
namespace {

constexpr int kCons = 8;                    // consumer warps
constexpr int kThreads = (kCons + 1) * 32;  // + one producer warp
constexpr int kG = kGemvGroup;              // tokens per group
constexpr int kPieceBytes = 1024;           // target bytes of one row piece
constexpr int kMaxStages = 8;
constexpr int kSmemLimit = 232448;          // 227 KB opt-in per CTA
constexpr int kBarrierBytes = 256;

template <int WF>
struct Fmt;
template <>
struct Fmt<MOE_W_F32> { static constexpr int kVec = 4, kBits = 32; };
template <>
struct Fmt<MOE_W_BF16> { static constexpr int kVec = 8, kBits = 16; };
template <>
struct Fmt<MOE_W_INT8_ROW> { static constexpr int kVec = 16, kBits = 8; };
template <>
struct Fmt<MOE_W_INT4_B32> { static constexpr int kVec = 32, kBits = 4; };

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

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, off);
  return v;
}

struct StreamArgs {
  const void* in;  // gate/up: x [T, H]; down: hbuf [P, I]
  const void* W0;  // gate/up: W_gate; down: W_down
  const void* W1;  // gate/up: W_up
  const float* s0;
  const float* s1;
  const int32_t* offsets;
  const int32_t* touched;
  const int32_t* group_base;
  const int32_t* meta;
  const int32_t* sorted_pair;
  const float* topk_w;  // down only
  void* out;            // gate/up: hbuf [P, I]; down: yp [P, H]
  uint32_t* flags;
  int R;          // output rows per expert (I for gate/up, H for down)
  int K;          // reduction length (H for gate/up, I for down)
  int k;          // slots per token
  int KC;         // elements per row piece (multiple of 64)
  int npieces;    // pieces per row
  int NS;         // ring stages
  int pitch;      // bytes per row slot in a stage
  int stage_bytes;
  int xs_off;     // shared-memory offsets
  int ring_off;
  int act;        // gate/up: moe_act
  int qsh;        // int4: log2 of the scale block (5 or 7)
};

// position in the CTA's contiguous range of (touched expert, row block, token group) items
struct Cursor {
  int ti, e, base, m, ng, rb, g;
  __device__ void load(const StreamArgs& a) {
    e = a.touched[ti];
    base = a.offsets[e];
    m = a.offsets[e + 1] - base;
    ng = (m + kG - 1) / kG;
  }
  __device__ void seek(const StreamArgs& a, int u, int nrb, int ntouched) {
    int lo = 0, hi = ntouched - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (a.group_base[mid] * nrb <= u) lo = mid;
      else hi = mid - 1;
    }
    ti = lo;
    load(a);
    const int r = u - a.group_base[ti] * nrb;
    rb = r / ng;
    g = r - rb * ng;
  }
  __device__ void next(const StreamArgs& a, int nrb) {
    if (++g == ng) {
      g = 0;
      if (++rb == nrb) {
        rb = 0;
        ++ti;
        load(a);
      }
    }
  }
};

// acc[q][g] += <row q of the warp's slots, x_g> over one piece; lanes stride
// the piece's 16-byte chunks.  Shared memory is read by 32-bit shared address.
// x is staged planar: for chunk index ci (V elements), float4 j of token g sits
// at xs + g*xrow + j*plane + ci*16 bytes, so a warp's reads are contiguous.
template <int WF, int NW, int GT>
__device__ __forceinline__ void dot_piece(const uint32_t (&rows)[NW], const float* const (&bscale)[NW],
                                          uint32_t xs, int xrow, int plane, int k0, int nch, int qsh,
                                          float (&acc)[NW][kG]) {
  constexpr int V = Fmt<WF>::kVec;
  for (int c = threadIdx.x & 31; c < nch; c += 32) {
    uint4 wv[NW];
#pragma unroll
    for (int q = 0; q < NW; ++q) wv[q] = ld_shared_v4(rows[q] + c * 16);
    const int ci = k0 / V + c;
    const uint32_t xc = xs + ci * 16;
    if constexpr (V <= 16) {
      float wf[NW][V];
#pragma unroll
      for (int q = 0; q < NW; ++q) decode<WF>(wv[q], wf[q]);
#pragma unroll
      for (int g = 0; g < GT; ++g) {
        float xv[V];
#pragma unroll
        for (int j = 0; j < V / 4; ++j) {
          const uint4 t = ld_shared_v4(xc + g * xrow + j * plane);
          xv[4 * j] = __uint_as_float(t.x);
          xv[4 * j + 1] = __uint_as_float(t.y);
          xv[4 * j + 2] = __uint_as_float(t.z);
          xv[4 * j + 3] = __uint_as_float(t.w);
        }
#pragma unroll
        for (int q = 0; q < NW; ++q) {
#pragma unroll
          for (int j = 0; j < V; ++j) acc[q][g] = fmaf(wf[q][j], xv[j], acc[q][g]);
        }
      }
    } else {
      const int kel = k0 + c * V;
#pragma unroll
      for (int q = 0; q < NW; ++q) {
        float wf[V];
        decode<WF>(wv[q], wf);
        const float s = __ldg(bscale[q] + (kel >> qsh));
#pragma unroll
        for (int g = 0; g < GT; ++g) {
          float part = 0.f;
#pragma unroll
          for (int j = 0; j < V / 4; ++j) {
            const uint4 t = ld_shared_v4(xc + g * xrow + j * plane);
            part = fmaf(wf[4 * j], __uint_as_float(t.x), part);
            part = fmaf(wf[4 * j + 1], __uint_as_float(t.y), part);
            part = fmaf(wf[4 * j + 2], __uint_as_float(t.z), part);
            part = fmaf(wf[4 * j + 3], __uint_as_float(t.w), part);
          }
          acc[q][g] = fmaf(s, part, acc[q][g]);
        }
      }
    }
  }
}

// MODE 0: gate/up (2 rows of each matrix per warp); MODE 1: down (4 rows per warp)
template <int MODE, int WF, bool IN_BF16, bool OUT_F32>
__global__ void __launch_bounds__(kThreads, 1) gemv_stream_kernel(const StreamArgs a) {
  pdl_wait();
  pdl_trigger();
  extern __shared__ __align__(128) uint8_t smem[];
  constexpr int NMAT = MODE == 0 ? 2 : 1;
  constexpr int RPW = MODE == 0 ? 2 : 4;
  constexpr int NW = NMAT * RPW;  // weight rows per warp
  constexpr int RS = RPW * kCons;  // output rows per item
  constexpr int kBits = Fmt<WF>::kBits;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem);
  uint64_t* empty = full + kMaxStages;
  float* xs = reinterpret_cast<float*>(smem + a.xs_off);
  uint8_t* ring = smem + a.ring_off;
  const int w = warp_id(), lane = lane_id();

  if (threadIdx.x == 0) {
    for (int i = 0; i < a.NS; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], kCons);
    }
    fence_mbar_init();
  }
  __syncthreads();

  const int ntouched = a.meta[0];
  const int nrb = a.R / RS;
  const int total = a.meta[2] * nrb;
  const int per = (total + gridDim.x - 1) / gridDim.x;
  const int u0 = blockIdx.x * per, u1 = min(total, u0 + per);
  if (u0 >= u1) return;
  const size_t row_bytes = (size_t)a.K * kBits / 8;

  if (w == kCons) {  // ---------------------------------------------------- producer
    if (lane != 0) return;
    Cursor cur;
    cur.seek(a, u0, nrb, ntouched);
    uint32_t it = 0;
    bool dead = false;
    for (int u = u0; u < u1; ++u) {
      for (int p = 0; p < a.npieces; ++p, ++it) {
        const int s = it % a.NS;
        const uint32_t round = it / a.NS;
        if (dead) continue;
        if (!mbar_wait(&empty[s], (round & 1u) ^ 1u)) {
          dead = true;
          raise_flag(a.flags, MOE_FLAG_TIMEOUT);
          continue;
        }
        const int k0 = p * a.KC;
        const uint32_t bytes = (uint32_t)min(a.KC, a.K - k0) * kBits / 8;
        mbar_arrive_expect_tx(&full[s], bytes * NMAT * RS);
        uint8_t* dst = ring + (size_t)s * a.stage_bytes;
#pragma unroll
        for (int mtx = 0; mtx < NMAT; ++mtx) {
          const uint8_t* W = static_cast<const uint8_t*>(mtx ? a.W1 : a.W0);
          const uint8_t* src = W + ((size_t)cur.e * a.R + (size_t)cur.rb * RS) * row_bytes + (size_t)k0 * kBits / 8;
          for (int r = 0; r < RS; ++r) bulk_g2s(dst + (mtx * RS + r) * a.pitch, src + r * row_bytes, bytes, &full[s]);
        }
      }
      if (u + 1 < u1) cur.next(a, nrb);
    }
    // keep this CTA alive until the copies of the last stages have landed
    const uint32_t first = it > (uint32_t)a.NS ? it - a.NS : 0u;
    for (uint32_t j = first; j < it && !dead; ++j)
      if (!mbar_wait(&full[j % a.NS], (j / a.NS) & 1u)) dead = true;
    return;
  }

  // ------------------------------------------------------------------------- consumers
  Cursor cur;
  cur.seek(a, u0, nrb, ntouched);
  uint32_t it = 0;
  bool dead = false;
  int staged_ti = -1, staged_g = -1;
  const int ct = threadIdx.x;  // 0 .. kCons*32-1
  for (int u = u0; u < u1; ++u) {
    const int g0 = cur.g * kG;
    const int G = min(kG, cur.m - g0);
    if (cur.ti != staged_ti || cur.g != staged_g) {
      named_bar_sync(1, kCons * 32);
      const int per_row = a.K / 4;
      for (int i = ct; i < kG * per_row; i += kCons * 32) {
        const int j = i / per_row, c = (i - j * per_row) * 4;
        float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
        if (j < G) {
          const int pos = cur.base + g0 + j;
          const size_t row = MODE == 0 ? (size_t)(a.sorted_pair[pos] / a.k) : (size_t)pos;
          if (IN_BF16) {
            const uint2 b = *reinterpret_cast<const uint2*>(static_cast<const uint16_t*>(a.in) + row * a.K + c);
            v = make_float4(__uint_as_float(b.x << 16), __uint_as_float(b.x & 0xFFFF0000u),
                            __uint_as_float(b.y << 16), __uint_as_float(b.y & 0xFFFF0000u));
          } else {
            v = *reinterpret_cast<const float4*>(static_cast<const float*>(a.in) + row * a.K + c);
          }
        }
        // planar: element c (a multiple of 4) -> plane (c % V) / 4, chunk c / V
        constexpr int V = Fmt<WF>::kVec;
        const int off = j * a.K + ((c % V) / 4) * (a.K / V) * 4 + (c / V) * 4;
        *reinterpret_cast<float4*>(xs + off) = v;
      }
      named_bar_sync(1, kCons * 32);
      staged_ti = cur.ti;
      staged_g = cur.g;
    }
    float acc[NW][kG];
#pragma unroll
    for (int q = 0; q < NW; ++q)
#pragma unroll
      for (int g = 0; g < kG; ++g) acc[q][g] = 0.f;
    const int row0 = cur.rb * RS + w * RPW;  // first output row of this warp
    const float* bsc[NW];
#pragma unroll
    for (int q = 0; q < NW; ++q) {
      const int mtx = q / RPW, rr = q % RPW;
      const float* S = mtx ? a.s1 : a.s0;
      bsc[q] = (WF == MOE_W_INT4_B32) ? S + ((size_t)cur.e * a.R + row0 + rr) * (a.K >> a.qsh) : nullptr;
    }
    for (int p = 0; p < a.npieces; ++p, ++it) {
      const int s = it % a.NS;
      const uint32_t round = it / a.NS;
      if (dead) continue;
      if (!mbar_wait(&full[s], round & 1u)) {
        dead = true;
        if (lane == 0) raise_flag(a.flags, MOE_FLAG_TIMEOUT);
        continue;
      }
      const uint32_t st = smem_u32(ring) + (uint32_t)(s * a.stage_bytes);
      uint32_t rows[NW];
#pragma unroll
      for (int q = 0; q < NW; ++q) rows[q] = st + ((q / RPW) * RS + w * RPW + (q % RPW)) * a.pitch;
      const int k0 = p * a.KC;
      const int nch = min(a.KC, a.K - k0) * kBits / 128;
      const uint32_t xsa = smem_u32(xs);
      const int xrow = a.K * 4, plane = (a.K / Fmt<WF>::kVec) * 16;
      if (G == 1)
        dot_piece<WF, NW, 1>(rows, bsc, xsa, xrow, plane, k0, nch, a.qsh, acc);
      else if (G == 2)
        dot_piece<WF, NW, 2>(rows, bsc, xsa, xrow, plane, k0, nch, a.qsh, acc);
      else
        dot_piece<WF, NW, kG>(rows, bsc, xsa, xrow, plane, k0, nch, a.qsh, acc);
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[s]);
    }
    if (!dead) {
#pragma unroll
      for (int q = 0; q < NW; ++q)
#pragma unroll
        for (int g = 0; g < kG; ++g) acc[q][g] = warp_sum(acc[q][g]);
      // lane (rr, g) writes output row row0 + rr for token g of the group
      if (lane < RPW * kG) {
        const int rr = lane / kG, g = lane % kG;
        if (g < G) {
          const int pos = cur.base + g0 + g;
          const int row = row0 + rr;
          float v = 0.f;
#pragma unroll
          for (int q = 0; q < RPW; ++q)
#pragma unroll
            for (int gg = 0; gg < kG; ++gg)
              if (q == rr && gg == g) {
                if (MODE == 0) {
                  float gv = acc[q][gg], uv = acc[RPW + q][gg];
                  if (WF == MOE_W_INT8_ROW) {
                    gv *= a.s0[(size_t)cur.e * a.R + row];
                    uv *= a.s1[(size_t)cur.e * a.R + row];
                  }
                  v = a.act == MOE_ACT_GELU_TANH ? gelu_tanh_mul(gv, uv) : silu_mul(gv, uv);
                } else {
                  v = acc[q][gg];
                  if (WF == MOE_W_INT8_ROW) v *= a.s0[(size_t)cur.e * a.R + row];
                }
              }
          if (MODE == 0) {
            if (OUT_F32)
              static_cast<float*>(a.out)[(size_t)pos * a.R + row] = v;
            else
              static_cast<uint16_t*>(a.out)[(size_t)pos * a.R + row] = f32_to_bf16(v);
          } else {
            const int pair = a.sorted_pair[pos];
            static_cast<float*>(a.out)[(size_t)pair * a.R + row] = a.topk_w[pair] * v;
          }
        }
      }
    }
    if (u + 1 < u1) cur.next(a, nrb);
  }
}

template <int MODE, int WF>
cudaError_t launch_wf(StreamArgs a, bool in_bf16, bool out_f32, int num_sms, cudaStream_t s) {
  constexpr int NMAT = MODE == 0 ? 2 : 1;
  constexpr int RS = (MODE == 0 ? 2 : 4) * kCons;
  constexpr int kBits = Fmt<WF>::kBits;
  const int per_piece = kPieceBytes * 8 / kBits;
  a.npieces = (a.K + per_piece - 1) / per_piece;
  a.KC = ((a.K + a.npieces - 1) / a.npieces + 63) / 64 * 64;
  a.npieces = (a.K + a.KC - 1) / a.KC;
  a.pitch = a.KC * kBits / 8;
  a.stage_bytes = NMAT * RS * a.pitch;
  a.xs_off = kBarrierBytes;
  a.ring_off = (kBarrierBytes + kG * a.K * 4 + 127) / 128 * 128;
  a.NS = (kSmemLimit - a.ring_off) / a.stage_bytes;
  if (a.NS > kMaxStages) a.NS = kMaxStages;
  if (a.NS < 2) return cudaErrorInvalidConfiguration;
  const size_t smem = (size_t)a.ring_off + (size_t)a.NS * a.stage_bytes;
  auto kern = in_bf16 ? (out_f32 ? gemv_stream_kernel<MODE, WF, true, true> : gemv_stream_kernel<MODE, WF, true, false>)
                      : (out_f32 ? gemv_stream_kernel<MODE, WF, false, true> : gemv_stream_kernel<MODE, WF, false, false>);
  cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (err != cudaSuccess) return err;
  return launch_k(kern, dim3(num_sms), dim3(kThreads), smem, s, a);
}

template <int MODE>
cudaError_t launch_mode(const moe_desc& d, const StreamArgs& a, bool in_bf16, bool out_f32, int num_sms,
                        cudaStream_t s) {
  switch (d.wfmt) {
    case MOE_W_F32: return launch_wf<MODE, MOE_W_F32>(a, in_bf16, out_f32, num_sms, s);
    case MOE_W_BF16: return launch_wf<MODE, MOE_W_BF16>(a, in_bf16, out_f32, num_sms, s);
    case MOE_W_INT8_ROW: return launch_wf<MODE, MOE_W_INT8_ROW>(a, in_bf16, out_f32, num_sms, s);
    default: return launch_wf<MODE, MOE_W_INT4_B32>(a, in_bf16, out_f32, num_sms, s);
  }
}

StreamArgs common_args(const moe_desc& d, const Workspace& ws, int k, uint32_t* flags) {
  StreamArgs a{};
  a.act = d.act;
  a.qsh = d.wfmt == MOE_W_INT4_B128 ? 7 : 5;
  a.offsets = ws.offsets;
  a.touched = ws.touched;
  a.group_base = ws.group_base;
  a.meta = ws.meta;
  a.sorted_pair = ws.sorted_pair;
  a.k = k;
  a.flags = flags;
  return a;
}

}  // namespace

// h is fp32 when the weights are fp32 (the fp32 layer stays fp32 end to end), bf16 otherwise
static bool h_is_f32(const moe_desc& d) { return d.wfmt == MOE_W_F32; }

cudaError_t launch_gemv_gateup(const moe_desc& d, const void* x, int k, const Workspace& ws, int num_sms,
                               uint32_t* flags, cudaStream_t s) {
  StreamArgs a = common_args(d, ws, k, flags);
  a.in = x;
  a.W0 = d.W_gate;
  a.W1 = d.W_up;
  a.s0 = d.s_gate;
  a.s1 = d.s_up;
  a.out = ws.hbuf;
  a.R = d.I;
  a.K = d.H;
  return launch_mode<0>(d, a, d.xfmt == MOE_X_BF16, h_is_f32(d), num_sms, s);
}

cudaError_t launch_gemv_down(const moe_desc& d, const float* topk_w, int k, const Workspace& ws, int num_sms,
                             uint32_t* flags, cudaStream_t s) {
  StreamArgs a = common_args(d, ws, k, flags);
  a.in = ws.hbuf;
  a.W0 = d.W_down;
  a.s0 = d.s_down;
  a.topk_w = topk_w;
  a.out = ws.yp;
  a.R = d.H;
  a.K = d.I;
  return launch_mode<1>(d, a, !h_is_f32(d), true, num_sms, s);
}

}  // namespace moe
