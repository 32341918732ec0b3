// Grouped expert GEMMs on the 5th-generation tensor cores (tcgen05 + TMEM + TMA).
//
// "only the 8 routed experts are computed for each token" (Qwen3-30B-A3B
// LiteRT-LM card, Conversion Notes): after the tokens are sorted by expert,
// every expert e owns a contiguous run of m_e rows.  Each unit of work is
// (expert e, block of 128 weight rows, chunk of up to 128 of e's tokens) and
// is computed swap-AB:  D[128 weight rows, N tokens] = W_blk[128, K] * X_e[N, K]^T,
// with M = 128 fixed and N = the chunk's token count rounded up to 16, so a
// ragged expert costs at most 15 padded columns instead of a padded 128-row tile.
//
//   gate/up:  h[pos, i] = SiLU(s_g D_gate[i, pos]) * (s_u D_up[i, pos])       (bf16 out)
//   down:     Yp[pair, r] = w_pair * s_d * D_down[r, pos]                       (fp32 out)
// Storage: bf16 weights go straight from TMA into the 128-byte-swizzled K-major
// layout the tensor core reads; int8 (per-row scale, Kimi-Linear LiteRT-LM
// details page, quantization bullet) is widened exactly to bf16 by dequant
// warps and its row scale applied in the epilogue; int4 block-32 (Qwen3 card,
// Available Artifacts table) is widened to q*s in bf16 by the dequant warps.
//
// Roles in a persistent CTA (one per SM), all on one list of units:
//   warp 0 lane 0   TMA producer (weights or raw quantised tiles, token tile)
//   warp 1          TMEM allocator; lane 0 issues tcgen05.mma
//   warps 4..7      epilogue: TMEM -> registers -> activation/scales -> global
//   warps 8..11     dequantisation (int8 / int4 only)
// Accumulators are double-buffered in TMEM so the epilogue of one unit
// overlaps the MMAs of the next.  Every wait is bounded (MOE_FLAG_TIMEOUT).
#include <cuda.h>

#include "common.cuh"
#include "internal.h"

namespace moe {
namespace {

constexpr int kBM = 128;  // weight rows per unit (MMA M)
constexpr int kBK = 64;   // K per stage (one 128-byte swizzle row of bf16)
constexpr int kMaxN = kTileN;  // tokens per unit
constexpr int kTileBytes = kBM * kBK * 2;  // 16 KB bf16 tile
constexpr int kMaxStages = 8;

struct GemmArgs {
  const float* s0;       // scales of W0 (int8: [E,R]; int4: [E,R,K/32])
  const float* s1;       // scales of W1 (gate/up only)
  const int32_t* offsets;
  const int32_t* touched;
  const int32_t* tile_base;
  const int32_t* meta;
  const int32_t* sorted_pair;
  const float* topk_w;   // down only
  void* out;             // gate/up: hbuf bf16 [P, R]; down: yp fp32 [P, H]
  uint32_t* flags;
  int R;                 // weight rows per expert (I for gate/up, H for down)
  int K;                 // reduction length
  int NS;                // pipeline stages
  int stage_bytes;
};

__device__ __forceinline__ void wait_or_die(uint64_t* bar, uint32_t parity, bool& dead, uint32_t* flags) {
  if (dead) return;
  if (!mbar_wait(bar, parity)) {
    dead = true;
    raise_flag(flags, MOE_FLAG_TIMEOUT);
  }
}

struct Unit {
  int e, base, m, ib, c, n_tok, n_mma;
};

// unit u -> (expert, weight-row block, token chunk); chunks fastest
__device__ __forceinline__ Unit decode_unit(const GemmArgs& a, int u, int nib, int ntouched) {
  int lo = 0, hi = ntouched - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (a.tile_base[mid] * nib <= u) lo = mid;
    else hi = mid - 1;
  }
  Unit t;
  t.e = a.touched[lo];
  t.base = a.offsets[t.e];
  t.m = a.offsets[t.e + 1] - t.base;
  const int nc = (t.m + kMaxN - 1) / kMaxN;
  const int r = u - a.tile_base[lo] * nib;
  t.ib = r / nc;
  t.c = r - t.ib * nc;
  t.n_tok = min(kMaxN, t.m - t.c * kMaxN);
  t.n_mma = (t.n_tok + 15) & ~15;
  return t;
}

// widen one 8-element chunk of a raw quantised row to bf16 (int8: exact q;
// int4: q * block scale, rounded to nearest even)
template <int WF>
__device__ __forceinline__ uint4 widen8(const uint8_t* raw_chunk, float scale) {
  uint4 o;
  if constexpr (WF == MOE_W_INT8_ROW) {
    const uint2 w = *reinterpret_cast<const uint2*>(raw_chunk);
    const uint32_t words[2] = {w.x, w.y};
    uint32_t outw[4];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
#pragma unroll
      for (int b = 0; b < 4; b += 2) {
        // q + 128 in the low mantissa bits of 2^23, minus (2^23 + 128): exact q
        const float f0 = __uint_as_float(0x4B000000u | (((words[h] >> (8 * b)) & 0xFFu) ^ 0x80u)) - 8388736.0f;
        const float f1 = __uint_as_float(0x4B000000u | (((words[h] >> (8 * b + 8)) & 0xFFu) ^ 0x80u)) - 8388736.0f;
        // |q| <= 128 has at most 8 significant bits: the top half of the fp32 is the exact bf16
        outw[h * 2 + b / 2] = __byte_perm(__float_as_uint(f0), __float_as_uint(f1), 0x7632);
      }
    }
    o = make_uint4(outw[0], outw[1], outw[2], outw[3]);
  } else {
    const uint32_t w = *reinterpret_cast<const uint32_t*>(raw_chunk);
    uint32_t outw[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float q0 = __uint_as_float(0x4B000000u | (((w >> (8 * j)) & 0xFu) ^ 0x8u)) - 8388616.0f;
      const float q1 = __uint_as_float(0x4B000000u | (((w >> (8 * j + 4)) & 0xFu) ^ 0x8u)) - 8388616.0f;
      outw[j] = pack_bf16x2(q0 * scale, q1 * scale);
    }
    o = make_uint4(outw[0], outw[1], outw[2], outw[3]);
  }
  return o;
}

template <int MODE, int WF>
struct Layout {
  static constexpr int NMAT = MODE == 0 ? 2 : 1;
  static constexpr bool kQuant = WF != MOE_W_BF16;
  static constexpr int kRawBytes = WF == MOE_W_INT8_ROW ? kBM * kBK : (WF == MOE_W_INT4_B32 ? kBM * kBK / 2 : 0);
  // stage: [A_0 .. A_{NMAT-1}] (bf16 16 KB each) [B tokens 16 KB] [raw_0 .. raw_{NMAT-1}]
  static constexpr int kA = 0;
  static constexpr int kB = NMAT * kTileBytes;
  static constexpr int kRaw = kB + kMaxN * kBK * 2;
  static constexpr int kStage = kRaw + NMAT * kRawBytes;
  static constexpr int kThreads = kQuant ? 384 : 256;
  static constexpr int kAccCols = NMAT * kMaxN;  // TMEM columns per accumulator buffer
  static constexpr int kTmemCols = 2 * kAccCols; // double-buffered (256 or 512)
};

template <int MODE, int WF>
__global__ void __launch_bounds__(Layout<MODE, WF>::kThreads, 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap tm_w0, const __grid_constant__ CUtensorMap tm_w1,
                   const __grid_constant__ CUtensorMap tm_b, const GemmArgs a) {
  using L = Layout<MODE, WF>;
  constexpr int NMAT = L::NMAT;
  extern __shared__ uint8_t smem_raw[];
  // 1024-byte aligned base for the swizzled tiles
  const uint32_t raw_base = smem_u32(smem_raw);
  const uint32_t pad = ((raw_base + 1023u) & ~1023u) - raw_base;
  uint8_t* smem = smem_raw + pad;
  uint8_t* stages = smem + 1024;  // first 1 KB: barriers and the TMEM address
  uint64_t* full = reinterpret_cast<uint64_t*>(smem);       // TMA landed (bf16: A+B; quant: raw+B)
  uint64_t* ready = full + kMaxStages;                      // quant: bf16 A written by dequant warps
  uint64_t* empty = ready + kMaxStages;                     // MMA finished reading the stage
  uint64_t* acc_full = empty + kMaxStages;                  // [2] accumulator complete
  uint64_t* acc_empty = acc_full + 2;                       // [2] epilogue drained the accumulator
  uint64_t* mma_done = acc_empty + 2;                       // final completion of all MMAs
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_done + 1);

  const int w = warp_id(), lane = lane_id();
  const int NS = a.NS;
  if (threadIdx.x == 0) {
    for (int i = 0; i < NS; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&ready[i], 4);
      mbar_init(&empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&acc_full[i], 1);
      mbar_init(&acc_empty[i], 4);
    }
    mbar_init(mma_done, 1);
    fence_mbar_init();
  }
  if (w == 1) tmem_alloc(tmem_slot, L::kTmemCols);
  if (threadIdx.x == 32) {
    prefetch_tmap(&tm_w0);
    if (NMAT == 2) prefetch_tmap(&tm_w1);
    prefetch_tmap(&tm_b);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  const int ntouched = a.meta[0];
  const int nib = a.R / kBM;
  const int total = ntouched > 0 ? a.meta[3] * nib : 0;
  const int nk = a.K / kBK;

  if (w == 0) {
    // ---------------------------------------------------------------- TMA producer
    if (lane == 0) {
      bool dead = false;
      uint32_t it = 0;
      for (int u = blockIdx.x; u < total; u += gridDim.x) {
        const Unit t = decode_unit(a, u, nib, ntouched);
        const int nbox = (t.n_tok + 31) / 32;
        const int brow = t.base + t.c * kMaxN;
        const int wrow = t.e * a.R + t.ib * kBM;
        for (int kb = 0; kb < nk; ++kb, ++it) {
          const int s = it % NS;
          wait_or_die(&empty[s], ((it / NS) & 1u) ^ 1u, dead, a.flags);
          if (dead) continue;
          uint8_t* st = stages + (size_t)s * a.stage_bytes;
          const uint32_t wbytes = L::kQuant ? L::kRawBytes : kTileBytes;
          mbar_arrive_expect_tx(&full[s], NMAT * wbytes + nbox * 32 * kBK * 2);
          // weights: bf16 straight into the swizzled A tile; quantised into the raw area
          const int wcol = WF == MOE_W_INT4_B32 ? kb * kBK / 2 : kb * kBK;  // int4: bytes
          tma_load_2d(L::kQuant ? st + L::kRaw : st + L::kA, &tm_w0, wcol, wrow, &full[s]);
          if (NMAT == 2)
            tma_load_2d(L::kQuant ? st + L::kRaw + L::kRawBytes : st + L::kA + kTileBytes, &tm_w1, wcol, wrow,
                        &full[s]);
          for (int j = 0; j < nbox; ++j) tma_load_2d(st + L::kB + j * 32 * kBK * 2, &tm_b, kb * kBK, brow + 32 * j, &full[s]);
        }
      }
      // stay until the last stages' copies have landed
      const uint32_t first = it > (uint32_t)NS ? it - NS : 0u;
      for (uint32_t j = first; j < it && !dead; ++j) wait_or_die(&full[j % NS], (j / NS) & 1u, dead, a.flags);
    }
  } else if (w == 1) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      bool dead = false;
      uint32_t it = 0, local = 0;
      const uint32_t stage0 = smem_u32(stages);
      for (int u = blockIdx.x; u < total; u += gridDim.x, ++local) {
        const Unit t = decode_unit(a, u, nib, ntouched);
        const uint32_t buf = local & 1u;
        wait_or_die(&acc_empty[buf], ((local >> 1) & 1u) ^ 1u, dead, a.flags);
        tc_fence_after();
        const uint32_t idesc = umma_idesc_bf16(kBM, t.n_mma);
        const uint32_t d0 = tmem_base + buf * L::kAccCols;
        for (int kb = 0; kb < nk; ++kb, ++it) {
          const int s = it % NS;
          const uint32_t par = (it / NS) & 1u;
          wait_or_die(L::kQuant ? &ready[s] : &full[s], par, dead, a.flags);
          if (L::kQuant) wait_or_die(&full[s], par, dead, a.flags);  // token tile landed too
          if (dead) continue;
          tc_fence_after();
          const uint32_t sa = stage0 + s * a.stage_bytes;
#pragma unroll
          for (int k = 0; k < kBK / 16; ++k) {
            const uint64_t bdesc = umma_desc_sw128(sa + L::kB + k * 32);
#pragma unroll
            for (int mtx = 0; mtx < NMAT; ++mtx)
              umma_bf16(d0 + mtx * kMaxN, umma_desc_sw128(sa + L::kA + mtx * kTileBytes + k * 32), bdesc, idesc,
                        (kb | k) != 0);
          }
          umma_commit(&empty[s]);
        }
        if (!dead) umma_commit(&acc_full[buf]);
      }
      if (!dead) {
        umma_commit(mma_done);
        wait_or_die(mma_done, 0, dead, a.flags);
      }
    }
  } else if (w >= 4 && w < 8) {
    // ---------------------------------------------------------------- epilogue
    const int q = w - 4;                // TMEM lanes 32q .. 32q+31
    const int row_in_blk = q * 32 + lane;
    bool dead = false;
    uint32_t local = 0;
    for (int u = blockIdx.x; u < total; u += gridDim.x, ++local) {
      const Unit t = decode_unit(a, u, nib, ntouched);
      const uint32_t buf = local & 1u;
      // one lane waits, the warp follows its verdict (the TMEM loads below are warp-collective)
      if (lane == 0) wait_or_die(&acc_full[buf], (local >> 1) & 1u, dead, a.flags);
      dead = __shfl_sync(0xFFFFFFFFu, dead ? 1 : 0, 0) != 0;
      __syncwarp();
      tc_fence_after();
      if (!dead) {
        const int row = t.ib * kBM + row_in_blk;
        const size_t grow = (size_t)t.e * a.R + row;
        const uint32_t tacc = tmem_base + ((uint32_t)(q * 32) << 16) + buf * L::kAccCols;
        const int pos0 = t.base + t.c * kMaxN;
        if (MODE == 0) {
          const float sg = WF == MOE_W_INT8_ROW ? a.s0[grow] : 1.f;
          const float su = WF == MOE_W_INT8_ROW ? a.s1[grow] : 1.f;
          uint16_t* h = static_cast<uint16_t*>(a.out);
          for (int n0 = 0; n0 < t.n_tok; n0 += 16) {
            uint32_t g[16], v[16];
            tmem_ld16(tacc + n0, g);
            tmem_ld16(tacc + kMaxN + n0, v);
            tmem_ld_wait();
#pragma unroll
            for (int j = 0; j < 16; ++j) {
              if (n0 + j < t.n_tok) {
                const float hv = silu_mul(__uint_as_float(g[j]) * sg, __uint_as_float(v[j]) * su);
                h[(size_t)(pos0 + n0 + j) * a.R + row] = f32_to_bf16(hv);
              }
            }
          }
        } else {
          const float sd = WF == MOE_W_INT8_ROW ? a.s0[grow] : 1.f;
          float* yp = static_cast<float*>(a.out);
          for (int n0 = 0; n0 < t.n_tok; n0 += 16) {
            uint32_t d[16];
            tmem_ld16(tacc + n0, d);
            tmem_ld_wait();
#pragma unroll
            for (int j = 0; j < 16; ++j) {
              if (n0 + j < t.n_tok) {
                const int pair = a.sorted_pair[pos0 + n0 + j];
                yp[(size_t)pair * a.R + row] = a.topk_w[pair] * sd * __uint_as_float(d[j]);
              }
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[buf]);
    }
  } else if (L::kQuant && w >= 8) {
    // ---------------------------------------------------------------- dequantisation
    const int ct = threadIdx.x - 256;  // 0..127
    bool dead = false;
    uint32_t it = 0;
    for (int u = blockIdx.x; u < total; u += gridDim.x) {
      const Unit t = decode_unit(a, u, nib, ntouched);
      for (int kb = 0; kb < nk; ++kb, ++it) {
        const int s = it % NS;
        wait_or_die(&full[s], (it / NS) & 1u, dead, a.flags);
        if (!dead) {
          uint8_t* st = stages + (size_t)s * a.stage_bytes;
#pragma unroll
          for (int mtx = 0; mtx < NMAT; ++mtx) {
            const uint8_t* raw = st + L::kRaw + mtx * L::kRawBytes;
            uint8_t* A = st + L::kA + mtx * kTileBytes;
            const float* S = mtx ? a.s1 : a.s0;
#pragma unroll 2
            for (int i = ct; i < kBM * 8; i += 128) {
              const int r = i >> 3, c8 = i & 7;
              float sc = 1.f;
              if (WF == MOE_W_INT4_B32)
                sc = __ldg(S + ((size_t)t.e * a.R + t.ib * kBM + r) * (a.K / 32) + kb * 2 + (c8 >> 2));
              const int rb = WF == MOE_W_INT8_ROW ? r * kBK + c8 * 8 : r * (kBK / 2) + c8 * 4;
              const uint4 v = widen8<WF>(raw + rb, sc);
              *reinterpret_cast<uint4*>(A + r * 128 + ((c8 ^ (r & 7)) << 4)) = v;
            }
          }
          fence_proxy_async_smem();
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&ready[s]);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (w == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, L::kTmemCols);
  }
}

// ------------------------------------------------------------------ host side

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

// 2-D map over a row-major [rows, cols] matrix; box = [box_cols, box_rows]
cudaError_t make_map(CUtensorMap* m, const void* base, CUtensorMapDataType dt, int elem_bytes, uint64_t cols,
                     uint64_t rows, uint32_t box_cols, uint32_t box_rows, CUtensorMapSwizzle swz) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return cudaErrorNotSupported;
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {cols * elem_bytes};
  const cuuint32_t box[2] = {box_cols, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(m, dt, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swz,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

cudaError_t weight_map(CUtensorMap* m, const void* W, int wfmt, int E, int R, int K) {
  const uint64_t rows = (uint64_t)E * R;
  if (wfmt == MOE_W_BF16)
    return make_map(m, W, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, K, rows, kBK, kBM, CU_TENSOR_MAP_SWIZZLE_128B);
  if (wfmt == MOE_W_INT8_ROW)
    return make_map(m, W, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, K, rows, kBK, kBM, CU_TENSOR_MAP_SWIZZLE_NONE);
  return make_map(m, W, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, K / 2, rows, kBK / 2, kBM, CU_TENSOR_MAP_SWIZZLE_NONE);
}

template <int MODE, int WF>
cudaError_t launch_gemm(const CUtensorMap& m0, const CUtensorMap& m1, const CUtensorMap& mb, GemmArgs a,
                        int num_sms, cudaStream_t s) {
  using L = Layout<MODE, WF>;
  a.stage_bytes = L::kStage;
  const int budget = 232448 - 2048;  // opt-in limit minus barriers and alignment slack
  a.NS = budget / L::kStage;
  if (a.NS > kMaxStages) a.NS = kMaxStages;
  const size_t smem = 2048 + (size_t)a.NS * L::kStage;
  auto kern = gemm_tc_kernel<MODE, WF>;
  cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (err != cudaSuccess) return err;
  kern<<<num_sms, L::kThreads, smem, s>>>(m0, m1, mb, a);
  return cudaGetLastError();
}

template <int MODE>
cudaError_t launch_by_format(int wfmt, const CUtensorMap& m0, const CUtensorMap& m1, const CUtensorMap& mb,
                             const GemmArgs& a, int num_sms, cudaStream_t s) {
  switch (wfmt) {
    case MOE_W_BF16: return launch_gemm<MODE, MOE_W_BF16>(m0, m1, mb, a, num_sms, s);
    case MOE_W_INT8_ROW: return launch_gemm<MODE, MOE_W_INT8_ROW>(m0, m1, mb, a, num_sms, s);
    default: return launch_gemm<MODE, MOE_W_INT4_B32>(m0, m1, mb, a, num_sms, s);
  }
}

GemmArgs common(const Workspace& ws, uint32_t* flags) {
  GemmArgs a{};
  a.offsets = ws.offsets;
  a.touched = ws.touched;
  a.tile_base = ws.tile_base;
  a.meta = ws.meta;
  a.sorted_pair = ws.sorted_pair;
  a.flags = flags;
  return a;
}

__global__ void __launch_bounds__(256) gather_rows_kernel(const uint16_t* __restrict__ x, int H, int k,
                                                          const int32_t* __restrict__ sorted_pair,
                                                          const int32_t* __restrict__ meta, uint16_t* __restrict__ xs) {
  const int P = meta[1];
  const int per_row = H / 8;  // 16-byte chunks
  const size_t n = (size_t)P * per_row;
  for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x) {
    const int pos = (int)(i / per_row), c = (int)(i - (size_t)pos * per_row) * 8;
    const int t = sorted_pair[pos] / k;
    *reinterpret_cast<uint4*>(xs + (size_t)pos * H + c) = *reinterpret_cast<const uint4*>(x + (size_t)t * H + c);
  }
}

}  // namespace

bool gemm_tc_supported(const moe_desc& d) {
  return d.xfmt == MOE_X_BF16 && d.wfmt != MOE_W_F32 && d.H % kBM == 0 && d.I % kBM == 0 && encode_fn() != nullptr;
}

cudaError_t launch_gather_rows(const moe_desc& d, const void* x, const Workspace& ws, int P, int num_sms,
                               cudaStream_t s) {
  const size_t n = (size_t)P * (d.H / 8);
  int blocks = (int)((n + 255) / 256);
  if (blocks > num_sms * 8) blocks = num_sms * 8;
  if (blocks < 1) blocks = 1;
  gather_rows_kernel<<<blocks, 256, 0, s>>>(static_cast<const uint16_t*>(x), d.H, d.k, ws.sorted_pair, ws.meta,
                                            static_cast<uint16_t*>(ws.xs));
  return cudaGetLastError();
}

cudaError_t launch_gemm_gateup(const moe_desc& d, const Workspace& ws, int P, int num_sms, uint32_t* flags,
                               cudaStream_t s) {
  CUtensorMap mg, mu, mb;
  cudaError_t e = weight_map(&mg, d.W_gate, d.wfmt, d.E, d.I, d.H);
  if (e == cudaSuccess) e = weight_map(&mu, d.W_up, d.wfmt, d.E, d.I, d.H);
  if (e == cudaSuccess)
    e = make_map(&mb, ws.xs, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, d.H, (uint64_t)P, kBK, 32, CU_TENSOR_MAP_SWIZZLE_128B);
  if (e != cudaSuccess) return e;
  GemmArgs a = common(ws, flags);
  a.s0 = d.s_gate;
  a.s1 = d.s_up;
  a.out = ws.hbuf;
  a.R = d.I;
  a.K = d.H;
  return launch_by_format<0>(d.wfmt, mg, mu, mb, a, num_sms, s);
}

cudaError_t launch_gemm_down(const moe_desc& d, const float* topk_w, const Workspace& ws, int P, int num_sms,
                             uint32_t* flags, cudaStream_t s) {
  CUtensorMap md, mb;
  cudaError_t e = weight_map(&md, d.W_down, d.wfmt, d.E, d.H, d.I);
  if (e == cudaSuccess)
    e = make_map(&mb, ws.hbuf, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, d.I, (uint64_t)P, kBK, 32,
                 CU_TENSOR_MAP_SWIZZLE_128B);
  if (e != cudaSuccess) return e;
  GemmArgs a = common(ws, flags);
  a.s0 = d.s_down;
  a.topk_w = topk_w;
  a.out = ws.yp;
  a.R = d.H;
  a.K = d.I;
  return launch_by_format<1>(d.wfmt, md, md, mb, a, num_sms, s);
}

}  // namespace moe
