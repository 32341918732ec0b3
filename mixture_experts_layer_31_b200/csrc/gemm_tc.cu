// Grouped expert GEMMs on the 5th-generation tensor cores (tcgen05 + TMEM + TMA).
//
// A token runs only through its 8 routed experts (Qwen3-30B-A3B LiteRT-LM
// card, Conversion Notes): after the tokens are sorted by expert,
// every expert e owns a contiguous run of m_e rows.  A unit of work is
// (expert e, block of output rows, chunk of up to `chunk` of e's tokens),
// computed swap-AB:  D[128 weight rows, N tokens] = A[128, K] * X_e[N, K]^T,
// M = 128 and N = the chunk's token count rounded up to 16 (<= 256), so a
// ragged expert pays at most 15 padded columns.
//
//   gate/up: M tile 0 = 128 rows of W_gate, M tile 1 = the same rows of W_up,
//            both against one token tile, so TMEM lane i holds both projections
//            of output row i:  h[pos, i] = SiLU(s_g D0[i, pos]) * (s_u D1[i, pos])
//   down:    1 or 2 M tiles of 128 W_down rows;  Yp[pair, r] = w_pair * s_d * D[r, pos]
//            (Yp in fp32, or bf16 when the launch asks for it: large bf16 batches)
// Storage: bf16 weights go straight from TMA into the 128-byte-swizzled
// K-major layout the tensor core reads; int8 rows (one scale per row and
// expert -- Kimi-Linear LiteRT-LM details, quantization bullet) are widened
// exactly to bf16 by dequant warps and scaled in the epilogue; int4 block-32
// (Qwen3 card, Available Artifacts table) is widened to q*s in bf16.
//
// Roles in a persistent CTA (one per SM), all walking one list of units that
// warp 0 lane 0 claims from a per-launch counter and publishes, decoded, through
// a small shared-memory queue:
//   warp 0 lane 0   scheduler and TMA producer: bf16 weight tiles and token boxes
//                   into one stage ring; quantised weights: raw tiles into their own ring
//   warp 1          TMEM allocator; lane 0 issues tcgen05.mma, commits stages
//   warp 2 lane 0   quantised weights only: TMA producer of the token boxes
//   warps 4..11     epilogue (two 4-warp groups): tcgen05.ld -> activation / scales -> global
//   warps 12..19    dequantisation (int8 / int4 only): one weight row per thread,
//                   widened to bf16 into a shared-memory A ring or, where that
//                   measured faster, into TMEM (the MMA then reads A from TMEM)
// Quantised weights keep two rings so that a raw tile's slot is refilled as
// soon as the dequant warps have widened it, not when the MMAs that use its
// bf16 copy finish: the weight stream runs as many stages ahead as the raw
// ring holds, while the token ring only needs to cover L2 latency.
// TMEM holds two accumulator buffers when they fit (with A in shared memory:
// chunks up to 128 tokens), so the epilogue of one unit overlaps the MMAs of the
// next; launch_gemm lays out the accumulators and widened A stages.  Every wait
// is bounded (MOE_FLAG_TIMEOUT).
// A launch may carry a second, dense problem (the shared expert of the MoE
// block: every token in order, weight 1, weights of its own) whose units follow
// the routed ones, so both share the persistent grid.
// The router's logits reuse the kernel as a third mode (MODE 2): dense
// x . W3^T over K splits, W3 the exact three-way bf16 split of the fp32 router
// weights.
// No cluster, no multicast.
#include <cuda.h>

#include "common.cuh"
#include "internal.h"

namespace moe {
namespace {

constexpr int kBM = 128;                   // MMA M (weight rows per tile)
constexpr int kBK = 64;                    // K per stage: one 128-byte swizzle row of bf16
constexpr int kTileBytes = kBM * kBK * 2;  // A tile, 16 KB
constexpr int kBoxRows = 32;               // token rows per TMA box
constexpr int kMaxStages = 16;
constexpr int kAStages = 2;                // quantised: bf16 A tiles between dequant and MMA
constexpr int kBarrierBytes = 2048;          // barriers, the unit queue, the TMEM address
constexpr int kUnitQ = 8;                  // expert GEMMs: unit ids in flight between the scheduler and the roles
constexpr int kSmemLimit = 232448;         // 227 KB opt-in

struct GemmArgs {
  const float* s0;  // scales of W0 (int8: [E,R]; int4: [E,R,K >> qsh])
  const float* s1;  // scales of W1 (gate/up)
  const int32_t* offsets;
  const int32_t* touched;
  const int32_t* tile_base;
  const int32_t* meta;
  const int32_t* sorted_pair;
  const float* topk_w;  // down only
  void* out;            // gate/up: hbuf bf16 [P, I]; down: yp fp32 [P, H]
  uint32_t* flags;
  int R;                // weight rows per expert and matrix (I for gate/up, H for down)
  int K;                // reduction length
  int chunk;            // tokens per chunk (multiple of 16, <= 256)
  int NS;               // stages of the main ring (bf16: A and B; quantised: B only)
  int stage_bytes;
  int b_off;            // B tile offset within a stage
  int RS;               // quantised: stages of the raw weight ring
  int raw_stage_bytes;  // quantised: bytes of one raw stage (MT raw tiles)
  int raw_ring_off;     // quantised: raw ring offset from the main ring's start
  int acc_stride;       // TMEM columns per M tile accumulator (power of two >= chunk)
  int nbuf;             // accumulator buffers (2: epilogue overlaps the next unit's MMAs)
  int tmem_cols;        // TMEM columns allocated
  int a_col0;           // quantised, A in TMEM: first TMEM column of the widened A stages
  int a_stride;         // and the TMEM columns from one A stage to the next
  // router logits (MODE 2): dense [T, E] = x [T, H] . W3 [E, 3H]^T over S splits of the K steps
  int T;
  int S;
  int Hx;               // columns of x (the K coordinate of x is taken modulo Hx)
  int act;              // gate/up: moe_act (SiLU or tanh-GELU)
  int out_bf16;         // down: the routed problem's per-pair outputs in bf16 (else fp32)
  int qsh;              // int4: log2 of the scale block (5: 32 columns, 7: 128)
  // optional second, dense problem in the same launch (the shared expert): every
  // one of Td tokens in token order with weight 1, expert 0 of weights with Rd rows
  // and Kd columns; its units follow the routed ones
  int dense_units;      // 0: none
  int Rd, Kd, Td, chunkd;
  const float* sd0;
  const float* sd1;
  void* outd;           // gate/up: h [Td, Rd] bf16; down: rows [Td, Rd] fp32
  // expert GEMMs: units past the first one of each CTA are claimed from this
  // counter (zeroed by the kernel that runs before the launch), so CTAs whose
  // units are cheap take more of them
  int* sched;
};

__device__ __forceinline__ void wait_or_die(uint64_t* bar, uint32_t parity, bool& dead, uint32_t* flags) {
  if (dead) return;
  if (!mbar_wait(bar, parity)) {
    dead = true;
    raise_flag(flags, MOE_FLAG_TIMEOUT);
  }
}

struct Unit {
  int e, base, ib, c, n_tok, n_mma;
  int k0, nk;  // K steps [k0, k0 + nk)
  int pos0;    // first sorted position (dense: first token) of the unit's chunk
  bool dense;  // a unit of the dense problem
};

// barriers [4 rings x kMaxStages, 2 x kAStages, acc_full/acc_empty x 2, mma_done,
// q_full/q_empty x kUnitQ], the unit queue (ids and decoded units), the TMEM address
static_assert((4 * kMaxStages + 2 * kAStages + 5 + 2 * kUnitQ) * 8 + kUnitQ * (4 + (int)sizeof(Unit)) + 4 <=
                  kBarrierBytes,
              "barrier region too small");

// The per-problem view a role needs for a unit.
struct ProbView {
  int R, K;
  const float* s0;
  const float* s1;
  void* out;
};

__device__ __forceinline__ ProbView view_of(const GemmArgs& a, const Unit& t) {
  if (t.dense) return ProbView{a.Rd, a.Kd, a.sd0, a.sd1, a.outd};
  return ProbView{a.R, a.K, a.s0, a.s1, a.out};
}

// units of the expert GEMMs (MODE 0/1): (expert, output-row block, token chunk),
// chunks fastest; of the router GEMM (MODE 2): (token chunk, expert block, K split)
template <int MODE>
__device__ __forceinline__ Unit decode_unit(const GemmArgs& a, int u, int nib, int ntouched, int routed) {
  Unit t;
  const int nk_all = a.K / kBK;
  t.dense = false;
  if (MODE != 2 && u >= routed) {
    // dense problem: (row block, token chunk), chunks fastest
    const int v = u - routed;
    const int nc = (a.Td + a.chunkd - 1) / a.chunkd;
    t.dense = true;
    t.e = 0;
    t.base = 0;
    t.ib = v / nc;
    t.c = v - t.ib * nc;
    t.pos0 = t.c * a.chunkd;
    t.n_tok = min(a.chunkd, a.Td - t.pos0);
    t.n_mma = (t.n_tok + 15) & ~15;
    t.k0 = 0;
    t.nk = a.Kd / kBK;
    return t;
  }
  if (MODE == 2) {
    const int s = u % a.S, r = u / a.S;
    t.ib = r % nib;
    t.c = s;
    t.e = 0;
    t.base = (r / nib) * a.chunk;
    t.n_tok = min(a.chunk, a.T - t.base);
    t.n_mma = (t.n_tok + 15) & ~15;
    t.k0 = s * nk_all / a.S;
    t.nk = (s + 1) * nk_all / a.S - t.k0;
    t.pos0 = t.base;
    return t;
  }
  int lo = 0, hi = ntouched - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (a.tile_base[mid] * nib <= u) lo = mid;
    else hi = mid - 1;
  }
  t.e = a.touched[lo];
  t.base = a.offsets[t.e];
  const int m = a.offsets[t.e + 1] - t.base;
  const int nc = (m + a.chunk - 1) / a.chunk;
  const int r = u - a.tile_base[lo] * nib;
  t.ib = r / nc;
  t.c = r - t.ib * nc;
  t.n_tok = min(a.chunk, m - t.c * a.chunk);
  t.n_mma = (t.n_tok + 15) & ~15;
  t.k0 = 0;
  t.nk = nk_all;
  t.pos0 = t.base + t.c * a.chunk;
  return t;
}

// lane 0's unit to the whole warp
__device__ __forceinline__ void shfl_unit(Unit& t) {
  t.e = __shfl_sync(0xFFFFFFFFu, t.e, 0);
  t.base = __shfl_sync(0xFFFFFFFFu, t.base, 0);
  t.ib = __shfl_sync(0xFFFFFFFFu, t.ib, 0);
  t.c = __shfl_sync(0xFFFFFFFFu, t.c, 0);
  t.n_tok = __shfl_sync(0xFFFFFFFFu, t.n_tok, 0);
  t.n_mma = __shfl_sync(0xFFFFFFFFu, t.n_mma, 0);
  t.k0 = __shfl_sync(0xFFFFFFFFu, t.k0, 0);
  t.nk = __shfl_sync(0xFFFFFFFFu, t.nk, 0);
  t.pos0 = __shfl_sync(0xFFFFFFFFu, t.pos0, 0);
  t.dense = __shfl_sync(0xFFFFFFFFu, t.dense ? 1 : 0, 0) != 0;
}

// Widen one 8-element chunk of a raw quantised row to bf16.
// int8: byte-permute (q + 128) into the low byte of the fp32 2^23 and subtract
// 2^23 + 128 -> exact q; |q| <= 128 has <= 8 significant bits, so the top half
// of that fp32 is the exact bf16.  int4: same for the nibble, then q * s
// rounded to nearest even.
template <int WF>
__device__ __forceinline__ uint4 widen8(const uint2 w, float scale) {
  uint32_t o[4];
  if constexpr (WF == MOE_W_INT8_ROW) {
    const uint32_t words[2] = {w.x ^ 0x80808080u, w.y ^ 0x80808080u};
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      float f[4];
#pragma unroll
      for (int b = 0; b < 4; ++b)
        f[b] = __uint_as_float(__byte_perm(words[h], 0x4B000000u, 0x7440u | b)) - 8388736.0f;
      o[2 * h] = __byte_perm(__float_as_uint(f[0]), __float_as_uint(f[1]), 0x7632);
      o[2 * h + 1] = __byte_perm(__float_as_uint(f[2]), __float_as_uint(f[3]), 0x7632);
    }
  } else {
    // int4: the subtraction and the scaling run on element pairs with the paired
    // fp32 instructions (the same roundings as one element at a time); fewer
    // instructions where the widening, not the tensor core, sets the pace
    const uint32_t lo = (w.x & 0x0F0F0F0Fu) ^ 0x08080808u;         // even elements, q + 8
    const uint32_t hi = ((w.x >> 4) & 0x0F0F0F0Fu) ^ 0x08080808u;  // odd elements
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      float v0, v1;
      add_mul_f32x2(__byte_perm(lo, 0x4B000000u, 0x7440u | j), __byte_perm(hi, 0x4B000000u, 0x7440u | j),
                    -8388616.0f, scale, v0, v1);
      o[j] = pack_bf16x2(v0, v1);
    }
  }
  return make_uint4(o[0], o[1], o[2], o[3]);
}

// TA (quantised weights only): the widened A tiles live in TMEM and the MMA
// reads A from there (tcgen05.mma [d], [a], b-desc) -- shared memory then
// carries only the raw bytes and the token tiles; otherwise they live in a
// shared-memory ring in the 128-byte swizzle.
template <int MODE, int WF, int MT, int TA>
struct Traits {
  static constexpr bool kQuant = WF != MOE_W_BF16;
  static constexpr bool kTmemA = kQuant && TA != 0;
  // gate/up: MT = 2 (gate tile, up tile) over 128 output rows; down: MT tiles of 128 rows
  static constexpr int kRows = MODE == 0 ? kBM : kBM * MT;  // output rows per unit
  static constexpr int kRawTile = WF == MOE_W_INT8_ROW ? kBM * kBK : (WF == MOE_W_INT4_B32 ? kBM * kBK / 2 : 0);
  static constexpr int kAcols = kTmemA ? MT * (kBK / 2) : 0;  // TMEM columns of one widened A stage
  static constexpr int kEpiWarps = 8;                     // two 4-warp groups
  static constexpr int kDequantWarps = kQuant ? 8 : 0;
  static constexpr int kDequant0 = 4 + kEpiWarps;         // first dequant warp
  static constexpr int kThreads = 32 * (4 + kEpiWarps + kDequantWarps);
  static constexpr int kGroupXchg = MODE == 0 ? 0 : 2 * 256 * 4;  // down: pair ids + weights per group
  static constexpr int kXchg = (2 * kGroupXchg + 1023) / 1024 * 1024;
  static constexpr int kARing = kQuant && !kTmemA ? kAStages * MT * kTileBytes : 0;  // shared-memory A ring
};

template <int MODE, int WF, int MT, int TA>
__global__ void __launch_bounds__(Traits<MODE, WF, MT, TA>::kThreads, 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap tm_w0, const __grid_constant__ CUtensorMap tm_w1,
                   const __grid_constant__ CUtensorMap tm_b, const __grid_constant__ CUtensorMap tm_w0d,
                   const __grid_constant__ CUtensorMap tm_w1d, const __grid_constant__ CUtensorMap tm_bd,
                   const GemmArgs a) {
  using Tr = Traits<MODE, WF, MT, TA>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_base = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((raw_base + 1023u) & ~1023u) - raw_base);  // 1024-aligned
  uint64_t* full = reinterpret_cast<uint64_t*>(smem);  // TMA landed (bf16: A and B; quantised: B)
  uint64_t* empty = full + kMaxStages;                 // MMAs finished reading the stage
  uint64_t* rfull = empty + kMaxStages;                // quantised: raw tiles landed
  uint64_t* rempty = rfull + kMaxStages;               // quantised: dequant warps done with the raw tiles
  uint64_t* ready = rempty + kMaxStages;               // [kAStages] quantised: bf16 A written
  uint64_t* a_empty = ready + kAStages;                // [kAStages] quantised: MMAs done with bf16 A
  uint64_t* acc_full = a_empty + kAStages;             // [2]
  uint64_t* acc_empty = acc_full + 2;                  // [2]
  uint64_t* mma_done = acc_empty + 2;
  uint64_t* q_full = mma_done + 1;                     // [kUnitQ] unit id published
  uint64_t* q_empty = q_full + kUnitQ;                 // [kUnitQ] every role has read it
  int* unit_q = reinterpret_cast<int*>(q_empty + kUnitQ);  // [kUnitQ] unit ids
  Unit* unit_tq = reinterpret_cast<Unit*>(unit_q + kUnitQ);  // [kUnitQ] the same units, decoded
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(unit_tq + kUnitQ);
  float* xchg = reinterpret_cast<float*>(smem + kBarrierBytes);
  uint8_t* a_ring = smem + kBarrierBytes + Tr::kXchg;  // quantised, A in shared memory: kAStages x MT bf16 A tiles
  uint8_t* stages = a_ring + Tr::kARing;
  uint8_t* raw_ring = stages + a.raw_ring_off;  // quantised only

  const int w = warp_id(), lane = lane_id();
  const int NS = a.NS, nbuf = a.nbuf;
  const uint32_t buf_cols = (uint32_t)(MT * a.acc_stride);
  if (threadIdx.x == 0) {
    for (int i = 0; i < NS; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    for (int i = 0; i < (Tr::kQuant ? a.RS : 0); ++i) {
      mbar_init(&rfull[i], 1);
      mbar_init(&rempty[i], Tr::kDequantWarps > 0 ? Tr::kDequantWarps : 1);
    }
    for (int i = 0; i < kAStages; ++i) {
      mbar_init(&ready[i], Tr::kDequantWarps > 0 ? Tr::kDequantWarps : 1);
      mbar_init(&a_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&acc_full[i], 1);
      mbar_init(&acc_empty[i], Tr::kEpiWarps);
    }
    mbar_init(mma_done, 1);
    // readers of a queue slot: the MMA warp, the epilogue warps and, for quantised
    // weights, the token producer and the dequant warps
    for (int i = 0; i < kUnitQ; ++i) {
      mbar_init(&q_full[i], 1);
      mbar_init(&q_empty[i], 1 + Tr::kEpiWarps + (Tr::kQuant ? 1 + Tr::kDequantWarps : 0));
    }
    fence_mbar_init();
  }
  if (w == 1) tmem_alloc(tmem_slot, (uint32_t)a.tmem_cols);
  if (threadIdx.x == 32) {
    prefetch_tmap(&tm_w0);
    if (MODE == 0) prefetch_tmap(&tm_w1);
    prefetch_tmap(&tm_b);
    if (a.dense_units > 0) {
      prefetch_tmap(&tm_w0d);
      if (MODE == 0) prefetch_tmap(&tm_w1d);
      prefetch_tmap(&tm_bd);
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  // the prologue above touches only this CTA's shared memory, TMEM and the tensor
  // maps; everything below reads what earlier launches wrote
  pdl_wait();
  pdl_trigger();

  const int ntouched = MODE == 2 ? 0 : a.meta[0];
  const int nib = (a.R + Tr::kRows - 1) / Tr::kRows;  // gate/up: the last block may be half (I % 128 == 64)
  const int routed = MODE == 2 ? nib * ((a.T + a.chunk - 1) / a.chunk) * a.S
                               : (ntouched > 0 ? a.meta[3] * nib : 0);
  const int total = routed + (MODE == 2 ? 0 : a.dense_units);

  // The sequence of units of this CTA.  Router (uniform units): blockIdx.x + i *
  // gridDim.x.  Expert GEMMs: the first unit is blockIdx.x, each later one is
  // claimed from a.sched by warp 0 lane 0 when it starts loading it, and
  // published through a small queue that every other role reads in order; -1
  // ends the sequence.
  // The scheduler decodes each unit once (a binary search over global memory)
  // and publishes it decoded, so the other roles read it from shared memory.
  auto publish_unit = [&](uint32_t i, bool& dead, Unit& t) -> int {
    if (MODE == 2) {
      const int u = blockIdx.x + (int)i * gridDim.x;
      if (u < total) t = decode_unit<MODE>(a, u, nib, ntouched, routed);
      return u < total ? u : -1;
    }
    const int slot = i % kUnitQ;
    wait_or_die(&q_empty[slot], ((i / kUnitQ) & 1u) ^ 1u, dead, a.flags);
    int u = i == 0 ? (int)blockIdx.x : (int)gridDim.x + atomicAdd(a.sched, 1);
    if (u >= total || dead) u = -1;
    if (u >= 0) {
      t = decode_unit<MODE>(a, u, nib, ntouched, routed);
      unit_tq[slot] = t;
    }
    unit_q[slot] = u;
    mbar_arrive(&q_full[slot]);  // release: readers that see the phase see the id and the unit
    return u;
  };
  auto read_unit = [&](uint32_t i, bool& dead, Unit& t) -> int {  // one lane per reading warp
    if (MODE == 2) {
      const int u = blockIdx.x + (int)i * gridDim.x;
      if (u < total) t = decode_unit<MODE>(a, u, nib, ntouched, routed);
      return u < total ? u : -1;
    }
    const int slot = i % kUnitQ;
    wait_or_die(&q_full[slot], (i / kUnitQ) & 1u, dead, a.flags);
    const int u = dead ? -1 : unit_q[slot];
    if (u >= 0) t = unit_tq[slot];
    mbar_arrive(&q_empty[slot]);
    return u;
  };

  if (w == 0 || (Tr::kQuant && w == 2)) {
    // ------------------------------------------------------------------ TMA producers
    // bf16: warp 0 loads A and B into one stage.  Quantised: warp 0 loads the raw
    // tiles into the raw ring, warp 2 the token boxes into the main ring.
    if (lane == 0) {
      const bool load_a = w == 0, load_b = !Tr::kQuant || w == 2;
      const bool raw = Tr::kQuant && load_a;
      const int ring = raw ? a.RS : NS;
      uint64_t* rf = raw ? rfull : full;
      uint64_t* re = raw ? rempty : empty;
      bool dead = false;
      uint32_t it = 0;
      int rs = 0;        // ring slot of K step `it`
      uint32_t rph = 0;  // and its phase parity
      const uint32_t abytes = load_a ? MT * (Tr::kQuant ? Tr::kRawTile : kTileBytes) : 0;
      for (uint32_t i = 0;; ++i) {
        Unit t{};
        const int u = w == 0 ? publish_unit(i, dead, t) : read_unit(i, dead, t);
        if (u < 0) break;
        const int nbox = load_b ? (t.n_tok + kBoxRows - 1) / kBoxRows : 0;
        const int brow = t.pos0;
        const int wrow0 = t.e * (t.dense ? a.Rd : a.R) + t.ib * Tr::kRows;
        const CUtensorMap* mw0 = t.dense ? &tm_w0d : &tm_w0;
        const CUtensorMap* mw1 = t.dense ? &tm_w1d : &tm_w1;
        const CUtensorMap* mb = t.dense ? &tm_bd : &tm_b;
        for (int kb = t.k0; kb < t.k0 + t.nk; ++kb, ++it) {
          const int s = rs;
          const uint32_t ph = rph;
          if (++rs == ring) { rs = 0; rph ^= 1u; }
          wait_or_die(&re[s], ph ^ 1u, dead, a.flags);
          if (dead) continue;
          mbar_arrive_expect_tx(&rf[s], abytes + nbox * kBoxRows * kBK * 2);
          if (load_a) {
            uint8_t* ad = raw ? raw_ring + (size_t)s * a.raw_stage_bytes : stages + (size_t)s * a.stage_bytes;
            const int wcol = WF == MOE_W_INT4_B32 ? kb * (kBK / 2) : kb * kBK;  // int4 maps count bytes
#pragma unroll
            for (int mt = 0; mt < MT; ++mt) {
              uint8_t* adst = ad + mt * (Tr::kQuant ? Tr::kRawTile : kTileBytes);
              if (MODE == 0)  // tile 0: 128 gate rows, tile 1: the same 128 up rows
                tma_load_2d(adst, mt ? mw1 : mw0, wcol, wrow0, &rf[s]);
              else            // 128 down rows per tile
                tma_load_2d(adst, mw0, wcol, wrow0 + mt * kBM, &rf[s]);
            }
          }
          if (load_b) {
            uint8_t* st = stages + (size_t)s * a.stage_bytes;
            const int bcol = MODE == 2 ? (kb * kBK) % a.Hx : kb * kBK;
            for (int j = 0; j < nbox; ++j)
              tma_load_2d(st + a.b_off + j * kBoxRows * kBK * 2, mb, bcol, brow + kBoxRows * j, &rf[s]);
          }
        }
      }
      // let the last loads land before the CTA can exit
      const uint32_t first = it > (uint32_t)ring ? it - ring : 0u;
      for (uint32_t j = first; j < it && !dead; ++j) wait_or_die(&rf[j % ring], (j / ring) & 1u, dead, a.flags);
    }
  } else if (w == 1) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      bool dead = false;
      uint32_t it = 0;
      int ms = 0;        // main-ring slot of K step `it`
      uint32_t mph = 0;  // and its phase parity
      const uint32_t stage0 = smem_u32(stages);
      const uint32_t a_ring0 = smem_u32(a_ring);
      for (uint32_t local = 0;; ++local) {
        Unit t{};
        const int u = read_unit(local, dead, t);
        if (u < 0) break;
        const uint32_t buf = local % nbuf;
        wait_or_die(&acc_empty[buf], ((local / nbuf) & 1u) ^ 1u, dead, a.flags);
        tc_fence_after();
        const uint32_t idesc = umma_idesc_bf16(kBM, t.n_mma);
        const uint32_t d = tmem_base + buf * buf_cols;
        for (int kb = 0; kb < t.nk; ++kb, ++it) {
          const int s = ms;
          const uint32_t ph = mph;
          if (++ms == NS) { ms = 0; mph ^= 1u; }
          const int ja = it % kAStages;
          if (Tr::kQuant) wait_or_die(&ready[ja], (it / kAStages) & 1u, dead, a.flags);
          wait_or_die(&full[s], ph, dead, a.flags);
          if (dead) continue;
          tc_fence_after();
          const uint32_t sb = stage0 + s * a.stage_bytes;
          const uint32_t sa = Tr::kQuant ? a_ring0 + ja * (MT * kTileBytes) : sb;
          const uint32_t ta = tmem_base + (uint32_t)(a.a_col0 + ja * a.a_stride);  // TMEM A: lane 0 of the stage
#pragma unroll
          for (int k = 0; k < kBK / 16; ++k) {
            const uint64_t bdesc = umma_desc_sw128(sb + a.b_off + k * 32);
#pragma unroll
            for (int mt = 0; mt < MT; ++mt) {
              if constexpr (Tr::kTmemA)  // A: 128 lanes x 8 columns of bf16 pairs per K = 16
                umma_bf16_ts(d + mt * a.acc_stride, ta + mt * (kBK / 2) + k * 8, bdesc, idesc, (kb | k) != 0);
              else
                umma_bf16(d + mt * a.acc_stride, umma_desc_sw128(sa + mt * kTileBytes + k * 32), bdesc, idesc,
                          (kb | k) != 0);
            }
          }
          umma_commit(&empty[s]);
          if (Tr::kQuant) umma_commit(&a_empty[ja]);
        }
        if (!dead) umma_commit(&acc_full[buf]);
      }
      if (!dead) {
        umma_commit(mma_done);
        wait_or_die(mma_done, 0, dead, a.flags);
      }
    }
  } else if (w >= 4 && w < 4 + Tr::kEpiWarps) {
    // ------------------------------------------------------------------ epilogue
    // Each thread owns one TMEM lane = one output row.  Gate/up and single-tile
    // down: the two groups split the unit's 16-column chunks (even / odd);
    // two-tile down: group g drains tile g.
    const int grp = (w - 4) >> 2;
    const int q = w & 3;  // TMEM lanes 32q .. 32q+31
    const bool split_cols = MODE != 1 || MT == 1;
    const int bar_x = 1 + 2 * grp, bar_v = 2 + 2 * grp;
    float* gx = xchg + grp * (Tr::kGroupXchg / 4);
    bool dead = false;
    for (uint32_t local = 0;; ++local) {
      int u = 0;
      Unit t{};
      if (lane == 0) u = read_unit(local, dead, t);
      u = __shfl_sync(0xFFFFFFFFu, u, 0);
      if (u < 0) break;
      shfl_unit(t);
      const uint32_t buf = local % nbuf;
      if (lane == 0) wait_or_die(&acc_full[buf], (local / nbuf) & 1u, dead, a.flags);
      if (MODE != 1) {
        dead = __shfl_sync(0xFFFFFFFFu, dead ? 1 : 0, 0) != 0;
        __syncwarp();
      } else {
        dead = named_bar_or(bar_v, 128, dead);  // the group stages shared pair ids below
      }
      tc_fence_after();
      const int tile = split_cols ? 0 : grp;
      const uint32_t tacc = tmem_base + ((uint32_t)(q * 32) << 16) + buf * buf_cols + tile * a.acc_stride;
      const int pos0 = t.pos0;
      const ProbView pv = view_of(a, t);
      const int c_first = split_cols ? grp * 16 : 0, c_step = split_cols ? 32 : 16;
      if (!dead) {
        if (MODE == 0) {
          const int row = t.ib * kBM + q * 32 + lane;
          const bool live = row < pv.R;
          const size_t grow = (size_t)t.e * pv.R + (live ? row : 0);
          const float sg = WF == MOE_W_INT8_ROW ? pv.s0[grow] : 1.f;
          const float su = WF == MOE_W_INT8_ROW ? pv.s1[grow] : 1.f;
          uint16_t* hout = static_cast<uint16_t*>(pv.out) + (size_t)pos0 * pv.R + row;
          const bool gelu = a.act == MOE_ACT_GELU_TANH;
          for (int n0 = c_first; n0 < t.n_tok; n0 += c_step) {
            uint32_t g[16], v[16];
            tmem_ld16(tacc + n0, g);
            tmem_ld16(tacc + a.acc_stride + n0, v);
            tmem_ld_wait();
            if (live) {
              // all 16 values first (independent chains), then the stores
              uint16_t hv[16];
              if (gelu) {
#pragma unroll
                for (int j = 0; j < 16; ++j)
                  hv[j] = f32_to_bf16(gelu_tanh_mul_fast(__uint_as_float(g[j]) * sg, __uint_as_float(v[j]) * su));
              } else {
#pragma unroll
                for (int j = 0; j < 16; ++j)
                  hv[j] = f32_to_bf16(silu_mul_fast(__uint_as_float(g[j]) * sg, __uint_as_float(v[j]) * su));
              }
              uint16_t* dst = hout + (size_t)n0 * pv.R;
              if (n0 + 16 <= t.n_tok) {
#pragma unroll
                for (int j = 0; j < 16; ++j) dst[(size_t)j * pv.R] = hv[j];
              } else {
#pragma unroll
                for (int j = 0; j < 16; ++j)
                  if (n0 + j < t.n_tok) dst[(size_t)j * pv.R] = hv[j];
              }
            }
          }
        } else if (MODE == 2) {
          // router logits: partial[s][t][e] (fp32), tokens along columns
          const int e = t.ib * kBM + q * 32 + lane;
          float* part = static_cast<float*>(a.out) + (size_t)t.c * a.T * a.R;
          for (int n0 = c_first; n0 < t.n_tok; n0 += c_step) {
            uint32_t v[16];
            tmem_ld16(tacc + n0, v);
            tmem_ld_wait();
            if (e < a.R) {
#pragma unroll
              for (int j = 0; j < 16; ++j)
                if (n0 + j < t.n_tok) part[(size_t)(t.base + n0 + j) * a.R + e] = __uint_as_float(v[j]);
            }
          }
        } else {
          // stage the unit's pair ids and routing weights (one round trip for all columns)
          int32_t* s_pair = reinterpret_cast<int32_t*>(gx);
          float* s_w = gx + 256;
          const int et = q * 32 + lane;
          for (int n = et; n < t.n_tok; n += 128) {
            // dense problem: the token itself, weight 1
            const int pair = t.dense ? pos0 + n : a.sorted_pair[pos0 + n];
            s_pair[n] = pair;
            s_w[n] = t.dense ? 1.f : a.topk_w[pair];
          }
          named_bar_sync(bar_x, 128);
          const int row = t.ib * Tr::kRows + tile * kBM + et;
          const float sd = WF == MOE_W_INT8_ROW ? pv.s0[(size_t)t.e * pv.R + row] : 1.f;
          float* yp = static_cast<float*>(pv.out);
          uint16_t* yb = static_cast<uint16_t*>(pv.out);
          const bool ob = a.out_bf16 && !t.dense;  // the dense problem's rows stay fp32
          auto put = [&](int pair, float v) {
            if (ob) yb[(size_t)pair * pv.R + row] = f32_to_bf16(v);
            else yp[(size_t)pair * pv.R + row] = v;
          };
          for (int n0 = c_first; n0 < t.n_tok; n0 += c_step) {
            uint32_t v[16];
            tmem_ld16(tacc + n0, v);
            tmem_ld_wait();
            if (n0 + 16 <= t.n_tok) {
              // whole chunk: pair ids and weights as 16-byte broadcasts, stores unpredicated
              const int4* p4 = reinterpret_cast<const int4*>(s_pair + n0);
              const float4* w4 = reinterpret_cast<const float4*>(s_w + n0);
#pragma unroll
              for (int j4 = 0; j4 < 4; ++j4) {
                const int4 p = p4[j4];
                const float4 wv = w4[j4];
                put(p.x, wv.x * sd * __uint_as_float(v[4 * j4 + 0]));
                put(p.y, wv.y * sd * __uint_as_float(v[4 * j4 + 1]));
                put(p.z, wv.z * sd * __uint_as_float(v[4 * j4 + 2]));
                put(p.w, wv.w * sd * __uint_as_float(v[4 * j4 + 3]));
              }
            } else {
#pragma unroll
              for (int j = 0; j < 16; ++j) {
                if (n0 + j < t.n_tok) put(s_pair[n0 + j], s_w[n0 + j] * sd * __uint_as_float(v[j]));
              }
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[buf]);
    }
  } else if (Tr::kQuant && w >= Tr::kDequant0) {
    // ------------------------------------------------------------------ dequantisation
    // One weight row per thread (two threads per row when the unit has 128 A rows):
    // thread ct owns row r = ct % (MT*128) of the unit's A rows and the 8-element
    // chunks [cg*kChunks, (cg+1)*kChunks) of it, cg = ct / (MT*128).  The raw tiles
    // arrive in the TMA's 64-byte (int8) or 32-byte (int4) swizzle, so a warp's 32
    // rows read their 16-byte pieces without bank conflicts, and the widened
    // chunks go to the 128-byte-swizzled bf16 tile the same way.  An int4 row
    // needs two block scales per K step (one per 32 columns), not one per chunk.
    constexpr int kDT = 32 * (Tr::kDequantWarps > 0 ? Tr::kDequantWarps : 8);  // dequant threads
    constexpr int kRowsA = MT * kBM;
    constexpr int kChunks = 8 * kRowsA / kDT;  // chunks per thread per K step (8 or 4)
    static_assert(kDT % kRowsA == 0 && kChunks >= 1 && kChunks <= 8, "dequant thread mapping");
    const int ct = threadIdx.x - 32 * Tr::kDequant0;
    const int r = ct % kRowsA, cg = ct / kRowsA;
    const int mt = r >> 7, rr = r & 127;
    const int c0 = cg * kChunks;  // first chunk of this thread
    bool dead = false;
    uint32_t it = 0;
    int rs = 0;        // raw-ring slot of K step `it`
    uint32_t rph = 0;  // and its phase parity
    for (uint32_t i = 0;; ++i) {
      int u = 0;
      Unit t{};
      if (lane == 0) u = read_unit(i, dead, t);
      u = __shfl_sync(0xFFFFFFFFu, u, 0);
      if (u < 0) break;
      shfl_unit(t);
      // int4: this row's block scales for the chunks of this thread, one K step ahead
      const ProbView pv = view_of(a, t);
      const float* S = (MODE == 0 && mt == 1) ? pv.s1 : pv.s0;
      int wr = MODE == 0 ? t.ib * kBM + rr : t.ib * Tr::kRows + mt * kBM + rr;
      if (wr >= pv.R) wr = pv.R - 1;  // rows past a half block are computed but never stored
      const float* srow = S + ((size_t)t.e * pv.R + wr) * (pv.K >> a.qsh);
      float s_next[2] = {1.f, 1.f};  // scales of chunks c0 and c0 + kChunks - 1 (the two 32-column halves)
      if (WF == MOE_W_INT4_B32) {
        s_next[0] = __ldg(srow + ((t.k0 * kBK + c0 * 8) >> a.qsh));
        s_next[1] = __ldg(srow + ((t.k0 * kBK + (c0 + kChunks - 1) * 8) >> a.qsh));
      }
      for (int kb = 0; kb < t.nk; ++kb, ++it) {
        const float s_lo = s_next[0], s_hi = s_next[1];
        if (WF == MOE_W_INT4_B32 && kb + 1 < t.nk) {
          s_next[0] = __ldg(srow + (((t.k0 + kb + 1) * kBK + c0 * 8) >> a.qsh));
          s_next[1] = __ldg(srow + (((t.k0 + kb + 1) * kBK + (c0 + kChunks - 1) * 8) >> a.qsh));
        }
        const int s = rs;
        const uint32_t ph = rph;
        if (++rs == a.RS) { rs = 0; rph ^= 1u; }
        const int ja = it % kAStages;
        // the row's raw bytes of this thread's chunks (16-byte pieces) are loaded as soon
        // as they have landed, before the wait for the A stage, so that the load latency
        // overlaps that wait
        wait_or_die(&rfull[s], ph, dead, a.flags);
        uint32_t q[kChunks * (WF == MOE_W_INT8_ROW ? 2 : 1)];
        if (!dead) {
          const uint8_t* raw = raw_ring + (size_t)s * a.raw_stage_bytes + mt * Tr::kRawTile;
          if constexpr (WF == MOE_W_INT8_ROW) {
            // 64-byte rows, piece p (chunks 2p, 2p+1) at (p ^ ((rr >> 1) & 3)) * 16
#pragma unroll
            for (int p = 0; p < kChunks / 2; ++p) {
              const int pp = c0 / 2 + p;
              const uint4 v = *reinterpret_cast<const uint4*>(raw + rr * 64 + ((pp ^ ((rr >> 1) & 3)) << 4));
              q[4 * p] = v.x; q[4 * p + 1] = v.y; q[4 * p + 2] = v.z; q[4 * p + 3] = v.w;
            }
          } else {
            // 32-byte rows, piece p (chunks 4p .. 4p+3) at (p ^ ((rr >> 2) & 1)) * 16
#pragma unroll
            for (int p = 0; p < (kChunks + 3) / 4; ++p) {
              const int pp = c0 / 4 + p;
              const uint4 v = *reinterpret_cast<const uint4*>(raw + rr * 32 + ((pp ^ ((rr >> 2) & 1)) << 4));
              q[4 * p] = v.x; q[4 * p + 1] = v.y; q[4 * p + 2] = v.z; q[4 * p + 3] = v.w;
            }
          }
        }
        wait_or_die(&a_empty[ja], ((it / kAStages) & 1u) ^ 1u, dead, a.flags);
        if constexpr (Tr::kTmemA) dead = __any_sync(0xFFFFFFFFu, dead);  // tcgen05.st below is warp-collective
        if (!dead) {
          uint8_t* A = a_ring + ja * (MT * kTileBytes) + mt * kTileBytes + rr * 128;
          if constexpr (Tr::kTmemA) {
            // the row's widened chunks are 4 * kChunks consecutive bf16-pair columns of
            // this thread's TMEM lane (lower K in the low half): one warp-wide store
            // into the warp's lane quarter (warp w reaches lanes 32 (w % 4) .. + 31,
            // and rr / 32 == w % 4 by the row mapping above)
            tc_fence_after();  // after a_empty: the MMAs that read this stage are complete
            uint32_t words[4 * kChunks];
#pragma unroll
            for (int j = 0; j < kChunks; ++j) {
              const uint2 raw8 = WF == MOE_W_INT8_ROW ? make_uint2(q[2 * j], q[2 * j + 1]) : make_uint2(q[j], 0u);
              const uint4 o = widen8<WF>(raw8, j * 2 < kChunks ? s_lo : s_hi);
              words[4 * j] = o.x;
              words[4 * j + 1] = o.y;
              words[4 * j + 2] = o.z;
              words[4 * j + 3] = o.w;
            }
            const uint32_t taddr = tmem_base + ((uint32_t)(rr & ~31) << 16) +
                                   (uint32_t)(a.a_col0 + ja * a.a_stride + mt * (kBK / 2) + c0 * 4);
#pragma unroll
            for (int h = 0; h < kChunks / 4; ++h) {
              uint32_t part[16];
#pragma unroll
              for (int i = 0; i < 16; ++i) part[i] = words[16 * h + i];
              tmem_st16(taddr + 16 * h, part);
            }
            if constexpr (kChunks % 4 != 0) {  // two chunks: 8 columns
              uint32_t part[8];
#pragma unroll
              for (int i = 0; i < 8; ++i) part[i] = words[4 * kChunks - 8 + i];
              tmem_st8(taddr + 4 * kChunks - 8, part);
            }
            tmem_st_wait();
            tc_fence_before();
          } else {
#pragma unroll
            for (int j = 0; j < kChunks; ++j) {
              const int c = c0 + j;
              const uint2 raw8 = WF == MOE_W_INT8_ROW ? make_uint2(q[2 * j], q[2 * j + 1]) : make_uint2(q[j], 0u);
              const float sc = j * 2 < kChunks ? s_lo : s_hi;
              *reinterpret_cast<uint4*>(A + ((c ^ (rr & 7)) << 4)) = widen8<WF>(raw8, sc);
            }
            fence_proxy_async_smem();
          }
        }
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&rempty[s]);  // the raw slot may be refilled
          mbar_arrive(&ready[ja]);
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (w == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, (uint32_t)a.tmem_cols);
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

cudaError_t weight_map(CUtensorMap* m, const void* W, int wfmt, int E, int R, int K, int box_rows) {
  const uint64_t rows = (uint64_t)E * R;
  if (wfmt == MOE_W_BF16)
    return make_map(m, W, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, K, rows, kBK, box_rows, CU_TENSOR_MAP_SWIZZLE_128B);
  if (wfmt == MOE_W_INT8_ROW)
    return make_map(m, W, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, K, rows, kBK, box_rows, CU_TENSOR_MAP_SWIZZLE_64B);
  return make_map(m, W, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, K / 2, rows, kBK / 2, box_rows, CU_TENSOR_MAP_SWIZZLE_32B);
}

uint32_t pow2_at_least(uint32_t v) {
  uint32_t p = 32;
  while (p < v) p <<= 1;
  return p;
}

// tensor maps of one launch: the routed problem's weights and token rows, and
// the dense problem's (copies of the routed ones when there is none)
struct Maps {
  CUtensorMap w0, w1, b, w0d, w1d, bd;
};

template <int MODE, int WF, int MT, int TA>
cudaError_t launch_gemm(const Maps& m, GemmArgs a, int chunk_max, int num_sms, cudaStream_t s) {
  using Tr = Traits<MODE, WF, MT, TA>;
  // stage: bf16 weights [A: MT x 16 KB][B]; quantised [B], with the raw tiles in a ring of
  // their own after the main ring (their bf16 A lives in the A ring or in TMEM).  Token
  // boxes are kBoxRows tall: B holds the chunk rounded up to whole boxes.  All sizes are
  // multiples of 1024 (4 KB boxes, 16/8/4 KB tiles).
  const int b_rows = (chunk_max + kBoxRows - 1) / kBoxRows * kBoxRows;
  a.b_off = Tr::kQuant ? 0 : MT * kTileBytes;
  a.stage_bytes = a.b_off + b_rows * kBK * 2;
  a.raw_stage_bytes = MT * Tr::kRawTile;
  // TMEM.  Shared-memory A: nbuf accumulator sets of MT tiles.  A in TMEM, two
  // layouts: "stacked" -- two accumulator sets, then the kAStages widened A stages --
  // while that fits (chunks up to 64 tokens with two tiles); otherwise, two tiles of
  // at most 192 tokens, "interleaved" -- one accumulator set, tile t at column 256 t
  // and A stage j in the 64 columns after it (192 + 256 j) -- so every region starts
  // on a multiple of 64 columns.
  a.acc_stride = (int)pow2_at_least((uint32_t)chunk_max);
  a.a_stride = Tr::kAcols;
  if (!Tr::kTmemA) {
    a.nbuf = 2 * MT * a.acc_stride <= 512 ? 2 : 1;
    a.tmem_cols = a.nbuf * MT * a.acc_stride;
    a.a_col0 = 0;
  } else if (2 * MT * a.acc_stride + kAStages * Tr::kAcols <= 512) {
    a.nbuf = 2;
    a.a_col0 = 2 * MT * a.acc_stride;
    a.tmem_cols = (int)pow2_at_least((uint32_t)(a.a_col0 + kAStages * Tr::kAcols));
  } else if (MT == 2 && kAStages == 2 && chunk_max <= 192) {
    a.nbuf = 1;
    a.acc_stride = 256;
    a.a_col0 = 192;
    a.a_stride = 256;
    a.tmem_cols = 512;
  } else {
    return cudaErrorInvalidConfiguration;
  }
  if (a.tmem_cols > 512) return cudaErrorInvalidConfiguration;
  const int fixed = 1024 + kBarrierBytes + Tr::kXchg + Tr::kARing;
  const int avail = kSmemLimit - fixed;
  if (Tr::kQuant) {
    // token ring: about 96 KB of boxes (L2-resident rows), 2..4 stages; the rest feeds the
    // raw weight ring (HBM latency)
    a.NS = (96 * 1024) / a.stage_bytes;
    a.NS = a.NS < 2 ? 2 : (a.NS > 4 ? 4 : a.NS);
    a.RS = (avail - a.NS * a.stage_bytes) / a.raw_stage_bytes;
    while (a.RS < 3 && a.NS > 2) a.RS = (avail - --a.NS * a.stage_bytes) / a.raw_stage_bytes;
    if (a.RS > kMaxStages) a.RS = kMaxStages;
    if (a.RS < 2) return cudaErrorInvalidConfiguration;
  } else {
    a.NS = avail / a.stage_bytes;
    if (a.NS > kMaxStages) a.NS = kMaxStages;
    a.RS = 0;
  }
  if (a.NS < 2) return cudaErrorInvalidConfiguration;
  a.raw_ring_off = a.NS * a.stage_bytes;
  const size_t smem = (size_t)fixed + (size_t)a.NS * a.stage_bytes + (size_t)a.RS * a.raw_stage_bytes;
  auto kern = gemm_tc_kernel<MODE, WF, MT, TA>;
  cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (err != cudaSuccess) return err;
  return launch_k(kern, dim3(num_sms), dim3(Tr::kThreads), smem, s, m.w0, m.w1, m.b, m.w0d, m.w1d, m.bd, a);
}

// Quantised weights widen into TMEM when two accumulator sets and the widened A
// stages fit in its 512 columns (chunks of at most 64 tokens: decode-sized
// batches, where it measured up to 11% faster for int4 and even for int8), and
// for gate/up with chunks of at most 192 tokens in the interleaved layout (one
// accumulator set: measured 8% faster on the int4 workload's 64-token experts).
// Otherwise -- the down projection beyond 64 tokens, and 256-token chunks -- A
// goes to shared memory, which keeps two accumulator sets where they fit: with
// A in TMEM the 256-token int8 prefill measured 4-11% slower at 192-token chunks.
template <int MODE, int WF, int MT>
cudaError_t launch_quant(const Maps& m, const GemmArgs& a, int chunk_max, int num_sms, cudaStream_t s) {
  const int acc = (int)pow2_at_least((uint32_t)chunk_max);  // TMEM columns of one tile's accumulator
  if (2 * MT * acc + kAStages * MT * (kBK / 2) <= 512 || (MODE == 0 && MT == 2 && chunk_max <= 192))
    return launch_gemm<MODE, WF, MT, 1>(m, a, chunk_max, num_sms, s);
  return launch_gemm<MODE, WF, MT, 0>(m, a, chunk_max, num_sms, s);
}

// gate/up always carries two M tiles (gate, up); down carries two 128-row tiles
// of W_down whenever H allows (each pipeline stage then moves 32 KB of weights:
// at decode sizes this streams the weights at about 93% of HBM bandwidth, one
// 16 KB tile per stage about 86%; at prefill sizes the token tile feeds 256
// weight rows)
template <int MODE>
cudaError_t launch_by_format(int wfmt, const Maps& m, GemmArgs a, int num_sms, cudaStream_t s) {
  const bool two = MODE == 0 || a.R % (2 * kBM) == 0;  // down: the dense problem has the same R (= H)
  // the dense problem's units: (row block of kRows, token chunk)
  const int rows = MODE == 0 || !two ? kBM : 2 * kBM;
  a.dense_units = a.Td > 0 ? ((a.Rd + rows - 1) / rows) * ((a.Td + a.chunkd - 1) / a.chunkd) : 0;
  const int chunk_max = a.dense_units > 0 && a.chunkd > a.chunk ? a.chunkd : a.chunk;
  switch (wfmt) {
    case MOE_W_BF16:
      return two ? launch_gemm<MODE, MOE_W_BF16, 2, 0>(m, a, chunk_max, num_sms, s)
                 : launch_gemm<MODE, MOE_W_BF16, 1, 0>(m, a, chunk_max, num_sms, s);
    case MOE_W_INT8_ROW:
      return two ? launch_quant<MODE, MOE_W_INT8_ROW, 2>(m, a, chunk_max, num_sms, s)
                 : launch_quant<MODE, MOE_W_INT8_ROW, 1>(m, a, chunk_max, num_sms, s);
    default:
      return two ? launch_quant<MODE, MOE_W_INT4_B32, 2>(m, a, chunk_max, num_sms, s)
                 : launch_quant<MODE, MOE_W_INT4_B32, 1>(m, a, chunk_max, num_sms, s);
  }
}

GemmArgs common(const Workspace& ws, int chunk, uint32_t* flags) {
  GemmArgs a{};
  a.offsets = ws.offsets;
  a.touched = ws.touched;
  a.tile_base = ws.tile_base;
  a.meta = ws.meta;
  a.sorted_pair = ws.sorted_pair;
  a.flags = flags;
  a.chunk = chunk;
  return a;
}

// also zeroes the unit counters of the two expert GEMMs that follow (meta[8], meta[9])
__global__ void __launch_bounds__(256) gather_rows_kernel(const uint16_t* __restrict__ x, int H, int k,
                                                          const int32_t* __restrict__ sorted_pair,
                                                          int32_t* __restrict__ meta, uint16_t* __restrict__ xs) {
  pdl_wait();
  pdl_trigger();
  if (blockIdx.x == 0 && threadIdx.x == 0) {
    meta[8] = 0;
    meta[9] = 0;
  }
  const int P = meta[1];
  // a warp copies a 128-chunk segment of one row (16-byte chunks): lane l takes
  // chunks l, l+32, l+64, l+96, all four loads in flight before the stores, and
  // every load and store instruction covers 512 contiguous bytes
  const int lane = threadIdx.x & 31;
  const int per_row = H / 8;
  const int nseg = (per_row + 127) / 128;
  const size_t items = (size_t)P * nseg;
  const size_t nwarps = ((size_t)gridDim.x * blockDim.x) >> 5;
  for (size_t it = ((size_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5; it < items; it += nwarps) {
    const int pos = (int)(it / nseg), seg = (int)(it - (size_t)pos * nseg);
    const int t = sorted_pair[pos] / k;
    const uint4* src = reinterpret_cast<const uint4*>(x + (size_t)t * H);
    uint4* dst = reinterpret_cast<uint4*>(xs + (size_t)pos * H);
    const int c0 = seg * 128 + lane;
    uint4 v[4];
#pragma unroll
    for (int q = 0; q < 4; ++q)
      if (c0 + 32 * q < per_row) v[q] = src[c0 + 32 * q];
#pragma unroll
    for (int q = 0; q < 4; ++q)
      if (c0 + 32 * q < per_row) dst[c0 + 32 * q] = v[q];
  }
}

// W3[e] = [hi | mid | lo] with hi = bf16(w), mid = bf16(w - hi), lo = bf16(w - hi - mid):
// each difference is exact in fp32 and the three parts reproduce w to ~2^-27
// relative, so bf16 x against W3 over 3H columns gives fp32-accurate logits
__global__ void __launch_bounds__(256) split3_kernel(const float* __restrict__ Wr, int E, int H,
                                                     uint16_t* __restrict__ W3) {
  pdl_wait();
  pdl_trigger();
  const int q4 = H / 4;  // float4 quads per row
  const int n = E * q4;
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x) {
    const int e = i / q4, h = (i - e * q4) * 4;
    const float4 w4 = *reinterpret_cast<const float4*>(Wr + (size_t)e * H + h);
    const float w[4] = {w4.x, w4.y, w4.z, w4.w};
    uint16_t p[3][4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      p[0][j] = f32_to_bf16(w[j]);
      const float r1 = w[j] - bf16_to_f32(p[0][j]);
      p[1][j] = f32_to_bf16(r1);
      p[2][j] = f32_to_bf16(r1 - bf16_to_f32(p[1][j]));
    }
    uint16_t* row = W3 + (size_t)e * 3 * H + h;
#pragma unroll
    for (int part = 0; part < 3; ++part)
      *reinterpret_cast<uint2*>(row + (size_t)part * H) =
          make_uint2((uint32_t)p[part][0] | ((uint32_t)p[part][1] << 16), (uint32_t)p[part][2] | ((uint32_t)p[part][3] << 16));
  }
}

}  // namespace

int router_tc_chunk(int T) {
  const int t = ((T > 0 ? T : 1) + 15) / 16 * 16;
  return t < kMaxTileN ? t : kMaxTileN;
}

// K splits of the tensor-core router: a function of T and H only, so a masked
// layer and its sliced twin sum identical partials in the same order.  Every
// split owns at least one of the 3H/64 K steps (a split with none would leave
// its TMEM accumulator unwritten).
int router_tc_splits(int T, int H) {
  const int chunks = (T + router_tc_chunk(T) - 1) / router_tc_chunk(T);
  const int nk_all = 3 * H / kBK;
  int S = 1;
  while (S < 8 && chunks * S * 2 <= 74 && S * 2 <= nk_all) S *= 2;
  return S;
}

bool router_tc_supported(const moe_desc& d) { return d.xfmt == MOE_X_BF16 && encode_fn() != nullptr; }

cudaError_t launch_router_split3(const moe_desc& d, void* W3, int num_sms, cudaStream_t s) {
  const size_t n = (size_t)d.E * d.H / 4;
  int blocks = (int)((n + 255) / 256);
  if (blocks > num_sms * 8) blocks = num_sms * 8;
  return launch_k(split3_kernel, dim3(blocks), dim3(256), 0, s, d.W_r, d.E, d.H, static_cast<uint16_t*>(W3));
}

cudaError_t launch_router_tc(const moe_desc& d, const void* x, int T, const void* W3, float* partial, int S,
                             int num_sms, uint32_t* flags, cudaStream_t s) {
  CUtensorMap ma, mb;
  cudaError_t e = make_map(&ma, W3, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, (uint64_t)3 * d.H, (uint64_t)d.E, kBK, kBM,
                           CU_TENSOR_MAP_SWIZZLE_128B);
  if (e == cudaSuccess)
    e = make_map(&mb, x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, d.H, (uint64_t)T, kBK, kBoxRows,
                 CU_TENSOR_MAP_SWIZZLE_128B);
  if (e != cudaSuccess) return e;
  GemmArgs a{};
  a.flags = flags;
  a.out = partial;
  a.R = d.E;
  a.K = 3 * d.H;
  a.chunk = router_tc_chunk(T);
  a.T = T;
  a.S = S;
  a.Hx = d.H;
  const Maps m{ma, ma, mb, ma, ma, mb};
  return launch_gemm<2, MOE_W_BF16, 1, 0>(m, a, a.chunk, num_sms, s);
}

// gate/up tiles 128 output rows of I (a multiple of 64; a half block is computed
// and not stored); down tiles 128 rows of H (K = I)
bool gemm_tc_supported(const moe_desc& d) {
  return d.xfmt == MOE_X_BF16 && d.wfmt != MOE_W_F32 && d.H % 128 == 0 && d.I % 64 == 0 && encode_fn() != nullptr;
}

cudaError_t launch_gather_rows(const moe_desc& d, const void* x, const Workspace& ws, int P, int num_sms,
                               cudaStream_t s) {
  const size_t warps = (size_t)P * ((d.H / 8 + 127) / 128);  // one warp per 128-chunk row segment
  int blocks = (int)((warps + 7) / 8);
  if (blocks > num_sms * 8) blocks = num_sms * 8;
  if (blocks < 1) blocks = 1;
  return launch_k(gather_rows_kernel, dim3(blocks), dim3(256), 0, s, static_cast<const uint16_t*>(x), d.H, d.k,
                    static_cast<const int32_t*>(ws.sorted_pair), ws.meta, static_cast<uint16_t*>(ws.xs));
}

cudaError_t launch_gemm_gateup(const moe_desc& d, const Workspace& ws, int P, int chunk, int num_sms,
                               uint32_t* flags, cudaStream_t s, const DenseGemm* dg) {
  Maps m;
  cudaError_t e = weight_map(&m.w0, d.W_gate, d.wfmt, d.E, d.I, d.H, kBM);
  if (e == cudaSuccess) e = weight_map(&m.w1, d.W_up, d.wfmt, d.E, d.I, d.H, kBM);
  if (e == cudaSuccess)
    e = make_map(&m.b, ws.xs, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, d.H, (uint64_t)P, kBK, kBoxRows,
                 CU_TENSOR_MAP_SWIZZLE_128B);
  if (e != cudaSuccess) return e;
  GemmArgs a = common(ws, chunk, flags);
  a.s0 = d.s_gate;
  a.s1 = d.s_up;
  a.out = ws.hbuf;
  a.R = d.I;
  a.K = d.H;
  a.act = d.act;
  a.qsh = d.wfmt == MOE_W_INT4_B128 ? 7 : 5;
  a.sched = ws.meta + 8;
  m.w0d = m.w0;
  m.w1d = m.w1;
  m.bd = m.b;
  if (dg) {  // the dense problem: its gate/up weights against the token rows in order
    const moe_desc& sd = *dg->d;
    e = weight_map(&m.w0d, sd.W_gate, sd.wfmt, 1, sd.I, sd.H, kBM);
    if (e == cudaSuccess) e = weight_map(&m.w1d, sd.W_up, sd.wfmt, 1, sd.I, sd.H, kBM);
    if (e == cudaSuccess)
      e = make_map(&m.bd, dg->b, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, sd.H, (uint64_t)dg->T, kBK, kBoxRows,
                   CU_TENSOR_MAP_SWIZZLE_128B);
    if (e != cudaSuccess) return e;
    a.Rd = sd.I;
    a.Kd = sd.H;
    a.Td = dg->T;
    a.chunkd = dg->chunk;
    a.sd0 = sd.s_gate;
    a.sd1 = sd.s_up;
    a.outd = dg->out;
  }
  return launch_by_format<0>(d.wfmt, m, a, num_sms, s);
}

cudaError_t launch_gemm_down(const moe_desc& d, const float* topk_w, const Workspace& ws, int P, int chunk,
                             int num_sms, uint32_t* flags, cudaStream_t s, const DenseGemm* dg, bool yp_bf16) {
  Maps m;
  cudaError_t e = weight_map(&m.w0, d.W_down, d.wfmt, d.E, d.H, d.I, 128);
  if (e == cudaSuccess)
    e = make_map(&m.b, ws.hbuf, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, d.I, (uint64_t)P, kBK, kBoxRows,
                 CU_TENSOR_MAP_SWIZZLE_128B);
  if (e != cudaSuccess) return e;
  GemmArgs a = common(ws, chunk, flags);
  a.s0 = d.s_down;
  a.topk_w = topk_w;
  a.out = ws.yp;
  a.out_bf16 = yp_bf16 ? 1 : 0;
  a.R = d.H;
  a.K = d.I;
  a.qsh = d.wfmt == MOE_W_INT4_B128 ? 7 : 5;
  a.sched = ws.meta + 9;
  m.w1 = m.w0;
  m.w0d = m.w0;
  m.w1d = m.w0;
  m.bd = m.b;
  if (dg) {  // the dense problem: its down weights against its h rows in token order
    const moe_desc& sd = *dg->d;
    e = weight_map(&m.w0d, sd.W_down, sd.wfmt, 1, sd.H, sd.I, 128);
    if (e == cudaSuccess)
      e = make_map(&m.bd, dg->b, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, sd.I, (uint64_t)dg->T, kBK, kBoxRows,
                   CU_TENSOR_MAP_SWIZZLE_128B);
    if (e != cudaSuccess) return e;
    m.w1d = m.w0d;
    a.Rd = sd.H;
    a.Kd = sd.I;
    a.Td = dg->T;
    a.chunkd = dg->chunk;
    a.sd0 = sd.s_down;
    a.outd = dg->out;
  }
  return launch_by_format<1>(d.wfmt, m, a, num_sms, s);
}

}  // namespace moe
