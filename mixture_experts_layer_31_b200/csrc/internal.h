// Host-side interface between the C ABI (moe_api.cu) and the kernel launchers.
#pragma once
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "moe.h"

namespace moe {

// Programmatic dependent launch, opt-in (MOE_PDL=1 in the environment; plain
// stream ordering otherwise): every kernel of this library may then start while
// the kernel before it on the stream is finishing (its CTAs take SMs as they free
// up and run their prologue); each waits (griddepcontrol.wait) before it reads
// or writes anything an earlier launch touches, and only then lets the next
// launch start, so results do not change.  Without the attribute the wait and
// the trigger are no-ops.
bool pdl_enabled();

// Launch one kernel on stream s and report the launch status.
template <typename... KArgs, typename... Args>
cudaError_t launch_k(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                     Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl_enabled() ? 1 : 0;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
  return e != cudaSuccess ? e : cudaGetLastError();
}

// Tokens are routed in chunks of this many (token, slot) pairs when building
// the expert-sorted order.
constexpr int kPairChunk = 1024;

// The weight-streaming path processes an expert's tokens in groups of this
// many (every group re-reads the expert's weights, mostly from L2).
constexpr int kGemvGroup = 4;

// The tensor-core path computes an expert's tokens in chunks of at most
// kMaxTileN (the N of one MMA tile).  A batch of T tokens routes at most T
// of them to one expert, so small batches use smaller chunks (and smaller
// pipeline stages): chunk = min(kMaxTileN, T rounded up to 16).
// Chunks above 128 tokens leave room for only one TMEM accumulator buffer (no
// epilogue overlap); batches averaging <= 96 tokens per expert use 128.
constexpr int kMaxTileN = 256;
inline int chunk_tokens(int T, int k, int E) {
  int t = ((T > 0 ? T : 1) + 15) / 16 * 16;
  if (t > kMaxTileN) t = kMaxTileN;
  if (t > 128 && (long long)T * k <= 96LL * E) t = 128;
  return t;
}
// the token chunk of a layer's grouped GEMMs
inline int gemm_chunk(const moe_desc& d, int T) { return chunk_tokens(T, d.k, d.E); }

// Split of the router's reduction over H into S partial sums (summed in a
// fixed order by the top-k kernel).  Depends on T only, so a masked layer and
// its sliced twin compute bit-identical logits.
int router_splits(int T);

// Device scratch carved from the caller's workspace.
struct Workspace {
  float* logits;      // [S, T, E] partial router logits
  int32_t* chunk_hist;  // [NC, E] pairs per expert per chunk (then chunk bases)
  int32_t* counts;    // [E]
  int32_t* offsets;   // [E + 1] start of each expert in the sorted order
  int32_t* touched;   // [E] experts with count > 0, ascending; touched[E] unused
  int32_t* meta;      // [16] device scalars: [0] touched experts, [1] valid pairs, [2] token groups,
                      //       [3] token chunks, [8] / [9] unit counters of the gate/up and down GEMMs,
                      //       [10] finished CTAs of the fused decode top-k
  int32_t* group_base;  // [E + 1] first token group of each touched expert (touched order)
  int32_t* tile_base;   // [E + 1] first token chunk of each touched expert
  int32_t* sorted_pair;  // [P] pair id (t * k + slot) at each sorted position
  void* hbuf;         // [P, I] activations between the two projections (bf16, or fp32 for fp32 weights)
  float* yp;          // [P, H] per-pair expert outputs times routing weight, indexed by pair id
                      //         (fp32; bf16 -- in the first half of the area -- when yp_bf16())
  void* xs;           // [P, H] bf16 tokens gathered in sorted order (tensor-core path)
  void* w3;           // [E, 3H] bf16 three-way split of W_r (tensor-core router)
  size_t total;
};

// forward_only: the layout of a forward pass given its routing, without the
// router-only regions (logits and w3 are then unusable)
Workspace carve_workspace(const moe_desc& d, int32_t T, void* base, bool forward_only = false);
// bytes of that forward-only layout
size_t forward_scratch_bytes(const moe_desc& d, int32_t T);
// moe_forward on a workspace of the full (forward_only = false) or the
// forward-only layout
moe_status forward_impl(const moe_desc* d, const void* x, int32_t T, const int32_t* topk_idx, const float* topk_w,
                        void* y, void* workspace, size_t ws_bytes, cudaStream_t stream, bool forward_only);

// set the calling thread's moe_last_error() message and return `code`
moe_status report_error(moe_status code, const char* message);

// launch bookkeeping (counting + optional event timing), defined in moe_api.cu
cudaError_t launch_done(const char* name, cudaStream_t s, void* begin_event);
void* launch_start(const char* name, cudaStream_t s);

// ---- launchers (each enqueues exactly one kernel) ----
cudaError_t launch_router_logits(const moe_desc& d, const void* x, int T, float* partial, int S,
                                 cudaStream_t s);
cudaError_t launch_router_topk(const moe_desc& d, const float* partial, int S, int T, int32_t* idx,
                               float* w, uint32_t* flags, cudaStream_t s);
// logits [T, E] = the S partials [S, T, E] summed in split order (as the top-k does)
cudaError_t launch_logits_sum(const float* partial, int S, int T, int E, float* logits, int num_sms,
                              cudaStream_t s);
bool small_sort_ok(int P, int E);
cudaError_t launch_small_sort(const int32_t* idx, int P, int E, int chunk, int32_t* counts, int32_t* offsets,
                              int32_t* touched, int32_t* group_base, int32_t* tile_base, int32_t* meta,
                              int32_t* sorted_pair, uint32_t* flags, cudaStream_t s);
cudaError_t launch_pair_histogram(const int32_t* idx, int P, int E, int32_t* chunk_hist,
                                  uint32_t* flags, cudaStream_t s);
cudaError_t launch_expert_scan(int NC, int E, int32_t* chunk_hist, int32_t* counts, int32_t* offsets,
                               int32_t* touched, int32_t* group_base, int32_t* tile_base, int chunk,
                               int32_t* meta, cudaStream_t s);
cudaError_t launch_pair_scatter(const int32_t* idx, int P, int E, const int32_t* chunk_hist,
                                int32_t* sorted_pair, cudaStream_t s);
cudaError_t launch_gemv_gateup(const moe_desc& d, const void* x, int k, const Workspace& ws,
                               int num_sms, uint32_t* flags, cudaStream_t s);
cudaError_t launch_gemv_down(const moe_desc& d, const float* topk_w, int k, const Workspace& ws,
                             int num_sms, uint32_t* flags, cudaStream_t s);
bool gemm_tc_supported(const moe_desc& d);
bool router_tc_supported(const moe_desc& d);
int router_tc_splits(int T, int H);
cudaError_t launch_router_split3(const moe_desc& d, void* W3, int num_sms, cudaStream_t s);
cudaError_t launch_router_tc(const moe_desc& d, const void* x, int T, const void* W3, float* partial, int S,
                             int num_sms, uint32_t* flags, cudaStream_t s);
cudaError_t launch_gather_rows(const moe_desc& d, const void* x, const Workspace& ws, int P, int num_sms,
                               cudaStream_t s);
// An optional second, dense problem run in the same grouped-GEMM launch (the
// shared expert): the one-expert layer *d applied to T token rows in order with
// weight 1; b = its input rows (gate/up: x [T, H]; down: its h [T, I]), out = its
// output rows (gate/up: h [T, I] bf16; down: [T, H] fp32); chunk its token chunk.
struct DenseGemm {
  const moe_desc* d;
  const void* b;
  void* out;
  int T;
  int chunk;
};
cudaError_t launch_gemm_gateup(const moe_desc& d, const Workspace& ws, int P, int chunk, int num_sms,
                               uint32_t* flags, cudaStream_t s, const DenseGemm* dg = nullptr);
cudaError_t launch_gemm_down(const moe_desc& d, const float* topk_w, const Workspace& ws, int P, int chunk,
                             int num_sms, uint32_t* flags, cudaStream_t s, const DenseGemm* dg = nullptr,
                             bool yp_bf16 = false);
// Large bf16 batches on the tensor-core path keep the per-pair expert outputs in
// bf16 (fp32 accumulation, one rounding): half the down projection's output
// bytes and half the combine's reads, where that traffic is a visible share of
// the layer.  Smaller batches keep them in fp32.
constexpr int kYpBf16MinT = 2048;
inline bool yp_bf16(const moe_desc& d, int T, int path) {
  return path == MOE_PATH_GEMM && d.xfmt == MOE_X_BF16 && T >= kYpBf16MinT;
}
// decode-sized batches (T <= 32): fp32 logits in one launch; with E <= 256 and
// T*k <= 8192 also top-k and the expert sort in one launch
bool decode_route_ok(const moe_desc& d, int T);
bool fused_route_sort_ok(const moe_desc& d, int T);
int decode_logit_splits(const moe_desc& d, int T);  // S: partial sums per logit (1, 2, 4 or 8)
// topk_done (optional): the fused top-k's completion counter, zeroed by this launch
constexpr int kMetaTopkDone = 10;
cudaError_t launch_decode_logits(const moe_desc& d, const void* x, int T, float* partial, int S, uint32_t* flags,
                                 cudaStream_t s, int32_t* topk_done = nullptr);
cudaError_t launch_topk_sort(const moe_desc& d, const float* partial, int S, int T, int32_t* idx, float* w,
                             int chunk, const Workspace& ws, uint32_t* flags, cudaStream_t s);
cudaError_t launch_expert_counts(const int32_t* idx, int64_t n, int E, uint64_t* counts, int num_sms,
                                 cudaStream_t s);
cudaError_t launch_combine(const moe_desc& d, const int32_t* idx, int T, const void* yp, bool yp_bf16, void* y,
                           cudaStream_t s, const float* ys = nullptr, const void* residual = nullptr);
cudaError_t launch_dense_plan(int T, int chunk, int32_t* counts, int32_t* offsets, int32_t* touched,
                              int32_t* group_base, int32_t* tile_base, int32_t* meta, int32_t* sorted_pair,
                              float* ones, cudaStream_t s);

}  // namespace moe
