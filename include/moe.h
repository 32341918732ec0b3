/*
 * moe.h -- C ABI of the B200 (sm_100a) routed mixture-of-experts layer.
 *
 * The layer, as the pages describe it:
 *   router   logits = W_r x (fp32); sigmoid scores with a selection bias, the
 *            top k chosen on score + bias, weights = the chosen SCORES
 *            renormalised and multiplied by a scale (2.446 for Kimi-Linear) --
 *            Kimi-Linear-48B-A3B LiteRT-LM details page, Conversion notes,
 *            mixture-of-experts bullet; the CMF code specialist page, step 1,
 *            names the same sigmoid router and its selection bias.  Or softmax,
 *            top k, renormalise (Qwen3-30B-A3B LiteRT-LM card, Conversion Notes).
 *   experts  only the k routed experts run for a token; each is a SiLU-gated
 *            FFN  o = W_down (SiLU(W_gate x) * (W_up x))  (Qwen3 card,
 *            Conversion Notes; the moe op's activation 'silu').
 *   combine  y = sum over the k slots of weight * o, in slot order.  The
 *            residual add stays outside the op (Qwen3 card, moe_fusion_guard
 *            bullet).
 *   storage  experts fp32, bf16, int8 with one fp32 scale per output row and
 *            expert (Kimi details page, quantization bullet), or int4 in blocks
 *            of 32 along the reduction axis with fp32 scales (Qwen3 card,
 *            Available Artifacts table).
 *   mask     an optional runtime expert mask: masked experts are never chosen;
 *            this equals slicing the router rows, the bias and the experts
 *            (CMF page, Defrag step).
 *
 * Conventions for every entry point:
 *   - All tensor pointers are DEVICE pointers owned by the caller, row-major,
 *     and must be 16-byte aligned (the workspace 256-byte aligned).  Nothing
 *     is allocated by moe_route / moe_forward: scratch comes from the caller's
 *     workspace (size from moe_workspace_size).
 *   - Work is enqueued asynchronously on `stream`; no entry point synchronises
 *     except moe_device_flags and moe_stage_times (documented there).
 *   - Arguments are validated on the host before anything is launched; a
 *     non-OK status means nothing was enqueued, and moe_last_error() returns a
 *     message for the calling thread.
 *   - Problems found in DATA on the device (an expert index out of range in
 *     caller-provided routing, fewer than k selectable experts, a non-finite
 *     router logit) cannot be reported synchronously; kernels set bits in a
 *     per-device sticky word read by moe_device_flags().  No kernel traps, and
 *     every wait inside a kernel is bounded in time (MOE_FLAG_TIMEOUT).
 *   - The current CUDA device is the one the pointers live on.
 */
#ifndef MOE_B200_H
#define MOE_B200_H

#include <stddef.h>
#include <stdint.h>

#include <cuda_runtime_api.h>

#if defined(__GNUC__)
#define MOE_API __attribute__((visibility("default")))
#else
#define MOE_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = 1,  /* null/misaligned pointer, bad size or enum value */
  MOE_ERR_UNSUPPORTED = 2,  /* valid but not built: e.g. an activation other than SiLU */
  MOE_ERR_WORKSPACE = 3,    /* workspace missing or smaller than moe_workspace_size */
  MOE_ERR_CUDA = 4          /* a CUDA launch or runtime call failed */
} moe_status;

typedef enum {
  MOE_ROUTER_SIGMOID_BIAS = 0, /* key = sigmoid(l) + b, weight from sigmoid(l) */
  MOE_ROUTER_SOFTMAX = 1       /* key = softmax(l) over active experts */
} moe_router_kind;

typedef enum {
  MOE_W_F32 = 0,
  MOE_W_BF16 = 1,
  MOE_W_INT8_ROW = 2, /* int8, one fp32 scale per (expert, output row) */
  MOE_W_INT4_B32 = 3, /* int4 two's complement, 2 per byte (low nibble = even
                         column), one fp32 scale per 32 columns */
  MOE_W_INT4_B128 = 4 /* the same nibbles, one fp32 scale per 128 columns (the
                         128-wide expert blocks of the Qwen3-30B-A3B LiteRT-LM
                         card's int4 notes); H and I multiples of 128 */
} moe_wfmt;

typedef enum { MOE_X_F32 = 0, MOE_X_BF16 = 1 } moe_xfmt;

typedef enum {
  MOE_ACT_SILU = 0,     /* h = g * sigmoid(g) * u */
  MOE_ACT_GELU_TANH = 1 /* h = g/2 * (1 + tanh(sqrt(2/pi) (g + 0.044715 g^3))) * u: the
                           moe op's other activation, 'gelu_tanh' (Kimi-Linear details
                           page, Runtime; Qwen3 card, Conversion Notes) */
} moe_act;

typedef enum {
  MOE_PATH_AUTO = 0, /* pick by tokens per expert and formats */
  MOE_PATH_GEMV = 1, /* weight-streaming split GEMV (any format) */
  MOE_PATH_GEMM = 2  /* tcgen05 grouped GEMM (bf16 x; bf16/int8/int4 weights) */
} moe_path;

/*
 * Layer description.  Shapes: x [T, H]; W_r [E, H] fp32; b [E] fp32 or NULL
 * (zero bias); expert_mask [E] uint8 (1 = active) or NULL (all active).
 *   W_gate, W_up : [E, I, H]   (int4: [E, I, H/2] bytes)
 *   W_down       : [E, H, I]   (int4: [E, H, I/2] bytes)
 *   s_gate, s_up : int8 [E, I];  int4 [E, I, H/32] (block 128: H/128);  otherwise NULL
 *   s_down       : int8 [E, H];  int4 [E, H, I/32] (block 128: I/128);  otherwise NULL
 * Limits: H, I multiples of 64 (of 128 for int4 block 128); 1 <= k <= 32;
 * k <= E <= 1024.
 */
typedef struct {
  int32_t H, I, E, k;
  int32_t router; /* moe_router_kind */
  int32_t act;    /* moe_act */
  int32_t wfmt;   /* moe_wfmt */
  int32_t xfmt;   /* moe_xfmt (also the dtype of y) */
  int32_t path;   /* moe_path */
  float scale;    /* multiplies the renormalised weights: 2.446 Kimi, 1 Qwen3 */
  const float* W_r;
  const float* b;
  const uint8_t* expert_mask;
  const void* W_gate;
  const void* W_up;
  const void* W_down;
  const float* s_gate;
  const float* s_up;
  const float* s_down;
} moe_desc;

/* Bytes of workspace moe_route and moe_forward need for T tokens (one buffer
 * serves both; calls on one stream may reuse it). */
MOE_API moe_status moe_workspace_size(const moe_desc* d, int32_t T, size_t* bytes);

/*
 * Router: topk_idx [T, k] int32 and topk_w [T, k] fp32, slots in descending
 * key order with ties to the lower expert index.  Logits are fp32 sums; the
 * softmax router selects on the logits, whose order equals the softmax's.
 * Tokens with fewer than k selectable experts get idx -1 / w 0 in the
 * unfilled slots and raise MOE_FLAG_TOO_FEW_ACTIVE.
 */
MOE_API moe_status moe_route(const moe_desc* d, const void* x, int32_t T, int32_t* topk_idx, float* topk_w,
                     void* workspace, size_t ws_bytes, cudaStream_t stream);

/*
 * The router logits l = W_r x that moe_route ranks: logits [T, E] fp32
 * (row-major, 4-byte aligned, caller-owned; every expert, masked ones too --
 * the mask acts on the keys, not on the logits).  Computed by the same kernels
 * moe_route runs for this T, with the partial sums added in the same fixed
 * order, so the values are exactly the ones moe_route (and moe_layer_forward)
 * form their keys from: sigmoid(l) + b, or l itself for the softmax router
 * (the router step of the Kimi-Linear LiteRT-LM details page, Conversion notes,
 * and of the Qwen3-30B-A3B LiteRT-LM card, Conversion Notes).  For callers that
 * need the logits themselves (auxiliary router losses, calibration) and for
 * checking the routing against an exact reference.  Workspace as for
 * moe_route; asynchronous on `stream`; errors as for moe_route.
 */
MOE_API moe_status moe_route_logits(const moe_desc* d, const void* x, int32_t T, float* logits, void* workspace,
                                    size_t ws_bytes, cudaStream_t stream);

/*
 * Experts + combine under a given routing (from moe_route or the caller):
 * y [T, H] in x's dtype, y[t] = sum_j topk_w[t, j] * FFN_{topk_idx[t, j]}(x[t])
 * summed in slot order in fp32, rounded once.  Slots whose index is outside
 * [0, E) contribute nothing and raise MOE_FLAG_BAD_EXPERT_INDEX.
 */
MOE_API moe_status moe_forward(const moe_desc* d, const void* x, int32_t T, const int32_t* topk_idx,
                       const float* topk_w, void* y, void* workspace, size_t ws_bytes,
                       cudaStream_t stream);

/*
 * moe_forward without a workspace argument, for callers that cannot allocate
 * device memory: a plugin host that owns every device buffer and hands the
 * library no allocator, or a latency-bound loop that must not call cudaMalloc
 * (which can synchronise the device) once it runs.  The pages describe no
 * such entry point; it has no counterpart there.
 *
 * Scratch comes from one static device array of MOE_NOALLOC_SCRATCH_BYTES
 * that this library holds on every GPU that loads it, until the process
 * exits.  Inputs and outputs are still the caller's, exactly as for
 * moe_forward, and the result is bit for bit moe_forward's (the same kernels
 * on the same data).  The forward pass alone needs less than
 * moe_workspace_size reports (that size also covers moe_route's logits and
 * its split router weights): sorted pairs, per-expert counts, the activations
 * between the projections and the per-pair outputs, about
 * T * k * (4 + 2 I + 6 H) bytes with bf16 activations -- some 115 tokens at
 * H = 2304, I = 2048, k = 8.  Larger problems are rejected with
 * MOE_ERR_WORKSPACE and a message naming both sizes; nothing is launched then.
 * No cudaMalloc/cudaFree or other allocating call is made (leave
 * moe_stage_timing off: the timing itself creates CUDA events).
 *
 * The first call on a device looks up the array's device address
 * (cudaGetSymbolAddress) with that device current; make that first call
 * before any stream capture.  Every call shares the one array and it keeps
 * the previous call's contents (nothing in it needs to start at zero: each
 * call writes what it reads), so calls whose work overlaps on the GPU --
 * several streams, or several host threads -- race on it and give wrong
 * results; order them on one stream.
 */
#define MOE_NOALLOC_SCRATCH_BYTES (16u << 20)
MOE_API moe_status moe_forward_noalloc(const moe_desc* d, const void* x, int32_t T, const int32_t* topk_idx,
                                       const float* topk_w, void* y, cudaStream_t stream);

/*
 * Route and forward in one call: the same results as moe_route followed by
 * moe_forward on the same arguments (topk_idx and topk_w are outputs here, as
 * for moe_route; the workspace is moe_workspace_size's).  Because the library
 * builds the routing itself, decode-sized batches (T <= 32, E <= 256) compute
 * the router logits in one kernel and the top-k together with the expert sort
 * in a second one, instead of four launches.  Larger batches run the two steps
 * as the separate entry points do.
 */
MOE_API moe_status moe_layer_forward(const moe_desc* d, const void* x, int32_t T, int32_t* topk_idx, float* topk_w,
                                     void* y, void* workspace, size_t ws_bytes, cudaStream_t stream);

/*
 * The whole MoE block: routed experts + shared expert + residual.
 *
 *   y[t] = sum_j w[t,j] FFN_{idx[t,j]}(x[t])  +  FFN_shared(x[t])  +  residual[t]
 *
 * The shared expert is one more gated FFN applied to every token with weight 1
 * (the Kimi-Linear APEX quantization page lists 256 routed experts and one shared one;
 * the shared expert runs beside the moe op -- Kimi-Linear LiteRT-LM details
 * page, Conversion notes).  It uses the routed experts' activation (d->act) and
 * activation dtype; its own intermediate size I and storage format.  The
 * residual add belongs to the block, outside the moe op (Qwen3-30B-A3B LiteRT-LM
 * card, Conversion Notes, moe_fusion_guard bullet); it is fused here into the
 * combine: after the k routed rows (slot order) the shared row and then the
 * residual are added in fp32, with one rounding to y's dtype.
 *
 * moe_shared_expert: weights of one expert in the layouts of moe_desc with E=1:
 *   W_gate, W_up [I, H] (int4: [I, H/2]); W_down [H, I] (int4: [H, I/2]);
 *   scales as for one routed expert of the same format, else NULL.
 *   I: multiple of 64 (of 128 for int4 block 128), <= 8192.
 * moe_block_workspace_size: bytes of device workspace moe_forward_block needs
 *   (256-byte aligned); shared may be NULL.
 * moe_forward_block: as moe_forward, plus shared (NULL: no shared expert) and
 *   residual ([T, H] in x's format, 16-byte aligned, or NULL: no residual).
 *   With both NULL the result equals moe_forward's bit for bit.  y may alias
 *   residual (each element is read before it is written, by the same thread).
 */
typedef struct {
  int32_t I;
  int32_t wfmt; /* moe_wfmt */
  const void* W_gate;
  const void* W_up;
  const void* W_down;
  const float* s_gate;
  const float* s_up;
  const float* s_down;
} moe_shared_expert;

MOE_API moe_status moe_block_workspace_size(const moe_desc* d, const moe_shared_expert* shared, int32_t T,
                                            size_t* bytes);
MOE_API moe_status moe_forward_block(const moe_desc* d, const moe_shared_expert* shared, const void* x, int32_t T,
                                     const int32_t* topk_idx, const float* topk_w, const void* residual, void* y,
                                     void* workspace, size_t ws_bytes, cudaStream_t stream);

/*
 * Routing statistics (CMF code specialist page, How it was made: Calibrate and
 * Defrag steps).
 *
 * moe_expert_counts: per-expert routing frequencies, accumulated across calls.
 *   topk_idx [T, k] int32 (device; routing from moe_route or the caller),
 *   counts [E] uint64 (device, caller-owned and zeroed once by the caller; each
 *   call adds, for every expert e, the number of entries of topk_idx equal to
 *   e).  Entries outside [0, E) are skipped, not flagged.  Only d->E and d->k
 *   are read from the descriptor.  Asynchronous on `stream`.  The adds are
 *   integer atomics, so calls adding into the same counts from several streams
 *   give the exact total in any order.
 *
 * moe_cover_set: host utility for the Defrag step.  counts [E] (HOST memory),
 *   cover in (0, 1].  Keeps the smallest set of experts whose counts reach
 *   cover * (sum of counts), taking experts by count descending with ties to
 *   the lower index.  Writes keep [E] (HOST, 1 = kept: usable directly as
 *   moe_desc.expert_mask once copied to the device), new_index [E] (HOST, the
 *   kept expert's position in the dense prefix that keeps the original index
 *   order, -1 for dropped experts; router rows, selection bias and experts are
 *   sliced in this order) and *n_keep.  All-zero counts keep no expert.
 *   Synchronous, no device work.
 */
MOE_API moe_status moe_expert_counts(const moe_desc* d, const int32_t* topk_idx, int32_t T, uint64_t* counts,
                                     cudaStream_t stream);
MOE_API moe_status moe_cover_set(const uint64_t* counts, int32_t E, double cover, uint8_t* keep,
                                 int32_t* new_index, int32_t* n_keep);

/*
 * Diagnostic (the pages have no counterpart): launches one small kernel whose
 * only waiting thread waits on a barrier that nothing completes.  After the
 * library's in-kernel wait bound (2 s of GPU time) it gives up, raises
 * MOE_FLAG_TIMEOUT in the device flags and returns; the context stays usable.
 * Shows on a given device that the library's waits end by themselves.
 * Asynchronous; read the result with moe_device_flags().
 */
MOE_API moe_status moe_selftest_bounded_wait(cudaStream_t stream);

/* Message for the last non-OK status returned on this thread ("" if none). */
MOE_API const char* moe_last_error(void);

/* Device data-error flags (bits below) of the current device.  Synchronises
 * the device.  clear != 0 resets the word after reading. */
#define MOE_FLAG_BAD_EXPERT_INDEX 0x1u
#define MOE_FLAG_TOO_FEW_ACTIVE 0x2u
#define MOE_FLAG_NONFINITE_LOGIT 0x4u
#define MOE_FLAG_TIMEOUT 0x8u /* a kernel's bounded wait expired; its outputs are incomplete */
MOE_API moe_status moe_device_flags(uint32_t* flags, int32_t clear);

/* Number of kernels this library has launched in this process. */
MOE_API uint64_t moe_launch_count(void);

/*
 * Optional per-kernel timing: when enabled, every kernel launch is bracketed
 * by CUDA events on its stream.  moe_stage_times() waits for those events and
 * returns, per kernel name, the number of launches and the summed duration in
 * ms since the previous call (then resets).  Off by default.
 */
typedef struct {
  char name[32];
  int32_t launches;
  float total_ms;
} moe_stage_time;
MOE_API moe_status moe_stage_timing(int32_t enable);
MOE_API moe_status moe_stage_times(moe_stage_time* out, int32_t capacity, int32_t* count);

/*
 * Restricts the per-kernel timing above to launches whose kernel name equals
 * `name` (at most 31 characters; NULL or "" times every launch again).  Each
 * timed launch adds two event records to its stream, and they cost time
 * between kernels; timing one kernel keeps that cost off the others.
 * Errors: MOE_ERR_INVALID_ARG if the name is too long.
 */
MOE_API moe_status moe_stage_timing_only(const char* name);

#ifdef __cplusplus
}
#endif
#endif /* MOE_B200_H */
