// C ABI of the routed-MoE library: argument validation, workspace carving,
// kernel dispatch, error reporting, launch accounting and optional per-kernel
// event timing.  Every step of the layer runs in this library's kernels; there
// is no host compute path.
#include <cuda_runtime.h>
#include <math.h>
#include <stdarg.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include <algorithm>
#include <atomic>
#include <mutex>
#include <string>
#include <vector>

#include <nvtx3/nvToolsExt.h>

#include "common.cuh"
#include "internal.h"
#include "moe.h"

namespace moe {

// ------------------------------------------------------------------ errors

static thread_local std::string g_err;

static moe_status fail(moe_status code, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_err = buf;
  return code;
}

moe_status report_error(moe_status code, const char* message) { return fail(code, "%s", message); }

static moe_status cuda_fail(cudaError_t e, const char* what) {
  return fail(MOE_ERR_CUDA, "%s: %s (%s)", what, cudaGetErrorName(e), cudaGetErrorString(e));
}

// ------------------------------------------------------------------ per-device state

static __device__ uint32_t g_device_flags;

struct DeviceState {
  bool ready = false;
  int num_sms = 0;
  uint32_t* flags = nullptr;  // device address of g_device_flags on this device
};
static std::mutex g_dev_mu;
static DeviceState g_dev[64];

static moe_status device_state(DeviceState** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= 64) return fail(MOE_ERR_UNSUPPORTED, "device ordinal %d out of range", dev);
  std::lock_guard<std::mutex> lk(g_dev_mu);
  DeviceState& st = g_dev[dev];
  if (!st.ready) {
    e = cudaDeviceGetAttribute(&st.num_sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceGetAttribute");
    e = cudaGetSymbolAddress(reinterpret_cast<void**>(&st.flags), g_device_flags);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(device flags)");
    st.ready = true;
  }
  *out = &st;
  return MOE_OK;
}

// ------------------------------------------------------------------ launch accounting

static std::atomic<uint64_t> g_launches{0};
static std::atomic<int> g_timing{0};

// Programmatic dependent launch is opt-in: MOE_PDL=1 in the environment (read
// once per process).  Plain stream ordering is the default.
bool pdl_enabled() {
  static const bool on = [] {
    const char* v = getenv("MOE_PDL");
    return v != nullptr && v[0] == '1';
  }();
  return on;
}
static char g_timing_only[32] = {0};  // "" = every launch; guarded by g_time_mu

struct Pending {
  char name[32];
  cudaEvent_t begin, end;
};
static std::mutex g_time_mu;
static std::vector<Pending> g_pending;
static std::vector<cudaEvent_t> g_event_pool;

static cudaEvent_t pool_event() {
  if (!g_event_pool.empty()) {
    cudaEvent_t ev = g_event_pool.back();
    g_event_pool.pop_back();
    return ev;
  }
  cudaEvent_t ev = nullptr;
  cudaEventCreate(&ev);
  return ev;
}

// every launch sits in an NVTX range named after the kernel's stage (visible to
// profilers; a no-op without one attached)
void* launch_start(const char* name, cudaStream_t s) {
  nvtxRangePushA(name);
  if (!g_timing.load(std::memory_order_relaxed)) return nullptr;
  std::lock_guard<std::mutex> lk(g_time_mu);
  if (g_timing_only[0] != 0 && strncmp(name, g_timing_only, sizeof(g_timing_only)) != 0) return nullptr;
  cudaEvent_t ev = pool_event();
  if (ev) cudaEventRecord(ev, s);
  return ev;
}

cudaError_t launch_done(const char* name, cudaStream_t s, void* begin_event) {
  cudaError_t err = cudaGetLastError();
  nvtxRangePop();
  g_launches.fetch_add(1, std::memory_order_relaxed);
  if (begin_event) {
    std::lock_guard<std::mutex> lk(g_time_mu);
    Pending p;
    snprintf(p.name, sizeof(p.name), "%s", name);
    p.begin = static_cast<cudaEvent_t>(begin_event);
    p.end = pool_event();
    if (p.end) {
      cudaEventRecord(p.end, s);
      g_pending.push_back(p);
    } else {
      g_event_pool.push_back(p.begin);
    }
  }
  return err;
}

#define MOE_LAUNCH(name, stream, call)                         \
  do {                                                         \
    void* _ev = launch_start(name, stream);                    \
    cudaError_t _e1 = (call);                                  \
    cudaError_t _e2 = launch_done(name, stream, _ev);          \
    if (_e1 != cudaSuccess) return cuda_fail(_e1, name);       \
    if (_e2 != cudaSuccess) return cuda_fail(_e2, name);       \
  } while (0)

// ------------------------------------------------------------------ validation

static bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

static moe_status validate_desc(const moe_desc* d) {
  if (!d) return fail(MOE_ERR_INVALID_ARG, "desc is NULL");
  if (d->H <= 0 || d->I <= 0 || d->E <= 0 || d->k <= 0)
    return fail(MOE_ERR_INVALID_ARG, "H, I, E, k must be positive (got %d, %d, %d, %d)", d->H, d->I, d->E, d->k);
  if (d->H % 64 || d->I % 64) return fail(MOE_ERR_INVALID_ARG, "H and I must be multiples of 64 (got %d, %d)", d->H, d->I);
  if (d->H > 8192 || d->I > 8192) return fail(MOE_ERR_UNSUPPORTED, "H and I are limited to 8192 (got %d, %d)", d->H, d->I);
  if (d->E > 1024) return fail(MOE_ERR_UNSUPPORTED, "E is limited to 1024 (got %d)", d->E);
  if (d->k > 32 || d->k > d->E) return fail(MOE_ERR_INVALID_ARG, "k must be <= min(E, 32) (got k=%d, E=%d)", d->k, d->E);
  if (d->router != MOE_ROUTER_SIGMOID_BIAS && d->router != MOE_ROUTER_SOFTMAX)
    return fail(MOE_ERR_INVALID_ARG, "unknown router kind %d", d->router);
  if (d->act != MOE_ACT_SILU && d->act != MOE_ACT_GELU_TANH)
    return fail(MOE_ERR_INVALID_ARG, "unknown activation %d", d->act);
  if (d->wfmt < MOE_W_F32 || d->wfmt > MOE_W_INT4_B128) return fail(MOE_ERR_INVALID_ARG, "unknown weight format %d", d->wfmt);
  if (d->wfmt == MOE_W_INT4_B128 && (d->H % 128 || d->I % 128))
    return fail(MOE_ERR_INVALID_ARG, "int4 block-128 weights need H and I multiples of 128 (got %d, %d)", d->H, d->I);
  if (d->xfmt != MOE_X_F32 && d->xfmt != MOE_X_BF16) return fail(MOE_ERR_INVALID_ARG, "unknown activation dtype %d", d->xfmt);
  if (d->path < MOE_PATH_AUTO || d->path > MOE_PATH_GEMM) return fail(MOE_ERR_INVALID_ARG, "unknown path %d", d->path);
  if (!isfinite(d->scale)) return fail(MOE_ERR_INVALID_ARG, "scale must be finite");
  if (!d->W_r || !aligned(d->W_r, 16)) return fail(MOE_ERR_INVALID_ARG, "W_r must be a non-NULL 16-byte aligned device pointer");
  if (!d->W_gate || !d->W_up || !d->W_down)
    return fail(MOE_ERR_INVALID_ARG, "W_gate, W_up and W_down must be non-NULL");
  if (!aligned(d->W_gate, 16) || !aligned(d->W_up, 16) || !aligned(d->W_down, 16))
    return fail(MOE_ERR_INVALID_ARG, "expert weights must be 16-byte aligned");
  const bool scaled = d->wfmt != MOE_W_F32 && d->wfmt != MOE_W_BF16;
  if (scaled && (!d->s_gate || !d->s_up || !d->s_down))
    return fail(MOE_ERR_INVALID_ARG, "int8/int4 weights need s_gate, s_up and s_down");
  if (scaled && (!aligned(d->s_gate, 4) || !aligned(d->s_up, 4) || !aligned(d->s_down, 4)))
    return fail(MOE_ERR_INVALID_ARG, "scales must be 4-byte aligned");
  return MOE_OK;
}

static moe_status validate_T(int32_t T, int k) {
  if (T < 0) return fail(MOE_ERR_INVALID_ARG, "T must be >= 0 (got %d)", T);
  if ((int64_t)T * k > (int64_t)1 << 30) return fail(MOE_ERR_UNSUPPORTED, "T*k above 2^30 (got T=%d, k=%d)", T, k);
  return MOE_OK;
}

// The tensor-core path needs bf16 activations, non-fp32 weights and 128-row tiles.
static bool gemm_capable(const moe_desc& d) { return gemm_tc_supported(d); }

// The path by tokens per expert.  The tensor-core GEMM streams the weights with
// TMA and serves decode as well as prefill; the SIMT weight-streaming GEMV serves
// fp32 layers, shapes the tensor cores cannot tile, and the smallest int4 batches:
// with at most one (token, slot) pair per kGemvPairsPerExpertInt4 experts on
// average the GEMV widens only the rows it multiplies (and no token tiles),
// which measured faster than the GEMM's full-tile dequantisation (1-4 tokens at
// the Qwen3-30B-A3B widths).  bf16 and int8 weights take the GEMM at every batch
// size: it measured at least as fast from one token up.
constexpr int kGemvPairsPerExpertInt4 = 4;  // GEMV while T * k * 4 <= E
static int choose_path(const moe_desc& d, int32_t T) {
  if (d.path == MOE_PATH_GEMV) return MOE_PATH_GEMV;
  if (d.path == MOE_PATH_GEMM) return MOE_PATH_GEMM;
  if (!gemm_capable(d)) return MOE_PATH_GEMV;
  const bool int4 = d.wfmt == MOE_W_INT4_B32 || d.wfmt == MOE_W_INT4_B128;
  if (int4 && (int64_t)T * d.k * kGemvPairsPerExpertInt4 <= d.E) return MOE_PATH_GEMV;
  return MOE_PATH_GEMM;
}

// ------------------------------------------------------------------ workspace

static size_t up256(size_t v) { return (v + 255) / 256 * 256; }

constexpr int kRegions = 13;

// forward_only: the router-only regions (partial logits, split router weights)
// take no space -- the layout of a forward pass that is given its routing
static void layout(const moe_desc& d, int32_t T, size_t off[kRegions], size_t* total, bool forward_only = false) {
  const size_t P = (size_t)T * d.k, E = d.E;
  const size_t S_simt = router_splits(T), S_tc = d.xfmt == MOE_X_BF16 ? router_tc_splits(T, d.H) : 0;
  size_t S = S_simt > S_tc ? S_simt : S_tc;
  if (T <= 32 && S < 8) S = 8;  // the decode router's splits (at most 8)
  const size_t w3_bytes = d.xfmt == MOE_X_BF16 ? (size_t)d.E * 3 * d.H * 2 : 0;
  const size_t NC = (P + kPairChunk - 1) / kPairChunk;
  const size_t hbytes = d.wfmt == MOE_W_F32 ? 4 : 2;
  const size_t xs_bytes = (d.xfmt == MOE_X_BF16 && d.wfmt != MOE_W_F32) ? P * d.H * 2 : 0;
  const size_t sizes[kRegions] = {forward_only ? 0 : S * T * E * 4, (NC ? NC : 1) * E * 4, E * 4, (E + 1) * 4,
                                  (E + 1) * 4, 16 * 4, P * 4, P * d.I * hbytes, P * d.H * 4, xs_bytes, (E + 1) * 4,
                                  (E + 1) * 4, forward_only ? 0 : w3_bytes};
  size_t o = 0;
  for (int i = 0; i < kRegions; ++i) {
    off[i] = o;
    o += up256(sizes[i]);
  }
  *total = o;
}

Workspace carve_workspace(const moe_desc& d, int32_t T, void* base, bool forward_only) {
  size_t off[kRegions], total;
  layout(d, T, off, &total, forward_only);
  char* b = static_cast<char*>(base);
  Workspace w;
  w.logits = reinterpret_cast<float*>(b + off[0]);
  w.chunk_hist = reinterpret_cast<int32_t*>(b + off[1]);
  w.counts = reinterpret_cast<int32_t*>(b + off[2]);
  w.offsets = reinterpret_cast<int32_t*>(b + off[3]);
  w.touched = reinterpret_cast<int32_t*>(b + off[4]);
  w.meta = reinterpret_cast<int32_t*>(b + off[5]);
  w.sorted_pair = reinterpret_cast<int32_t*>(b + off[6]);
  w.hbuf = b + off[7];
  w.yp = reinterpret_cast<float*>(b + off[8]);
  w.xs = b + off[9];
  w.group_base = reinterpret_cast<int32_t*>(b + off[10]);
  w.tile_base = reinterpret_cast<int32_t*>(b + off[11]);
  w.w3 = b + off[12];
  w.total = total;
  return w;
}

size_t forward_scratch_bytes(const moe_desc& d, int32_t T) {
  size_t off[kRegions], need;
  layout(d, T, off, &need, true);
  return need;
}

static moe_status check_ws(const moe_desc& d, int32_t T, void* ws, size_t ws_bytes, bool forward_only = false) {
  size_t off[kRegions], need;
  layout(d, T, off, &need, forward_only);
  if (!ws) return fail(MOE_ERR_WORKSPACE, "workspace is NULL (need %zu bytes)", need);
  if (!aligned(ws, 256)) return fail(MOE_ERR_WORKSPACE, "workspace must be 256-byte aligned");
  if (ws_bytes < need) return fail(MOE_ERR_WORKSPACE, "workspace too small: %zu bytes given, %zu needed", ws_bytes, need);
  return MOE_OK;
}

}  // namespace moe

using namespace moe;

// ====================================================================== C ABI

extern "C" moe_status moe_workspace_size(const moe_desc* d, int32_t T, size_t* bytes) {
  g_err.clear();
  moe_status st = validate_desc(d);
  if (st != MOE_OK) return st;
  if ((st = validate_T(T, d->k)) != MOE_OK) return st;
  if (!bytes) return fail(MOE_ERR_INVALID_ARG, "bytes is NULL");
  size_t off[kRegions];
  layout(*d, T, off, bytes);
  return MOE_OK;
}

static moe_status route_partial_logits(const moe_desc* d, const void* x, int32_t T, const Workspace& ws,
                                       DeviceState* dev, cudaStream_t stream, int* S_out);

extern "C" moe_status moe_route(const moe_desc* d, const void* x, int32_t T, int32_t* topk_idx, float* topk_w,
                                void* workspace, size_t ws_bytes, cudaStream_t stream) {
  g_err.clear();
  moe_status st = validate_desc(d);
  if (st != MOE_OK) return st;
  if ((st = validate_T(T, d->k)) != MOE_OK) return st;
  if (T == 0) return MOE_OK;
  if (!x || !aligned(x, 16)) return fail(MOE_ERR_INVALID_ARG, "x must be a non-NULL 16-byte aligned device pointer");
  if (!topk_idx || !topk_w || !aligned(topk_idx, 4) || !aligned(topk_w, 4))
    return fail(MOE_ERR_INVALID_ARG, "topk_idx and topk_w must be non-NULL, 4-byte aligned");
  if ((st = check_ws(*d, T, workspace, ws_bytes)) != MOE_OK) return st;
  DeviceState* dev = nullptr;
  if ((st = device_state(&dev)) != MOE_OK) return st;
  const Workspace ws = carve_workspace(*d, T, workspace);
  int S = 0;
  if ((st = route_partial_logits(d, x, T, ws, dev, stream, &S)) != MOE_OK) return st;
  MOE_LAUNCH("router_topk", stream, launch_router_topk(*d, ws.logits, S, T, topk_idx, topk_w, dev->flags, stream));
  return MOE_OK;
}

extern "C" moe_status moe_route_logits(const moe_desc* d, const void* x, int32_t T, float* logits, void* workspace,
                                       size_t ws_bytes, cudaStream_t stream) {
  g_err.clear();
  moe_status st = validate_desc(d);
  if (st != MOE_OK) return st;
  if ((st = validate_T(T, d->k)) != MOE_OK) return st;
  if (T == 0) return MOE_OK;
  if (!x || !aligned(x, 16)) return fail(MOE_ERR_INVALID_ARG, "x must be a non-NULL 16-byte aligned device pointer");
  if (!logits || !aligned(logits, 4)) return fail(MOE_ERR_INVALID_ARG, "logits must be non-NULL, 4-byte aligned");
  if ((st = check_ws(*d, T, workspace, ws_bytes)) != MOE_OK) return st;
  DeviceState* dev = nullptr;
  if ((st = device_state(&dev)) != MOE_OK) return st;
  const Workspace ws = carve_workspace(*d, T, workspace);
  int S = 0;
  if ((st = route_partial_logits(d, x, T, ws, dev, stream, &S)) != MOE_OK) return st;
  MOE_LAUNCH("router_logits_sum", stream, launch_logits_sum(ws.logits, S, T, d->E, logits, dev->num_sms, stream));
  return MOE_OK;
}

// the router's partial logits [S, T, E] into ws.logits, by the kernels moe_route
// uses for this T; *S_out = S
static moe_status route_partial_logits(const moe_desc* d, const void* x, int32_t T, const Workspace& ws,
                                       DeviceState* dev, cudaStream_t stream, int* S_out) {
  int S;
  if (decode_route_ok(*d, T)) {
    // decode-sized batch: fp32 logits from fp32 W_r in one launch, every H-split
    // summed inside it
    S = decode_logit_splits(*d, T);
    MOE_LAUNCH("router_decode_logits", stream, launch_decode_logits(*d, x, T, ws.logits, S, dev->flags, stream));
  } else if (router_tc_supported(*d)) {
    // tensor cores: fp32-accurate logits from bf16 x against the exact three-way bf16 split of W_r
    S = router_tc_splits(T, d->H);
    MOE_LAUNCH("router_split3", stream, launch_router_split3(*d, ws.w3, dev->num_sms, stream));
    MOE_LAUNCH("router_logits_tc", stream,
               launch_router_tc(*d, x, T, ws.w3, ws.logits, S, dev->num_sms, dev->flags, stream));
  } else {
    S = router_splits(T);
    MOE_LAUNCH("router_logits", stream, launch_router_logits(*d, x, T, ws.logits, S, stream));
  }
  *S_out = S;
  return MOE_OK;
}

// the routed experts: expert-sorted order (unless already built), gate/up, down;
// leaves w * FFN rows in ws.yp (bf16 when yp_bf16(*d, T, path), else fp32)
static moe_status run_routed(const moe_desc* d, const void* x, int32_t T, const int32_t* topk_idx,
                             const float* topk_w, const Workspace& ws, int path, DeviceState* dev,
                             cudaStream_t stream, bool sorted = false, const DenseGemm* dense_up = nullptr,
                             const DenseGemm* dense_down = nullptr) {
  const int P = T * d->k;
  const int NC = (P + kPairChunk - 1) / kPairChunk;
  if (sorted) {
    // the plan was built together with the routing
  } else if (small_sort_ok(P, d->E)) {
    MOE_LAUNCH("small_sort", stream,
               launch_small_sort(topk_idx, P, d->E, gemm_chunk(*d, T), ws.counts, ws.offsets, ws.touched,
                                 ws.group_base, ws.tile_base, ws.meta, ws.sorted_pair, dev->flags, stream));
  } else {
    MOE_LAUNCH("pair_histogram", stream, launch_pair_histogram(topk_idx, P, d->E, ws.chunk_hist, dev->flags, stream));
    MOE_LAUNCH("expert_scan", stream,
               launch_expert_scan(NC, d->E, ws.chunk_hist, ws.counts, ws.offsets, ws.touched, ws.group_base,
                                  ws.tile_base, gemm_chunk(*d, T), ws.meta, stream));
    MOE_LAUNCH("pair_scatter", stream, launch_pair_scatter(topk_idx, P, d->E, ws.chunk_hist, ws.sorted_pair, stream));
  }
  if (path == MOE_PATH_GEMM) {
    MOE_LAUNCH("gather_rows", stream, launch_gather_rows(*d, x, ws, P, dev->num_sms, stream));
    const int chunk = gemm_chunk(*d, T);
    MOE_LAUNCH("gemm_gateup", stream,
               launch_gemm_gateup(*d, ws, P, chunk, dev->num_sms, dev->flags, stream, dense_up));
    MOE_LAUNCH("gemm_down", stream,
               launch_gemm_down(*d, topk_w, ws, P, chunk, dev->num_sms, dev->flags, stream, dense_down,
                                yp_bf16(*d, T, path)));
  } else {
    MOE_LAUNCH("gemv_gateup", stream, launch_gemv_gateup(*d, x, d->k, ws, dev->num_sms, dev->flags, stream));
    MOE_LAUNCH("gemv_down", stream, launch_gemv_down(*d, topk_w, d->k, ws, dev->num_sms, dev->flags, stream));
  }
  return MOE_OK;
}

static moe_status check_io(const void* x, const void* y, const int32_t* topk_idx, const float* topk_w) {
  if (!x || !aligned(x, 16)) return fail(MOE_ERR_INVALID_ARG, "x must be a non-NULL 16-byte aligned device pointer");
  if (!y || !aligned(y, 16)) return fail(MOE_ERR_INVALID_ARG, "y must be a non-NULL 16-byte aligned device pointer");
  if (!topk_idx || !topk_w || !aligned(topk_idx, 4) || !aligned(topk_w, 4))
    return fail(MOE_ERR_INVALID_ARG, "topk_idx and topk_w must be non-NULL, 4-byte aligned");
  return MOE_OK;
}

static const char* kNoTensorCores =
    "tensor-core path needs bf16 activations, bf16/int8/int4 weights and H, I multiples of 128";

// moe_forward's work; forward_only carves the workspace without the
// router-only regions (the layout forward_scratch_bytes sizes)
moe_status moe::forward_impl(const moe_desc* d, const void* x, int32_t T, const int32_t* topk_idx,
                             const float* topk_w, void* y, void* workspace, size_t ws_bytes, cudaStream_t stream,
                             bool forward_only) {
  g_err.clear();
  moe_status st = validate_desc(d);
  if (st != MOE_OK) return st;
  if ((st = validate_T(T, d->k)) != MOE_OK) return st;
  if (T == 0) return MOE_OK;
  if ((st = check_io(x, y, topk_idx, topk_w)) != MOE_OK) return st;
  if ((st = check_ws(*d, T, workspace, ws_bytes, forward_only)) != MOE_OK) return st;
  const int path = choose_path(*d, T);
  if (path == MOE_PATH_GEMM && !gemm_capable(*d)) return fail(MOE_ERR_UNSUPPORTED, "%s", kNoTensorCores);
  DeviceState* dev = nullptr;
  if ((st = device_state(&dev)) != MOE_OK) return st;
  const Workspace ws = carve_workspace(*d, T, workspace, forward_only);
  if ((st = run_routed(d, x, T, topk_idx, topk_w, ws, path, dev, stream)) != MOE_OK) return st;
  MOE_LAUNCH("combine", stream, launch_combine(*d, topk_idx, T, ws.yp, yp_bf16(*d, T, path), y, stream));
  return MOE_OK;
}

extern "C" moe_status moe_forward(const moe_desc* d, const void* x, int32_t T, const int32_t* topk_idx,
                                  const float* topk_w, void* y, void* workspace, size_t ws_bytes,
                                  cudaStream_t stream) {
  return forward_impl(d, x, T, topk_idx, topk_w, y, workspace, ws_bytes, stream, false);
}

// ------------------------------------------------------------------ route and forward in one call

extern "C" moe_status moe_layer_forward(const moe_desc* d, const void* x, int32_t T, int32_t* topk_idx,
                                        float* topk_w, void* y, void* workspace, size_t ws_bytes,
                                        cudaStream_t stream) {
  g_err.clear();
  moe_status st = validate_desc(d);
  if (st != MOE_OK) return st;
  if ((st = validate_T(T, d->k)) != MOE_OK) return st;
  if (!fused_route_sort_ok(*d, T)) {
    // larger batches: the two steps as moe_route and moe_forward run them
    if ((st = moe_route(d, x, T, topk_idx, topk_w, workspace, ws_bytes, stream)) != MOE_OK) return st;
    return moe_forward(d, x, T, topk_idx, topk_w, y, workspace, ws_bytes, stream);
  }
  if ((st = check_io(x, y, topk_idx, topk_w)) != MOE_OK) return st;
  if ((st = check_ws(*d, T, workspace, ws_bytes)) != MOE_OK) return st;
  const int path = choose_path(*d, T);
  if (path == MOE_PATH_GEMM && !gemm_capable(*d)) return fail(MOE_ERR_UNSUPPORTED, "%s", kNoTensorCores);
  DeviceState* dev = nullptr;
  if ((st = device_state(&dev)) != MOE_OK) return st;
  const Workspace ws = carve_workspace(*d, T, workspace);
  const int S = decode_logit_splits(*d, T);
  MOE_LAUNCH("router_decode_logits", stream,
             launch_decode_logits(*d, x, T, ws.logits, S, dev->flags, stream, ws.meta + kMetaTopkDone));
  MOE_LAUNCH("router_topk_sort", stream,
             launch_topk_sort(*d, ws.logits, S, T, topk_idx, topk_w, gemm_chunk(*d, T), ws, dev->flags,
                              stream));
  if ((st = run_routed(d, x, T, topk_idx, topk_w, ws, path, dev, stream, true)) != MOE_OK) return st;
  MOE_LAUNCH("combine", stream, launch_combine(*d, topk_idx, T, ws.yp, yp_bf16(*d, T, path), y, stream));
  return MOE_OK;
}

// ------------------------------------------------------------------ the block: shared expert + residual

// the shared expert as a one-expert layer: every token routed to expert 0 with weight 1
static moe_desc shared_as_layer(const moe_desc& d, const moe_shared_expert& sh) {
  moe_desc s = d;
  s.E = 1;
  s.k = 1;
  s.I = sh.I;
  s.wfmt = sh.wfmt;
  s.b = nullptr;
  s.expert_mask = nullptr;
  s.W_gate = sh.W_gate;
  s.W_up = sh.W_up;
  s.W_down = sh.W_down;
  s.s_gate = sh.s_gate;
  s.s_up = sh.s_up;
  s.s_down = sh.s_down;
  return s;
}

static moe_status validate_shared(const moe_desc& d, const moe_shared_expert* sh) {
  if (!sh) return MOE_OK;
  if (sh->I < 64 || sh->I % 64) return fail(MOE_ERR_INVALID_ARG, "shared expert I must be a positive multiple of 64 (got %d)", sh->I);
  if (sh->I > 8192) return fail(MOE_ERR_UNSUPPORTED, "shared expert I is limited to 8192 (got %d)", sh->I);
  const moe_desc s = shared_as_layer(d, *sh);
  moe_status st = validate_desc(&s);
  if (st != MOE_OK) return fail(st, "shared expert: %s", g_err.c_str());
  return MOE_OK;
}

// block workspace: the routed layer's, then the shared expert's (as a one-expert
// layer over T tokens), then T unit weights
static void block_layout(const moe_desc& d, const moe_shared_expert* sh, int32_t T, size_t* shared_off,
                         size_t* ones_off, size_t* total) {
  size_t off[kRegions], routed = 0, shared = 0;
  layout(d, T, off, &routed);
  if (sh) {
    const moe_desc s = shared_as_layer(d, *sh);
    layout(s, T, off, &shared);
  }
  *shared_off = routed;
  *ones_off = routed + shared;
  *total = routed + shared + (sh ? up256((size_t)T * 4) : 0);
}

extern "C" moe_status moe_block_workspace_size(const moe_desc* d, const moe_shared_expert* shared, int32_t T,
                                               size_t* bytes) {
  g_err.clear();
  moe_status st = validate_desc(d);
  if (st != MOE_OK) return st;
  if ((st = validate_T(T, d->k)) != MOE_OK) return st;
  if ((st = validate_shared(*d, shared)) != MOE_OK) return st;
  if (!bytes) return fail(MOE_ERR_INVALID_ARG, "bytes is NULL");
  size_t so, oo;
  block_layout(*d, shared, T, &so, &oo, bytes);
  return MOE_OK;
}

extern "C" moe_status moe_forward_block(const moe_desc* d, const moe_shared_expert* shared, const void* x,
                                        int32_t T, const int32_t* topk_idx, const float* topk_w,
                                        const void* residual, void* y, void* workspace, size_t ws_bytes,
                                        cudaStream_t stream) {
  g_err.clear();
  moe_status st = validate_desc(d);
  if (st != MOE_OK) return st;
  if ((st = validate_T(T, d->k)) != MOE_OK) return st;
  if ((st = validate_shared(*d, shared)) != MOE_OK) return st;
  if (T == 0) return MOE_OK;
  if ((st = check_io(x, y, topk_idx, topk_w)) != MOE_OK) return st;
  if (residual && !aligned(residual, 16)) return fail(MOE_ERR_INVALID_ARG, "residual must be 16-byte aligned");
  size_t shared_off, ones_off, need;
  block_layout(*d, shared, T, &shared_off, &ones_off, &need);
  if (!workspace) return fail(MOE_ERR_WORKSPACE, "workspace is NULL (need %zu bytes)", need);
  if (!aligned(workspace, 256)) return fail(MOE_ERR_WORKSPACE, "workspace must be 256-byte aligned");
  if (ws_bytes < need) return fail(MOE_ERR_WORKSPACE, "workspace too small: %zu bytes given, %zu needed", ws_bytes, need);
  const int path = choose_path(*d, T);
  if (path == MOE_PATH_GEMM && !gemm_capable(*d)) return fail(MOE_ERR_UNSUPPORTED, "%s", kNoTensorCores);
  moe_desc sd{};
  int spath = MOE_PATH_GEMV;
  if (shared) {
    sd = shared_as_layer(*d, *shared);
    spath = choose_path(sd, T);
    if (spath == MOE_PATH_GEMM && !gemm_capable(sd)) return fail(MOE_ERR_UNSUPPORTED, "shared expert: %s", kNoTensorCores);
  }
  DeviceState* dev = nullptr;
  if ((st = device_state(&dev)) != MOE_OK) return st;
  const Workspace ws = carve_workspace(*d, T, workspace);
  const float* ys = nullptr;
  if (shared && path == MOE_PATH_GEMM && spath == MOE_PATH_GEMM && sd.wfmt == d->wfmt) {
    // the shared expert's units ride in the routed experts' grouped-GEMM launches
    const Workspace ss = carve_workspace(sd, T, static_cast<char*>(workspace) + shared_off);
    const int chunk = gemm_chunk(sd, T);
    const DenseGemm up{&sd, x, ss.hbuf, T, chunk};
    const DenseGemm down{&sd, ss.hbuf, ss.yp, T, chunk};
    if ((st = run_routed(d, x, T, topk_idx, topk_w, ws, path, dev, stream, false, &up, &down)) != MOE_OK) return st;
    MOE_LAUNCH("combine", stream,
               launch_combine(*d, topk_idx, T, ws.yp, yp_bf16(*d, T, path), y, stream, ss.yp, residual));
    return MOE_OK;
  }
  if ((st = run_routed(d, x, T, topk_idx, topk_w, ws, path, dev, stream)) != MOE_OK) return st;
  if (shared) {
    Workspace ss = carve_workspace(sd, T, static_cast<char*>(workspace) + shared_off);
    float* ones = reinterpret_cast<float*>(static_cast<char*>(workspace) + ones_off);
    const int chunk = gemm_chunk(sd, T);
    MOE_LAUNCH("shared_plan", stream,
               launch_dense_plan(T, chunk, ss.counts, ss.offsets, ss.touched, ss.group_base, ss.tile_base, ss.meta,
                                 ss.sorted_pair, ones, stream));
    if (spath == MOE_PATH_GEMM) {
      ss.xs = const_cast<void*>(x);  // token order is the sorted order: x serves as the gathered rows
      MOE_LAUNCH("shared_gateup", stream, launch_gemm_gateup(sd, ss, T, chunk, dev->num_sms, dev->flags, stream));
      MOE_LAUNCH("shared_down", stream, launch_gemm_down(sd, ones, ss, T, chunk, dev->num_sms, dev->flags, stream));
    } else {
      MOE_LAUNCH("shared_gateup", stream, launch_gemv_gateup(sd, x, 1, ss, dev->num_sms, dev->flags, stream));
      MOE_LAUNCH("shared_down", stream, launch_gemv_down(sd, ones, 1, ss, dev->num_sms, dev->flags, stream));
    }
    ys = ss.yp;
  }
  MOE_LAUNCH("combine", stream,
             launch_combine(*d, topk_idx, T, ws.yp, yp_bf16(*d, T, path), y, stream, ys, residual));
  return MOE_OK;
}

// ------------------------------------------------------------------ routing statistics

extern "C" moe_status moe_expert_counts(const moe_desc* d, const int32_t* topk_idx, int32_t T, uint64_t* counts,
                                        cudaStream_t stream) {
  g_err.clear();
  if (!d) return fail(MOE_ERR_INVALID_ARG, "descriptor is NULL");
  if (d->E < 1 || d->E > 1024) return fail(MOE_ERR_INVALID_ARG, "E must be in [1, 1024] (got %d)", d->E);
  if (d->k < 1 || d->k > 32) return fail(MOE_ERR_INVALID_ARG, "k must be in [1, 32] (got %d)", d->k);
  moe_status st = validate_T(T, d->k);
  if (st != MOE_OK) return st;
  if (!counts || !aligned(counts, 8)) return fail(MOE_ERR_INVALID_ARG, "counts must be a non-NULL 8-byte aligned device pointer");
  if (T == 0) return MOE_OK;
  if (!topk_idx || !aligned(topk_idx, 4)) return fail(MOE_ERR_INVALID_ARG, "topk_idx must be non-NULL, 4-byte aligned");
  DeviceState* dev = nullptr;
  if ((st = device_state(&dev)) != MOE_OK) return st;
  MOE_LAUNCH("expert_counts", stream,
             launch_expert_counts(topk_idx, (int64_t)T * d->k, d->E, counts, dev->num_sms, stream));
  return MOE_OK;
}

extern "C" moe_status moe_cover_set(const uint64_t* counts, int32_t E, double cover, uint8_t* keep,
                                    int32_t* new_index, int32_t* n_keep) {
  g_err.clear();
  if (!counts || !keep || !new_index || !n_keep) return fail(MOE_ERR_INVALID_ARG, "NULL argument");
  if (E < 1) return fail(MOE_ERR_INVALID_ARG, "E must be >= 1 (got %d)", E);
  if (!(cover > 0.0 && cover <= 1.0)) return fail(MOE_ERR_INVALID_ARG, "cover must lie in (0, 1] (got %g)", cover);
  std::vector<int32_t> order((size_t)E);
  uint64_t total = 0;
  for (int32_t e = 0; e < E; ++e) {
    order[e] = e;
    total += counts[e];
  }
  std::stable_sort(order.begin(), order.end(), [&](int32_t a, int32_t b) { return counts[a] > counts[b]; });
  const double target = cover * (double)total;
  int32_t m = 0;
  uint64_t mass = 0;
  while (m < E && (double)mass < target) mass += counts[order[m++]];
  std::fill(keep, keep + E, (uint8_t)0);
  for (int32_t i = 0; i < m; ++i) keep[order[i]] = 1;
  int32_t next = 0;
  for (int32_t e = 0; e < E; ++e) new_index[e] = keep[e] ? next++ : -1;
  *n_keep = m;
  return MOE_OK;
}

// ------------------------------------------------------------------ diagnostics

namespace moe {
namespace {
// one thread waits on an mbarrier that nothing completes: the library's bounded
// wait gives up, the kernel raises MOE_FLAG_TIMEOUT and returns
__global__ void bounded_wait_selftest_kernel(uint32_t* flags) {
  pdl_wait();
  pdl_trigger();
  __shared__ __align__(8) uint64_t never;
  if (threadIdx.x == 0) {
    mbar_init(&never, 1);
    fence_mbar_init();
    if (!mbar_wait(&never, 0)) raise_flag(flags, MOE_FLAG_TIMEOUT);
  }
}
}  // namespace
}  // namespace moe

extern "C" moe_status moe_selftest_bounded_wait(cudaStream_t stream) {
  g_err.clear();
  DeviceState* dev = nullptr;
  moe_status st = device_state(&dev);
  if (st != MOE_OK) return st;
  MOE_LAUNCH("selftest_bounded_wait", stream, launch_k(bounded_wait_selftest_kernel, dim3(1), dim3(32), 0, stream,
                                                        dev->flags));
  return MOE_OK;
}

extern "C" const char* moe_last_error(void) { return g_err.c_str(); }

extern "C" moe_status moe_device_flags(uint32_t* flags, int32_t clear) {
  g_err.clear();
  if (!flags) return fail(MOE_ERR_INVALID_ARG, "flags is NULL");
  DeviceState* dev = nullptr;
  moe_status st = device_state(&dev);
  if (st != MOE_OK) return st;
  cudaError_t e = cudaDeviceSynchronize();
  if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceSynchronize");
  e = cudaMemcpy(flags, dev->flags, sizeof(uint32_t), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(e, "reading device flags");
  if (clear) {
    e = cudaMemset(dev->flags, 0, sizeof(uint32_t));
    if (e == cudaSuccess) e = cudaDeviceSynchronize();
    if (e != cudaSuccess) return cuda_fail(e, "clearing device flags");
  }
  return MOE_OK;
}

extern "C" uint64_t moe_launch_count(void) { return g_launches.load(); }

extern "C" moe_status moe_stage_timing(int32_t enable) {
  g_timing.store(enable ? 1 : 0);
  return MOE_OK;
}

extern "C" moe_status moe_stage_timing_only(const char* name) {
  g_err.clear();
  if (name != nullptr && strlen(name) >= sizeof(g_timing_only))
    return fail(MOE_ERR_INVALID_ARG, "kernel name longer than %d characters", (int)sizeof(g_timing_only) - 1);
  std::lock_guard<std::mutex> lk(g_time_mu);
  snprintf(g_timing_only, sizeof(g_timing_only), "%s", name ? name : "");
  return MOE_OK;
}

extern "C" moe_status moe_stage_times(moe_stage_time* out, int32_t capacity, int32_t* count) {
  g_err.clear();
  if (!count || (capacity > 0 && !out)) return fail(MOE_ERR_INVALID_ARG, "out/count is NULL");
  std::lock_guard<std::mutex> lk(g_time_mu);
  std::vector<moe_stage_time> agg;
  cudaError_t first = cudaSuccess;
  for (const Pending& p : g_pending) {
    float ms = 0.f;
    cudaError_t e = cudaEventSynchronize(p.end);
    if (e == cudaSuccess) e = cudaEventElapsedTime(&ms, p.begin, p.end);
    if (e != cudaSuccess && first == cudaSuccess) first = e;
    size_t i = 0;
    for (; i < agg.size(); ++i)
      if (strncmp(agg[i].name, p.name, sizeof(p.name)) == 0) break;
    if (i == agg.size()) {
      moe_stage_time t;
      memset(&t, 0, sizeof(t));
      snprintf(t.name, sizeof(t.name), "%s", p.name);
      agg.push_back(t);
    }
    agg[i].launches += 1;
    agg[i].total_ms += ms;
    g_event_pool.push_back(p.begin);
    g_event_pool.push_back(p.end);
  }
  g_pending.clear();
  *count = (int32_t)agg.size();
  for (int32_t i = 0; i < capacity && i < (int32_t)agg.size(); ++i) out[i] = agg[i];
  if (first != cudaSuccess) return cuda_fail(first, "stage timing events");
  return MOE_OK;
}
