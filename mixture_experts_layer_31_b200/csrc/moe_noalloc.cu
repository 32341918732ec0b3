// moe_forward_noalloc: moe_forward for callers that cannot allocate device
// memory.  Some hosts give a kernel library no allocator at all (plugin
// interfaces whose engine owns every device buffer), and some callers must not
// call cudaMalloc once they are running (it can synchronise the device and
// stall a latency-bound decode loop, or fail under a memory pool the host has
// already sized).  For them the scratch of the forward pass (expert histogram,
// sorted pair order, the activations between the two projections and the
// per-pair outputs) lives in one file-scope device array of fixed size instead
// of a caller workspace.
//
// The array is a static __device__ object: every GPU that loads this library
// holds MOE_NOALLOC_SCRATCH_BYTES of it until the process exits.  In host code
// its name is only a host-side stand-in, so its device address is looked up
// with cudaGetSymbolAddress once per device (under a lock, with that device
// current) on the first call made on that device, and that address is what the
// kernels receive.
#include <cuda_runtime.h>

#include <stdio.h>

#include <mutex>

#include "internal.h"
#include "moe.h"

namespace moe {
namespace {

static __device__ __align__(256) unsigned char g_noalloc_scratch[MOE_NOALLOC_SCRATCH_BYTES];

struct ScratchSlot {
  bool ready = false;
  void* ptr = nullptr;
};
std::mutex g_scratch_mu;
ScratchSlot g_scratch[64];

// device address of the scratch array on the current device (set up on first use)
cudaError_t scratch_address(void** out, int* dev_out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lk(g_scratch_mu);
  ScratchSlot& s = g_scratch[dev];
  if (!s.ready) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return e;
    s.ptr = p;
    s.ready = true;
  }
  *out = s.ptr;
  *dev_out = dev;
  return cudaSuccess;
}

}  // namespace
}  // namespace moe

extern "C" moe_status moe_forward_noalloc(const moe_desc* d, const void* x, int32_t T, const int32_t* topk_idx,
                                          const float* topk_w, void* y, cudaStream_t stream) {
  size_t full = 0;
  moe_status st = moe_workspace_size(d, T, &full);  // validates the descriptor and T
  if (st != MOE_OK) return st;
  if (T == 0) return MOE_OK;
  // the forward pass alone: the routing is given, so the router's regions of
  // moe_workspace_size's layout are left out
  const size_t need = moe::forward_scratch_bytes(*d, T);
  if (need > (size_t)MOE_NOALLOC_SCRATCH_BYTES) {
    char msg[256];
    snprintf(msg, sizeof(msg),
             "moe_forward_noalloc: this problem needs %zu bytes of scratch but the library's static scratch "
             "holds %zu; use moe_forward with a caller workspace",
             need, (size_t)MOE_NOALLOC_SCRATCH_BYTES);
    return moe::report_error(MOE_ERR_WORKSPACE, msg);
  }
  void* scratch = nullptr;
  int dev = 0;
  cudaError_t e = moe::scratch_address(&scratch, &dev);
  if (e != cudaSuccess) {
    char msg[256];
    snprintf(msg, sizeof(msg), "moe_forward_noalloc: cudaGetSymbolAddress of the static scratch failed: %s",
             cudaGetErrorString(e));
    return moe::report_error(MOE_ERR_CUDA, msg);
  }
  return moe::forward_impl(d, x, T, topk_idx, topk_w, y, scratch, (size_t)MOE_NOALLOC_SCRATCH_BYTES, stream, true);
}
