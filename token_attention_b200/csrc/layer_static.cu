// layer_static.cu -- mta_layer_fwd for callers that cannot allocate device memory.
//
// Some callers of this library cannot hand it a workspace: for example a host
// runtime that only receives device pointers to its own inputs and outputs
// from another component and has no device allocator of its own, or code that
// must not call cudaMalloc in the middle of a latency-sensitive loop because
// the allocation may synchronise the device.  For them the layer's scratch
// (the error word, the QKV buffer, the attention output and the normalised
// output) lives in one static device buffer inside the library.
//
// The buffer is a file-scope __device__ array of MTA_STATIC_SCRATCH_BYTES.
// Every GPU that loads the library holds it until the process exits.  Its
// device address is looked up once per device, on the first call made while
// that device is current; make that first call before any stream capture.
// All calls on a device share the buffer and it keeps the last call's
// contents; the layer clears the error word at the start of every call and
// overwrites everything else before reading it.  Calls whose execution
// overlaps on the GPU (different streams, or several host threads) race on
// the buffer: order them on one stream.
#include <cuda_runtime.h>

#include <mutex>

#include "mta.h"

namespace mta {
size_t layer_base_workspace_bytes(const mta_cfg *cfg);  // mta_api.cu
}  // namespace mta

namespace {

__device__ __align__(256) unsigned char g_layer_scratch[MTA_STATIC_SCRATCH_BYTES];

constexpr int kMaxDevices = 128;
std::mutex g_scratch_mutex;
void *g_scratch_ptr[kMaxDevices];  // device address of g_layer_scratch, per device

// Address of this device's copy of the static buffer (looked up once).
mta_status scratch_for_current_device(void **ptr) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return MTA_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return MTA_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_scratch_mutex);
  if (!g_scratch_ptr[dev]) {
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_layer_scratch) != cudaSuccess || p == nullptr) return MTA_ERR_CUDA;
    g_scratch_ptr[dev] = p;
  }
  *ptr = g_scratch_ptr[dev];
  return MTA_OK;
}

}  // namespace

extern "C" mta_status mta_layer_fwd_static(const void *x, const void *Wqkv, const float *theta,
                                           const float *w_head, const mta_gn *gn, const void *Wo,
                                           const mta_cfg *cfg, void *out) {
  if (!cfg) return MTA_ERR_INVALID;
  // the fixed scratch must fit; the contraction kernel's operands are used
  // where the rest of the buffer holds them, else the layer takes another kernel
  const size_t need = mta::layer_base_workspace_bytes(cfg);
  mta_cfg c = *cfg;
  if (need == 0) {
    // invalid configuration: let the layer's own checks report the precise status
    c.workspace = nullptr;
    c.workspace_bytes = 0;
    return mta_layer_fwd(x, Wqkv, theta, w_head, gn, Wo, &c, out);
  }
  if (need > static_cast<size_t>(MTA_STATIC_SCRATCH_BYTES)) return MTA_ERR_WORKSPACE;
  void *scratch = nullptr;
  const mta_status s = scratch_for_current_device(&scratch);
  if (s != MTA_OK) return s;
  c.workspace = scratch;
  c.workspace_bytes = MTA_STATIC_SCRATCH_BYTES;
  return mta_layer_fwd(x, Wqkv, theta, w_head, gn, Wo, &c, out);
}
