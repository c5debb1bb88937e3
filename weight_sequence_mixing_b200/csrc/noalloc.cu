// ttt_forward_noalloc: the forward pass for callers that cannot allocate device
// memory.  The workspace is a file-scope static device array owned by this
// library instead of a buffer the caller passes in.
//
// Who needs it: code that runs where allocation is not allowed or not safe --
// inside a host framework that owns every allocation on the device (a plugin or
// an embedding runtime with its own allocator and no allocation hooks for us), on
// a latency-critical path where a cudaMalloc could block on device-wide
// synchronisation, or while another component is capturing work into a CUDA graph
// that must not contain allocations.  Such a caller still owns its inputs and
// outputs; it only cannot provide the scratch buffer the layer needs.
#include <mutex>

#include "../../include/ttt.h"
#include "ttt_plan.cuh"

namespace ttt {
namespace {

// The scratch every call of ttt_forward_noalloc on a device shares.  Every GPU
// that loads this library holds one copy of it until the process exits.
static __device__ __align__(256) unsigned char g_noalloc_scratch[TTT_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 256;
std::mutex g_mu;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of this device's copy of the scratch array, resolved once per
// device with that device current.  In host code `g_noalloc_scratch` names a
// host-side stand-in, never the device memory, so it must not be passed to a kernel.
int scratch_for_current_device(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return TTT_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return TTT_ERR_CUDA;
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return TTT_OK;
}

}  // namespace
}  // namespace ttt

extern "C" int ttt_forward_noalloc(ttt_handle* h, const void* Q, const void* K, const void* V, const float* eta,
                                   const float* W0, void* O, float* W_out, unsigned* status_out, void* stream) {
  using namespace ttt;
  if (!h || !Q || !K || !V || !W0 || !O) return TTT_ERR_INVALID_ARG;
  const void* ptrs[] = {Q, K, V, eta, W0, O, W_out, status_out};
  for (const void* p : ptrs)
    if (p && (reinterpret_cast<uintptr_t>(p) & 3) != 0) return TTT_ERR_INVALID_ARG;
  const void* aligned16[] = {Q, K, V, eta, W0, O, W_out};
  for (const void* p : aligned16)
    if (p && (reinterpret_cast<uintptr_t>(p) & 15) != 0) return TTT_ERR_INVALID_ARG;
  if (h->plan.ws_bytes > TTT_NOALLOC_SCRATCH_BYTES) return TTT_ERR_WORKSPACE;  // layer too large for the scratch
  void* scratch = nullptr;
  int r = scratch_for_current_device(&scratch);
  if (r != TTT_OK) return r;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  Io io{Q, K, V, eta, W0, O, W_out};
  // plan_run clears the status word and every buffer that must start at zero
  // (momentum) before use, so a call never sees a previous call's state.
  r = plan_run(h->plan, io, scratch, st);
  if (r != TTT_OK) return r;
  if (status_out && cudaMemcpyAsync(status_out, scratch, sizeof(unsigned), cudaMemcpyDeviceToDevice, st) != cudaSuccess)
    return TTT_ERR_CUDA;
  return TTT_OK;
}
