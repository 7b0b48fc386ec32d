// recsa_prefill_static: the tensor-core window prefill with its scratch in a
// fixed device array instead of a caller workspace.
//
// Some callers cannot hand the library any device memory beyond the tensors
// of the call: a runtime whose device memory is entirely planned ahead and
// owned by its own arena, or a plain C host that has no device allocator on
// its call path.  For them this entry point keeps the window partials (an fp32
// row of head_dim + 2 per query head) in a file-scope device array of kStaticFloats floats
// (4 MiB), which every GPU that loads the library holds until the process
// exits.  Nothing here calls cudaMalloc, cudaFree or any allocating routine.
#include <mutex>

#include "recsa_internal.cuh"

namespace recsa {
namespace {

// batch * n_q * n_q_heads * (head_dim + 2) must not exceed this (4 MiB of fp32).
constexpr size_t kStaticFloats = size_t(1) << 20;

__device__ __align__(256) float g_prefill_scratch[kStaticFloats];

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mutex;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device.  The host-side
// symbol is only a stand-in for it.  Outside stream capture the address is
// looked up on every call (a host-side table lookup), so a call after a
// device reset, which reloads the module, gets the array's new address.
// During capture the address recorded by the last call outside capture is
// used, and a device never set up that way is refused.
cudaError_t scratch_address(cudaStream_t s, void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
  e = cudaStreamIsCapturing(s, &cap);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lock(g_scratch_mutex);
  if (cap == cudaStreamCaptureStatusNone) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_prefill_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_ptr[dev] = p;
  } else if (!g_scratch_ptr[dev]) {
    return cudaErrorStreamCaptureUnsupported;
  }
  *out = g_scratch_ptr[dev];
  return cudaSuccess;
}

}  // namespace

size_t prefill_static_bytes() { return kStaticFloats * sizeof(float); }

cudaError_t launch_prefill_static(const Params& p, const void* Q, const void* K, const void* V,
                                  const void* tree, int64_t q_start, int32_t n_q, void* O,
                                  int32_t* trace, cudaStream_t s) {
  if (p.mode != RECSA_MODE_RECSA) return cudaErrorNotSupported;   // other modes: own kernels
  void* ml = nullptr;
  cudaError_t e = scratch_address(s, &ml);
  if (e != cudaSuccess) return e;
  // The window kernel writes every partial row of the range before the tree
  // kernel reads it, so the array needs no clearing between calls.
  e = launch_prefill_window(p, Q, K, V, tree, q_start, n_q, ml, s);
  const void* wml = ml;
  if (e == cudaErrorNotSupported) {
    cudaGetLastError();
    wml = nullptr;   // geometry outside the window kernel: the tree kernel attends it
  } else if (e != cudaSuccess) {
    return e;
  }
  return launch_prefill_warp(p, Q, K, V, tree, q_start, n_q, O, trace, wml, s);
}

}  // namespace recsa
