// Allocation-free variant of muon_ns_batched.
//
// Some callers cannot allocate device memory when they need the
// orthogonalisation: a host that has handed the whole GPU to its own caching
// allocator (a raw cudaMalloc would fail or fragment its pool), a loop that
// forbids allocation after start-up for predictable latency, or a plugin that
// is handed input and output pointers but no allocator.  For them this entry
// point takes its workspace from a fixed array in the library's own device
// memory instead of a caller buffer.
//
// The array is a file-scope __device__ object, so every GPU that loads the
// library holds MUON_NOALLOC_SCRATCH_BYTES of it until the process exits.
// Host code must not use the array's name as a device address (on the host it
// is only a stand-in symbol): its device address is looked up with
// cudaGetSymbolAddress while the device is current.
#include <mutex>

#include "../../include/muon.h"

namespace {

__device__ __align__(256) unsigned char g_noalloc_scratch[MUON_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
void* g_scratch_ptr[kMaxDevices] = {};
std::mutex g_scratch_mu;

// Device address of the scratch array on the current device (null on error).
// Outside a stream capture the address is looked up on every call (cheap), so
// a device reset, which unloads the module and may move the array, cannot
// leave a stale pointer behind.  During a capture the lookup (which may load
// the module) is not allowed, so the address cached by the last uncaptured
// call on this device is used; without one the call fails.
void* scratch_for_current_device(cudaStream_t stream) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(stream, &cap) != cudaSuccess) return nullptr;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (cap == cudaStreamCaptureStatusNone) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess) return nullptr;
    g_scratch_ptr[dev] = ptr;
  }
  return g_scratch_ptr[dev];
}

}  // namespace

extern "C" MUON_API int muon_ns_batched_noalloc(void* const* X, int count, int rows, int cols, int dtype,
                                                const muon_ns_params* ns, int* status_per_matrix, void* stream) {
  if (!X || count < 0 || rows <= 0 || cols <= 0 || !ns) return MUON_ERR_INVALID;
  if (count == 0) return MUON_OK;
  // One matrix must fit; more are processed in chunks that fit.
  const size_t need_one = muon_ns_workspace_size(1, rows, cols, ns);
  if (need_one == 0) return MUON_ERR_INVALID;
  if (need_one > (size_t)MUON_NOALLOC_SCRATCH_BYTES) return MUON_ERR_WORKSPACE;
  void* ws = scratch_for_current_device(reinterpret_cast<cudaStream_t>(stream));
  if (ws == nullptr) return MUON_ERR_CUDA;
  return muon_ns_batched(X, count, rows, cols, dtype, ns, ws, (size_t)MUON_NOALLOC_SCRATCH_BYTES, status_per_matrix,
                         stream);
}
