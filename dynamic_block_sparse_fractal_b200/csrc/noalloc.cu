// sparse_attn_forward_noalloc: plan + forward for callers that may not
// allocate device memory themselves. The workspace is a fixed array in the
// library's own device image instead of a caller-provided buffer.
#include <cuda_runtime.h>

#include <cstddef>
#include <mutex>

#include "../../include/sparse_attn.h"

namespace {

constexpr size_t kScratchBytes = SA_NOALLOC_SCRATCH_BYTES;
constexpr int kMaxDevices = 64;

// One copy per GPU that loads this library, held until the process exits.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kScratchBytes];

// Device addresses of g_noalloc_scratch per device. In host code the symbol
// itself is only a host-side handle, never a device address. The address is
// looked up again on every call made outside stream capture (a device reset
// reloads the module, and the array may then sit elsewhere); a call made
// while its stream is being captured cannot look it up and uses the address
// the last uncaptured call on that device found.
void* g_scratch_ptr[kMaxDevices] = {};
std::mutex g_scratch_mu;

sa_status scratch_for_current_device(cudaStream_t stream, void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return SA_ERR_CUDA;
  cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(stream, &cap) != cudaSuccess) return SA_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (cap == cudaStreamCaptureStatusNone) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr)
      return SA_ERR_CUDA;
    g_scratch_ptr[dev] = p;
  } else if (g_scratch_ptr[dev] == nullptr) {
    return SA_ERR_CUDA;  // first call on this device inside a capture
  }
  *out = g_scratch_ptr[dev];
  return SA_OK;
}

}  // namespace

extern "C" sa_status sparse_attn_forward_noalloc(const sa_desc* desc, const void* q,
                                                 const void* k, const void* v, void* out,
                                                 void* stream) {
  size_t need = 0;
  sa_status st = sparse_attn_workspace_size(desc, &need);
  if (st != SA_OK) return st;
  if (need > kScratchBytes) return SA_ERR_WORKSPACE;
  void* ws = nullptr;
  st = scratch_for_current_device(static_cast<cudaStream_t>(stream), &ws);
  if (st != SA_OK) return st;
  st = sparse_attn_plan(desc, q, k, ws, kScratchBytes, stream);
  if (st != SA_OK) return st;
  return sparse_attn_fwd(desc, q, k, v, ws, kScratchBytes, out, stream);
}
