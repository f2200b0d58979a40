// Full forward with a built-in, fixed-size scratch buffer, for callers that
// cannot allocate device memory themselves.
//
// Some callers have no way to call cudaMalloc or to hand the library a
// workspace: code that runs inside another runtime's memory pool or allocator
// policy, plug-in hosts that forbid allocations after start-up, or tools that
// only ever pass pointers to buffers they were given.  For them this file
// provides rehyat_hybrid_attn_fwd_noalloc: the same computation as
// rehyat_hybrid_attn_fwd, with the workspace taken from a file-scope
// __device__ array instead of the caller.  Inputs and outputs are still the
// caller's.
#include <cuda_runtime.h>

#include <mutex>

#include "rehyat.h"

namespace rehyat {
namespace {

// 32 MiB: enough for the 320x480 Wan layer (one batch, 12 heads, 21 slices,
// D = D' = 128 needs about 22 MiB of workspace); larger problems are refused.
constexpr size_t kScratchBytes = size_t(32) << 20;

// Every GPU that loads this library holds this array until the process exits.
__device__ __align__(256) unsigned char g_noalloc_scratch[kScratchBytes];

constexpr int kMaxDevices = 128;
void* g_scratch_addr[kMaxDevices] = {};  // last address looked up per device ordinal
std::mutex g_scratch_mutex;

// The array's name is a host-side stand-in in host code, not a device
// address; the real address comes from cudaGetSymbolAddress with the device
// current.  It is looked up again on every call made outside stream capture
// (cheap next to the forward), so a context created anew on the device
// (after cudaDeviceReset, or another context made current) gets the array's
// address in that context.  A call on a capturing stream cannot look it up
// safely (the first lookup may load the module, which would break the
// capture), so it uses the address of the last uncaptured call on the
// device, and is refused when there was none.
rehyat_status scratch_for_current_device(cudaStream_t stream, void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return REHYAT_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return REHYAT_ERR_UNSUPPORTED;
  cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(stream, &cap) != cudaSuccess) return REHYAT_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_scratch_mutex);
  if (cap != cudaStreamCaptureStatusNone) {
    if (g_scratch_addr[dev] == nullptr) return REHYAT_ERR_INVALID_ARG;
    *out = g_scratch_addr[dev];
    return REHYAT_OK;
  }
  void* ptr = nullptr;
  if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess || ptr == nullptr)
    return REHYAT_ERR_CUDA;
  g_scratch_addr[dev] = ptr;
  *out = ptr;
  return REHYAT_OK;
}

}  // namespace
}  // namespace rehyat

extern "C" rehyat_status rehyat_hybrid_attn_fwd_noalloc(const rehyat_params* p, const void* q,
                                                        const void* k, const void* v,
                                                        const rehyat_phi* phi, void* y,
                                                        const rehyat_debug* dbg,
                                                        void* stream) {
  const size_t need = rehyat_workspace_bytes(p);
  if (need == 0)  // invalid params: let the regular entry point name the error
    return rehyat_hybrid_attn_fwd(p, q, k, v, phi, y, nullptr, 0, dbg, stream);
  if (need > rehyat::kScratchBytes) return REHYAT_ERR_SCRATCH_LIMIT;
  void* scratch = nullptr;
  const rehyat_status st =
      rehyat::scratch_for_current_device(static_cast<cudaStream_t>(stream), &scratch);
  if (st != REHYAT_OK) return st;
  return rehyat_hybrid_attn_fwd(p, q, k, v, phi, y, scratch, rehyat::kScratchBytes, dbg, stream);
}
