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
void* g_scratch_addr[kMaxDevices] = {};  // device address per device ordinal
std::mutex g_scratch_mutex;

// The array's name is a host-side stand-in in host code, not a device
// address; the real address comes from cudaGetSymbolAddress, once per
// device, with that device current.
rehyat_status scratch_for_current_device(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return REHYAT_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return REHYAT_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_scratch_mutex);
  if (g_scratch_addr[dev] == nullptr) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess || ptr == nullptr)
      return REHYAT_ERR_CUDA;
    g_scratch_addr[dev] = ptr;
  }
  *out = g_scratch_addr[dev];
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
  const rehyat_status st = rehyat::scratch_for_current_device(&scratch);
  if (st != REHYAT_OK) return st;
  return rehyat_hybrid_attn_fwd(p, q, k, v, phi, y, scratch, rehyat::kScratchBytes, dbg, stream);
}
