// Full forward on host-resident q, k, v, y: the runtime that overlaps the
// PCIe copies with the kernels.
//
// Every (batch, head) of ReHyAt's chunked hybrid attention is independent
// ("ReHyAt: Recurrent Hybrid Attention for Video Diffusion Transformers",
// papernotes.org note, Method, Key designs 1-4: the softmax window, the
// linear state and the joint normalisation are all per head), so the heads
// are processed in slabs of consecutive heads of one batch element.  Slab s
// uses device slot s mod kSlots: its q, k, v are uploaded on a copy stream,
// its forward runs on the caller's stream, and its y is downloaded on a
// second copy stream, so the upload of slab s + 1, the forward of slab s and
// the download of slab s - 1 proceed together (PCIe is full duplex).
// Events order the three streams; each slot is reused only after the
// forward has read its inputs and the download has read its output.  The
// first and the last slab of a call take half the heads (rounded up): the
// first upload and the last download overlap nothing, so shorter ones start
// the kernels earlier and end the call sooner.
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>
#include <vector>

#include "internal.h"

namespace rehyat {
namespace {

constexpr int kSlots = 3;
constexpr size_t kAlign = 256;
size_t align_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }
int elem_size(int dtype) { return dtype == REHYAT_BF16 ? 2 : 4; }

// The two copy streams of each device, created on first use and kept for
// the life of the process (non-blocking: they never wait on stream 0).
constexpr int kMaxDevices = 64;
cudaStream_t g_copy_streams[kMaxDevices][2];
std::mutex g_copy_mutex;

cudaError_t copy_streams(cudaStream_t* up, cudaStream_t* down) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_copy_mutex);
  for (int i = 0; i < 2; ++i)
    if (!g_copy_streams[dev][i]) {
      e = cudaStreamCreateWithFlags(&g_copy_streams[dev][i], cudaStreamNonBlocking);
      if (e != cudaSuccess) return e;
    }
  *up = g_copy_streams[dev][0];
  *down = g_copy_streams[dev][1];
  return cudaSuccess;
}

struct SlabLayout {
  int per_slab;         // heads per slab
  size_t in_bytes;      // q, k or v of one slab
  size_t out_bytes;     // y of one slab
  size_t slot_bytes;    // q, k, v, y of one slot
  size_t fwd_bytes;     // workspace of one slab's forward
  size_t total;
};

rehyat_params slab_params(const rehyat_params* p, int heads) {
  rehyat_params s = *p;
  s.batch = 1;
  s.heads = heads;
  return s;
}

// One slab: heads [h0, h0 + hn) of batch element b.
struct Slab {
  int b, h0, hn;
};

// The slabs of a call in order: per_slab heads each within a batch element,
// except that the first slab of the call and the last one hold
// ceil(per_slab / 2) heads.
std::vector<Slab> slab_list(int batch, int heads, int per_slab) {
  const int ramp = (per_slab + 1) / 2;
  std::vector<Slab> out;
  for (int b = 0; b < batch; ++b)
    for (int h = 0; h < heads;) {
      int hn = out.empty() ? ramp : per_slab;
      hn = heads - h < hn ? heads - h : hn;
      out.push_back(Slab{b, h, hn});
      h += hn;
    }
  Slab& last = out.back();
  if (last.hn > ramp) {
    const Slab tail{last.b, last.h0 + last.hn - ramp, ramp};
    last.hn -= ramp;
    out.push_back(tail);
  }
  return out;
}

SlabLayout slab_layout(const rehyat_params* p, int heads_per_slab) {
  SlabLayout L{};
  L.per_slab = heads_per_slab > 0 && heads_per_slab < p->heads ? heads_per_slab : p->heads;
  const size_t tokens = static_cast<size_t>(p->T) * p->Hs * p->Ws * p->D;
  L.in_bytes = align_up(tokens * L.per_slab * elem_size(p->in_dtype));
  L.out_bytes = align_up(tokens * L.per_slab * elem_size(p->out_dtype));
  L.slot_bytes = 3 * L.in_bytes + L.out_bytes;
  const rehyat_params sp = slab_params(p, L.per_slab);
  L.fwd_bytes = align_up(rehyat_workspace_bytes(&sp));
  L.total = kSlots * L.slot_bytes + L.fwd_bytes;
  return L;
}

}  // namespace
}  // namespace rehyat

using namespace rehyat;

extern "C" {

size_t rehyat_host_workspace_bytes(const rehyat_params* p, int heads_per_slab) {
  if (rehyat_workspace_bytes(p) == 0) return 0;  // invalid params
  return slab_layout(p, heads_per_slab).total;
}

rehyat_status rehyat_hybrid_attn_fwd_host(const rehyat_params* p, const void* q, const void* k,
                                          const void* v, const rehyat_phi* phi, void* y,
                                          int heads_per_slab, void* workspace, size_t ws_bytes,
                                          void* stream) {
  if (rehyat_workspace_bytes(p) == 0) return REHYAT_ERR_INVALID_ARG;
  if (!q || !k || !v || !y || !phi || !workspace) return REHYAT_ERR_INVALID_ARG;
  if (!phi->Wq || !phi->bq || !phi->Wk || !phi->bk) return REHYAT_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(workspace) & 15) return REHYAT_ERR_MISALIGNED;
  const SlabLayout L = slab_layout(p, heads_per_slab);
  if (ws_bytes < L.total) return REHYAT_ERR_WORKSPACE;
  cudaStream_t up = nullptr, down = nullptr;
  if (copy_streams(&up, &down) != cudaSuccess) return REHYAT_ERR_CUDA;
  const cudaStream_t s = static_cast<cudaStream_t>(stream);

  cudaEvent_t start, loaded[kSlots], computed[kSlots], drained[kSlots];
  cudaEvent_t* all[1 + 3 * kSlots];
  int nev = 0;
  all[nev++] = &start;
  for (int i = 0; i < kSlots; ++i) {
    all[nev++] = &loaded[i];
    all[nev++] = &computed[i];
    all[nev++] = &drained[i];
  }
  int made = 0;
  cudaError_t e = cudaSuccess;
  for (; made < nev && e == cudaSuccess; ++made)
    e = cudaEventCreateWithFlags(all[made], cudaEventDisableTiming);
  if (e != cudaSuccess) made -= 1;

  const size_t tokens = static_cast<size_t>(p->T) * p->Hs * p->Ws * p->D;
  const size_t head_in = tokens * elem_size(p->in_dtype);
  const size_t head_out = tokens * elem_size(p->out_dtype);
  const size_t phiW = static_cast<size_t>(p->D) * p->Dp;  // floats of W per head (both parts)
  char* ws = static_cast<char*>(workspace);
  char* fwd_ws = ws + kSlots * L.slot_bytes;
  std::vector<Slab> slabs;
  try {
    slabs = slab_list(p->batch, p->heads, L.per_slab);
  } catch (...) {  // host allocation failure
    e = cudaErrorMemoryAllocation;
  }
  const int nslabs = static_cast<int>(slabs.size());
  rehyat_status st = REHYAT_OK;

  // The copy streams start after the work already on the caller's stream.
  if (e == cudaSuccess) e = cudaEventRecord(start, s);
  if (e == cudaSuccess) e = cudaStreamWaitEvent(up, start, 0);
  if (e == cudaSuccess) e = cudaStreamWaitEvent(down, start, 0);
  for (int sl = 0; sl < nslabs && e == cudaSuccess && st == REHYAT_OK; ++sl) {
    const int slot = sl % kSlots;
    const int b = slabs[sl].b, h0 = slabs[sl].h0, hn = slabs[sl].hn;
    const size_t head_index = static_cast<size_t>(b) * p->heads + h0;
    char* dq = ws + slot * L.slot_bytes;
    char* dk = dq + L.in_bytes;
    char* dv = dk + L.in_bytes;
    char* dy = dv + L.in_bytes;
    // Upload: the slot's inputs were last read by the forward of slab sl - kSlots.
    if (sl >= kSlots) e = cudaStreamWaitEvent(up, computed[slot], 0);
    const size_t nin = head_in * hn;
    if (e == cudaSuccess)
      e = cudaMemcpyAsync(dq, static_cast<const char*>(q) + head_index * head_in, nin,
                          cudaMemcpyHostToDevice, up);
    if (e == cudaSuccess)
      e = cudaMemcpyAsync(dk, static_cast<const char*>(k) + head_index * head_in, nin,
                          cudaMemcpyHostToDevice, up);
    if (e == cudaSuccess)
      e = cudaMemcpyAsync(dv, static_cast<const char*>(v) + head_index * head_in, nin,
                          cudaMemcpyHostToDevice, up);
    if (e == cudaSuccess) e = cudaEventRecord(loaded[slot], up);
    // Forward: after the upload, and after the slot's y of slab sl - kSlots
    // has been downloaded.
    if (e == cudaSuccess) e = cudaStreamWaitEvent(s, loaded[slot], 0);
    if (e == cudaSuccess && sl >= kSlots) e = cudaStreamWaitEvent(s, drained[slot], 0);
    if (e != cudaSuccess) break;
    const rehyat_params sp = slab_params(p, hn);
    const rehyat_phi sphi = {phi->Wq + h0 * phiW, phi->bq + static_cast<size_t>(h0) * p->Dp,
                             phi->Wk + h0 * phiW, phi->bk + static_cast<size_t>(h0) * p->Dp};
    st = rehyat_hybrid_attn_fwd(&sp, dq, dk, dv, &sphi, dy, fwd_ws, L.fwd_bytes, nullptr, stream);
    if (st != REHYAT_OK) break;
    e = cudaEventRecord(computed[slot], s);
    // Download.
    if (e == cudaSuccess) e = cudaStreamWaitEvent(down, computed[slot], 0);
    if (e == cudaSuccess)
      e = cudaMemcpyAsync(static_cast<char*>(y) + head_index * head_out, dy, head_out * hn,
                          cudaMemcpyDeviceToHost, down);
    if (e == cudaSuccess) e = cudaEventRecord(drained[slot], down);
  }
  // The caller's stream ends after the last upload and the last download,
  // on an error too, so that synchronising it covers every copy this call
  // enqueued (a refused or failed slab may leave an upload in flight).
  if (made > 0) {
    cudaError_t j = cudaEventRecord(start, up);
    if (j == cudaSuccess) j = cudaStreamWaitEvent(s, start, 0);
    if (j == cudaSuccess) j = cudaEventRecord(start, down);
    if (j == cudaSuccess) j = cudaStreamWaitEvent(s, start, 0);
    if (e == cudaSuccess) e = j;
  }
  // Events may be destroyed with work pending; their resources are released
  // once it completes.
  for (int i = 0; i < made; ++i) cudaEventDestroy(*all[i]);
  if (st != REHYAT_OK) return st;
  return e == cudaSuccess ? REHYAT_OK : REHYAT_ERR_CUDA;
}

}  // extern "C"
