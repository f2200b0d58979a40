// General feature map of ReHyAt (fp32 CUDA-core kernel).
//
// Source: "ReHyAt: Recurrent Hybrid Attention for Video Diffusion
// Transformers" (papernotes.org note), Method, Key design 3: a light per-head
// embedding network (grouped 1x1 convolution = per-head linear map, with a
// nonlinearity) produces psi, which is cut into P equal parts; part i is
// raised to the i-th power: phi = [psi_1^1, ..., psi_P^P].  Here
//   psi = GELU(x W_a + b_a) W_b + b_b,  GELU(u) = u * Phi(u) (exact form),
// per head, with hidden width D_h.  The output feeds rehyat_hybrid_attn_fwd_phi.
//
// One block per (32 tokens, b*h): the token tile and the hidden activations
// sit in shared memory; W_a and W_b stream through L1/L2 (read along their
// output columns, coalesced).
#include <cuda_bf16.h>
#include <math.h>
#include <stdint.h>

#include "internal.h"

namespace rehyat {
namespace {

constexpr int kMlpRows = 32;
constexpr int kMlpThreads = 256;

__device__ __forceinline__ float load_xv(const void* base, long long i, int bf16) {
  if (bf16) {
    const unsigned short b = reinterpret_cast<const unsigned short*>(base)[i];
    return __uint_as_float(static_cast<unsigned>(b) << 16);
  }
  return reinterpret_cast<const float*>(base)[i];
}

__global__ void __launch_bounds__(kMlpThreads) phi_mlp_kernel(PhiMlpArgs a) {
  extern __shared__ float sm[];
  float* xs = sm;                        // [32][D]
  float* hs = xs + kMlpRows * a.D;       // [32][Dh]
  const int bh = blockIdx.y, h = bh % a.heads;
  const long long r0 = static_cast<long long>(blockIdx.x) * kMlpRows;
  const long long rowbase = static_cast<long long>(bh) * a.N;
  const int nrows = static_cast<int>(min(static_cast<long long>(kMlpRows), a.N - r0));
  for (int i = threadIdx.x; i < kMlpRows * a.D; i += kMlpThreads) {
    const int r = i / a.D, d = i % a.D;
    xs[i] = r < nrows ? load_xv(a.x, (rowbase + r0 + r) * a.D + d, a.in_bf16) : 0.f;
  }
  __syncthreads();
  // Hidden layer: thread t computes column j = t mod 256 (+256 ...) for all rows.
  const float* Wa = a.Wa + static_cast<long long>(h) * a.D * a.Dh;
  const float* ba = a.ba + static_cast<long long>(h) * a.Dh;
  for (int j = threadIdx.x; j < a.Dh; j += kMlpThreads) {
    float acc[kMlpRows];
    const float bj = __ldg(ba + j);
#pragma unroll
    for (int r = 0; r < kMlpRows; ++r) acc[r] = bj;
    for (int d = 0; d < a.D; ++d) {
      const float w = __ldg(Wa + static_cast<long long>(d) * a.Dh + j);
#pragma unroll
      for (int r = 0; r < kMlpRows; ++r) acc[r] = fmaf(xs[r * a.D + d], w, acc[r]);
    }
#pragma unroll
    for (int r = 0; r < kMlpRows; ++r) {
      const float u = acc[r];
      hs[r * a.Dh + j] = 0.5f * u * (1.f + erff(u * 0.70710678118654752f));
    }
  }
  __syncthreads();
  // Output layer and the part powers.
  const float* Wb = a.Wb + static_cast<long long>(h) * a.Dh * a.Dp;
  const float* bb = a.bb + static_cast<long long>(h) * a.Dp;
  const int width = a.Dp / a.parts;
  for (int f = threadIdx.x; f < a.Dp; f += kMlpThreads) {
    float acc[kMlpRows];
    const float bf = __ldg(bb + f);
#pragma unroll
    for (int r = 0; r < kMlpRows; ++r) acc[r] = bf;
    for (int j = 0; j < a.Dh; ++j) {
      const float w = __ldg(Wb + static_cast<long long>(j) * a.Dp + f);
#pragma unroll
      for (int r = 0; r < kMlpRows; ++r) acc[r] = fmaf(hs[r * a.Dh + j], w, acc[r]);
    }
    const int power = f / width + 1;
#pragma unroll
    for (int r = 0; r < kMlpRows; ++r) {
      if (r < nrows) {
        float v = acc[r];
        for (int i = 1; i < power; ++i) v *= acc[r];
        const long long o = (rowbase + r0 + r) * a.Dp + f;
        if (a.phi_bf16)
          static_cast<__nv_bfloat16*>(a.phi)[o] = __float2bfloat16_rn(v);
        else
          static_cast<float*>(a.phi)[o] = v;
      }
    }
  }
}

}  // namespace

cudaError_t launch_phi_mlp(const PhiMlpArgs& a, cudaStream_t s) {
  const size_t smem = sizeof(float) * kMlpRows * (a.D + a.Dh);
  cudaError_t e = cudaFuncSetAttribute(phi_mlp_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  dim3 grid(static_cast<unsigned>((a.N + kMlpRows - 1) / kMlpRows), a.BH);
  phi_mlp_kernel<<<grid, kMlpThreads, smem, s>>>(a);
  return cudaGetLastError();
}

}  // namespace rehyat
