// Gradient of ReHyAt's hybrid attention with respect to the feature-map
// parameters W_q, b_q, W_k, b_k (fp32 CUDA-core kernels).
//
// Source: "ReHyAt: Recurrent Hybrid Attention for Video Diffusion
// Transformers" (papernotes.org note), Method, Key designs 1-5: the forward's
// joint normalisation y = (a^S + phi_q(q) S_L) / (n^S + phi_q(q) z_L) and the
// first training stage (Key design 5), which updates only phi_q and phi_k.
// With g = dL/dy, den = n^S + n^L (the forward's joint denominator):
//   dL/dphi_q(q_i) = (S_L,t g_i - z_L,t (g_i . y_i)) / den_i      (chunk t of i)
//   G_t = sum_{i in t} phi_q(q_i) g_i^T / den_i,  h_t = -sum_{i in t} phi_q(q_i) (g_i.y_i)/den_i
//   dL/dphi_k(k_j) = Ghat_s v_j + hhat_s, Ghat_s = sum of G_t over the chunks t
//                    whose linear set holds slice s (likewise hhat_s)
//   through phi = [(x W_1 + b_1)^2, (x W_2 + b_2)^2]: du = 2 u * dphi,
//   dW = sum x^T du, db = sum du, over every token and the batch.
// Passes (each CTA works on one feature piece of at most 128 features):
//   1. q pass, per (b*h, piece, chunk, row range): u_q, dphi_q, du_q; partial
//      dW_q, db_q, G_t, h_t of its rows;
//   2. Ghat pass: G_t, h_t per chunk from its row-range partials, then per
//      (b*h, piece, slice) Ghat_s, hhat_s as the sum over the chunks whose
//      linear set holds the slice;
//   3. k pass, per (b*h, piece, slice, row range): u_k, dphi_k, du_k; partial
//      dW_k, db_k;
//   4. reduction of the partials over the batch, chunks/slices and row
//      ranges in a fixed order (deterministic), into the parameter layouts.
#include <cuda_bf16.h>
#include <stdint.h>

#include "internal.h"
#include "layout.cuh"

namespace rehyat {
namespace {

constexpr int kRows = 32;        // token rows per tile
constexpr int kPiece = 128;      // features per CTA (one piece)
constexpr int kBwdThreads = 256;

__device__ __forceinline__ float load_x(const void* base, long long i, int bf16) {
  if (bf16) {
    const unsigned short b = reinterpret_cast<const unsigned short*>(base)[i];
    return __uint_as_float(static_cast<unsigned>(b) << 16);
  }
  return reinterpret_cast<const float*>(base)[i];
}

// Parameter layouts: W [h][2][D][Dp/2], b [h][2][Dp/2]; feature f of the
// concatenated map is column f mod Dp/2 of part f / (Dp/2).
__device__ __forceinline__ long long w_at(int h, int D, int Dp, int d, int f) {
  const int half = Dp >> 1, part = f >= half;
  return (static_cast<long long>(h * 2 + part) * D + d) * half + (f - part * half);
}
__device__ __forceinline__ long long b_at(int h, int Dp, int f) {
  const int half = Dp >> 1, part = f >= half;
  return static_cast<long long>(h * 2 + part) * half + (f - part * half);
}

// Shared-memory tile products for a 32-row tile and a piece of pw <= 128
// features, 256 threads.  out[r][c] (r < 32, c < 128) for thread t covers
// rows 4*(t/32) .. +3 and columns t%32 + 32*i, i < 4.
template <int D>
__device__ __forceinline__ void tile_times(const float* X /*[32][D]*/, const float* M /*[D][128]*/,
                                           float acc[4][4]) {
  const int rg = (threadIdx.x >> 5) * 4, lane = threadIdx.x & 31;
#pragma unroll 4
  for (int d = 0; d < D; ++d) {
    float x[4], m[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) x[i] = X[(rg + i) * D + d];
#pragma unroll
    for (int i = 0; i < 4; ++i) m[i] = M[d * kPiece + lane + 32 * i];
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
      for (int b = 0; b < 4; ++b) acc[a][b] = fmaf(x[a], m[b], acc[a][b]);
  }
}

// Outer-product accumulation over the tile's rows: acc[j][i] += sum_r
// A[r][a0 + j] * B[r][c0 + 16 i] for an 8 x 8 block per thread; A is [32][lda],
// B is [32][ldb].  Thread t: a0 = 8 * (t / 16), c0 = t % 16.
__device__ __forceinline__ void tile_outer(const float* A, int lda, const float* B, int ldb,
                                           float acc[8][8]) {
  const int a0 = (threadIdx.x >> 4) * 8, c0 = threadIdx.x & 15;
#pragma unroll 2
  for (int r = 0; r < kRows; ++r) {
    float a[8], b[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) a[j] = A[r * lda + a0 + j];
#pragma unroll
    for (int i = 0; i < 8; ++i) b[i] = B[r * ldb + c0 + 16 * i];
#pragma unroll
    for (int j = 0; j < 8; ++j)
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[j][i] = fmaf(a[j], b[i], acc[j][i]);
  }
}

struct BwdParams {
  const void *q, *k, *v;
  const float *y, *dy, *den;
  const float *Wq, *bq, *Wk, *bk;
  const float *SL, *zL;          // linear-set state per chunk (SL in the image layout)
  float *qpart;                  // [BH*FP][nchunks][QS][D*pw + pw + pw*D + pw]
  float *ghat;                   // [BH*FP][T][pw*D + pw]
  float *kpart;                  // [BH*FP][T][KS][D*pw + pw]
  int BH, heads, T, HW, D, Dp, Tc, To, causal, nchunks, in_bf16, QS, KS, FP;
};

__device__ __forceinline__ long long qpart_size(int D) {
  return 2LL * D * kPiece + 2LL * kPiece;
}

// ---------------------------------------------------------------- pass 1
template <int D>
__global__ void __launch_bounds__(kBwdThreads, 1) phi_bwd_q_kernel(BwdParams P) {
  extern __shared__ float sm[];
  float* Ws = sm;                        // [D][128]  W_q piece
  float* SLT = Ws + D * kPiece;          // [D][128]  S_L piece, transposed
  float* Xs = SLT + D * kPiece;          // [32][D]   q tile
  float* Es = Xs + kRows * D;            // [32][D]   dy / den
  float* Us = Es + kRows * D;            // [32][128] u_q, then phi_q
  float* Ds = Us + kRows * kPiece;       // [32][128] dphi_q, then du_q
  float* zl = Ds + kRows * kPiece;       // [128]
  float* bs = zl + kPiece;               // [128]
  float* rr = bs + kPiece;               // [32]     (dy . y) / den
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int qs = blockIdx.x, t = blockIdx.y;
  const int bh = blockIdx.z / P.FP, pf = blockIdx.z % P.FP, h = bh % P.heads;
  const int Dp = P.Dp, pw = Dp < kPiece ? Dp : kPiece, f0 = pf * pw;
  // Rows of chunk t, split into QS ranges.
  const int first = t * P.Tc, end = min(P.T, first + P.Tc);
  const long long c0 = static_cast<long long>(first) * P.HW, c1 = static_cast<long long>(end) * P.HW;
  const long long span = (c1 - c0 + P.QS - 1) / P.QS;
  const long long r0 = c0 + qs * span, r1 = min(c1, r0 + span);
  const long long N = static_cast<long long>(P.T) * P.HW;
  const long long rowbase = static_cast<long long>(bh) * N;

  for (int i = tid; i < D * kPiece; i += kBwdThreads) {
    const int d = i / kPiece, c = i % kPiece;
    Ws[i] = c < pw ? __ldg(P.Wq + w_at(h, D, Dp, d, f0 + c)) : 0.f;
    SLT[i] = c < pw ? __ldg(P.SL + (static_cast<long long>(bh) * P.nchunks + t) * Dp * D +
                            sl_index(f0 + c, d, D, Dp))
                    : 0.f;
  }
  for (int c = tid; c < kPiece; c += kBwdThreads) {
    zl[c] = c < pw ? __ldg(P.zL + (static_cast<long long>(bh) * P.nchunks + t) * Dp + f0 + c) : 0.f;
    bs[c] = c < pw ? __ldg(P.bq + b_at(h, Dp, f0 + c)) : 0.f;
  }
  float accW[8][8], accG[8][8];  // dW_q [d][c] and G [c][d] blocks
#pragma unroll
  for (int j = 0; j < 8; ++j)
#pragma unroll
    for (int i = 0; i < 8; ++i) accW[j][i] = accG[j][i] = 0.f;
  float accb = 0.f, acch = 0.f;  // db_q[c], h[c] for c = tid < 128

  for (long long tr0 = r0; tr0 < r1; tr0 += kRows) {
    __syncthreads();
    // Tile loads; rows past r1 are zero (they then contribute nothing).
    for (int i = tid; i < kRows * D; i += kBwdThreads) {
      const int r = i / D, d = i % D;
      const long long row = tr0 + r;
      const bool ok = row < r1;
      const long long gi = (rowbase + row) * D + d;
      Xs[i] = ok ? load_x(P.q, gi, P.in_bf16) : 0.f;
      Es[i] = ok ? __ldg(P.dy + gi) / __ldg(P.den + rowbase + row) : 0.f;
    }
    // (dy . y) / den per row: warp w handles rows 4w .. 4w+3.
    for (int r = warp * 4; r < warp * 4 + 4; ++r) {
      const long long row = tr0 + r;
      float s = 0.f;
      if (row < r1)
        for (int d = lane; d < D; d += 32)
          s = fmaf(__ldg(P.dy + (rowbase + row) * D + d), __ldg(P.y + (rowbase + row) * D + d), s);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
      if (lane == 0) rr[r] = row < r1 ? s / __ldg(P.den + rowbase + row) : 0.f;
    }
    __syncthreads();
    {
      // u = q W + b and dphi = e S_L^T - r z_L for this thread's 4 x 4 outputs.
      float u[4][4] = {}, g[4][4] = {};
      tile_times<D>(Xs, Ws, u);
      tile_times<D>(Es, SLT, g);
      const int rg = warp * 4;
#pragma unroll
      for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int b = 0; b < 4; ++b) {
          const int c = lane + 32 * b;
          const float uu = u[a][b] + bs[c];
          const float dphi = g[a][b] - rr[rg + a] * zl[c];
          Us[(rg + a) * kPiece + c] = uu * uu;         // phi_q
          Ds[(rg + a) * kPiece + c] = 2.f * uu * dphi;  // du_q
        }
    }
    __syncthreads();
    // dW_q[d][c] += sum_r q[r][d] du[r][c];  G[c][d] += sum_r phi[r][c] e[r][d]
    tile_outer(Xs, D, Ds, kPiece, accW);
    tile_outer(Us, kPiece, Es, D, accG);
    if (tid < kPiece) {
      for (int r = 0; r < kRows; ++r) {
        accb += Ds[r * kPiece + tid];
        acch -= Us[r * kPiece + tid] * rr[r];
      }
    }
  }
  // Partials of this CTA: [dW (D x 128)] [db (128)] [G (128 x D)] [h (128)].
  float* out = P.qpart + ((static_cast<long long>(blockIdx.z) * P.nchunks + t) * P.QS + qs) *
                             qpart_size(D);
  const int a0 = (tid >> 4) * 8, cc = tid & 15;
  if (a0 < D) {
#pragma unroll
    for (int j = 0; j < 8; ++j)
#pragma unroll
      for (int i = 0; i < 8; ++i) out[(a0 + j) * kPiece + cc + 16 * i] = accW[j][i];
  }
  float* outG = out + D * kPiece + kPiece;
  // accG rows are features (a0 + j < 128), columns d = cc + 16 i.
#pragma unroll
  for (int j = 0; j < 8; ++j)
#pragma unroll
    for (int i = 0; i < 8; ++i)
      if (cc + 16 * i < D) outG[(a0 + j) * D + cc + 16 * i] = accG[j][i];
  if (tid < kPiece) {
    out[D * kPiece + tid] = accb;
    outG[kPiece * D + tid] = acch;
  }
}

// ---------------------------------------------------------------- pass 2
// Pass 2 in two parallel steps.  (a) One thread per (element, chunk): G_t
// (and h_t) as the sum of its QS partials, stored in place of partial 0.
// grid (ceil(n/256), nchunks, BH*FP).
__global__ void phi_bwd_gsum_kernel(BwdParams P) {
  const int D = P.D;
  const long long n = static_cast<long long>(kPiece) * D + kPiece;
  const long long e = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (e >= n) return;
  const long long psz = qpart_size(D);
  float* g = P.qpart + (static_cast<long long>(blockIdx.z) * P.nchunks + blockIdx.y) * P.QS * psz +
             static_cast<long long>(D) * kPiece + kPiece + e;
  float acc = 0.f;
  for (int qs = 0; qs < P.QS; ++qs) acc += g[qs * psz];
  g[0] = acc;
}

// (b) One thread per (element, slice): Ghat_s = the sum of G_t over the
// chunks whose linear set holds s, in chunk order.  grid (ceil(n/256), T, BH*FP).
__global__ void phi_bwd_gsel_kernel(BwdParams P) {
  const int D = P.D;
  const long long n = static_cast<long long>(kPiece) * D + kPiece;
  const long long e = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (e >= n) return;
  const int s = blockIdx.y;
  const long long psz = qpart_size(D);
  const float* g = P.qpart + static_cast<long long>(blockIdx.z) * P.nchunks * P.QS * psz +
                   static_cast<long long>(D) * kPiece + kPiece + e;
  float acc = 0.f;
  for (int t = 0; t < P.nchunks; ++t) {
    const int first = t * P.Tc, end = min(P.T, first + P.Tc);
    const int w = max(first - P.To, 0);
    if (P.causal ? s < w : (s < w || s >= end)) acc += g[static_cast<long long>(t) * P.QS * psz];
  }
  P.ghat[(static_cast<long long>(blockIdx.z) * P.T + s) * n + e] = acc;
}

// Both steps in one launch when a (b, h) has at most kGhatChunks chunks: a
// block takes kGhatCols consecutive elements; its threads first form G_t of
// every chunk for them (the sum of the QS partials, in order) in shared
// memory, then Ghat_s of every slice (chunks in order).  The same sums in the
// same order as (a) and (b), with each partial read once.  A thread owns four
// consecutive elements (16-byte loads and stores; partial sizes, offsets and
// the element count per (b, h) are multiples of four floats) and issues four
// partials' loads before it adds them, in order.
constexpr int kGhatChunks = 48, kGhatCols = 128, kGhatVec = kGhatCols / 4;
__global__ void __launch_bounds__(256) phi_bwd_ghat_fused_kernel(BwdParams P) {
  __shared__ float4 G[kGhatChunks][kGhatVec];
  const int D = P.D;
  const long long n = static_cast<long long>(kPiece) * D + kPiece;
  const long long e0 = static_cast<long long>(blockIdx.x) * kGhatCols;
  const long long psz = qpart_size(D);
  const float* g = P.qpart + static_cast<long long>(blockIdx.z) * P.nchunks * P.QS * psz +
                   static_cast<long long>(D) * kPiece + kPiece + e0;
  auto add4 = [](float4& a, const float4 b) {
    a.x += b.x;
    a.y += b.y;
    a.z += b.z;
    a.w += b.w;
  };
  for (int idx = threadIdx.x; idx < P.nchunks * kGhatVec; idx += blockDim.x) {
    const int t = idx / kGhatVec, j4 = idx % kGhatVec;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    if (e0 + 4 * j4 < n) {
      const float* src = g + static_cast<long long>(t) * P.QS * psz + 4 * j4;
      for (int qs0 = 0; qs0 < P.QS; qs0 += 4) {
        float4 x[4];
#pragma unroll
        for (int u = 0; u < 4; ++u)
          if (qs0 + u < P.QS) x[u] = __ldg(reinterpret_cast<const float4*>(src + (qs0 + u) * psz));
#pragma unroll
        for (int u = 0; u < 4; ++u)
          if (qs0 + u < P.QS) add4(acc, x[u]);
      }
    }
    G[t][j4] = acc;
  }
  __syncthreads();
  float* out = P.ghat + static_cast<long long>(blockIdx.z) * P.T * n + e0;
  for (int idx = threadIdx.x; idx < P.T * kGhatVec; idx += blockDim.x) {
    const int s = idx / kGhatVec, j4 = idx % kGhatVec;
    if (e0 + 4 * j4 >= n) continue;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int t = 0; t < P.nchunks; ++t) {
      const int first = t * P.Tc, end = min(P.T, first + P.Tc);
      const int w = max(first - P.To, 0);
      if (P.causal ? s < w : (s < w || s >= end)) add4(acc, G[t][j4]);
    }
    *reinterpret_cast<float4*>(out + static_cast<long long>(s) * n + 4 * j4) = acc;
  }
}

// Ghat pass.
void launch_ghat(const BwdParams& bp, cudaStream_t s) {
  const long long ng = static_cast<long long>(kPiece) * bp.D + kPiece;
  const unsigned gx = static_cast<unsigned>((ng + 255) / 256);
  if (bp.nchunks <= kGhatChunks) {
    const unsigned gb = static_cast<unsigned>((ng + kGhatCols - 1) / kGhatCols);
    phi_bwd_ghat_fused_kernel<<<dim3(gb, 1, bp.BH * bp.FP), 256, 0, s>>>(bp);
    return;
  }
  phi_bwd_gsum_kernel<<<dim3(gx, bp.nchunks, bp.BH * bp.FP), 256, 0, s>>>(bp);
  phi_bwd_gsel_kernel<<<dim3(gx, bp.T, bp.BH * bp.FP), 256, 0, s>>>(bp);
}

// ---------------------------------------------------------------- pass 3
template <int D>
__global__ void __launch_bounds__(kBwdThreads, 1) phi_bwd_k_kernel(BwdParams P) {
  extern __shared__ float sm[];
  float* Ws = sm;                        // [D][128]  W_k piece
  float* GT = Ws + D * kPiece;           // [D][128]  Ghat piece, transposed
  float* Xs = GT + D * kPiece;           // [32][D]   k tile
  float* Vs = Xs + kRows * D;            // [32][D]   v tile
  float* Ds = Vs + kRows * D;            // [32][128] du_k
  float* hs = Ds + kRows * kPiece;       // [128]
  float* bs = hs + kPiece;               // [128]
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int ks = blockIdx.x, s = blockIdx.y;
  const int bh = blockIdx.z / P.FP, pf = blockIdx.z % P.FP, h = bh % P.heads;
  const int Dp = P.Dp, pw = Dp < kPiece ? Dp : kPiece, f0 = pf * pw;
  const long long span = (P.HW + P.KS - 1) / P.KS;
  const long long r0 = static_cast<long long>(s) * P.HW + ks * span;
  const long long r1 = min(static_cast<long long>(s + 1) * P.HW, r0 + span);
  const long long N = static_cast<long long>(P.T) * P.HW;
  const long long rowbase = static_cast<long long>(bh) * N;
  const float* gh = P.ghat + (static_cast<long long>(blockIdx.z) * P.T + s) *
                                 (static_cast<long long>(kPiece) * D + kPiece);
  for (int i = tid; i < D * kPiece; i += kBwdThreads) {
    const int d = i / kPiece, c = i % kPiece;
    Ws[i] = c < pw ? __ldg(P.Wk + w_at(h, D, Dp, d, f0 + c)) : 0.f;
    GT[i] = gh[c * D + d];  // Ghat[c][d]
  }
  for (int c = tid; c < kPiece; c += kBwdThreads) {
    hs[c] = gh[kPiece * D + c];
    bs[c] = c < pw ? __ldg(P.bk + b_at(h, Dp, f0 + c)) : 0.f;
  }
  float accW[8][8];
#pragma unroll
  for (int j = 0; j < 8; ++j)
#pragma unroll
    for (int i = 0; i < 8; ++i) accW[j][i] = 0.f;
  float accb = 0.f;
  for (long long tr0 = r0; tr0 < r1; tr0 += kRows) {
    __syncthreads();
    for (int i = tid; i < kRows * D; i += kBwdThreads) {
      const int r = i / D, d = i % D;
      const long long row = tr0 + r;
      const bool ok = row < r1;
      const long long gi = (rowbase + row) * D + d;
      Xs[i] = ok ? load_x(P.k, gi, P.in_bf16) : 0.f;
      Vs[i] = ok ? load_x(P.v, gi, P.in_bf16) : 0.f;
    }
    __syncthreads();
    {
      float u[4][4] = {}, g[4][4] = {};
      tile_times<D>(Xs, Ws, u);
      tile_times<D>(Vs, GT, g);
      const int rg = warp * 4;
#pragma unroll
      for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int b = 0; b < 4; ++b) {
          const int c = lane + 32 * b;
          const bool ok = tr0 + rg + a < r1;  // padded rows: u = b, but dphi must be 0
          const float dphi = ok ? g[a][b] + hs[c] : 0.f;
          Ds[(rg + a) * kPiece + c] = 2.f * (u[a][b] + bs[c]) * dphi;
        }
    }
    __syncthreads();
    tile_outer(Xs, D, Ds, kPiece, accW);
    if (tid < kPiece)
      for (int r = 0; r < kRows; ++r) accb += Ds[r * kPiece + tid];
  }
  float* out = P.kpart + ((static_cast<long long>(blockIdx.z) * P.T + s) * P.KS + ks) *
                             (static_cast<long long>(D) * kPiece + kPiece);
  const int a0 = (tid >> 4) * 8, cc = tid & 15;
  if (a0 < D) {
#pragma unroll
    for (int j = 0; j < 8; ++j)
#pragma unroll
      for (int i = 0; i < 8; ++i) out[(a0 + j) * kPiece + cc + 16 * i] = accW[j][i];
  }
  if (tid < kPiece) out[D * kPiece + tid] = accb;
}

// ---------------------------------------------------------------- pass 4
// One thread per four consecutive parameter elements of one head (four
// features of one W row, or of b, inside one feature piece: D' and the piece
// width are multiples of four): the sum over batch, chunks (slices) and row
// ranges of the partials, in a fixed order, read as 16-byte vectors with
// eight partials' loads in flight before they are added.
// grid (ceil(heads * (D*Dp + Dp) / 1024), 2): y = 0 -> (W_q, b_q), 1 -> (W_k, b_k).
__global__ void phi_bwd_reduce_kernel(BwdParams P, float* dWq, float* dbq, float* dWk, float* dbk,
                                      int batch) {
  const int D = P.D, Dp = P.Dp, pw = Dp < kPiece ? Dp : kPiece;
  const long long per_head = static_cast<long long>(D) * Dp + Dp;
  const long long e = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) * 4;
  if (e >= per_head * P.heads) return;
  const int h = static_cast<int>(e / per_head);
  const long long rem = e % per_head;
  const bool is_b = rem >= static_cast<long long>(D) * Dp;
  const int f = is_b ? static_cast<int>(rem - static_cast<long long>(D) * Dp)
                     : static_cast<int>(rem % Dp);
  const int d = is_b ? 0 : static_cast<int>(rem / Dp);
  const int pf = f / pw, c = f % pw;
  const bool qside = blockIdx.y == 0;
  const int nsets = qside ? P.nchunks * P.QS : P.T * P.KS;
  const long long psz = qside ? qpart_size(D) : static_cast<long long>(D) * kPiece + kPiece;
  const float* base = qside ? P.qpart : P.kpart;
  const long long off = is_b ? static_cast<long long>(D) * kPiece + c
                             : static_cast<long long>(d) * kPiece + c;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  auto add4 = [&](const float4 x) {
    acc.x += x.x;
    acc.y += x.y;
    acc.z += x.z;
    acc.w += x.w;
  };
  for (int b = 0; b < batch; ++b) {
    const long long z = static_cast<long long>(b * P.heads + h) * P.FP + pf;
    const float* src = base + z * nsets * psz + off;
    int i = 0;
    for (; i + 8 <= nsets; i += 8) {
      float4 x[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) x[u] = __ldg(reinterpret_cast<const float4*>(src + (i + u) * psz));
#pragma unroll
      for (int u = 0; u < 8; ++u) add4(x[u]);
    }
    for (; i < nsets; ++i) add4(__ldg(reinterpret_cast<const float4*>(src + i * psz)));
  }
  const float v[4] = {acc.x, acc.y, acc.z, acc.w};
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    if (is_b)
      (qside ? dbq : dbk)[b_at(h, Dp, f + u)] = v[u];
    else
      (qside ? dWq : dWk)[w_at(h, D, Dp, d, f + u)] = v[u];
  }
}

template <int D>
cudaError_t launch_bwd_d(const BwdParams& bp, const PhiBwdArgs& a, cudaStream_t s) {
  const size_t smq = sizeof(float) * (2 * D * kPiece + 2 * kRows * D + 2 * kRows * kPiece +
                                      2 * kPiece + kRows);
  const size_t smk = sizeof(float) * (2 * D * kPiece + 2 * kRows * D + kRows * kPiece +
                                      2 * kPiece);
  cudaError_t e = cudaFuncSetAttribute(phi_bwd_q_kernel<D>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smq));
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(phi_bwd_k_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(smk));
  if (e != cudaSuccess) return e;
  phi_bwd_q_kernel<D><<<dim3(bp.QS, bp.nchunks, bp.BH * bp.FP), kBwdThreads, smq, s>>>(bp);
  launch_ghat(bp, s);
  phi_bwd_k_kernel<D><<<dim3(bp.KS, bp.T, bp.BH * bp.FP), kBwdThreads, smk, s>>>(bp);
  const long long nr = (static_cast<long long>(D) * bp.Dp + bp.Dp) * bp.heads;
  phi_bwd_reduce_kernel<<<dim3(static_cast<unsigned>((nr / 4 + 255) / 256), 2), 256, 0, s>>>(
      bp, a.dWq, a.dbq, a.dWk, a.dbk, a.batch);
  return cudaGetLastError();
}

}  // namespace

void phi_bwd_split(int T, int Tc, int HW, int* QS, int* KS) {
  // Row ranges per chunk (QS) and per slice (KS) of about 1000 rows.
  const int chunk_rows = (Tc < T ? Tc : T) * HW;
  *QS = (chunk_rows + 1023) / 1024;
  *KS = (HW + 1023) / 1024;
}

size_t phi_bwd_partial_floats(int BH, int T, int nchunks, int D, int Dp, int QS, int KS) {
  const size_t FP = Dp > kPiece ? Dp / kPiece : 1;
  const size_t z = static_cast<size_t>(BH) * FP;
  const size_t qsz = 2 * static_cast<size_t>(D) * kPiece + 2 * kPiece;
  const size_t gsz = static_cast<size_t>(kPiece) * D + kPiece;
  const size_t ksz = static_cast<size_t>(D) * kPiece + kPiece;
  return z * (static_cast<size_t>(nchunks) * QS * qsz + static_cast<size_t>(T) * gsz +
              static_cast<size_t>(T) * KS * ksz);
}

size_t phi_bwd_ghat_offset_floats(int BH, int nchunks, int D, int Dp, int QS) {
  const size_t FP = Dp > kPiece ? Dp / kPiece : 1;
  return static_cast<size_t>(BH) * FP * nchunks * QS *
         (2 * static_cast<size_t>(D) * kPiece + 2 * kPiece);
}

cudaError_t launch_phi_bwd(const PhiBwdArgs& a, cudaStream_t s) {
  BwdParams bp;
  bp.q = a.q; bp.k = a.k; bp.v = a.v;
  bp.y = a.y; bp.dy = a.dy; bp.den = a.den;
  bp.Wq = a.Wq; bp.bq = a.bq; bp.Wk = a.Wk; bp.bk = a.bk;
  bp.SL = a.SL; bp.zL = a.zL;
  bp.BH = a.batch * a.heads; bp.heads = a.heads; bp.T = a.T; bp.HW = a.HW; bp.D = a.D;
  bp.Dp = a.Dp; bp.Tc = a.Tc; bp.To = a.To; bp.causal = a.causal; bp.nchunks = a.nchunks;
  bp.in_bf16 = a.in_bf16;
  phi_bwd_split(a.T, a.Tc, a.HW, &bp.QS, &bp.KS);
  bp.FP = a.Dp > kPiece ? a.Dp / kPiece : 1;
  const size_t z = static_cast<size_t>(bp.BH) * bp.FP;
  bp.qpart = a.partials;
  bp.ghat = bp.qpart + z * a.nchunks * bp.QS * (2 * static_cast<size_t>(a.D) * kPiece + 2 * kPiece);
  bp.kpart = bp.ghat + z * a.T * (static_cast<size_t>(kPiece) * a.D + kPiece);
  if (a.tc) {
    // q and k passes on tcgen05; the Ghat and reduction passes as below.
    PhiBwdTcArgs t = {};
    t.BH = bp.BH; t.heads = bp.heads; t.T = bp.T; t.HW = bp.HW; t.Tc = bp.Tc;
    t.nchunks = bp.nchunks;
    t.x = a.q; t.gh = a.gh; t.r = a.r; t.w_img = a.wq_img; t.b = a.bq;
    t.M = a.SL; t.vec = a.zL; t.part = bp.qpart; t.splits = bp.QS; t.q_side = 1;
    t.dx = a.dq; t.dv = nullptr;
    cudaError_t e = launch_phi_bwd_tc(t, s);
    if (e != cudaSuccess) return e;
    launch_ghat(bp, s);
    t.x = a.k; t.v = a.v; t.w_img = a.wk_img; t.b = a.bk; t.M = bp.ghat; t.vec = nullptr;
    t.part = bp.kpart; t.splits = bp.KS; t.q_side = 0;
    t.dx = a.dk; t.dv = a.dv;
    e = launch_phi_bwd_tc(t, s);
    if (e != cudaSuccess) return e;
    const long long nr = (static_cast<long long>(a.D) * bp.Dp + bp.Dp) * bp.heads;
    phi_bwd_reduce_kernel<<<dim3(static_cast<unsigned>((nr / 4 + 255) / 256), 2), 256, 0, s>>>(
        bp, a.dWq, a.dbq, a.dWk, a.dbk, a.batch);
    return cudaGetLastError();
  }
  switch (a.D) {
    case 32: return launch_bwd_d<32>(bp, a, s);
    case 64: return launch_bwd_d<64>(bp, a, s);
    case 128: return launch_bwd_d<128>(bp, a, s);
  }
  return cudaErrorInvalidValue;
}

}  // namespace rehyat
