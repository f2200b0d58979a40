// Full backward of ReHyAt's chunked hybrid attention on fp32 CUDA cores:
// dL/dq, dL/dk, dL/dv (every shape and input dtype the forward takes).
//
// Source: "ReHyAt: Recurrent Hybrid Attention for Video Diffusion
// Transformers" (papernotes.org note), Method, Key designs 1-5.  Key design 5's
// second training stage fine-tunes the whole converted model, so gradients
// flow through q, k and v.  For a query i of chunk t (window W_t, linear set
// L_t), with g = dL/dy, den = n^S + n^L, gh_i = g_i / den_i and
// r_i = (g_i . y_i) / den_i:
//   e_ij = exp(s_ij - c_i), s_ij = scale q_i.k_j, c_i = max_{j in W_t} s_ij
//   dS_ij = e_ij (gh_i.v_j - r_i) - [j = j*_i] Dc_i,   Dc_i = sum_j e_ij (gh_i.v_j - r_i)
//     (the last term is the gradient through the maximum c_i: the linear
//     branch is not multiplied by exp(-c_i), so c_i is part of the function)
//   dq_i = scale sum_j dS_ij k_j + sum_p du_q,p W_q,p^T
//   dk_j = scale sum_i dS_ij q_i + sum_p du_k,p W_k,p^T
//   dv_j = sum_i e_ij gh_i + Ghat_s^T phi_k(k_j)
//   du_q = 2 u_q * (S_L gh - r z_L),  du_k = 2 u_k * (Ghat_s v + hhat_s)
// with Ghat_s, hhat_s the gradients of the linear-set states summed over the
// chunks whose linear set holds slice s (the feature-map backward's Ghat
// pass computes them).  j*_i is the window key with the largest logit as
// recomputed here in fp32 (the lowest index among equal ones); it differs
// from the forward's only where two logits tie to within rounding, where
// the function has a kink and either key gives a valid gradient.
//
// Kernels:
//   bwd_dq_kernel   per (b*h, chunk, 32 query rows): streams the window's
//                   keys in tiles of 32 (S, dP, dS on CUDA cores), dq, and
//                   per row r_i, Dc_i, j*_i for the next kernel;
//   bwd_dkv_kernel  per (b*h, 32 key rows): streams the query tiles of the
//                   chunks whose window holds a key of the tile, dk and dv.
// Both add the linear branch's part in their epilogue.  No atomics: every
// output element is written once, so repeated calls agree bit for bit.
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include <cuda_bf16.h>

#include "internal.h"
#include "layout.cuh"

namespace rehyat {
namespace {

constexpr int kT = 32;            // rows per tile (queries or keys)
constexpr int kThr = 256;
constexpr int kGhatPiece = 128;   // feature piece of the Ghat blocks

__device__ __forceinline__ float ldx(const void* base, long long i, int bf16) {
  if (bf16) {
    const unsigned short b = reinterpret_cast<const unsigned short*>(base)[i];
    return __uint_as_float(static_cast<unsigned>(b) << 16);
  }
  return reinterpret_cast<const float*>(base)[i];
}

// W [h][2][D][Dp/2]: feature f of the concatenated map is column f mod Dp/2
// of part f / (Dp/2).
__device__ __forceinline__ long long w_idx(int h, int D, int Dp, int d, int f) {
  const int half = Dp >> 1, part = f >= half;
  return (static_cast<long long>(h * 2 + part) * D + d) * half + (f - part * half);
}
__device__ __forceinline__ long long b_idx(int h, int Dp, int f) {
  const int half = Dp >> 1, part = f >= half;
  return static_cast<long long>(h * 2 + part) * half + (f - part * half);
}

// Reductions over the 8 threads of a row group (lanes 8g .. 8g+7 of a warp).
constexpr int kNone = 0x7fffffff;
__device__ __forceinline__ int group_min(int v) {
#pragma unroll
  for (int o = 1; o < 8; o <<= 1) v = min(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ float group_max(float v) {
#pragma unroll
  for (int o = 1; o < 8; o <<= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ float group_sum(float v) {
#pragma unroll
  for (int o = 1; o < 8; o <<= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// ---------------------------------------------------------------- dq
template <int D>
__global__ void __launch_bounds__(kThr) bwd_dq_kernel(AttnBwdParams P) {
  constexpr int DS = D + 1;  // padded smem rows
  extern __shared__ float sm[];
  float* Qs = sm;                  // [32][D]
  float* Gs = Qs + kT * D;         // [32][D]  gh = dy / den
  float* Ks = Gs + kT * D;         // [32][D+1]
  float* Vs = Ks + kT * DS;        // [32][D+1]
  float* Ss = Vs + kT * DS;        // [32][33] dS tile
  float* Us = Ss + kT * 33;        // [32][Dp] du_q (epilogue)
  float* rowc = Us + kT * P.Dp;    // [32] c
  float* rowr = rowc + kT;         // [32] r
  const int tid = threadIdx.x, lane = tid & 31;
  const int t = blockIdx.y, bh = blockIdx.z, h = bh % P.heads;
  const int first = t * P.Tc, end = min(P.T, first + P.Tc), w = max(first - P.To, 0);
  const long long N = static_cast<long long>(P.T) * P.HW;
  const long long q0 = static_cast<long long>(first) * P.HW + static_cast<long long>(blockIdx.x) * kT;
  const long long qend = static_cast<long long>(end) * P.HW;
  if (q0 >= qend) return;
  const long long base = static_cast<long long>(bh) * N;
  const long long k0 = static_cast<long long>(w) * P.HW, kend = qend;
  const int row = tid >> 3, sub = tid & 7;  // S mapping: row, keys 4 sub .. 4 sub + 3

  // Query tile, gh, c, r.
  for (int i = tid; i < kT * D; i += kThr) {
    const int rr = i / D, d = i % D;
    const long long g = q0 + rr;
    float qv = 0.f, gv = 0.f;
    if (g < qend) {
      qv = ldx(P.q, (base + g) * D + d, P.in_bf16);
      gv = P.dy[(base + g) * D + d] / P.den[base + g];
    }
    Qs[i] = qv;
    Gs[i] = gv;
  }
  {
    // r = (dy . y) / den: the 8 threads of a row group split the columns.
    const long long g = q0 + row;
    float acc = 0.f;
    if (g < qend)
      for (int d = sub; d < D; d += 8) acc += P.dy[(base + g) * D + d] * P.y[(base + g) * D + d];
    acc = group_sum(acc);
    if (sub == 0) {
      rowr[row] = g < qend ? acc / P.den[base + g] : 0.f;
      rowc[row] = g < qend ? P.c[base + g] : 0.f;
    }
  }
  __syncthreads();
  const float c_row = rowc[row], r_row = rowr[row];
  float Dc = 0.f;
  float best = -INFINITY;  // largest logit so far and its key (relative to k0)
  int jstar = kNone;
  // dq accumulators: thread (row, sub) owns columns sub + 8 m.
  float acc[D / 8];
#pragma unroll
  for (int m = 0; m < D / 8; ++m) acc[m] = 0.f;

  for (long long kt = k0; kt < kend; kt += kT) {
    for (int i = tid; i < kT * D; i += kThr) {
      const int rr = i / D, d = i % D;
      const long long g = kt + rr;
      const bool in = g < kend;
      Ks[rr * DS + d] = in ? ldx(P.k, (base + g) * D + d, P.in_bf16) : 0.f;
      Vs[rr * DS + d] = in ? ldx(P.v, (base + g) * D + d, P.in_bf16) : 0.f;
    }
    __syncthreads();
    float s[4], dp[4];
#pragma unroll
    for (int m = 0; m < 4; ++m) s[m] = dp[m] = 0.f;
#pragma unroll 8
    for (int d = 0; d < D; ++d) {
      const float qd = Qs[row * D + d], gd = Gs[row * D + d];
#pragma unroll
      for (int m = 0; m < 4; ++m) {
        s[m] = fmaf(qd, Ks[(4 * sub + m) * DS + d], s[m]);
        dp[m] = fmaf(gd, Vs[(4 * sub + m) * DS + d], dp[m]);
      }
    }
    float tmax = -INFINITY;
    int targ = kNone;
#pragma unroll
    for (int m = 0; m < 4; ++m) {
      const long long g = kt + 4 * sub + m;
      float ds = 0.f;
      if (g < kend) {
        const float sc = s[m] * P.scale;
        ds = expf(sc - c_row) * (dp[m] - r_row);
        if (sc > tmax) {
          tmax = sc;
          targ = static_cast<int>(g - k0);
        }
      }
      Dc += ds;
      Ss[row * 33 + 4 * sub + m] = ds;
    }
    // The tile's largest logit of the row and its first key; it replaces the
    // running one only if strictly larger (earlier keys win ties).
    const float gmax = group_max(tmax);
    targ = group_min(tmax == gmax ? targ : kNone);
    if (gmax > best) {
      best = gmax;
      jstar = targ;
    }
    __syncthreads();
#pragma unroll 4
    for (int kk = 0; kk < kT; ++kk) {
      const float ds = Ss[row * 33 + kk];
#pragma unroll
      for (int m = 0; m < D / 8; ++m) acc[m] = fmaf(ds, Ks[kk * DS + sub + 8 * m], acc[m]);
    }
    __syncthreads();
  }
  Dc = group_sum(Dc);
  const long long g = q0 + row;
  const bool valid = g < qend;
  // Softmax part, with the maximum's term: dq -= scale Dc k_{j*}.
  const long long js = jstar == kNone ? -1 : k0 + jstar;
#pragma unroll
  for (int m = 0; m < D / 8; ++m) {
    const float kj = (valid && js >= 0) ? ldx(P.k, (base + js) * D + sub + 8 * m, P.in_bf16) : 0.f;
    acc[m] = P.scale * (acc[m] - Dc * kj);
  }
  if (valid && sub == 0) {
    P.r[base + g] = r_row;
    P.Dc[base + g] = Dc;
    P.jstar[base + g] = static_cast<int>(js);
  }
  // Linear branch: du_q = 2 u_q * (S_L gh - r z_L) into Us, then
  // dq += sum_f du_q[f] W_q[d][f].
  const int Dp = P.Dp;
  const long long sl0 = (static_cast<long long>(bh) * P.nchunks + t) * Dp * D;
  for (int i = tid; i < kT * Dp; i += kThr) {
    const int rr = i / Dp, f = i % Dp;
    float u = P.bq[b_idx(h, Dp, f)], dphi = 0.f;
    for (int d = 0; d < D; ++d) {
      u = fmaf(Qs[rr * D + d], P.Wq[w_idx(h, D, Dp, d, f)], u);
      dphi = fmaf(P.SL[sl0 + sl_index(f, d, D, Dp)], Gs[rr * D + d], dphi);
    }
    dphi -= rowr[rr] * P.zL[(static_cast<long long>(bh) * P.nchunks + t) * Dp + f];
    Us[i] = 2.f * u * dphi;
  }
  __syncthreads();
#pragma unroll
  for (int m = 0; m < D / 8; ++m) {
    const int d = sub + 8 * m;
    float lin = 0.f;
    for (int f = 0; f < Dp; ++f) lin = fmaf(Us[row * Dp + f], P.Wq[w_idx(h, D, Dp, d, f)], lin);
    if (valid) P.dq[(base + g) * D + d] = acc[m] + lin;
  }
}

// ---------------------------------------------------------------- dk, dv
template <int D>
__global__ void __launch_bounds__(kThr) bwd_dkv_kernel(AttnBwdParams P) {
  constexpr int DS = D + 1;
  extern __shared__ float sm[];
  float* Ks = sm;                  // [32][D+1]
  float* Vs = Ks + kT * DS;        // [32][D+1]
  float* Qs = Vs + kT * DS;        // [32][D]
  float* Gs = Qs + kT * D;         // [32][D]
  float* Es = Gs + kT * D;         // [32 keys][33] e
  float* Ds = Es + kT * 33;        // [32 keys][33] dS
  float* qr = Ds + kT * 33;        // [32] r
  float* qc = qr + kT;             // [32] c
  float* qD = qc + kT;             // [32] Dc
  int* qj = reinterpret_cast<int*>(qD + kT);  // [32] j*
  float* Us = reinterpret_cast<float*>(qj + kT);  // [32][Dp] du_k (epilogue)
  float* Fs = Us + kT * P.Dp;      // [32][Dp] phi_k (epilogue)
  const int tid = threadIdx.x;
  const int bh = blockIdx.y, h = bh % P.heads;
  const long long N = static_cast<long long>(P.T) * P.HW;
  const long long j0 = static_cast<long long>(blockIdx.x) * kT;
  if (j0 >= N) return;
  const long long j1 = min(N, j0 + kT);
  const long long base = static_cast<long long>(bh) * N;
  const int kr = tid >> 3, sub = tid & 7;  // key row kr, queries 4 sub .. 4 sub + 3

  for (int i = tid; i < kT * D; i += kThr) {
    const int rr = i / D, d = i % D;
    const long long g = j0 + rr;
    Ks[rr * DS + d] = g < j1 ? ldx(P.k, (base + g) * D + d, P.in_bf16) : 0.f;
    Vs[rr * DS + d] = g < j1 ? ldx(P.v, (base + g) * D + d, P.in_bf16) : 0.f;
  }
  float dk[D / 8], dv[D / 8];
#pragma unroll
  for (int m = 0; m < D / 8; ++m) dk[m] = dv[m] = 0.f;
  const int s_lo = static_cast<int>(j0 / P.HW), s_hi = static_cast<int>((j1 - 1) / P.HW);
  const long long key = j0 + kr;
  for (int t = 0; t < P.nchunks; ++t) {
    const int first = t * P.Tc, end = min(P.T, first + P.Tc), w = max(first - P.To, 0);
    if (!(w <= s_hi && end > s_lo)) continue;  // no key of the tile in this window
    const long long wk0 = static_cast<long long>(w) * P.HW, wk1 = static_cast<long long>(end) * P.HW;
    const bool key_in = key < j1 && key >= wk0 && key < wk1;
    for (long long qt = static_cast<long long>(first) * P.HW; qt < wk1; qt += kT) {
      __syncthreads();  // previous tile's smem reads are done
      for (int i = tid; i < kT * D; i += kThr) {
        const int rr = i / D, d = i % D;
        const long long g = qt + rr;
        float qv = 0.f, gv = 0.f;
        if (g < wk1) {
          qv = ldx(P.q, (base + g) * D + d, P.in_bf16);
          gv = P.dy[(base + g) * D + d] / P.den[base + g];
        }
        Qs[i] = qv;
        Gs[i] = gv;
      }
      if (tid < kT) {
        const long long g = qt + tid;
        const bool in = g < wk1;
        qr[tid] = in ? P.r[base + g] : 0.f;
        qc[tid] = in ? P.c[base + g] : 0.f;
        qD[tid] = in ? P.Dc[base + g] : 0.f;
        qj[tid] = in ? P.jstar[base + g] : -1;
      }
      __syncthreads();
      float s[4], dp[4];
#pragma unroll
      for (int m = 0; m < 4; ++m) s[m] = dp[m] = 0.f;
#pragma unroll 8
      for (int d = 0; d < D; ++d) {
        const float kd = Ks[kr * DS + d], vd = Vs[kr * DS + d];
#pragma unroll
        for (int m = 0; m < 4; ++m) {
          s[m] = fmaf(Qs[(4 * sub + m) * D + d], kd, s[m]);
          dp[m] = fmaf(Gs[(4 * sub + m) * D + d], vd, dp[m]);
        }
      }
#pragma unroll
      for (int m = 0; m < 4; ++m) {
        const int qi = 4 * sub + m;
        float e = 0.f, ds = 0.f;
        if (key_in && qt + qi < wk1) {
          e = expf(s[m] * P.scale - qc[qi]);
          ds = e * (dp[m] - qr[qi]);
          if (qj[qi] == key) ds -= qD[qi];
        }
        Es[kr * 33 + qi] = e;
        Ds[kr * 33 + qi] = ds;
      }
      __syncthreads();
#pragma unroll 4
      for (int qi = 0; qi < kT; ++qi) {
        const float e = Es[kr * 33 + qi], ds = Ds[kr * 33 + qi];
#pragma unroll
        for (int m = 0; m < D / 8; ++m) {
          dv[m] = fmaf(e, Gs[qi * D + sub + 8 * m], dv[m]);
          dk[m] = fmaf(ds, Qs[qi * D + sub + 8 * m], dk[m]);
        }
      }
    }
  }
  __syncthreads();
  // Linear branch of each key row j (slice s): u_k, phi_k, du_k =
  // 2 u_k * (Ghat_s v_j + hhat_s); dk += sum_f du_k[f] W_k[d][f],
  // dv += sum_f Ghat_s[f][d] phi_k[f].
  const int Dp = P.Dp, pw = Dp < kGhatPiece ? Dp : kGhatPiece;
  const long long gn = static_cast<long long>(kGhatPiece) * D + kGhatPiece;
  for (int i = tid; i < kT * Dp; i += kThr) {
    const int rr = i / Dp, f = i % Dp;
    const long long g = j0 + rr;
    float u = 0.f, dphi = 0.f;
    if (g < j1) {
      const int sl = static_cast<int>(g / P.HW);
      const int pf = f / pw, fl = f - pf * pw;
      const float* gb = P.ghat + ((static_cast<long long>(bh) * P.FP + pf) * P.T + sl) * gn;
      u = P.bk[b_idx(h, Dp, f)];
      dphi = gb[static_cast<long long>(kGhatPiece) * D + fl];
      for (int d = 0; d < D; ++d) {
        u = fmaf(Ks[rr * DS + d], P.Wk[w_idx(h, D, Dp, d, f)], u);
        dphi = fmaf(gb[static_cast<long long>(fl) * D + d], Vs[rr * DS + d], dphi);
      }
    }
    Us[i] = 2.f * u * dphi;
    Fs[i] = u * u;
  }
  __syncthreads();
  if (key < j1) {
    const int sl = static_cast<int>(key / P.HW);
#pragma unroll
    for (int m = 0; m < D / 8; ++m) {
      const int d = sub + 8 * m;
      float lk = 0.f, lv = 0.f;
      for (int f = 0; f < Dp; ++f) {
        const int pf = f / pw, fl = f - pf * pw;
        const float* gb = P.ghat + ((static_cast<long long>(bh) * P.FP + pf) * P.T + sl) * gn;
        lk = fmaf(Us[kr * Dp + f], P.Wk[w_idx(h, D, Dp, d, f)], lk);
        lv = fmaf(gb[static_cast<long long>(fl) * D + d], Fs[kr * Dp + f], lv);
      }
      P.dk[(base + key) * D + d] = P.scale * dk[m] + lk;
      P.dv[(base + key) * D + d] = dv[m] + lv;
    }
  }
}

// ---------------------------------------------------------------- TC path
// Per query row (D = 128): r = (dy . y) / den and gh = bf16(dy / den), the
// A operand of the tensor-core products.  One warp per row, four columns
// per lane.
__global__ void __launch_bounds__(256) bwd_prep_kernel(const float* __restrict__ y,
                                                       const float* __restrict__ dy,
                                                       const float* __restrict__ den,
                                                       float* __restrict__ r,
                                                       uint2* __restrict__ gh, long long rows) {
  const long long row = static_cast<long long>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  const float4 g = reinterpret_cast<const float4*>(dy + row * 128)[lane];
  const float4 yy = reinterpret_cast<const float4*>(y + row * 128)[lane];
  float acc = g.x * yy.x + g.y * yy.y + g.z * yy.z + g.w * yy.w;
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  const float dn = den[row];
  if (lane == 0) r[row] = acc / dn;
  const float e0 = g.x / dn, e1 = g.y / dn, e2 = g.z / dn, e3 = g.w / dn;
  const __nv_bfloat162 lo = __floats2bfloat162_rn(e0, e1), hi = __floats2bfloat162_rn(e2, e3);
  gh[row * 32 + lane] = make_uint2(*reinterpret_cast<const uint32_t*>(&lo),
                                   *reinterpret_cast<const uint32_t*>(&hi));
}

// Linear branch of dq for 32 query rows of one chunk (added to dq):
// du_q = 2 u_q * (S_L gh - r z_L), dq += sum_f du_q[f] W_q[d][f].
template <int D>
__global__ void __launch_bounds__(kThr) bwd_lin_q_kernel(AttnBwdParams P) {
  extern __shared__ float sm[];
  float* Qs = sm;                  // [32][D]
  float* Gs = Qs + kT * D;         // [32][D] gh
  float* Us = Gs + kT * D;         // [32][Dp] du_q
  float* rowr = Us + kT * P.Dp;    // [32]
  const int tid = threadIdx.x;
  const int t = blockIdx.y, bh = blockIdx.z, h = bh % P.heads;
  const int first = t * P.Tc, end = min(P.T, first + P.Tc);
  const long long N = static_cast<long long>(P.T) * P.HW;
  const long long q0 = static_cast<long long>(first) * P.HW + static_cast<long long>(blockIdx.x) * kT;
  const long long qend = static_cast<long long>(end) * P.HW;
  if (q0 >= qend) return;
  const long long base = static_cast<long long>(bh) * N;
  const int Dp = P.Dp;
  for (int i = tid; i < kT * D; i += kThr) {
    const int rr = i / D, d = i % D;
    const long long g = q0 + rr;
    const bool in = g < qend;
    Qs[i] = in ? ldx(P.q, (base + g) * D + d, P.in_bf16) : 0.f;
    Gs[i] = in ? P.dy[(base + g) * D + d] / P.den[base + g] : 0.f;
  }
  if (tid < kT) rowr[tid] = q0 + tid < qend ? P.r[base + q0 + tid] : 0.f;
  __syncthreads();
  const long long sl0 = (static_cast<long long>(bh) * P.nchunks + t) * Dp * D;
  for (int i = tid; i < kT * Dp; i += kThr) {
    const int rr = i / Dp, f = i % Dp;
    float u = P.bq[b_idx(h, Dp, f)], dphi = 0.f;
    for (int d = 0; d < D; ++d) {
      u = fmaf(Qs[rr * D + d], P.Wq[w_idx(h, D, Dp, d, f)], u);
      dphi = fmaf(P.SL[sl0 + sl_index(f, d, D, Dp)], Gs[rr * D + d], dphi);
    }
    dphi -= rowr[rr] * P.zL[(static_cast<long long>(bh) * P.nchunks + t) * Dp + f];
    Us[i] = 2.f * u * dphi;
  }
  __syncthreads();
  const int row = tid >> 3, sub = tid & 7;
  const long long g = q0 + row;
  if (g >= qend) return;
#pragma unroll
  for (int m = 0; m < D / 8; ++m) {
    const int d = sub + 8 * m;
    float lin = 0.f;
    for (int f = 0; f < Dp; ++f) lin = fmaf(Us[row * Dp + f], P.Wq[w_idx(h, D, Dp, d, f)], lin);
    P.dq[(base + g) * D + d] += lin;
  }
}

// Linear branch of dk, dv for 32 key rows (added to dk, dv): u_k, phi_k,
// du_k = 2 u_k * (Ghat_s v + hhat_s); dk += du_k W_k^T, dv += Ghat_s^T phi_k.
template <int D>
__global__ void __launch_bounds__(kThr) bwd_lin_kv_kernel(AttnBwdParams P) {
  extern __shared__ float sm[];
  float* Ks = sm;                  // [32][D]
  float* Vs = Ks + kT * D;         // [32][D]
  float* Us = Vs + kT * D;         // [32][Dp] du_k
  float* Fs = Us + kT * P.Dp;      // [32][Dp] phi_k
  const int tid = threadIdx.x;
  const int bh = blockIdx.y, h = bh % P.heads;
  const long long N = static_cast<long long>(P.T) * P.HW;
  const long long j0 = static_cast<long long>(blockIdx.x) * kT;
  if (j0 >= N) return;
  const long long j1 = min(N, j0 + kT);
  const long long base = static_cast<long long>(bh) * N;
  const int Dp = P.Dp, pw = Dp < kGhatPiece ? Dp : kGhatPiece;
  const long long gn = static_cast<long long>(kGhatPiece) * D + kGhatPiece;
  for (int i = tid; i < kT * D; i += kThr) {
    const int rr = i / D, d = i % D;
    const long long g = j0 + rr;
    Ks[i] = g < j1 ? ldx(P.k, (base + g) * D + d, P.in_bf16) : 0.f;
    Vs[i] = g < j1 ? ldx(P.v, (base + g) * D + d, P.in_bf16) : 0.f;
  }
  __syncthreads();
  for (int i = tid; i < kT * Dp; i += kThr) {
    const int rr = i / Dp, f = i % Dp;
    const long long g = j0 + rr;
    float u = 0.f, dphi = 0.f;
    if (g < j1) {
      const int sl = static_cast<int>(g / P.HW);
      const int pf = f / pw, fl = f - pf * pw;
      const float* gb = P.ghat + ((static_cast<long long>(bh) * P.FP + pf) * P.T + sl) * gn;
      u = P.bk[b_idx(h, Dp, f)];
      dphi = gb[static_cast<long long>(kGhatPiece) * D + fl];
      for (int d = 0; d < D; ++d) {
        u = fmaf(Ks[rr * D + d], P.Wk[w_idx(h, D, Dp, d, f)], u);
        dphi = fmaf(gb[static_cast<long long>(fl) * D + d], Vs[rr * D + d], dphi);
      }
    }
    Us[i] = 2.f * u * dphi;
    Fs[i] = u * u;
  }
  __syncthreads();
  const int kr = tid >> 3, sub = tid & 7;
  const long long key = j0 + kr;
  if (key >= j1) return;
  const int sl = static_cast<int>(key / P.HW);
#pragma unroll
  for (int m = 0; m < D / 8; ++m) {
    const int d = sub + 8 * m;
    float lk = 0.f, lv = 0.f;
    for (int f = 0; f < Dp; ++f) {
      const int pf = f / pw, fl = f - pf * pw;
      const float* gb = P.ghat + ((static_cast<long long>(bh) * P.FP + pf) * P.T + sl) * gn;
      lk = fmaf(Us[kr * Dp + f], P.Wk[w_idx(h, D, Dp, d, f)], lk);
      lv = fmaf(gb[static_cast<long long>(fl) * D + d], Fs[kr * Dp + f], lv);
    }
    P.dk[(base + key) * D + d] += lk;
    P.dv[(base + key) * D + d] += lv;
  }
}

template <int D>
cudaError_t launch_bwd_simt_d(const AttnBwdParams& p, cudaStream_t s) {
  const size_t smq = sizeof(float) * (2 * kT * D + 2 * kT * (D + 1) + kT * 33 +
                                      static_cast<size_t>(kT) * p.Dp + 2 * kT);
  const size_t smk = sizeof(float) * (2 * kT * (D + 1) + 2 * kT * D + 2 * kT * 33 + 4 * kT +
                                      2 * static_cast<size_t>(kT) * p.Dp);
  cudaError_t e = cudaFuncSetAttribute(bwd_dq_kernel<D>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smq));
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(bwd_dkv_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(smk));
  if (e != cudaSuccess) return e;
  const int chunk_rows = (p.Tc < p.T ? p.Tc : p.T) * p.HW;
  const dim3 gq((chunk_rows + kT - 1) / kT, p.nchunks, p.BH);
  bwd_dq_kernel<D><<<gq, kThr, smq, s>>>(p);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const long long N = static_cast<long long>(p.T) * p.HW;
  const dim3 gk(static_cast<unsigned>((N + kT - 1) / kT), p.BH);
  bwd_dkv_kernel<D><<<gk, kThr, smk, s>>>(p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_bwd_prep(const float* y, const float* dy, const float* den, float* r,
                            void* gh_bf16, long long rows, cudaStream_t s) {
  bwd_prep_kernel<<<static_cast<unsigned>((rows + 7) / 8), 256, 0, s>>>(
      y, dy, den, r, static_cast<uint2*>(gh_bf16), rows);
  return cudaGetLastError();
}

cudaError_t launch_attn_bwd_tc_kernels(const AttnBwdParams& p, const void* gh_bf16,
                                       bool accumulate, cudaStream_t s) {
  AttnBwdTcArgs a;
  a.q = p.q; a.k = p.k; a.v = p.v; a.gh = gh_bf16;
  a.c = p.c; a.r = p.r; a.Dc = p.Dc; a.jstar = p.jstar;
  a.dq = p.dq; a.dk = p.dk; a.dv = p.dv;
  a.BH = p.BH; a.T = p.T; a.HW = p.HW; a.Tc = p.Tc; a.To = p.To; a.nchunks = p.nchunks;
  a.accumulate = accumulate ? 1 : 0;
  a.scale = p.scale;
  cudaError_t e = launch_attn_bwd_dq_tc(a, s);
  if (e != cudaSuccess) return e;
  return launch_attn_bwd_dkv_tc(a, s);
}

cudaError_t launch_attn_bwd_tc_softmax(const AttnBwdParams& p, void* gh_bf16, bool accumulate,
                                       cudaStream_t s) {
  const long long rows = static_cast<long long>(p.T) * p.HW * p.BH;
  const cudaError_t e = launch_bwd_prep(p.y, p.dy, p.den, p.r, gh_bf16, rows, s);
  if (e != cudaSuccess) return e;
  return launch_attn_bwd_tc_kernels(p, gh_bf16, accumulate, s);
}

cudaError_t launch_attn_bwd_lin_simt(const AttnBwdParams& p, cudaStream_t s) {
  // The linear branch's parts, added to dq, dk, dv.
  constexpr int D = 128;
  cudaError_t e;
  const long long N = static_cast<long long>(p.T) * p.HW;
  const size_t smq = sizeof(float) * (2 * kT * D + static_cast<size_t>(kT) * p.Dp + kT);
  const size_t smk = sizeof(float) * (2 * kT * D + 2 * static_cast<size_t>(kT) * p.Dp);
  if ((e = cudaFuncSetAttribute(bwd_lin_q_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                static_cast<int>(smq))) != cudaSuccess)
    return e;
  if ((e = cudaFuncSetAttribute(bwd_lin_kv_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                static_cast<int>(smk))) != cudaSuccess)
    return e;
  const int chunk_rows = (p.Tc < p.T ? p.Tc : p.T) * p.HW;
  bwd_lin_q_kernel<D><<<dim3((chunk_rows + kT - 1) / kT, p.nchunks, p.BH), kThr, smq, s>>>(p);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  bwd_lin_kv_kernel<D><<<dim3(static_cast<unsigned>((N + kT - 1) / kT), p.BH), kThr, smk, s>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_attn_bwd_simt(const AttnBwdParams& p, cudaStream_t s) {
  switch (p.D) {
    case 32: return launch_bwd_simt_d<32>(p, s);
    case 64: return launch_bwd_simt_d<64>(p, s);
    case 128: return launch_bwd_simt_d<128>(p, s);
  }
  return cudaErrorInvalidValue;
}

}  // namespace rehyat
