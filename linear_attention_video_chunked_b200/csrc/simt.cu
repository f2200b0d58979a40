// fp32 CUDA-core kernels for ReHyAt's chunked hybrid attention.
//
// They cover every supported shape (D in {32, 64, 128}, Dp in {32..256}) and
// both input dtypes, compute in fp32 throughout, and are the exact-fp32 path
// (the tensor-core kernels round P and phi to narrower types).
//
// Source of the arithmetic: "ReHyAt: Recurrent Hybrid Attention for Video
// Diffusion Transformers" (papernotes.org note), Method, Key designs 1-4:
// window softmax with stabiliser c_t, linear branch phi_q(q) (sum phi_k v^T),
// joint normalisation, overlap set, causal set and chunk-wise state.
#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <math.h>

#include "internal.h"
#include "layout.cuh"

namespace rehyat {

// Rows whose joint denominator n^S + n^L fell below 2^-10 n^S (non-positive,
// NaN, or cancelled to ~10 bits) in a forward with phi given, since the last
// reset (see rehyat_denominator_report).
__device__ unsigned long long rehyat_simt_den_rows = 0;

namespace {

// Element i of a given feature map: fp32, or bf16 when bf16 is set.
__device__ __forceinline__ float ld_phi(const void* phi, int bf16, long long i) {
  return bf16 ? __bfloat162float(__ldg(static_cast<const __nv_bfloat16*>(phi) + i))
              : __ldg(static_cast<const float*>(phi) + i);
}


constexpr float kLn2 = 0.69314718055994530942f;

__device__ __forceinline__ float load_in(const void* base, long long i, int bf16) {
  if (bf16) {
    unsigned short b = reinterpret_cast<const unsigned short*>(base)[i];
    return __uint_as_float(static_cast<unsigned>(b) << 16);
  }
  return reinterpret_cast<const float*>(base)[i];
}

// Round an fp32 value to the nearest bf16 value (ties to even), kept as fp32.
__device__ __forceinline__ float round_bf16(float x) {
  return __bfloat162float(__float2bfloat16_rn(x));
}

__device__ __forceinline__ float load_w(const float* W, long long i, int w_bf16) {
  float w = __ldg(W + i);
  return w_bf16 ? round_bf16(w) : w;
}

__device__ __forceinline__ void store_out(void* base, long long i, float x, int bf16) {
  if (bf16)
    reinterpret_cast<__nv_bfloat16*>(base)[i] = __float2bfloat16_rn(x);
  else
    reinterpret_cast<float*>(base)[i] = x;
}

// phi feature f of part W[h][f / half][:, f % half]: column index helpers.
__device__ __forceinline__ long long w_index(int h, int D, int Dp, int d, int f) {
  const int half = Dp >> 1;
  const int part = f >= half;
  const int col = f - part * half;
  return ((static_cast<long long>(h) * 2 + part) * D + d) * half + col;
}
__device__ __forceinline__ long long b_index(int h, int Dp, int f) {
  const int half = Dp >> 1;
  const int part = f >= half;
  return (static_cast<long long>(h) * 2 + part) * half + (f - part * half);
}

// ---------------------------------------------------------------------------
// Window softmax + linear readout + joint normalisation.
// Block: 128 threads = 32 query rows x 4 lanes; key tiles of 32.
// ---------------------------------------------------------------------------
constexpr int kBQ = 32;
constexpr int kBK = 32;

template <int D>
__global__ void __launch_bounds__(128) attn_simt_kernel(AttnParams P) {
  extern __shared__ float smem[];
  float* Qs = smem;                        // [kBQ][D]
  float* Ks = Qs + kBQ * D;                // [kBK][D + 1]
  float* Vs = Ks + kBK * (D + 1);          // [kBK][D]
  float* Ps = Vs + kBK * D;                // [kBQ][kBK + 1]
  float* Fq = Qs + kBQ * D;                // [kBQ][Dp], reuses Ks.. after the loop

  const int tid = threadIdx.x;
  const int r = tid >> 2;
  const int lane4 = tid & 3;
  const int t = blockIdx.y;
  const int bh = blockIdx.z;
  const int h = bh % P.heads;

  // Query rows and key ranges of this chunk.
  long long q_first, q_end;
  const void *ka, *va, *kb = nullptr, *vb = nullptr;
  long long ka_off, na, kb_off = 0, nb = 0;
  if (P.seen == nullptr) {
    const int first = t * P.Tc;
    const int end = min(P.T, first + P.Tc);
    const int w = max(first - P.To, 0);
    q_first = static_cast<long long>(first) * P.HW;
    q_end = static_cast<long long>(end) * P.HW;
    ka = P.k; va = P.v;
    ka_off = bh * P.rows_per_bh + static_cast<long long>(w) * P.HW;
    na = static_cast<long long>(end - w) * P.HW;
  } else {
    const long long seen = *P.seen;
    const long long r_slices = seen < P.To ? seen : P.To;
    q_first = 0;
    q_end = static_cast<long long>(P.nq_slices) * P.HW;
    ka = P.rk; va = P.rv;
    ka_off = bh * P.ring_rows_per_bh;
    na = r_slices * P.HW;
    kb = P.k; vb = P.v;
    kb_off = bh * P.rows_per_bh;
    nb = q_end;
  }
  const long long row0 = q_first + static_cast<long long>(blockIdx.x) * kBQ;
  if (row0 >= q_end) return;
  const int nrows = static_cast<int>(min(static_cast<long long>(kBQ), q_end - row0));
  const long long qrow_base = bh * P.rows_per_bh + row0;

  for (int i = tid; i < kBQ * D; i += 128) {
    const int rr = i / D, d = i % D;
    Qs[i] = rr < nrows ? load_in(P.q, (qrow_base + rr) * D + d, P.in_bf16) : 0.f;
  }

  float o[D / 4];
#pragma unroll
  for (int c = 0; c < D / 4; ++c) o[c] = 0.f;
  float m = -INFINITY, l = 0.f;

  for (int range = 0; range < 2; ++range) {
    const void* kp = range == 0 ? ka : kb;
    const void* vp = range == 0 ? va : vb;
    const long long off = range == 0 ? ka_off : kb_off;
    const long long n = range == 0 ? na : nb;
    for (long long kt = 0; kt < n; kt += kBK) {
      __syncthreads();
      for (int i = tid; i < kBK * D; i += 128) {
        const int j = i / D, d = i % D;
        const bool ok = kt + j < n;
        const long long gi = (off + kt + j) * D + d;
        Ks[j * (D + 1) + d] = ok ? load_in(kp, gi, P.in_bf16) : 0.f;
        Vs[j * D + d] = ok ? load_in(vp, gi, P.in_bf16) : 0.f;
      }
      __syncthreads();
      float s[kBK / 4];
      float mt = -INFINITY;
#pragma unroll
      for (int i = 0; i < kBK / 4; ++i) {
        const int j = lane4 + 4 * i;
        float acc = 0.f;
#pragma unroll 8
        for (int d = 0; d < D; ++d) acc = fmaf(Qs[r * D + d], Ks[j * (D + 1) + d], acc);
        s[i] = (kt + j < n) ? acc * P.scale_log2 : -INFINITY;
        mt = fmaxf(mt, s[i]);
      }
      mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, 1));
      mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, 2));
      const float m_new = fmaxf(m, mt);
      const float alpha = exp2f(m - m_new);
      float lsum = 0.f;
#pragma unroll
      for (int i = 0; i < kBK / 4; ++i) {
        const float pv = exp2f(s[i] - m_new);
        Ps[r * (kBK + 1) + lane4 + 4 * i] = pv;
        lsum += pv;
      }
      l = l * alpha + lsum;
      m = m_new;
      __syncwarp();
#pragma unroll
      for (int c = 0; c < D / 4; ++c) {
        const int col = lane4 + 4 * c;
        float acc = o[c] * alpha;
#pragma unroll 8
        for (int j = 0; j < kBK; ++j) acc = fmaf(Ps[r * (kBK + 1) + j], Vs[j * D + col], acc);
        o[c] = acc;
      }
    }
  }
  l += __shfl_xor_sync(0xffffffffu, l, 1);
  l += __shfl_xor_sync(0xffffffffu, l, 2);

  // Linear branch: phi_q(q) . S^L and phi_q(q) . z^L.
  float aL[D / 4];
  float nL = 0.f;
#pragma unroll
  for (int c = 0; c < D / 4; ++c) aL[c] = 0.f;
  if (!P.full_softmax) {
    __syncthreads();
    const int Dp = P.Dp;
    const float* SL = P.SL + (static_cast<long long>(bh) * P.nchunks + t) * Dp * D;
    const float* zL = P.zL + (static_cast<long long>(bh) * P.nchunks + t) * Dp;
    for (int f = lane4; f < Dp; f += 4) {
      float ph;
      if (P.phi_q) {  // phi_q(q) given
        ph = r < nrows ? ld_phi(P.phi_q, P.phi_bf16, (qrow_base + r) * Dp + f) : 0.f;
      } else {
        float psi = __ldg(P.bq + b_index(h, Dp, f));
        for (int d = 0; d < D; ++d)
          psi = fmaf(Qs[r * D + d], load_w(P.Wq, w_index(h, D, Dp, d, f), P.w_bf16), psi);
        ph = psi * psi;
      }
      Fq[r * Dp + f] = ph;
      nL = fmaf(ph, __ldg(zL + f), nL);
    }
    nL += __shfl_xor_sync(0xffffffffu, nL, 1);
    nL += __shfl_xor_sync(0xffffffffu, nL, 2);
    __syncwarp();
    for (int f = 0; f < Dp; ++f) {
      const float ph = Fq[r * Dp + f];
#pragma unroll
      for (int c = 0; c < D / 4; ++c)
        aL[c] = fmaf(ph, __ldg(SL + sl_index(f, lane4 + 4 * c, D, Dp)), aL[c]);
    }
  }

  if (r < nrows) {
    const long long row = qrow_base + r;
    const float den = l + nL;
    // A signed phi (degree-1 parts) can drive n^L towards -n^S: count the
    // rows, the output stays as the formula gives it.
    if (P.phi_q && lane4 == 0 && !(den >= ldexpf(l, -10)))
      atomicAdd(&rehyat_simt_den_rows, 1ull);
#pragma unroll
    for (int c = 0; c < D / 4; ++c) {
      const int col = lane4 + 4 * c;
      store_out(P.y, row * D + col, __fdiv_rn(o[c] + aL[c], den), P.out_bf16);
      if (P.dbg_aS) P.dbg_aS[row * D + col] = o[c];
      if (P.dbg_aL) P.dbg_aL[row * D + col] = aL[c];
    }
    if (lane4 == 0) {
      if (P.dbg_nS) P.dbg_nS[row] = l;
      if (P.dbg_nL) P.dbg_nL[row] = nL;
      if (P.dbg_c) P.dbg_c[row] = m * kLn2;
    }
  }
}

// ---------------------------------------------------------------------------
// Per-slice state P_i = sum phi_k(k) v^T, z_i = sum phi_k(k).
// Block: 256 threads = 64 features x 4 lanes; grid (nslots, BH, Dp/64).
// ---------------------------------------------------------------------------
constexpr int kTok = 16;
constexpr int kFeat = 64;

template <int D>
__global__ void __launch_bounds__(256) partials_simt_kernel(PartialParams P) {
  __shared__ float Kt[kTok][D + 1];
  __shared__ float Vt[kTok][D];
  __shared__ float Ft[kTok][kFeat + 1];
  const int tid = threadIdx.x;
  const int fl = tid >> 2;
  const int lane4 = tid & 3;
  const int slot = blockIdx.x;
  const int bh = blockIdx.y;
  const int f0 = blockIdx.z * kFeat;
  const int h = bh % P.heads;
  const int Dp = P.Dp;

  const void *kp, *vp;
  long long base;  // first row of the slice
  if (P.seen == nullptr) {
    kp = P.k; vp = P.v;
    base = bh * P.rows_per_bh + static_cast<long long>(slot) * P.HW;
  } else {
    const long long seen = *P.seen;
    const long long r = seen < P.To ? seen : P.To;
    const long long after = seen + P.nq_slices;
    const long long r2 = after < P.To ? after : P.To;
    const long long leave = r + P.nq_slices - r2;
    if (slot >= leave) return;
    const long long g = seen - r + slot;
    if (g < seen) {
      kp = P.rk; vp = P.rv;
      base = bh * P.ring_rows_per_bh + (g % P.To) * P.HW;
    } else {
      kp = P.k; vp = P.v;
      base = bh * P.rows_per_bh + (g - seen) * P.HW;
    }
  }

  float acc[D / 4];
#pragma unroll
  for (int c = 0; c < D / 4; ++c) acc[c] = 0.f;
  float zacc = 0.f;

  for (int j0 = 0; j0 < P.HW; j0 += kTok) {
    __syncthreads();
    for (int i = tid; i < kTok * D; i += 256) {
      const int j = i / D, d = i % D;
      const bool ok = j0 + j < P.HW;
      const long long gi = (base + j0 + j) * D + d;
      Kt[j][d] = ok ? load_in(kp, gi, P.in_bf16) : 0.f;
      Vt[j][d] = ok ? load_in(vp, gi, P.in_bf16) : 0.f;
    }
    __syncthreads();
    // phi_k for kTok tokens x kFeat features (4 values per thread).
    for (int i = tid; i < kTok * kFeat; i += 256) {
      const int j = i / kFeat, fq = i % kFeat;
      const int f = f0 + fq;
      float ph = 0.f;
      if (f < Dp && j0 + j < P.HW) {
        if (P.phi_k) {  // phi_k(k) given (full forward: rows as in k)
          ph = ld_phi(P.phi_k, P.phi_bf16, (base + j0 + j) * Dp + f);
        } else {
          float psi = __ldg(P.bk + b_index(h, Dp, f));
          for (int d = 0; d < D; ++d)
            psi = fmaf(Kt[j][d], load_w(P.Wk, w_index(h, D, Dp, d, f), P.w_bf16), psi);
          ph = psi * psi;
        }
      }
      Ft[j][fq] = ph;
    }
    __syncthreads();
#pragma unroll 4
    for (int j = 0; j < kTok; ++j) {
      const float ph = Ft[j][fl];
      zacc += ph;
#pragma unroll
      for (int c = 0; c < D / 4; ++c) acc[c] = fmaf(ph, Vt[j][lane4 + 4 * c], acc[c]);
    }
  }
  const int f = f0 + fl;
  if (f < Dp) {
    // Per-slice states are stored in the S^L image layout.
    float* Pout = P.P + (static_cast<long long>(bh) * P.nslots + slot) * Dp * D +
                  sl_feature_base(f, D, Dp);
#pragma unroll
    for (int c = 0; c < D / 4; ++c) Pout[sl_column_offset(f, lane4 + 4 * c)] = acc[c];
    if (lane4 == 0) P.z[(static_cast<long long>(bh) * P.nslots + slot) * Dp + f] = zacc;
  }
}

// ---------------------------------------------------------------------------
// Chunk scan: one thread per state element, sequential over slices.
// ---------------------------------------------------------------------------
__global__ void scan_kernel(const float* __restrict__ P, const float* __restrict__ z,
                            float* __restrict__ SL, float* __restrict__ zL, int T, int Tc,
                            int To, int nchunks, int Dp, int D, int causal) {
  // Launched as a programmatic dependent of the per-slice state kernel: wait
  // for that grid (and its writes) before reading P, z.
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const long long PD = static_cast<long long>(Dp) * D;
  const long long e = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int bh = blockIdx.y;
  const float* src;
  float* dst;
  long long stride;
  if (e < PD) {
    // Per-slice states and S^L share the image layout: element e of each.
    src = P + bh * T * PD + e;
    dst = SL + bh * nchunks * PD + e;
    stride = PD;
  } else if (e < PD + Dp) {
    src = z + static_cast<long long>(bh) * T * Dp + (e - PD);
    dst = zL + static_cast<long long>(bh) * nchunks * Dp + (e - PD);
    stride = Dp;
  } else {
    return;
  }
  // Slices are read in batches of 8 independent loads (the walk over slices
  // is otherwise one dependent load at a time), then folded in order; chunk
  // t receives the prefix when it reaches its window start w_t and, in the
  // bidirectional form, the suffix from its end end_t on.
  constexpr int kBatch = 8;
  float v[kBatch];
  float pre = 0.f;
  int tp = 0;
  while (tp < nchunks && max(tp * Tc - To, 0) == 0) dst[static_cast<long long>(tp++) * stride] = 0.f;
  for (int s0 = 0; s0 < T && tp < nchunks; s0 += kBatch) {
#pragma unroll
    for (int i = 0; i < kBatch; ++i)
      v[i] = s0 + i < T ? src[static_cast<long long>(s0 + i) * stride] : 0.f;
#pragma unroll
    for (int i = 0; i < kBatch; ++i) {
      pre += v[i];  // = sum over slices < s0 + i + 1
      while (tp < nchunks && max(tp * Tc - To, 0) == s0 + i + 1)
        dst[static_cast<long long>(tp++) * stride] = pre;
    }
  }
  if (!causal) {
    float suf = 0.f;
    int ts = nchunks - 1;
    while (ts >= 0 && min(T, (ts + 1) * Tc) >= T) --ts;  // nothing after the last chunk
    for (int s1 = T; s1 > 0 && ts >= 0; s1 -= kBatch) {
#pragma unroll
      for (int i = 0; i < kBatch; ++i)
        v[i] = s1 - 1 - i >= 0 ? src[static_cast<long long>(s1 - 1 - i) * stride] : 0.f;
#pragma unroll
      for (int i = 0; i < kBatch; ++i) {
        suf += v[i];  // = sum over slices >= s1 - 1 - i
        while (ts >= 0 && min(T, (ts + 1) * Tc) == s1 - 1 - i)
          dst[static_cast<long long>(ts--) * stride] += suf;
      }
    }
  }
}

// Chunk scan for T <= kScanRegs slices: each thread reads its four elements
// of every per-slice state once into registers, then writes each chunk's
// linear-set sum as a plain sum, in slice order, over the slices of that
// chunk's linear set (slices < w_t, and in the bidirectional form also
// slices >= end_t): no total-minus-window subtraction, and P is read once
// instead of once per direction.  Four elements per thread share the
// per-slice set tests.
constexpr int kScanRegs = 32;
__global__ void scan_regs_kernel(const float4* __restrict__ P, const float4* __restrict__ z,
                                 float4* __restrict__ SL, float4* __restrict__ zL, int T, int Tc,
                                 int To, int nchunks, int Dp, int D, int causal) {
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const long long PD4 = static_cast<long long>(Dp) * D / 4;
  const long long e = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int bh = blockIdx.y;
  const float4* src;
  float4* dst;
  long long stride;
  if (e < PD4) {
    src = P + bh * T * PD4 + e;
    dst = SL + bh * nchunks * PD4 + e;
    stride = PD4;
  } else if (e < PD4 + Dp / 4) {
    src = z + static_cast<long long>(bh) * T * (Dp / 4) + (e - PD4);
    dst = zL + static_cast<long long>(bh) * nchunks * (Dp / 4) + (e - PD4);
    stride = Dp / 4;
  } else {
    return;
  }
  float4 v[kScanRegs];
#pragma unroll
  for (int i = 0; i < kScanRegs; ++i)
    v[i] = i < T ? src[static_cast<long long>(i) * stride] : make_float4(0.f, 0.f, 0.f, 0.f);
  for (int t = 0; t < nchunks; ++t) {
    const int first = t * Tc, end = min(T, first + Tc), w = max(first - To, 0);
    const int lim = causal ? T : end;  // slices >= lim join the linear set
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int i = 0; i < kScanRegs; ++i)
      if (i < w || (i >= lim && i < T)) {
        acc.x += v[i].x;
        acc.y += v[i].y;
        acc.z += v[i].z;
        acc.w += v[i].w;
      }
    dst[static_cast<long long>(t) * stride] = acc;
  }
}

// Chunk scan for at most kScanAcc chunks (any T): each thread keeps one
// accumulator per chunk for its four elements and streams the per-slice
// states in slice order, kScanBatch slices' loads in flight at a time, adding
// each slice to the accumulators of the chunks whose linear set holds it.
// The sums are the same as scan_regs_kernel's (each chunk's slices in slice
// order, no subtraction), and P is read once, but a thread holds the
// accumulators and one batch instead of every slice, so six blocks fit on an
// SM and the whole grid of the bench layer is resident in one wave.
constexpr int kScanAcc = 8, kScanBatch = 4;
__global__ void __launch_bounds__(128, 6)
    scan_stream_kernel(const float4* __restrict__ P, const float4* __restrict__ z,
                       float4* __restrict__ SL, float4* __restrict__ zL, int T, int Tc, int To,
                       int nchunks, int Dp, int D, int causal) {
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const long long PD4 = static_cast<long long>(Dp) * D / 4;
  const long long e = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int bh = blockIdx.y;
  const float4* src;
  float4* dst;
  long long stride;
  if (e < PD4) {
    src = P + bh * T * PD4 + e;
    dst = SL + bh * nchunks * PD4 + e;
    stride = PD4;
  } else if (e < PD4 + Dp / 4) {
    src = z + static_cast<long long>(bh) * T * (Dp / 4) + (e - PD4);
    dst = zL + static_cast<long long>(bh) * nchunks * (Dp / 4) + (e - PD4);
    stride = Dp / 4;
  } else {
    return;
  }
  float4 acc[kScanAcc];
#pragma unroll
  for (int t = 0; t < kScanAcc; ++t) acc[t] = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int s0 = 0; s0 < T; s0 += kScanBatch) {
    float4 v[kScanBatch];
#pragma unroll
    for (int u = 0; u < kScanBatch; ++u)
      v[u] = s0 + u < T ? src[static_cast<long long>(s0 + u) * stride]
                        : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int u = 0; u < kScanBatch; ++u) {
      const int sl = s0 + u;
#pragma unroll
      for (int t = 0; t < kScanAcc; ++t) {
        const int first = t * Tc, end = min(T, first + Tc), w = max(first - To, 0);
        const int lim = causal ? T : end;  // slices >= lim join the linear set
        if (t < nchunks && sl < T && (sl < w || sl >= lim)) {
          acc[t].x += v[u].x;
          acc[t].y += v[u].y;
          acc[t].z += v[u].z;
          acc[t].w += v[u].w;
        }
      }
    }
  }
#pragma unroll
  for (int t = 0; t < kScanAcc; ++t)
    if (t < nchunks) dst[static_cast<long long>(t) * stride] = acc[t];
}

// ---------------------------------------------------------------------------
// Streaming helpers.
// ---------------------------------------------------------------------------
__device__ __forceinline__ long long leaving_slices(long long seen, int To, int n) {
  const long long r = seen < To ? seen : To;
  const long long after = seen + n;
  const long long r2 = after < To ? after : To;
  return r + n - r2;
}

// End of a streaming step, one launch (grid (nadd + nring, BH)):
//  * blocks [0, nadd): (s, z) += the states of the slices that left the
//    window this step (per-slot states from the fold, same image layout);
//  * blocks [nadd, nadd + nring): the chunk slices that stay in the window
//    are copied into their ring slots (slice g in slot g mod T_o), 16-byte
//    vectors, kRingBlocksPerSlice blocks per chunk slice;
//  * the slice counter advances by nq, written by the last block to finish
//    (a completion count in the state header), after every block has read
//    the old value.
constexpr int kRingBlocksPerSlice = 16;

__global__ void step_finish_kernel(const float* __restrict__ P, const float* __restrict__ zp,
                                   float* __restrict__ s_state, float* __restrict__ z_state,
                                   long long* seen, unsigned* done, int Dp, int D, int To,
                                   int nq, int nslots, int nadd, const uint4* __restrict__ k,
                                   const uint4* __restrict__ v, uint4* __restrict__ rk,
                                   uint4* __restrict__ rv, long long slice_vecs) {
  const long long sn = *seen;
  const int bh = blockIdx.y;
  if (static_cast<int>(blockIdx.x) < nadd) {
    const long long PD = static_cast<long long>(Dp) * D;
    const long long e = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
    const long long leave = leaving_slices(sn, To, nq);
    if (e < PD) {
      const long long se = bh * PD + e;
      float acc = s_state[se];
      for (long long i = 0; i < leave; ++i) acc += P[(bh * nslots + i) * PD + e];
      s_state[se] = acc;
    } else if (e < PD + Dp) {
      const long long f = e - PD;
      float acc = z_state[static_cast<long long>(bh) * Dp + f];
      for (long long i = 0; i < leave; ++i) acc += zp[(bh * nslots + i) * Dp + f];
      z_state[static_cast<long long>(bh) * Dp + f] = acc;
    }
  } else {
    const int rb = blockIdx.x - nadd;
    const long long after = sn + nq;
    const long long keep = after < To ? after : To;
    const int slice = rb / kRingBlocksPerSlice;  // chunk slice of this block
    const int part = rb % kRingBlocksPerSlice;
    const long long g = sn + slice;              // its global slice index
    if (g >= after - keep) {                     // it stays in the window
      const uint4* ks = k + (static_cast<long long>(bh) * nq + slice) * slice_vecs;
      const uint4* vs = v + (static_cast<long long>(bh) * nq + slice) * slice_vecs;
      uint4* kd = rk + (static_cast<long long>(bh) * To + (g % To)) * slice_vecs;
      uint4* vd = rv + (static_cast<long long>(bh) * To + (g % To)) * slice_vecs;
      for (long long i = static_cast<long long>(part) * blockDim.x + threadIdx.x; i < slice_vecs;
           i += static_cast<long long>(blockDim.x) * kRingBlocksPerSlice) {
        kd[i] = ks[i];
        vd[i] = vs[i];
      }
    }
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();
    const unsigned nblocks = gridDim.x * gridDim.y;
    if (atomicAdd(done, 1u) == nblocks - 1) {
      *seen = sn + nq;
      *done = 0;
      __threadfence();
    }
  }
}

// E4M3 copies of q and k for the fp8 softmax variant: eight bf16 values in,
// eight E4M3 bytes out per thread and array (round to nearest even,
// saturating at +-448).
__device__ __forceinline__ uint2 bf16x8_to_e4m3(uint4 v) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  uint32_t out[2] = {0, 0};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float lo = __uint_as_float(w[i] << 16), hi = __uint_as_float(w[i] & 0xFFFF0000u);
    const __nv_fp8x2_storage_t p = __nv_cvt_float2_to_fp8x2(make_float2(lo, hi), __NV_SATFINITE,
                                                            __NV_E4M3);
    out[i >> 1] |= static_cast<uint32_t>(p) << (16 * (i & 1));
  }
  return make_uint2(out[0], out[1]);
}

__global__ void e4m3_kernel(const uint4* __restrict__ a, const uint4* __restrict__ b,
                            uint2* __restrict__ a8, uint2* __restrict__ b8, long long n8) {
  for (long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; i < n8;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    a8[i] = bf16x8_to_e4m3(__ldg(a + i));
    b8[i] = bf16x8_to_e4m3(__ldg(b + i));
  }
}

// bf16 copy of phi weights in the tensor-core image layout; blockIdx.y
// selects the matrix (0: W_q, 1: W_k).
__global__ void w_image_kernel(const float* __restrict__ Wq, __nv_bfloat16* __restrict__ out_q,
                               const float* __restrict__ Wk, __nv_bfloat16* __restrict__ out_k,
                               int heads, int D, int Dp) {
  // The per-slice state kernel that follows may start now; it waits for
  // this grid before its first read of the W_k image.
  asm volatile("griddepcontrol.launch_dependents;");
  const float* Wsrc = blockIdx.y == 0 ? Wq : Wk;
  __nv_bfloat16* out = blockIdx.y == 0 ? out_q : out_k;
  const long long per_head = static_cast<long long>(Dp) * D;
  const long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= per_head * heads) return;
  const int h = static_cast<int>(i / per_head);
  const int rem = static_cast<int>(i % per_head);
  const int d = rem / Dp, f = rem % Dp;
  out[h * per_head + wimg_index(f, d, D, Dp)] = __float2bfloat16_rn(Wsrc[w_index(h, D, Dp, d, f)]);
}

template <int D>
cudaError_t launch_attn_simt_d(const AttnParams& p, cudaStream_t s) {
  const int fl_loop = kBQ * D + kBK * (D + 1) + kBK * D + kBQ * (kBK + 1);
  const int fl_tail = kBQ * D + kBQ * p.Dp;
  const size_t bytes = sizeof(float) * static_cast<size_t>(fl_loop > fl_tail ? fl_loop : fl_tail);
  cudaError_t e = cudaFuncSetAttribute(attn_simt_kernel<D>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(bytes));
  if (e != cudaSuccess) return e;
  int qrows_max;  // rows of the largest chunk
  if (p.seen) qrows_max = p.nq_slices * p.HW;
  else qrows_max = (p.Tc < p.T ? p.Tc : p.T) * p.HW;
  dim3 grid((qrows_max + kBQ - 1) / kBQ, p.nchunks, p.BH);
  attn_simt_kernel<D><<<grid, 128, bytes, s>>>(p);
  return cudaGetLastError();
}

template <int D>
cudaError_t launch_partials_simt_d(const PartialParams& p, cudaStream_t s) {
  dim3 grid(p.nslots, p.BH, (p.Dp + kFeat - 1) / kFeat);
  partials_simt_kernel<D><<<grid, 256, 0, s>>>(p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attn_simt(const AttnParams& p, cudaStream_t s) {
  switch (p.D) {
    case 32: return launch_attn_simt_d<32>(p, s);
    case 64: return launch_attn_simt_d<64>(p, s);
    case 128: return launch_attn_simt_d<128>(p, s);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_partials_simt(const PartialParams& p, cudaStream_t s) {
  switch (p.D) {
    case 32: return launch_partials_simt_d<32>(p, s);
    case 64: return launch_partials_simt_d<64>(p, s);
    case 128: return launch_partials_simt_d<128>(p, s);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_scan(const float* P, const float* z, float* SL, float* zL, int BH, int T,
                        int Tc, int To, int nchunks, int Dp, int D, int causal,
                        cudaStream_t s) {
  const long long n = static_cast<long long>(Dp) * D + Dp;
  // Programmatic dependent launch: the grid is scheduled while the state
  // kernel before it still runs, and waits for it on the device.
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>((n + 255) / 256), BH);
  cfg.blockDim = dim3(256);
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if ((nchunks <= kScanAcc || T <= kScanRegs) && Dp % 4 == 0) {
    const long long n4 = static_cast<long long>(Dp) * D / 4 + Dp / 4;
    cfg.gridDim = dim3(static_cast<unsigned>((n4 + 127) / 128), BH);
    cfg.blockDim = dim3(128);
    return cudaLaunchKernelEx(&cfg, nchunks <= kScanAcc ? scan_stream_kernel : scan_regs_kernel,
                              reinterpret_cast<const float4*>(P),
                              reinterpret_cast<const float4*>(z), reinterpret_cast<float4*>(SL),
                              reinterpret_cast<float4*>(zL), T, Tc, To, nchunks, Dp, D, causal);
  }
  return cudaLaunchKernelEx(&cfg, scan_kernel, P, z, SL, zL, T, Tc, To, nchunks, Dp, D, causal);
}

cudaError_t launch_step_finish(const float* P, const float* zp, float* s_state, float* z_state,
                               long long* seen, unsigned* done, int BH, int Dp, int D, int To,
                               int nq_slices, int nslots, const void* k, const void* v, void* rk,
                               void* rv, int HW, int elem_bytes, cudaStream_t s) {
  const long long n = static_cast<long long>(Dp) * D + Dp;
  const int nadd = static_cast<int>((n + 255) / 256);
  const int nring = To > 0 ? nq_slices * kRingBlocksPerSlice : 0;
  const long long slice_vecs = static_cast<long long>(HW) * D * elem_bytes / 16;
  dim3 grid(nadd + nring, BH);
  step_finish_kernel<<<grid, 256, 0, s>>>(
      P, zp, s_state, z_state, seen, done, Dp, D, To, nq_slices, nslots, nadd,
      static_cast<const uint4*>(k), static_cast<const uint4*>(v), static_cast<uint4*>(rk),
      static_cast<uint4*>(rv), slice_vecs);
  return cudaGetLastError();
}

cudaError_t launch_e4m3(const void* a, const void* b, void* a8, void* b8, long long n,
                        cudaStream_t s) {
  const long long n8 = n / 8;
  const int blocks = static_cast<int>(n8 / 256 + 1 < 4096 ? n8 / 256 + 1 : 4096);
  e4m3_kernel<<<blocks, 256, 0, s>>>(static_cast<const uint4*>(a), static_cast<const uint4*>(b),
                                     static_cast<uint2*>(a8), static_cast<uint2*>(b8), n8);
  return cudaGetLastError();
}

cudaError_t launch_w_images(const float* Wq, void* out_q, const float* Wk, void* out_k,
                            int heads, int D, int Dp, cudaStream_t s) {
  const long long n = static_cast<long long>(heads) * D * Dp;
  dim3 grid(static_cast<unsigned>((n + 255) / 256), Wk != nullptr ? 2 : 1);
  w_image_kernel<<<grid, 256, 0, s>>>(Wq, static_cast<__nv_bfloat16*>(out_q), Wk,
                                      static_cast<__nv_bfloat16*>(out_k), heads, D, Dp);
  return cudaGetLastError();
}

cudaError_t read_den_rows_simt(unsigned long long* rows, int reset) {
  cudaError_t e = cudaMemcpyFromSymbol(rows, rehyat_simt_den_rows, sizeof(*rows));
  if (e != cudaSuccess || !reset) return e;
  const unsigned long long zero = 0;
  return cudaMemcpyToSymbol(rehyat_simt_den_rows, &zero, sizeof(zero));
}

}  // namespace rehyat
