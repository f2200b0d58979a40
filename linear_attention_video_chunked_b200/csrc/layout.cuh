// Memory layouts shared by the kernels of librehyat.so.
//
// Tensor-core operands live in shared memory in the 128-byte-swizzled,
// K-major form that TMA writes and tcgen05.mma reads: a "box" is a run of
// 128-byte rows; within each 1024-byte atom (eight rows) the 16-byte chunk c
// of row r sits at chunk position c ^ (r & 7).  Operands that are not loaded
// by a tensor map are stored in global memory already in this form (an
// "image"), so a single bulk copy puts them in place.
#pragma once
#include <stdint.h>

namespace rehyat {

// Width of one feature piece of the linear readout (the tensor-core tail
// processes the D' features in pieces of at most 128).
__host__ __device__ __forceinline__ int piece_width(int Dp) { return Dp < 128 ? Dp : 128; }

// S^L (and the streaming s): logical [Dp][D] fp32, stored per feature piece
// as a K-major tf32 operand [D rows][piece features]: boxes of 32 features,
// each box D rows x 128 bytes.
__host__ __device__ __forceinline__ long long sl_index(int f, int d, int D, int Dp) {
  const int pw = piece_width(Dp);
  const int piece = f / pw;
  const int fl = f - piece * pw;
  const int box = fl >> 5;
  const int chunk = (fl >> 2) & 7;
  const int w = fl & 3;
  return static_cast<long long>(piece) * D * pw + static_cast<long long>(box) * D * 32 +
         d * 32 + ((chunk ^ (d & 7)) << 2) + w;
}

// sl_index split into a part that depends on the feature only and the
// offset of column d within the feature's run (for writers that walk d with
// f fixed); piece widths are multiples of 32 whenever D' has several pieces.
__host__ __device__ __forceinline__ long long sl_feature_base(int f, int D, int Dp) {
  const int pw = piece_width(Dp);
  const int piece = f / pw;
  const int fl = f - piece * pw;
  return static_cast<long long>(piece) * D * pw + static_cast<long long>(fl >> 5) * D * 32 +
         (fl & 3);
}
__host__ __device__ __forceinline__ int sl_column_offset(int f, int d) {
  return d * 32 + ((((f >> 2) & 7) ^ (d & 7)) << 2);
}

// Inverse of sl_index: the (feature, column) stored at image offset o.
__host__ __device__ __forceinline__ void sl_coords(long long o, int D, int Dp, int* f, int* d) {
  const int pw = piece_width(Dp);
  const long long piece = o / (static_cast<long long>(D) * pw);
  const int r1 = static_cast<int>(o - piece * D * pw);
  const int box = r1 / (D * 32);
  const int r2 = r1 - box * D * 32;
  const int dd = r2 >> 5;
  const int r3 = r2 & 31;
  const int chunk = (r3 >> 2) ^ (dd & 7);
  *d = dd;
  *f = static_cast<int>(piece) * pw + box * 32 + chunk * 4 + (r3 & 3);
}

// phi_q weights of one head: logical W[d][f] (f over both parts), stored per
// feature piece as a K-major bf16 operand [piece features][D]: boxes of 64
// D-elements, each box pw rows x 128 bytes.
__host__ __device__ __forceinline__ long long wimg_index(int f, int d, int D, int Dp) {
  const int pw = piece_width(Dp);
  const int piece = f / pw;
  const int n = f - piece * pw;
  const int box = d >> 6;
  const int chunk = (d >> 3) & 7;
  const int w = d & 7;
  return static_cast<long long>(piece) * pw * D + static_cast<long long>(box) * pw * 64 +
         n * 64 + ((chunk ^ (n & 7)) << 3) + w;
}

// A K-major bf16 operand [N rows][K] (K a multiple of 128) stored as pieces
// of 128 K-elements (two 64-element boxes) by rp = min(N, 128) rows, piece
// (kp, np) at ((kp * (N / rp) + np) * 2 * rp * 64); within a piece, box b
// of row r at (b * rp + r) * 64.  Used for the two weight matrices of the
// general feature map: W_a^T as [D_h][D] and W_b^T as [D'][D_h].
__host__ __device__ __forceinline__ long long kpiece_img_index(int n, int k, int N) {
  const int rp = N < 128 ? N : 128;
  const int np = n / rp, r = n - np * rp;
  const int kp = k >> 7, kk = k & 127;
  const int box = kk >> 6, chunk = (kk >> 3) & 7, w = kk & 7;
  return (static_cast<long long>(kp) * (N / rp) + np) * 2 * rp * 64 +
         static_cast<long long>(box) * rp * 64 + r * 64 + ((chunk ^ (r & 7)) << 3) + w;
}

}  // namespace rehyat
