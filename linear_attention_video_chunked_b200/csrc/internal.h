// Internal declarations shared by the translation units of librehyat.so.
// Not part of the C ABI (see include/rehyat.h for that).
#pragma once
#include <cuda_runtime.h>
#include <stdint.h>

#include "rehyat.h"

namespace rehyat {

// Softmax window + linear readout + joint normalisation for the query rows of
// one or more chunks ("Key designs 1, 2 and 4" of the ReHyAt note).
//
// Two modes:
//  * full  (seen == nullptr): chunk t = blockIdx.y covers query rows
//    [t*Tc*HW, min(T,(t+1)*Tc)*HW) of q; keys are rows [w_t*HW, end_t*HW) of
//    k, v with w_t = max(t*Tc - To, 0).
//  * step  (seen != nullptr): one chunk of nq_slices slices; keys are ring
//    rows [0, min(To, *seen)*HW) followed by all rows of k, v.
// The linear state of chunk t is SL + (bh*nchunks + t)*Dp*D (image layout,
// layout.cuh sl_index), zL + (bh*nchunks + t)*Dp.  full_softmax skips the
// linear branch.
struct AttnParams {
  const void *q, *k, *v;
  long long rows_per_bh;     // rows of q/k/v (and y) per (b, h)
  const void *rk, *rv;       // ring keys/values [BH][To*HW][D] (step mode)
  long long ring_rows_per_bh;
  const long long* seen;     // device slice counter (step mode) or nullptr
  const float *SL, *zL;      // linear-set state per chunk
  const float *Wq, *bq;      // phi_q parameters, fp32 [h][2][D][Dp/2], [h][2][Dp/2]
  const void* wq_img;        // bf16 phi_q weight image per head (tensor-core path) or nullptr
  const void* phi_q;         // phi_q(q) given as [BH][rows][Dp] (then Wq, bq unused) or nullptr
  int phi_bf16;              // the given phi_q is bf16 (else fp32)
  const void *q8, *k8;       // E4M3 copies of q, k for the softmax logits (fp8 variant) or nullptr
  void* y;
  float *dbg_aS, *dbg_nS, *dbg_c, *dbg_aL, *dbg_nL;
  int BH, heads, T, HW, D, Dp, Tc, To, nchunks, nq_slices;
  int in_bf16, out_bf16, w_bf16, full_softmax;
  int one_tile;              // tensor-core path: force the one-query-tile kernel
  float scale_log2;          // logit scale * log2(e)
  // Step mode, two-tile tensor-core kernel: with ksplit > 1 the pairs of
  // query tiles past the first kwhole (in (b*h, pair) order; the pairs that
  // hold only tile A always run whole) run as ksplit CTAs over consecutive
  // pieces of the key window, which leave their partial a^S, maximum and row
  // sum in part (attn_split_part_bytes) and count themselves in
  // part_cnt[split pair] (zero between launches); the last piece to arrive
  // merges all pieces in order and writes y.
  int ksplit, kwhole;
  float* part;
  unsigned* part_cnt;
};

// Key-window split of a streaming step's attention (tc_kernels.cu) for a
// chunk of nq_slices slices on a device with `sms` SMs: pieces per split
// pair (1 = no split) and the number of two-tile pairs run whole.
struct StepSplit {
  int ksplit, whole;
};
StepSplit attn_step_split(int BH, int HW, int nq_slices, int To, int sms);
size_t attn_split_part_bytes(int BH, int HW, int nq_slices, StepSplit sp);

// Per-slice linear state: P_i = sum_{rows of slice i} phi_k(k) v^T ([Dp][D])
// and z_i = sum phi_k(k) ([Dp]).
//  * full mode (seen == nullptr): slice i = rows [i*HW, (i+1)*HW) of k, v,
//    for i in [0, nslots).
//  * step mode: slot i holds the i-th slice leaving the softmax window; its
//    global index is g = seen - r + i with r = min(To, seen); it lives in the
//    ring (slot g % To) if g < seen, else in the chunk (slice g - seen).
//    Slots past the number of leaving slices are skipped.
struct PartialParams {
  const void *k, *v;
  long long rows_per_bh;
  const void *rk, *rv;
  long long ring_rows_per_bh;
  const long long* seen;
  const float *Wk, *bk;
  const void* phi_k;         // phi_k(k) given as [BH][rows][Dp] (then Wk, bk unused) or nullptr
  int phi_bf16;              // the given phi_k is bf16 (else fp32)
  float *P, *z;              // [BH][nslots][Dp][D], [BH][nslots][Dp]
  int BH, heads, HW, D, Dp, To, nslots, nq_slices;
  int in_bf16, w_bf16;
};

// Gradient of the feature-map parameters (phi_bwd.cu).  q, k, v in the
// forward's input dtype; y, dy, den fp32; SL, zL the linear-set state per
// chunk as the forward's state pass leaves it; partials: a scratch array of
// phi_bwd_partial_floats(...) floats.  Outputs overwrite dWq, dbq, dWk, dbk.
struct PhiBwdArgs {
  const void *q, *k, *v;
  const float *y, *dy, *den;
  const float *Wq, *bq, *Wk, *bk;
  const float *SL, *zL;
  const void *wq_img, *wk_img;  // bf16 weight images (tensor-core passes) or nullptr
  float *partials;
  float *dWq, *dbq, *dWk, *dbk;
  // Tensor-core passes only: the linear branch's token gradients are
  // written to dq, dk, dv when non-null (the full backward, which then adds
  // the softmax branch's).
  float *dq, *dk, *dv;
  // Tensor-core passes only: r = g . y / den per row and gh = bf16(g / den)
  // [BH][N][D], as bwd_prep_kernel writes them.
  const float* r;
  const void* gh;
  int batch, heads, T, HW, D, Dp, Tc, To, causal, nchunks, in_bf16;
  int tc;                       // run the q and k passes on tcgen05
};
// One tensor-core pass of the feature-map backward (tc_phi_bwd.cuh; bf16
// inputs, D = D' = 128), writing the CUDA-core passes' partial layout.
struct PhiBwdTcArgs {
  const void *x, *v;          // q or k (the pass's rows), and v (k pass), bf16 [BH][N][128]
  const void* gh;             // q pass: bf16 g / den [BH][N][128] (bwd_prep_kernel)
  const float* r;             // q pass: g . y / den per row [BH][N] (bwd_prep_kernel)
  const void* w_img;          // bf16 image of W_q or W_k, [heads][Dp * D]
  const float* b;             // b_q or b_k [heads][Dp]
  const float* M;             // q: S_L per chunk (image layout); k: Ghat^T blocks per slice
  const float* vec;           // q: z_L per chunk (k: hhat, inside the Ghat block)
  float* part;                // partial blocks of the pass (the q pass's G blocks as [d][f])
  // Optional token gradients of the linear branch, written (fp32
  // [BH][N][128]; null = not computed): q pass dx = dq = du_q W_q; k pass
  // dx = dk = du_k W_k and dv = phi_k(k) Ghat_s.
  float *dx, *dv;
  int BH, heads, T, HW, Tc, nchunks, splits, q_side;
};
bool tc_phi_bwd_eligible(int in_bf16, int D, int Dp);
cudaError_t launch_phi_bwd_tc(const PhiBwdTcArgs& a, cudaStream_t s);

void phi_bwd_split(int T, int Tc, int HW, int* QS, int* KS);
size_t phi_bwd_partial_floats(int BH, int T, int nchunks, int D, int Dp, int QS, int KS);
cudaError_t launch_phi_bwd(const PhiBwdArgs& a, cudaStream_t s);

// Offset (in floats) of the Ghat blocks inside the partials array of
// launch_phi_bwd: per (b*h, feature piece of 128, slice) a [128][D] block
// Ghat_s (feature-major) followed by hhat_s [128].
size_t phi_bwd_ghat_offset_floats(int BH, int nchunks, int D, int Dp, int QS);

// Full backward of the hybrid attention (attn_bwd.cu): dq, dk, dv given the
// forward's inputs, y, dy = dL/dy, the stabiliser c and the joint
// denominator den per query, the linear-set state per chunk (SL image
// layout, zL) and the Ghat blocks of the feature-map backward.  r, Dc, jstar
// are per-query scratch [BH][N] the dq kernel writes and the dk/dv kernel
// reads.
struct AttnBwdParams {
  const void *q, *k, *v;
  const float *y, *dy, *c, *den;
  const float *Wq, *bq, *Wk, *bk;
  const float *SL, *zL, *ghat;
  float *r, *Dc;
  int* jstar;
  float *dq, *dk, *dv;
  int BH, heads, T, HW, D, Dp, Tc, To, causal, nchunks, in_bf16, FP;
  float scale;
};
cudaError_t launch_attn_bwd_simt(const AttnBwdParams& p, cudaStream_t s);
// Tensor-core path (bf16, D = 128): prep (r, gh = bf16(dy / den) into
// gh_bf16, [BH][N][128]) and the dq and dk/dv kernels of tc_attn_bwd.cuh
// (the softmax branch); the linear branch's parts are added afterwards.
bool tc_attn_bwd_eligible(int in_bf16, int D);
struct AttnBwdTcArgs {
  const void *q, *k, *v, *gh;  // bf16 [BH][N][128]
  const float *c, *r;          // per query [BH][N]: stabiliser, (g . y) / den
  float* Dc;                   // per query: written by the dq kernel, read by dk/dv
  int* jstar;                  // per query: arg-max key (absolute row), likewise
  float *dq, *dk, *dv;         // fp32 [BH][N][128]: overwritten, or added to if accumulate
  int BH, T, HW, Tc, To, nchunks;
  int accumulate;
  float scale;
};
cudaError_t launch_attn_bwd_dq_tc(const AttnBwdTcArgs& a, cudaStream_t s);
cudaError_t launch_attn_bwd_dkv_tc(const AttnBwdTcArgs& a, cudaStream_t s);
// prep, then the dq and dk/dv kernels; with accumulate they add into dq,
// dk, dv (which then hold the linear branch's parts already).
cudaError_t launch_attn_bwd_tc_softmax(const AttnBwdParams& p, void* gh_bf16, bool accumulate,
                                       cudaStream_t s);
// The dq and dk/dv kernels alone, after launch_bwd_prep.
cudaError_t launch_attn_bwd_tc_kernels(const AttnBwdParams& p, const void* gh_bf16,
                                       bool accumulate, cudaStream_t s);
// r = dy . y / den per row and gh = bf16(dy / den) for D = 128 rows.
cudaError_t launch_bwd_prep(const float* y, const float* dy, const float* den, float* r,
                            void* gh_bf16, long long rows, cudaStream_t s);
// The linear branch's token gradients on CUDA cores, added to dq, dk, dv
// (D = 128; used when the feature-map passes do not run on tensor cores).
cudaError_t launch_attn_bwd_lin_simt(const AttnBwdParams& p, cudaStream_t s);

// General feature map (phi_mlp.cu): phi = [psi_1^1 .. psi_P^P],
// psi = GELU(x W_a + b_a) W_b + b_b per head; x [BH][N][D] (in dtype),
// phi [BH][N][Dp] fp32.
struct PhiMlpArgs {
  const void* x;
  const float *Wa, *ba, *Wb, *bb;
  void* phi;                 // fp32, or bf16 when phi_bf16
  int phi_bf16;
  long long N;
  int BH, heads, D, Dh, Dp, parts, in_bf16;
};
cudaError_t launch_phi_mlp(const PhiMlpArgs& a, cudaStream_t s);
// Tensor-core version (bf16 x, D = 128, D_h a multiple of 128, D' in
// {64, 128}, x and phi 16-byte aligned, shared memory permitting); images
// holds phi_mlp_image_bytes of bf16 weight images it writes first.
bool tc_phi_mlp_eligible(const PhiMlpArgs& a);
size_t phi_mlp_image_bytes(int heads, int Dh, int Dp);
cudaError_t launch_phi_mlp_tc(const PhiMlpArgs& a, void* images, cudaStream_t s);

// ---- SIMT (fp32 CUDA-core) kernels: every supported shape, both dtypes.
cudaError_t launch_attn_simt(const AttnParams& p, cudaStream_t s);
cudaError_t launch_partials_simt(const PartialParams& p, cudaStream_t s);

// bf16 images of the phi weights (layout.cuh, wimg_index) for the
// tensor-core kernels: out [heads][Dp*D] each.  Wk/out_k may be null.
// E4M3 copies of two bf16 arrays of n elements each (round to nearest even,
// saturating at +-448), n a multiple of 8; pointers 16-byte aligned.
cudaError_t launch_e4m3(const void* a, const void* b, void* a8, void* b8, long long n,
                        cudaStream_t s);

cudaError_t launch_w_images(const float* Wq, void* out_q, const float* Wk, void* out_k,
                            int heads, int D, int Dp, cudaStream_t s);
bool tc_attn_eligible(int in_bf16, int D, int Dp);

// Tensor-core per-slice state (bf16, D = 128, Dp in {64, 128}); wk_img is
// the bf16 image of W_k.
bool tc_state_eligible(int in_bf16, int D, int Dp);
cudaError_t launch_state_tc(const PartialParams& p, const void* wk_img, cudaStream_t s);

// Linear-set state per chunk from the per-slice states (full mode).
// causal: S^L_t = sum_{i < w_t} P_i.  bidirectional: S^L_t = sum_{i < w_t} P_i
// + sum_{i >= end_t} P_i (prefix plus suffix, no subtraction).  P is plain
// [Dp][D]; S^L is written in the image layout (layout.cuh, sl_index).
cudaError_t launch_scan(const float* P, const float* z, float* SL, float* zL,
                        int BH, int T, int Tc, int To, int nchunks, int Dp,
                        int D, int causal, cudaStream_t s);

// Streaming helpers (step mode; all read the device slice counter).
// End of a streaming step: fold the leaving slices' states into (s, z), copy
// the staying chunk slices into the ring, advance the slice counter (done:
// a zeroed completion count in the state header, reset by the kernel).
cudaError_t launch_step_finish(const float* P, const float* zp, float* s_state, float* z_state,
                               long long* seen, unsigned* done, int BH, int Dp, int D, int To,
                               int nq_slices, int nslots, const void* k, const void* v, void* rk,
                               void* rv, int HW, int elem_bytes, cudaStream_t s);

// ---- tcgen05 / TMA kernels (bf16, D = 128).  Return cudaErrorNotSupported
// when the shape is outside what they handle.
bool tc_attn_supported(const AttnParams& p);
cudaError_t launch_attn_tc(const AttnParams& p, cudaStream_t s);

}  // namespace rehyat
