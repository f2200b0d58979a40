// C ABI of librehyat.so: argument checks, workspace/state layout, dispatch.
// The method and every entry point are documented in include/rehyat.h.
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include "internal.h"

namespace rehyat {
namespace {

constexpr size_t kAlign = 256;

size_t align_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int elem_bytes(int dtype) { return dtype == REHYAT_BF16 ? 2 : 4; }

rehyat_status check_params(const rehyat_params* p) {
  if (!p) return REHYAT_ERR_INVALID_ARG;
  if (p->batch < 1 || p->heads < 1 || p->T < 1 || p->Hs < 1 || p->Ws < 1 || p->Tc < 1 ||
      p->To < 0)
    return REHYAT_ERR_INVALID_ARG;
  if (p->causal != 0 && p->causal != 1) return REHYAT_ERR_INVALID_ARG;
  if ((p->in_dtype != REHYAT_F32 && p->in_dtype != REHYAT_BF16) ||
      (p->out_dtype != REHYAT_F32 && p->out_dtype != REHYAT_BF16))
    return REHYAT_ERR_INVALID_ARG;
  if (!(p->scale >= 0.f) || isinf(p->scale)) return REHYAT_ERR_INVALID_ARG;
  if (p->D != 32 && p->D != 64 && p->D != 128) return REHYAT_ERR_UNSUPPORTED;
  if (p->Dp != 32 && p->Dp != 64 && p->Dp != 128 && p->Dp != 256) return REHYAT_ERR_UNSUPPORTED;
  // Index arithmetic: rows per (b, h) and grid sizes must fit in 32 bits.
  const long long HW = static_cast<long long>(p->Hs) * p->Ws;
  const long long N = HW * p->T;
  if (N * p->D >= (1LL << 31) || static_cast<long long>(p->batch) * p->heads >= 65535)
    return REHYAT_ERR_UNSUPPORTED;
  // The fp8 softmax variant runs on the two-query-tile tensor-core kernel only.
  if ((p->flags & REHYAT_FLAG_FP8_QK) &&
      (p->in_dtype != REHYAT_BF16 || p->D != 128 || p->Dp > 128 ||
       (p->flags & (REHYAT_FLAG_FORCE_SIMT | REHYAT_FLAG_ONE_TILE))))
    return REHYAT_ERR_UNSUPPORTED;
  return REHYAT_OK;
}

// Entry points without an fp8 softmax variant.
rehyat_status no_fp8(const rehyat_params* p) {
  return (p && (p->flags & REHYAT_FLAG_FP8_QK)) ? REHYAT_ERR_UNSUPPORTED : REHYAT_OK;
}

int nchunks_of(const rehyat_params* p) { return (p->T + p->Tc - 1) / p->Tc; }

struct FwdWorkspace {
  size_t P_off, z_off, SL_off, zL_off, wimg_off, wkimg_off, q8_off, k8_off, total;
};

// phi_q or phi_k weight image (bf16, all heads) for the tensor-core kernels.
size_t wimg_bytes(const rehyat_params* p) {
  return static_cast<size_t>(p->heads) * p->Dp * p->D * 2;
}

FwdWorkspace fwd_layout(const rehyat_params* p) {
  const size_t BH = static_cast<size_t>(p->batch) * p->heads;
  const size_t PD = static_cast<size_t>(p->Dp) * p->D;
  FwdWorkspace w;
  w.P_off = 0;
  w.z_off = align_up(w.P_off + BH * p->T * PD * sizeof(float));
  w.SL_off = align_up(w.z_off + BH * p->T * p->Dp * sizeof(float));
  w.zL_off = align_up(w.SL_off + BH * nchunks_of(p) * PD * sizeof(float));
  w.wimg_off = align_up(w.zL_off + BH * nchunks_of(p) * p->Dp * sizeof(float));
  w.wkimg_off = align_up(w.wimg_off + wimg_bytes(p));
  w.q8_off = w.k8_off = w.total = align_up(w.wkimg_off + wimg_bytes(p));
  if (p->flags & REHYAT_FLAG_FP8_QK) {  // E4M3 copies of q and k
    const size_t n8 = BH * p->T * static_cast<size_t>(p->Hs) * p->Ws * p->D;
    w.k8_off = align_up(w.q8_off + n8);
    w.total = align_up(w.k8_off + n8);
  }
  return w;
}

// Whether the tensor-core attention kernel (and its weight image) is used.
bool tc_path(const rehyat_params* p) {
  return !(p->flags & REHYAT_FLAG_FORCE_SIMT) &&
         tc_attn_eligible(p->in_dtype == REHYAT_BF16, p->D, p->Dp);
}

// Whether the tensor-core per-slice state kernel is used.
bool tc_state_path(const rehyat_params* p) {
  return !(p->flags & REHYAT_FLAG_FORCE_SIMT) &&
         tc_state_eligible(p->in_dtype == REHYAT_BF16, p->D, p->Dp);
}

// Whether the feature-map backward's q and k passes run on tensor cores.
bool phi_bwd_on_tc(const rehyat_params* p) {
  return tc_path(p) && tc_phi_bwd_eligible(p->in_dtype == REHYAT_BF16, p->D, p->Dp);
}

// Feature-map backward workspace: the forward's layout, then the q and k
// passes' partials ...
size_t phi_bwd_base_bytes(const rehyat_params* p) {
  if (check_params(p) != REHYAT_OK || no_fp8(p) != REHYAT_OK) return 0;
  int QS, KS;
  phi_bwd_split(p->T, p->Tc, p->Hs * p->Ws, &QS, &KS);
  const size_t parts = phi_bwd_partial_floats(p->batch * p->heads, p->T, nchunks_of(p), p->D,
                                              p->Dp, QS, KS);
  return fwd_layout(p).total + align_up(parts * sizeof(float));
}

// ... and, for the tensor-core passes' shapes (bf16, D = D' = 128), r and
// bf16 g / den per row for the q pass.
size_t phi_bwd_prep_bytes(const rehyat_params* p) {
  if ((p->flags & REHYAT_FLAG_FORCE_SIMT) || p->in_dtype != REHYAT_BF16 || p->D != 128 ||
      p->Dp != 128)
    return 0;
  const size_t rows = static_cast<size_t>(p->batch) * p->heads * p->T * p->Hs * p->Ws;
  return align_up(rows * sizeof(float)) + align_up(rows * p->D * 2);
}

// Per-slice states on the path these params select.
cudaError_t run_partials(const rehyat_params* p, const PartialParams& pp, const void* wk_img,
                         cudaStream_t s) {
  if (tc_state_path(p)) return launch_state_tc(pp, wk_img, s);
  return launch_partials_simt(pp, s);
}

struct StateLayout {
  size_t s_off, z_off, cnt_off, rk_off, rv_off, total;
};

int device_sm_count() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) {
    cudaGetLastError();
    return 148;
  }
  return n;
}

// Pieces of the key window per pair of query tiles in a streaming step of
// nslices slices (the two-tile tensor-core kernel only; 1 = no split).
StepSplit step_split(const rehyat_params* p, int nslices) {
  if (!tc_path(p) || (p->flags & REHYAT_FLAG_ONE_TILE)) return StepSplit{1, 0};
  return attn_step_split(p->batch * p->heads, p->Hs * p->Ws, nslices, p->To, device_sm_count());
}

size_t step_pairs(const rehyat_params* p) {
  const size_t qrows = static_cast<size_t>(p->Tc) * p->Hs * p->Ws;
  return (qrows + 255) / 256;
}

// Streaming state header (kAlign bytes, zeroed by rehyat_state_init): the
// int64 count of slices consumed at offset 0, and at kStepDoneOffset the
// uint32 completion count the step-finish kernel uses (0 between steps).
constexpr size_t kStepDoneOffset = 64;

StateLayout state_layout(const rehyat_params* p) {
  const size_t BH = static_cast<size_t>(p->batch) * p->heads;
  const size_t HW = static_cast<size_t>(p->Hs) * p->Ws;
  StateLayout s;
  s.s_off = kAlign;  // header: slice counter, step completion count
  s.z_off = align_up(s.s_off + BH * p->Dp * p->D * sizeof(float));
  // Arrival counters of the split attention, one per (b, h, pair of query
  // tiles); zeroed with the state and left zero by every step.
  s.cnt_off = align_up(s.z_off + BH * p->Dp * sizeof(float));
  s.rk_off = align_up(s.cnt_off + BH * step_pairs(p) * sizeof(unsigned));
  const size_t ring = BH * p->To * HW * p->D * elem_bytes(p->in_dtype);
  s.rv_off = align_up(s.rk_off + ring);
  s.total = align_up(s.rv_off + ring);
  return s;
}

struct StepWorkspace {
  size_t P_off, z_off, wimg_off, wkimg_off, part_off, total;
  int nslots;
};

StepWorkspace step_layout(const rehyat_params* p) {
  const size_t BH = static_cast<size_t>(p->batch) * p->heads;
  StepWorkspace w;
  w.nslots = p->To + p->Tc;  // at most this many slices leave per step
  w.P_off = 0;
  w.z_off = align_up(BH * w.nslots * static_cast<size_t>(p->Dp) * p->D * sizeof(float));
  w.wimg_off = align_up(w.z_off + BH * w.nslots * p->Dp * sizeof(float));
  w.wkimg_off = align_up(w.wimg_off + wimg_bytes(p));
  w.part_off = align_up(w.wkimg_off + wimg_bytes(p));
  size_t part = 0;  // split attention partials, for any chunk length <= T_c
  for (int n = 1; n <= p->Tc; ++n) {
    const size_t b = attn_split_part_bytes(static_cast<int>(BH), p->Hs * p->Ws, n,
                                           step_split(p, n));
    part = b > part ? b : part;
  }
  w.total = align_up(w.part_off + part);
  return w;
}

float logit_scale(const rehyat_params* p) {
  return p->scale > 0.f ? p->scale : 1.0f / sqrtf(static_cast<float>(p->D));
}

AttnParams base_attn(const rehyat_params* p, const void* q, const void* k, const void* v,
                     const rehyat_phi* phi, void* y, const rehyat_debug* dbg) {
  AttnParams a = {};
  a.q = q; a.k = k; a.v = v;
  a.Wq = phi ? phi->Wq : nullptr;
  a.bq = phi ? phi->bq : nullptr;
  a.y = y;
  if (dbg) {
    a.dbg_aS = dbg->aS; a.dbg_nS = dbg->nS; a.dbg_c = dbg->c;
    a.dbg_aL = dbg->aL; a.dbg_nL = dbg->nL;
  }
  a.BH = p->batch * p->heads;
  a.heads = p->heads;
  a.T = p->T;
  a.HW = p->Hs * p->Ws;
  a.D = p->D;
  a.Dp = p->Dp;
  a.Tc = p->Tc;
  a.To = p->To;
  a.in_bf16 = p->in_dtype == REHYAT_BF16;
  a.out_bf16 = p->out_dtype == REHYAT_BF16;
  a.w_bf16 = a.in_bf16;
  a.one_tile = (p->flags & REHYAT_FLAG_ONE_TILE) != 0;
  a.scale_log2 = logit_scale(p) * 1.4426950408889634f;
  return a;
}

rehyat_status check_phi(const rehyat_phi* phi) {
  if (!phi || !phi->Wq || !phi->bq || !phi->Wk || !phi->bk) return REHYAT_ERR_INVALID_ARG;
  if (!aligned16(phi->Wq) || !aligned16(phi->Wk) || (reinterpret_cast<uintptr_t>(phi->bq) & 3) ||
      (reinterpret_cast<uintptr_t>(phi->bk) & 3))
    return REHYAT_ERR_MISALIGNED;
  return REHYAT_OK;
}

rehyat_status check_dbg(const rehyat_debug* dbg) {
  if (!dbg) return REHYAT_OK;
  const void* ptrs[5] = {dbg->aS, dbg->nS, dbg->c, dbg->aL, dbg->nL};
  for (const void* q : ptrs)
    if (q && (reinterpret_cast<uintptr_t>(q) & 3)) return REHYAT_ERR_MISALIGNED;
  return REHYAT_OK;
}

rehyat_status to_status(cudaError_t e) { return e == cudaSuccess ? REHYAT_OK : REHYAT_ERR_CUDA; }

bool use_tc(const rehyat_params* p, const AttnParams& a) {
  if (p->flags & REHYAT_FLAG_FORCE_SIMT) return false;
  return tc_attn_supported(a);
}

cudaError_t run_attn(const rehyat_params* p, const AttnParams& a, cudaStream_t s) {
  if (a.q8 != nullptr)  // the fp8 variant exists on the tensor-core kernel only
    return use_tc(p, a) ? launch_attn_tc(a, s) : cudaErrorNotSupported;
  if (use_tc(p, a)) return launch_attn_tc(a, s);
  return launch_attn_simt(a, s);
}

// Per-slice states and the linear-set state per chunk into the workspace
// laid out by fwd_layout (weight images, per-slice state kernel, chunk scan);
// arguments already checked.
// With phi_k given ([BH][N][Dp], fp32 or with REHYAT_FLAG_PHI_BF16 bf16),
// phi is unused (may be null).
rehyat_status state_pass(const rehyat_params* p, const void* k, const void* v,
                         const rehyat_phi* phi, char* ws, cudaStream_t s,
                         const void* phi_k = nullptr) {
  const FwdWorkspace w = fwd_layout(p);
  float* P = reinterpret_cast<float*>(ws + w.P_off);
  float* z = reinterpret_cast<float*>(ws + w.z_off);
  float* SL = reinterpret_cast<float*>(ws + w.SL_off);
  float* zL = reinterpret_cast<float*>(ws + w.zL_off);
  const int BH = p->batch * p->heads;
  const int HW = p->Hs * p->Ws;

  PartialParams pp = {};
  pp.k = k; pp.v = v;
  pp.rows_per_bh = static_cast<long long>(p->T) * HW;
  pp.Wk = phi_k ? nullptr : phi->Wk;
  pp.bk = phi_k ? nullptr : phi->bk;
  pp.phi_k = phi_k;
  pp.phi_bf16 = (p->flags & REHYAT_FLAG_PHI_BF16) ? 1 : 0;
  pp.P = P; pp.z = z;
  pp.BH = BH; pp.heads = p->heads; pp.HW = HW; pp.D = p->D; pp.Dp = p->Dp; pp.To = p->To;
  pp.nslots = p->T;
  pp.in_bf16 = p->in_dtype == REHYAT_BF16;
  pp.w_bf16 = pp.in_bf16;
  cudaError_t e = cudaSuccess;
  if (!phi_k && (tc_path(p) || tc_state_path(p)))
    e = launch_w_images(phi->Wq, ws + w.wimg_off, phi->Wk, ws + w.wkimg_off, p->heads, p->D,
                        p->Dp, s);
  if (e != cudaSuccess) return to_status(e);
  e = run_partials(p, pp, ws + w.wkimg_off, s);
  if (e != cudaSuccess) return to_status(e);
  return to_status(launch_scan(P, z, SL, zL, BH, p->T, p->Tc, p->To, nchunks_of(p), p->Dp,
                               p->D, p->causal, s));
}

// Checks and marshals the feature-map call; REHYAT_OK and *a filled, or the error.
rehyat_status mlp_args(const rehyat_params* p, const void* x, const rehyat_phi_mlp* mlp,
                       void* phi, PhiMlpArgs* a) {
  rehyat_status st = check_params(p);
  if (st != REHYAT_OK) return st;
  if ((st = no_fp8(p)) != REHYAT_OK) return st;
  if (!x || !mlp || !phi || !mlp->Wa || !mlp->ba || !mlp->Wb || !mlp->bb)
    return REHYAT_ERR_INVALID_ARG;
  if (mlp->parts < 1 || p->Dp % mlp->parts != 0 || mlp->Dh < 1) return REHYAT_ERR_INVALID_ARG;
  if (mlp->Dh > 512) return REHYAT_ERR_UNSUPPORTED;
  const void* ptrs[6] = {x, phi, mlp->Wa, mlp->ba, mlp->Wb, mlp->bb};
  for (const void* q : ptrs)
    if (reinterpret_cast<uintptr_t>(q) & 3) return REHYAT_ERR_MISALIGNED;
  a->x = x; a->Wa = mlp->Wa; a->ba = mlp->ba; a->Wb = mlp->Wb; a->bb = mlp->bb; a->phi = phi;
  a->N = static_cast<long long>(p->T) * p->Hs * p->Ws;
  a->BH = p->batch * p->heads; a->heads = p->heads; a->D = p->D; a->Dh = mlp->Dh;
  a->Dp = p->Dp; a->parts = mlp->parts; a->in_bf16 = p->in_dtype == REHYAT_BF16;
  a->phi_bf16 = (p->flags & REHYAT_FLAG_PHI_BF16) ? 1 : 0;
  return REHYAT_OK;
}

bool mlp_tc(const rehyat_params* p, const PhiMlpArgs& a) {
  return !(p->flags & REHYAT_FLAG_FORCE_SIMT) && tc_phi_mlp_eligible(a);
}
}  // namespace
}  // namespace rehyat

using namespace rehyat;

extern "C" {

int rehyat_version(void) { return 100; }

int rehyat_attn_path(const rehyat_params* p) {
  if (check_params(p) != REHYAT_OK) return -1;
  return tc_path(p) ? 1 : 0;
}

const char* rehyat_status_string(rehyat_status s) {
  switch (s) {
    case REHYAT_OK: return "ok";
    case REHYAT_ERR_INVALID_ARG: return "invalid argument";
    case REHYAT_ERR_UNSUPPORTED: return "unsupported shape";
    case REHYAT_ERR_MISALIGNED: return "pointer not 16-byte aligned";
    case REHYAT_ERR_WORKSPACE: return "workspace or state too small";
    case REHYAT_ERR_CUDA: return "CUDA launch error";
    case REHYAT_ERR_SCRATCH_LIMIT: return "problem needs more than the built-in 32 MiB scratch";
  }
  return "unknown status";
}

size_t rehyat_workspace_bytes(const rehyat_params* p) {
  if (check_params(p) != REHYAT_OK) return 0;
  return fwd_layout(p).total;
}

rehyat_status rehyat_fwd_state(const rehyat_params* p, const void* k, const void* v,
                               const rehyat_phi* phi, void* workspace, size_t ws_bytes,
                               void* stream) {
  rehyat_status st = check_params(p);
  if (st != REHYAT_OK) return st;
  if (!k || !v || !workspace) return REHYAT_ERR_INVALID_ARG;
  if ((st = check_phi(phi)) != REHYAT_OK) return st;
  if (!aligned16(k) || !aligned16(v) || !aligned16(workspace)) return REHYAT_ERR_MISALIGNED;
  if (ws_bytes < fwd_layout(p).total) return REHYAT_ERR_WORKSPACE;
  return state_pass(p, k, v, phi, static_cast<char*>(workspace),
                    static_cast<cudaStream_t>(stream));
}

rehyat_status rehyat_fwd_attn(const rehyat_params* p, const void* q, const void* k,
                              const void* v, const rehyat_phi* phi, void* y,
                              void* workspace, size_t ws_bytes, const rehyat_debug* dbg,
                              void* stream) {
  rehyat_status st = check_params(p);
  if (st != REHYAT_OK) return st;
  if (!q || !k || !v || !y || !workspace) return REHYAT_ERR_INVALID_ARG;
  if ((st = check_phi(phi)) != REHYAT_OK) return st;
  if ((st = check_dbg(dbg)) != REHYAT_OK) return st;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(y) || !aligned16(workspace))
    return REHYAT_ERR_MISALIGNED;
  const FwdWorkspace w = fwd_layout(p);
  if (ws_bytes < w.total) return REHYAT_ERR_WORKSPACE;
  char* ws = static_cast<char*>(workspace);
  AttnParams a = base_attn(p, q, k, v, phi, y, dbg);
  a.rows_per_bh = static_cast<long long>(p->T) * p->Hs * p->Ws;
  a.SL = reinterpret_cast<const float*>(ws + w.SL_off);
  a.zL = reinterpret_cast<const float*>(ws + w.zL_off);
  a.nchunks = nchunks_of(p);
  if (tc_path(p)) a.wq_img = ws + w.wimg_off;
  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (p->flags & REHYAT_FLAG_FP8_QK) {
    const cudaError_t e = launch_e4m3(q, k, ws + w.q8_off, ws + w.k8_off,
                                      static_cast<long long>(a.BH) * a.rows_per_bh * p->D, s);
    if (e != cudaSuccess) return to_status(e);
    a.q8 = ws + w.q8_off;
    a.k8 = ws + w.k8_off;
  }
  return to_status(run_attn(p, a, s));
}

rehyat_status rehyat_hybrid_attn_fwd(const rehyat_params* p, const void* q, const void* k,
                                     const void* v, const rehyat_phi* phi, void* y,
                                     void* workspace, size_t ws_bytes,
                                     const rehyat_debug* dbg, void* stream) {
  // Check everything both stages need before enqueueing either.
  rehyat_status st = check_params(p);
  if (st != REHYAT_OK) return st;
  if (!q || !k || !v || !y || !workspace) return REHYAT_ERR_INVALID_ARG;
  if ((st = check_phi(phi)) != REHYAT_OK) return st;
  if ((st = check_dbg(dbg)) != REHYAT_OK) return st;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(y) || !aligned16(workspace))
    return REHYAT_ERR_MISALIGNED;
  if (ws_bytes < fwd_layout(p).total) return REHYAT_ERR_WORKSPACE;
  st = rehyat_fwd_state(p, k, v, phi, workspace, ws_bytes, stream);
  if (st != REHYAT_OK) return st;
  return rehyat_fwd_attn(p, q, k, v, phi, y, workspace, ws_bytes, dbg, stream);
}

rehyat_status rehyat_softmax_attn_fwd(const rehyat_params* p, const void* q, const void* k,
                                      const void* v, void* y, void* stream) {
  rehyat_status st = check_params(p);
  if (st != REHYAT_OK) return st;
  if ((st = no_fp8(p)) != REHYAT_OK) return st;
  if (!q || !k || !v || !y) return REHYAT_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(y))
    return REHYAT_ERR_MISALIGNED;
  // One chunk spanning all T slices, no overlap, no linear branch.
  rehyat_params full = *p;
  full.Tc = p->T;
  full.To = 0;
  AttnParams a = base_attn(&full, q, k, v, nullptr, y, nullptr);
  a.rows_per_bh = static_cast<long long>(p->T) * p->Hs * p->Ws;
  a.nchunks = 1;
  a.full_softmax = 1;
  return to_status(run_attn(&full, a, static_cast<cudaStream_t>(stream)));
}

size_t rehyat_state_bytes(const rehyat_params* p) {
  if (check_params(p) != REHYAT_OK || no_fp8(p) != REHYAT_OK) return 0;
  return state_layout(p).total;
}

size_t rehyat_step_workspace_bytes(const rehyat_params* p) {
  if (check_params(p) != REHYAT_OK || no_fp8(p) != REHYAT_OK) return 0;
  return step_layout(p).total;
}

int rehyat_step_key_split(const rehyat_params* p, int nslices) {
  if (check_params(p) != REHYAT_OK || no_fp8(p) != REHYAT_OK || nslices < 1 || nslices > p->Tc)
    return 0;
  return step_split(p, nslices).ksplit;
}

rehyat_status rehyat_state_init(const rehyat_params* p, void* state, void* stream) {
  rehyat_status st = check_params(p);
  if (st != REHYAT_OK) return st;
  if ((st = no_fp8(p)) != REHYAT_OK) return st;
  if (!state) return REHYAT_ERR_INVALID_ARG;
  if (!aligned16(state)) return REHYAT_ERR_MISALIGNED;
  const StateLayout L = state_layout(p);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  // Header (counter = 0) and s, z = 0.  The ring needs no clearing: only
  // slots written since the last reset are ever read.
  return to_status(cudaMemsetAsync(state, 0, L.rk_off, s));
}

rehyat_status rehyat_chunk_step(const rehyat_params* p, const void* q, const void* k,
                                const void* v, int nslices, const rehyat_phi* phi, void* state,
                                void* y, void* workspace, size_t ws_bytes,
                                const rehyat_debug* dbg, void* stream) {
  rehyat_status st = check_params(p);
  if (st != REHYAT_OK) return st;
  if ((st = no_fp8(p)) != REHYAT_OK) return st;
  if (p->causal != 1) return REHYAT_ERR_INVALID_ARG;
  if (nslices < 1 || nslices > p->Tc) return REHYAT_ERR_INVALID_ARG;
  if (!q || !k || !v || !y || !state || !workspace) return REHYAT_ERR_INVALID_ARG;
  if ((st = check_phi(phi)) != REHYAT_OK) return st;
  if ((st = check_dbg(dbg)) != REHYAT_OK) return st;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(y) || !aligned16(state) ||
      !aligned16(workspace))
    return REHYAT_ERR_MISALIGNED;
  const StepWorkspace w = step_layout(p);
  if (ws_bytes < w.total) return REHYAT_ERR_WORKSPACE;
  const StateLayout L = state_layout(p);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  char* stb = static_cast<char*>(state);
  long long* seen = reinterpret_cast<long long*>(stb);
  float* s_state = reinterpret_cast<float*>(stb + L.s_off);
  float* z_state = reinterpret_cast<float*>(stb + L.z_off);
  void* rk = stb + L.rk_off;
  void* rv = stb + L.rv_off;
  char* ws = static_cast<char*>(workspace);
  float* P = reinterpret_cast<float*>(ws + w.P_off);
  float* zp = reinterpret_cast<float*>(ws + w.z_off);
  const int BH = p->batch * p->heads;
  const int HW = p->Hs * p->Ws;
  const long long nrows = static_cast<long long>(nslices) * HW;

  // 1. Softmax over ring + chunk, linear branch from (s, z), joint norm.
  AttnParams a = base_attn(p, q, k, v, phi, y, dbg);
  a.rows_per_bh = nrows;
  a.rk = rk; a.rv = rv;
  a.ring_rows_per_bh = static_cast<long long>(p->To) * HW;
  a.seen = seen;
  a.SL = s_state; a.zL = z_state;
  a.nchunks = 1;
  a.nq_slices = nslices;
  const StepSplit sp = step_split(p, nslices);
  a.ksplit = sp.ksplit;
  a.kwhole = sp.whole;
  if (a.ksplit > 1) {
    // The partials of this call's split must fit the workspace's region.
    const size_t need = attn_split_part_bytes(BH, HW, nslices, sp);
    if (need == 0 || w.part_off + need > ws_bytes) return REHYAT_ERR_WORKSPACE;
    a.part = reinterpret_cast<float*>(ws + w.part_off);
    a.part_cnt = reinterpret_cast<unsigned*>(stb + L.cnt_off);
  }
  cudaError_t e = cudaSuccess;
  if (tc_path(p) || tc_state_path(p)) {
    e = launch_w_images(phi->Wq, ws + w.wimg_off, phi->Wk, ws + w.wkimg_off, p->heads, p->D,
                        p->Dp, s);
    if (e != cudaSuccess) return to_status(e);
  }
  if (tc_path(p)) a.wq_img = ws + w.wimg_off;
  e = run_attn(p, a, s);
  if (e != cudaSuccess) return to_status(e);

  // 2. Fold the slices that leave the softmax window into (s, z).
  PartialParams pp = {};
  pp.k = k; pp.v = v;
  pp.rows_per_bh = nrows;
  pp.rk = rk; pp.rv = rv;
  pp.ring_rows_per_bh = a.ring_rows_per_bh;
  pp.seen = seen;
  pp.Wk = phi->Wk; pp.bk = phi->bk;
  pp.P = P; pp.z = zp;
  pp.BH = BH; pp.heads = p->heads; pp.HW = HW; pp.D = p->D; pp.Dp = p->Dp; pp.To = p->To;
  pp.nslots = w.nslots;
  pp.nq_slices = nslices;
  pp.in_bf16 = p->in_dtype == REHYAT_BF16;
  pp.w_bf16 = pp.in_bf16;
  e = run_partials(p, pp, ws + w.wkimg_off, s);
  if (e != cudaSuccess) return to_status(e);
  // 3. Add them into (s, z), keep the newest T_o slices in the ring and
  // advance the counter, in one launch.
  unsigned* done = reinterpret_cast<unsigned*>(stb + kStepDoneOffset);
  return to_status(launch_step_finish(P, zp, s_state, z_state, seen, done, BH, p->Dp, p->D,
                                      p->To, nslices, w.nslots, k, v, rk, rv, HW,
                                      elem_bytes(p->in_dtype), s));
}

rehyat_status rehyat_hybrid_attn_fwd_phi(const rehyat_params* p, const void* q, const void* k,
                                         const void* v, const void* phi_q, const void* phi_k,
                                         void* y, void* workspace, size_t ws_bytes,
                                         const rehyat_debug* dbg, void* stream) {
  rehyat_status st = check_params(p);
  if (st != REHYAT_OK) return st;
  if ((st = no_fp8(p)) != REHYAT_OK) return st;
  if (!q || !k || !v || !phi_q || !phi_k || !y || !workspace) return REHYAT_ERR_INVALID_ARG;
  if ((st = check_dbg(dbg)) != REHYAT_OK) return st;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(y) || !aligned16(phi_q) ||
      !aligned16(phi_k) || !aligned16(workspace))
    return REHYAT_ERR_MISALIGNED;
  const FwdWorkspace w = fwd_layout(p);
  if (ws_bytes < w.total) return REHYAT_ERR_WORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  char* ws = static_cast<char*>(workspace);
  if ((st = state_pass(p, k, v, nullptr, ws, s, phi_k)) != REHYAT_OK) return st;
  AttnParams a = base_attn(p, q, k, v, nullptr, y, dbg);
  a.phi_q = phi_q;
  a.phi_bf16 = (p->flags & REHYAT_FLAG_PHI_BF16) ? 1 : 0;
  a.rows_per_bh = static_cast<long long>(p->T) * p->Hs * p->Ws;
  a.SL = reinterpret_cast<const float*>(ws + w.SL_off);
  a.zL = reinterpret_cast<const float*>(ws + w.zL_off);
  a.nchunks = nchunks_of(p);
  return to_status(run_attn(p, a, s));
}

size_t rehyat_feature_map_mlp_workspace_bytes(const rehyat_params* p, const rehyat_phi_mlp* mlp,
                                              const void* x, const void* phi) {
  PhiMlpArgs a;
  if (mlp_args(p, x, mlp, const_cast<void*>(phi), &a) != REHYAT_OK || !mlp_tc(p, a)) return 0;
  return align_up(phi_mlp_image_bytes(a.heads, a.Dh, a.Dp));
}

rehyat_status rehyat_feature_map_mlp(const rehyat_params* p, const void* x,
                                     const rehyat_phi_mlp* mlp, void* phi, void* workspace,
                                     size_t ws_bytes, void* stream) {
  PhiMlpArgs a;
  const rehyat_status st = mlp_args(p, x, mlp, phi, &a);
  if (st != REHYAT_OK) return st;
  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (!mlp_tc(p, a)) return to_status(launch_phi_mlp(a, s));
  if (!workspace || ws_bytes < phi_mlp_image_bytes(a.heads, a.Dh, a.Dp))
    return REHYAT_ERR_WORKSPACE;
  if (!aligned16(workspace)) return REHYAT_ERR_MISALIGNED;
  return to_status(launch_phi_mlp_tc(a, workspace, s));
}

size_t rehyat_phi_bwd_workspace_bytes(const rehyat_params* p) {
  const size_t b = rehyat::phi_bwd_base_bytes(p);
  return b == 0 ? 0 : b + rehyat::phi_bwd_prep_bytes(p);
}

}  // extern "C"

namespace rehyat {
namespace {

// The feature-map backward; with dq, dk, dv non-null and the tensor-core
// passes in use, it also writes the linear branch's token gradients to them.
// The tensor-core q pass reads r and bf16 g / den per row: r_pre, gh_pre
// when the caller has them (the full backward), else computed into the
// workspace after the base region.
rehyat_status phi_bwd_impl(const rehyat_params* p, const void* q, const void* k, const void* v,
                           const float* y, const float* dy, const float* den,
                           const rehyat_phi* phi, const rehyat_phi_grad* grad, void* workspace,
                           size_t ws_bytes, void* stream, float* dq, float* dk, float* dv,
                           bool* added, const float* r_pre = nullptr,
                           const void* gh_pre = nullptr) {
  rehyat_status st = check_params(p);
  if (st != REHYAT_OK) return st;
  if ((st = no_fp8(p)) != REHYAT_OK) return st;
  if (!q || !k || !v || !y || !dy || !den || !grad || !workspace) return REHYAT_ERR_INVALID_ARG;
  if (!grad->dWq || !grad->dbq || !grad->dWk || !grad->dbk) return REHYAT_ERR_INVALID_ARG;
  if ((st = check_phi(phi)) != REHYAT_OK) return st;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(y) || !aligned16(dy) ||
      !aligned16(workspace) || (reinterpret_cast<uintptr_t>(den) & 3) ||
      (reinterpret_cast<uintptr_t>(grad->dWq) & 3) || (reinterpret_cast<uintptr_t>(grad->dbq) & 3) ||
      (reinterpret_cast<uintptr_t>(grad->dWk) & 3) || (reinterpret_cast<uintptr_t>(grad->dbk) & 3))
    return REHYAT_ERR_MISALIGNED;
  const size_t base = phi_bwd_base_bytes(p);
  const bool have_prep = r_pre != nullptr && gh_pre != nullptr;
  if (ws_bytes < base + (have_prep ? 0 : phi_bwd_prep_bytes(p))) return REHYAT_ERR_WORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  char* ws = static_cast<char*>(workspace);
  // The linear-set state of every chunk, as the forward computes it (or, with
  // REHYAT_FLAG_FWD_STATE, as the forward left it in this workspace).
  if (!(p->flags & REHYAT_FLAG_FWD_STATE) && (st = state_pass(p, k, v, phi, ws, s)) != REHYAT_OK)
    return st;
  const FwdWorkspace w = fwd_layout(p);
  PhiBwdArgs a;
  a.q = q; a.k = k; a.v = v; a.y = y; a.dy = dy; a.den = den;
  a.Wq = phi->Wq; a.bq = phi->bq; a.Wk = phi->Wk; a.bk = phi->bk;
  a.SL = reinterpret_cast<const float*>(ws + w.SL_off);
  a.zL = reinterpret_cast<const float*>(ws + w.zL_off);
  a.partials = reinterpret_cast<float*>(ws + w.total);
  a.dWq = grad->dWq; a.dbq = grad->dbq; a.dWk = grad->dWk; a.dbk = grad->dbk;
  a.batch = p->batch; a.heads = p->heads; a.T = p->T; a.HW = p->Hs * p->Ws; a.D = p->D;
  a.Dp = p->Dp; a.Tc = p->Tc; a.To = p->To; a.causal = p->causal; a.nchunks = nchunks_of(p);
  a.in_bf16 = p->in_dtype == REHYAT_BF16;
  // Tensor-core q and k passes where the weight images exist (bf16, D = D' = 128).
  a.tc = phi_bwd_on_tc(p);
  a.wq_img = a.tc ? ws + w.wimg_off : nullptr;
  a.wk_img = a.tc ? ws + w.wkimg_off : nullptr;
  a.dq = a.tc ? dq : nullptr;
  a.dk = a.tc ? dk : nullptr;
  a.dv = a.tc ? dv : nullptr;
  a.r = r_pre;
  a.gh = gh_pre;
  if (a.tc && !have_prep) {
    const long long rows = static_cast<long long>(p->batch) * p->heads * p->T * p->Hs * p->Ws;
    float* r = reinterpret_cast<float*>(ws + base);
    void* gh = ws + base + align_up(static_cast<size_t>(rows) * sizeof(float));
    const cudaError_t e = launch_bwd_prep(y, dy, den, r, gh, rows, s);
    if (e != cudaSuccess) return to_status(e);
    a.r = r;
    a.gh = gh;
  }
  if (added) *added = a.tc && dq != nullptr;
  return to_status(launch_phi_bwd(a, s));
}

}  // namespace
}  // namespace rehyat

extern "C" {

rehyat_status rehyat_phi_bwd(const rehyat_params* p, const void* q, const void* k, const void* v,
                             const float* y, const float* dy, const float* den,
                             const rehyat_phi* phi, const rehyat_phi_grad* grad,
                             void* workspace, size_t ws_bytes, void* stream) {
  return rehyat::phi_bwd_impl(p, q, k, v, y, dy, den, phi, grad, workspace, ws_bytes, stream,
                              nullptr, nullptr, nullptr, nullptr);
}

size_t rehyat_hybrid_attn_bwd_workspace_bytes(const rehyat_params* p) {
  const size_t phi_ws = rehyat::phi_bwd_base_bytes(p);
  if (phi_ws == 0) return 0;
  const size_t rows = static_cast<size_t>(p->batch) * p->heads * p->T * p->Hs * p->Ws;
  // Shapes the tensor-core path takes (bf16, D = 128): a bf16 copy of dy / den.
  const size_t gh = (p->in_dtype == REHYAT_BF16 && p->D == 128) ? align_up(rows * p->D * 2) : 0;
  return phi_ws + 3 * align_up(rows * sizeof(float)) + gh;
}

rehyat_status rehyat_hybrid_attn_bwd(const rehyat_params* p, const void* q, const void* k,
                                     const void* v, const rehyat_phi* phi, const float* y,
                                     const float* dy, const float* c, const float* den,
                                     float* dq, float* dk, float* dv,
                                     const rehyat_phi_grad* grad, void* workspace,
                                     size_t ws_bytes, void* stream) {
  rehyat_status st = check_params(p);
  if (st != REHYAT_OK) return st;
  if ((st = no_fp8(p)) != REHYAT_OK) return st;
  if (!q || !k || !v || !y || !dy || !c || !den || !dq || !dk || !dv || !grad || !workspace)
    return REHYAT_ERR_INVALID_ARG;
  if (!grad->dWq || !grad->dbq || !grad->dWk || !grad->dbk) return REHYAT_ERR_INVALID_ARG;
  if ((st = check_phi(phi)) != REHYAT_OK) return st;
  auto a4 = [](const void* x) { return (reinterpret_cast<uintptr_t>(x) & 3) == 0; };
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(y) || !aligned16(dy) ||
      !aligned16(workspace) || !aligned16(dq) || !aligned16(dk) || !aligned16(dv) || !a4(c) ||
      !a4(den) || !a4(grad->dWq) || !a4(grad->dbq) || !a4(grad->dWk) || !a4(grad->dbk))
    return REHYAT_ERR_MISALIGNED;
  if (ws_bytes < rehyat_hybrid_attn_bwd_workspace_bytes(p)) return REHYAT_ERR_WORKSPACE;
  char* ws = static_cast<char*>(workspace);
  const FwdWorkspace w = fwd_layout(p);
  const int BH = p->batch * p->heads, HW = p->Hs * p->Ws;
  int QS, KS;
  phi_bwd_split(p->T, p->Tc, HW, &QS, &KS);
  const float* partials = reinterpret_cast<const float*>(ws + w.total);
  const size_t rows = static_cast<size_t>(BH) * p->T * HW;
  char* scratch = ws + phi_bwd_base_bytes(p);
  AttnBwdParams a;
  a.q = q; a.k = k; a.v = v; a.y = y; a.dy = dy; a.c = c; a.den = den;
  a.Wq = phi->Wq; a.bq = phi->bq; a.Wk = phi->Wk; a.bk = phi->bk;
  a.SL = reinterpret_cast<const float*>(ws + w.SL_off);
  a.zL = reinterpret_cast<const float*>(ws + w.zL_off);
  a.ghat = partials + phi_bwd_ghat_offset_floats(BH, nchunks_of(p), p->D, p->Dp, QS);
  a.r = reinterpret_cast<float*>(scratch);
  a.Dc = reinterpret_cast<float*>(scratch + align_up(rows * sizeof(float)));
  a.jstar = reinterpret_cast<int*>(scratch + 2 * align_up(rows * sizeof(float)));
  a.dq = dq; a.dk = dk; a.dv = dv;
  a.BH = BH; a.heads = p->heads; a.T = p->T; a.HW = HW; a.D = p->D; a.Dp = p->Dp;
  a.Tc = p->Tc; a.To = p->To; a.causal = p->causal; a.nchunks = nchunks_of(p);
  a.in_bf16 = p->in_dtype == REHYAT_BF16;
  a.FP = p->Dp > 128 ? p->Dp / 128 : 1;
  a.scale = p->scale > 0.f ? p->scale : 1.0f / sqrtf(static_cast<float>(p->D));
  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  const size_t phi_ws = phi_bwd_base_bytes(p);
  if (!(p->flags & REHYAT_FLAG_FORCE_SIMT) && tc_attn_bwd_eligible(a.in_bf16, p->D)) {
    // Softmax branch on tensor cores.  Where the feature-map passes run on
    // tensor cores too they go first and write the linear branch's token
    // gradients to dq, dk, dv (one plain store per element), and the softmax
    // kernels add theirs in their epilogues; otherwise the softmax kernels
    // write and CUDA-core kernels add the linear parts after the
    // feature-map backward.  All read the same r and bf16 dy / den rows.
    void* gh = scratch + 3 * align_up(rows * sizeof(float));
    cudaError_t e = launch_bwd_prep(y, dy, den, a.r, gh, static_cast<long long>(rows), s);
    if (e != cudaSuccess) return to_status(e);
    if (phi_bwd_on_tc(p)) {
      bool added = false;
      if ((st = phi_bwd_impl(p, q, k, v, y, dy, den, phi, grad, workspace, phi_ws, stream, dq,
                             dk, dv, &added, a.r, gh)) != REHYAT_OK)
        return st;
      if (!added) return REHYAT_ERR_CUDA;
      return to_status(launch_attn_bwd_tc_kernels(a, gh, true, s));
    }
    if ((e = launch_attn_bwd_tc_kernels(a, gh, false, s)) != cudaSuccess) return to_status(e);
    if ((st = phi_bwd_impl(p, q, k, v, y, dy, den, phi, grad, workspace, phi_ws, stream, nullptr,
                           nullptr, nullptr, nullptr, a.r, gh)) != REHYAT_OK)
      return st;
    return to_status(launch_attn_bwd_lin_simt(a, s));
  }
  // CUDA cores: the feature-map backward first (S_L, z_L and the Ghat blocks
  // the token gradients use), then dq and dk/dv with the linear parts fused.
  if ((st = phi_bwd_impl(p, q, k, v, y, dy, den, phi, grad, workspace, phi_ws, stream, nullptr,
                         nullptr, nullptr, nullptr)) != REHYAT_OK)
    return st;
  return to_status(launch_attn_bwd_simt(a, s));
}

}  // extern "C"
