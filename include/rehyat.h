/*
 * rehyat.h -- C ABI of librehyat.so: ReHyAt temporally chunked hybrid
 * attention (forward), for NVIDIA B200 (sm_100a).
 *
 * Method: "ReHyAt: Recurrent Hybrid Attention for Video Diffusion
 * Transformers" (papernotes.org note of the CVPR 2026 paper), Method, Key
 * designs 1-4.  Notation:
 *   B batch, heads h, T latent slices of Hs x Ws tokens (HW = Hs*Ws),
 *   N = T*HW tokens in time-major order (slice, row, column), D head width,
 *   Dp = D' the total feature width of phi, T_c slices per chunk, T_o overlap
 *   slices.  Chunk t holds slices [t*T_c, min(T,(t+1)*T_c)); its softmax keys
 *   start w_t = max(t*T_c - T_o, 0) slices in (Key design 2).
 *
 *   For a query i of chunk t, with softmax set S_t = keys of slices
 *   [w_t, end_t) and linear set L_t (bidirectional: every other token;
 *   causal: tokens of slices < w_t; Key designs 1 and 4):
 *     c_i   = max_{j in S_t} (q_i . k_j) * scale           (stabiliser)
 *     a^S_i = sum_{j in S_t} exp((q_i . k_j) * scale - c_i) v_j,
 *     n^S_i = sum_{j in S_t} exp((q_i . k_j) * scale - c_i)
 *     a^L_i = phi_q(q_i) . (sum_{j in L_t} phi_k(k_j) v_j^T),
 *     n^L_i = phi_q(q_i) . (sum_{j in L_t} phi_k(k_j))
 *     y_i   = (a^S_i + a^L_i) / (n^S_i + n^L_i)               (joint norm)
 *   phi(x) = [(x W_1 + b_1)^2, (x W_2 + b_2)^2] (Key design 3, degree-2 form).
 *
 * Conventions shared by every entry point:
 *   - Ownership: the caller allocates and owns every buffer (inputs, outputs,
 *     phi parameters, workspace, streaming state).  The library never
 *     allocates device memory, frees or synchronises; all work is enqueued on
 *     `stream` (a cudaStream_t passed as void*; NULL = the legacy default
 *     stream).  Exceptions, stated at each: rehyat_hybrid_attn_fwd_host
 *     creates two copy streams per device on first use (kept for the life of
 *     the process) and a few events per call; rehyat_device_error_flags
 *     synchronises the device.
 *   - All pointers are device pointers unless stated, 16-byte aligned.
 *   - Errors: arguments are checked before any launch; a bad argument
 *     returns a status and enqueues nothing.  A launch failure returns
 *     REHYAT_ERR_CUDA.  Faults during execution surface at the caller's next
 *     synchronisation.  The library never aborts or exits.
 *   - Determinism: no atomics in any reduction; repeated calls on the same
 *     inputs give bit-identical results.
 */
#ifndef REHYAT_H
#define REHYAT_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define REHYAT_API __attribute__((visibility("default")))
#else
#define REHYAT_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  REHYAT_OK = 0,
  REHYAT_ERR_INVALID_ARG = 1,  /* null pointer, non-positive size, bad enum */
  REHYAT_ERR_UNSUPPORTED = 2,  /* D or Dp outside the supported set */
  REHYAT_ERR_MISALIGNED = 3,   /* a pointer not 16-byte aligned */
  REHYAT_ERR_WORKSPACE = 4,    /* workspace or state smaller than required */
  REHYAT_ERR_CUDA = 5,         /* a CUDA launch or query failed */
  REHYAT_ERR_SCRATCH_LIMIT = 6 /* problem needs more workspace than the fixed
                                  scratch of rehyat_hybrid_attn_fwd_noalloc */
} rehyat_status;

typedef enum { REHYAT_F32 = 0, REHYAT_BF16 = 1 } rehyat_dtype;

/* Flags for rehyat_params.flags. */
#define REHYAT_FLAG_FORCE_SIMT 1 /* use the fp32 CUDA-core kernels even where a
                                    tensor-core kernel exists (testing aid) */
#define REHYAT_FLAG_ONE_TILE 2   /* tensor-core attention: use the one-query-tile
                                    kernel instead of the two-tile kernel (closed-
                                    form phi only; testing aid) */
#define REHYAT_FLAG_FP8_QK 4     /* fp8 softmax branch: the logits q.k^T are formed
                                    from q and k rounded to E4M3 (round to nearest
                                    even, saturating at +-448, unit scale) on the
                                    tensor cores (kind::f8f6f4); P.V, the feature
                                    maps and the linear branch keep bf16.  Full
                                    forward only (rehyat_hybrid_attn_fwd, the
                                    split stages, the no-alloc and host-buffer
                                    variants), bf16
                                    inputs, D = 128, Dp <= 128; every other entry
                                    point returns REHYAT_ERR_UNSUPPORTED with it.
                                    The workspace grows by the two E4M3 copies
                                    (2 * B * h * N * D bytes), which
                                    rehyat_fwd_attn writes. */
#define REHYAT_FLAG_PHI_BF16 8   /* feature-map arrays in bf16 instead of fp32:
                                    the output of rehyat_feature_map_mlp (phi
                                    rounded to nearest even) and the phi_q,
                                    phi_k inputs of rehyat_hybrid_attn_fwd_phi.
                                    Halves the maps' memory traffic; the
                                    tensor-core forward rounds phi_k to bf16
                                    anyway.  Ignored by other entry points. */
#define REHYAT_FLAG_FWD_STATE 16 /* backward entry points (rehyat_phi_bwd,
                                    rehyat_hybrid_attn_bwd): the workspace is
                                    the one the forward ran on
                                    (rehyat_hybrid_attn_fwd, or rehyat_fwd_state,
                                    with the same k, v, phi and params apart
                                    from this flag), unchanged since, so it
                                    already holds the per-chunk linear-set
                                    states S_L, z_L and the weight images; the
                                    backward reads them instead of recomputing
                                    them (the forward's state stage).  Size the
                                    workspace with the backward's
                                    *_workspace_bytes: the forward accepts the
                                    larger buffer and uses its front part, which
                                    the backward's layout shares.  A workspace
                                    that does not hold that state gives wrong
                                    gradients; nothing detects it.  Ignored by
                                    other entry points. */

typedef struct {
  int batch, heads;   /* B >= 1, h >= 1 */
  int T, Hs, Ws;      /* latent slices and slice height/width, all >= 1 */
  int D;              /* head width: 32, 64 or 128 */
  int Dp;             /* total phi width D': 32, 64, 128 or 256 */
  int Tc, To;         /* chunk slices (>= 1) and overlap slices (>= 0) */
  int causal;         /* 0 bidirectional, 1 causal (Key design 4) */
  int in_dtype;       /* rehyat_dtype of q, k, v (and of the streaming ring) */
  int out_dtype;      /* rehyat_dtype of y */
  float scale;        /* softmax logit scale; 0 means 1/sqrt(D) */
  int flags;          /* REHYAT_FLAG_* */
} rehyat_params;

/* phi parameters, fp32 device arrays, per head:
 *   W: [heads][2][D][Dp/2]  (part 0 = W_1, part 1 = W_2), row-major
 *   b: [heads][2][Dp/2]
 * In bf16 mode (in_dtype == REHYAT_BF16) the W matrices are rounded to bf16
 * for the tensor-core products; b is added in fp32. */
typedef struct {
  const float *Wq, *bq, *Wk, *bk;
} rehyat_phi;

/* Optional branch partials, fp32 device arrays ([B][h][N][D] for aS, aL;
 * [B][h][N] for nS, c, nL).  Any member may be NULL.  c is the stabiliser in
 * natural-log units; aS, nS are relative to it. */
typedef struct {
  float *aS, *nS, *c, *aL, *nL;
} rehyat_debug;

/* ---------------------------------------------------------------------- */
/* Full-sequence forward (bidirectional or non-recursive causal form).     */

/* Bytes of workspace rehyat_hybrid_attn_fwd needs for these params (0 if the
 * params are invalid).  Holds the per-slice states sum phi_k(k) v^T and
 * sum phi_k(k) and the per-chunk linear-set states. */
REHYAT_API size_t rehyat_workspace_bytes(const rehyat_params* p);

/* y = ReHyAt hybrid attention of (q, k, v), all [B][h][N][D] contiguous.
 *   q, k, v : in_dtype;  y : out_dtype;  phi : see rehyat_phi (struct in
 *   host memory, arrays on the device);  workspace: >= ws_bytes bytes of
 *   device memory that the call may overwrite;  dbg: NULL or partials.
 * Source: Key designs 1-4 of the ReHyAt note (equations for y, a^S, a^L,
 * the overlap set and the causal set). */
REHYAT_API rehyat_status rehyat_hybrid_attn_fwd(const rehyat_params* p, const void* q,
                                     const void* k, const void* v,
                                     const rehyat_phi* phi, void* y,
                                     void* workspace, size_t ws_bytes,
                                     const rehyat_debug* dbg, void* stream);

/* The same forward in two stages on one stream (rehyat_hybrid_attn_fwd is
 * exactly rehyat_fwd_state followed by rehyat_fwd_attn on one workspace):
 *   rehyat_fwd_state: per-slice sums phi_k(k) v^T, phi_k(k) and the
 *     per-chunk linear-set state (bidirectional: all slices outside the
 *     chunk's softmax window; causal: the slices before it), into workspace;
 *   rehyat_fwd_attn: window softmax, phi_q readout of the workspace state
 *     and joint normalisation, into y.
 * Lets a caller time or overlap the stages, or reuse one state for several
 * query sets over the same keys. */
REHYAT_API rehyat_status rehyat_fwd_state(const rehyat_params* p, const void* k,
                                          const void* v, const rehyat_phi* phi,
                                          void* workspace, size_t ws_bytes,
                                          void* stream);
REHYAT_API rehyat_status rehyat_fwd_attn(const rehyat_params* p, const void* q,
                                         const void* k, const void* v,
                                         const rehyat_phi* phi, void* y,
                                         void* workspace, size_t ws_bytes,
                                         const rehyat_debug* dbg, void* stream);

/* The full forward without a caller-supplied workspace, for callers that
 * cannot allocate device memory (code running under another runtime's
 * allocator or memory pool, plug-in hosts that forbid allocation after
 * start-up, tools that only pass along buffers they were given).  The
 * paper has no counterpart: this is a packaging variant of
 * rehyat_hybrid_attn_fwd, with identical arguments minus the workspace and
 * identical results.
 *   - Scratch: a 32 MiB __device__ array inside the library.  Every GPU that
 *     loads the library holds it until the process exits.  Problems whose
 *     rehyat_workspace_bytes exceeds 32 MiB return REHYAT_ERR_SCRATCH_LIMIT
 *     and enqueue nothing (e.g. one 21x20x30 layer with 12 heads fits, the
 *     batch-2 21x30x52 layer does not).
 *   - Allocates nothing: no cudaMalloc/cudaFree and no allocating library
 *     call.  Every call made outside stream capture looks up the array's
 *     device address (cudaGetSymbolAddress, with the device current), so
 *     the address stays right after cudaDeviceReset or when another context
 *     is made current.  A call on a capturing stream reuses the address of
 *     the last uncaptured call on that device: make one uncaptured call on
 *     each device (and again after a cudaDeviceReset) before capturing.  A
 *     captured call with no earlier uncaptured one returns
 *     REHYAT_ERR_INVALID_ARG and touches neither the capture nor the GPU.
 *   - The array is shared by every call on a device and keeps the last
 *     call's contents (each call overwrites all of it that it reads, so no
 *     clearing is needed).  Calls that overlap on the GPU (other streams,
 *     other host threads) race on it: serialise them. */
REHYAT_API rehyat_status rehyat_hybrid_attn_fwd_noalloc(const rehyat_params* p, const void* q,
                                                        const void* k, const void* v,
                                                        const rehyat_phi* phi, void* y,
                                                        const rehyat_debug* dbg,
                                                        void* stream);

/* Plain softmax attention over all N keys (no chunking, no linear branch):
 * the dense comparator the ReHyAt note measures against (Experiments,
 * efficiency).  Uses batch, heads, T, Hs, Ws, D, in/out dtype and scale of
 * p; ignores Tc, To, causal and phi. */
REHYAT_API rehyat_status rehyat_softmax_attn_fwd(const rehyat_params* p, const void* q,
                                      const void* k, const void* v, void* y,
                                      void* stream);

/* ---------------------------------------------------------------------- */
/* Streaming: the causal chunk-wise RNN (Key design 4).                     */

/* Bytes of the opaque streaming state: the running s [B][h][Dp][D] and
 * z [B][h][Dp] (fp32), a ring holding the keys and values of the last T_o
 * slices (in_dtype), and a device-side count of slices consumed (with a
 * completion count and the split attention's arrival counters, all zero
 * between steps).  Constant for any number of steps; a copy taken between
 * steps restores the stream exactly.  After a step that set a bit in
 * rehyat_device_error_flags the state must be re-initialised. */
REHYAT_API size_t rehyat_state_bytes(const rehyat_params* p);

/* Reset a state to the start of a video: s = 0, z = 0, empty ring. */
REHYAT_API rehyat_status rehyat_state_init(const rehyat_params* p, void* state,
                                void* stream);

/* Workspace bytes rehyat_chunk_step needs on the current device.  With the
 * two-tile tensor-core attention the step may split each pair of query
 * tiles' key window over several CTAs so that the chunk fills the device's
 * SMs; the split is chosen from the shape and the device's SM count, and
 * its partials (fp32 a^S, maximum and row sum per query row and piece) live
 * here. */
REHYAT_API size_t rehyat_step_workspace_bytes(const rehyat_params* p);

/* Pieces the key window of each pair of query tiles is split into by
 * rehyat_chunk_step for a chunk of `nslices` slices on the current device
 * (1: no split; 0: p or nslices invalid).  A split runs the pieces as
 * separate CTAs and merges their partial softmax sums exactly (the row
 * maximum is the maximum of the pieces' maxima), in piece order. */
REHYAT_API int rehyat_step_key_split(const rehyat_params* p, int nslices);

/* One step of the chunk-wise RNN: consumes the next `nslices` latent slices
 * (1 <= nslices <= Tc; the last chunk of a video may be shorter) given as
 * q, k, v [B][h][nslices*HW][D] (in_dtype) and writes their outputs y
 * (same shape, out_dtype).  Softmax keys are the ring (up to T_o earlier
 * slices) plus the chunk; the linear branch reads the state.  Afterwards the
 * slices that leave the softmax window are added into (s, z) and the ring
 * keeps the newest T_o slices.  p->causal must be 1. */
REHYAT_API rehyat_status rehyat_chunk_step(const rehyat_params* p, const void* q,
                                const void* k, const void* v, int nslices,
                                const rehyat_phi* phi, void* state, void* y,
                                void* workspace, size_t ws_bytes,
                                const rehyat_debug* dbg, void* stream);

/* ---------------------------------------------------------------------- */
/* General feature maps (Key design 3: phi_q, phi_k from a light per-head
 * embedding network whose output psi is cut into P equal parts, part i
 * raised to the i-th power, phi = [psi_1^1, ..., psi_P^P]).                */

/* The same forward as rehyat_hybrid_attn_fwd with the feature maps given as
 * arrays: phi_q = phi_q(q), phi_k = phi_k(k), [B][h][N][Dp] in fp32 (bf16
 * with REHYAT_FLAG_PHI_BF16), 16-byte aligned (any map, e.g.
 * rehyat_feature_map_mlp's).  phi values may be
 * negative (a degree-1 part), so n^L may be negative; y is the joint
 * normalisation as written, without clamping the denominator.  Workspace as
 * rehyat_workspace_bytes(p); other arguments and errors as for
 * rehyat_hybrid_attn_fwd. */
REHYAT_API rehyat_status rehyat_hybrid_attn_fwd_phi(const rehyat_params* p, const void* q,
                                                    const void* k, const void* v,
                                                    const void* phi_q, const void* phi_k,
                                                    void* y, void* workspace, size_t ws_bytes,
                                                    const rehyat_debug* dbg, void* stream);

/* ---------------------------------------------------------------------- */
/* Host-resident tensors.  The forward is per (batch, head) (Key designs
 * 1-4: window softmax, linear state and joint normalisation never mix
 * heads), so it can run in slabs of consecutive heads while the next slab's
 * inputs are uploaded and the previous slab's output is downloaded.      */

/* Device workspace bytes for rehyat_hybrid_attn_fwd_host with slabs of
 * heads_per_slab heads (<= 0 or >= heads: one slab per batch element): three
 * slots of q, k, v, y for one slab plus one slab's forward workspace
 * (0 if p is invalid). */
REHYAT_API size_t rehyat_host_workspace_bytes(const rehyat_params* p, int heads_per_slab);

/* rehyat_hybrid_attn_fwd with q, k, v (p->in_dtype) and y (p->out_dtype) in
 * HOST memory, same [B][h][N][D] layouts; phi and workspace on the device.
 * Host buffers should be page-locked (cudaHostAlloc / cudaHostRegister):
 * pageable memory still works but its copies do not overlap.  Slabs are
 * runs of heads_per_slab consecutive heads of one batch element, in (batch,
 * head) order, except that the first and the last slab of the call take
 * ceil(heads_per_slab / 2) heads (their upload and download overlap no
 * kernel, so shorter ones shorten the call).  Slab s goes through device
 * slot s mod 3: upload on an internal copy stream, the
 * forward on `stream`, download on a second internal copy stream, ordered
 * by events.  The copies start after the work already on `stream`, and
 * `stream` waits for the last download: synchronising `stream` makes y
 * valid on the host.  The copy streams are created on first use per device
 * and kept.  Results equal rehyat_hybrid_attn_fwd's bit for bit.  Errors as
 * for rehyat_hybrid_attn_fwd; REHYAT_ERR_WORKSPACE if ws_bytes <
 * rehyat_host_workspace_bytes; workspace 16-byte aligned.  A slab refused or
 * failed after its upload was enqueued returns that status with `stream`
 * still made to wait for every copy already enqueued, so synchronising
 * `stream` before reusing the host buffers is enough on every path. */
REHYAT_API rehyat_status rehyat_hybrid_attn_fwd_host(const rehyat_params* p, const void* q,
                                                     const void* k, const void* v,
                                                     const rehyat_phi* phi, void* y,
                                                     int heads_per_slab, void* workspace,
                                                     size_t ws_bytes, void* stream);

/* Per-head 2-layer MLP feature map, fp32 device arrays:
 *   Wa [heads][D][Dh], ba [heads][Dh], Wb [heads][Dh][Dp], bb [heads][Dp];
 *   psi = GELU(x Wa + ba) Wb + bb with GELU(u) = u * Phi(u) (exact form),
 *   phi = [psi_1^1, ..., psi_P^P] over P = parts equal parts (Dp % parts == 0). */
typedef struct {
  const float *Wa, *ba, *Wb, *bb;
  int Dh, parts;
} rehyat_phi_mlp;

/* Workspace bytes rehyat_feature_map_mlp needs for these shapes (0 when it
 * runs on CUDA cores, or if p or mlp is invalid).  The tensor-core path
 * (bf16 x, D = 128, Dh a multiple of 128 with Dh * 256 + Dp * Dh * 2 <=
 * 198,656, Dp in {64, 128}, x, phi, ba and bb 16-byte aligned, no
 * REHYAT_FLAG_FORCE_SIMT) keeps bf16 images of Wa and Wb there. */
REHYAT_API size_t rehyat_feature_map_mlp_workspace_bytes(const rehyat_params* p,
                                                         const rehyat_phi_mlp* mlp,
                                                         const void* x, const void* phi);

/* phi [B][h][N][Dp] (fp32, or bf16 with REHYAT_FLAG_PHI_BF16) of x
 * [B][h][N][D] (p->in_dtype), N = T*Hs*Ws,
 * heads and shapes from p (Tc, To, causal unused).  Dh <= 512.  Pointers
 * 4-byte aligned; workspace (caller-owned, 16-byte aligned, may be NULL when
 * the size above is 0) of at least rehyat_feature_map_mlp_workspace_bytes
 * bytes.  Tensor-core path: x, W_a, GELU(.) and W_b enter the products as
 * bf16 (fp32 accumulation, b_a, b_b and the powers in fp32; erf inside GELU
 * from Abramowitz & Stegun 7.1.28, |error| <= 3e-7); CUDA-core path: fp32
 * throughout (erff).  REHYAT_ERR_INVALID_ARG for parts < 1 or Dp % parts != 0;
 * REHYAT_ERR_WORKSPACE if ws_bytes is too small. */
REHYAT_API rehyat_status rehyat_feature_map_mlp(const rehyat_params* p, const void* x,
                                                const rehyat_phi_mlp* mlp, void* phi,
                                                void* workspace, size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------------- */
/* Backward for the feature maps (Key design 5: the first training stage,
 * block-wise attention distillation, updates only phi_q and phi_k).       */

/* Gradients of the phi parameters, fp32 device arrays laid out like
 * rehyat_phi: dWq, dWk [heads][2][D][Dp/2], dbq, dbk [heads][2][Dp/2]. */
typedef struct {
  float *dWq, *dbq, *dWk, *dbk;
} rehyat_phi_grad;

/* Workspace bytes rehyat_phi_bwd needs (0 if p is invalid). */
REHYAT_API size_t rehyat_phi_bwd_workspace_bytes(const rehyat_params* p);

/* dL/dW_q, dL/db_q, dL/dW_k, dL/db_k of a scalar loss L, given the forward's
 * inputs q, k, v (in_dtype, [B][h][N][D]), its output y (fp32), the upstream
 * gradient dy = dL/dy (fp32, same shape) and den [B][h][N] (fp32), the
 * forward's joint denominator n^S + n^L per query (the nS + nL of
 * rehyat_debug).  The full forward's form is used (p->causal selects it).
 * With g = dy:  dL/dphi_q(q_i) = (S_L g_i - z_L (g_i.y_i)) / den_i;  a key j
 * in the linear set of chunk t receives G_t v_j + h_t with
 * G_t = sum_i phi_q(q_i) g_i^T / den_i, h_t = -sum_i phi_q(q_i)(g_i.y_i)/den_i;
 * through phi = [(xW_1+b_1)^2, (xW_2+b_2)^2], du = 2u * dphi, dW = sum x^T du,
 * db = sum du, summed over the batch (parameters are per head).  The
 * gradients are overwritten, not accumulated; fp32 arithmetic; the
 * reductions run in a fixed order, so repeated calls agree bit for bit.
 * Pointers: q, k, v, y, dy, workspace 16-byte aligned; den and the gradient
 * arrays 4-byte aligned.  Errors as for rehyat_hybrid_attn_fwd.
 * The call first recomputes the forward's linear-set state into the
 * workspace; with REHYAT_FLAG_FWD_STATE it takes that state from the
 * forward's workspace instead (same results bit for bit). */
REHYAT_API rehyat_status rehyat_phi_bwd(const rehyat_params* p, const void* q, const void* k,
                                        const void* v, const float* y, const float* dy,
                                        const float* den, const rehyat_phi* phi,
                                        const rehyat_phi_grad* grad, void* workspace,
                                        size_t ws_bytes, void* stream);

/* Workspace bytes rehyat_hybrid_attn_bwd needs (0 if p is invalid). */
REHYAT_API size_t rehyat_hybrid_attn_bwd_workspace_bytes(const rehyat_params* p);

/* Full backward of the forward of rehyat_hybrid_attn_fwd (either form):
 * dL/dq, dL/dk, dL/dv and dL/dW_q, dL/db_q, dL/dW_k, dL/db_k of a scalar
 * loss L, for the second training stage of the ReHyAt note (Method, Key
 * design 5: the whole converted model is fine-tuned, so gradients pass
 * through q, k and v).
 * Inputs: the forward's q, k, v (in_dtype, [B][h][N][D]) and phi; its output
 * y (fp32); dy = dL/dy (fp32, same shape); per query [B][h][N] fp32 the
 * stabiliser c (the forward's row maximum of the scaled logits over the
 * window, rehyat_debug.c) and den = n^S + n^L (rehyat_debug.nS + nL).
 * Math (chain rule through Key designs 1-4; gh = dy/den, r = dy.y/den):
 *   dS_ij = e_ij (gh_i.v_j - r_i) - [j = j*_i] Dc_i,  e_ij = exp(s_ij - c_i),
 *   Dc_i = sum_j e_ij (gh_i.v_j - r_i)  (c_i is the window maximum and the
 *   linear branch is not scaled by exp(-c_i), so the gradient also flows
 *   through the maximum, to its key j*_i: the window key with the largest
 *   logit as recomputed in fp32, the lowest index among equal ones),
 *   dq_i = scale sum_j dS_ij k_j + du_q W_q^T,  dk_j = scale sum_i dS_ij q_i
 *   + du_k W_k^T,  dv_j = sum_i e_ij gh_i + Ghat_s^T phi_k(k_j), where
 *   du_q = 2u_q * (S_L gh - r z_L), du_k = 2u_k * (Ghat_s v_j + hhat_s), Ghat_s
 *   the sum of the linear-set state gradients over the chunks whose linear
 *   set holds slice s; the parameter gradients are those of rehyat_phi_bwd.
 * Outputs (overwritten, not accumulated): dq, dk, dv fp32 [B][h][N][D];
 * grad's four arrays as for rehyat_phi_bwd.  bf16 inputs with D = 128 run
 * the softmax branch on tensor cores (S, dP and the dq, dk, dv products in
 * bf16 with fp32 accumulation: P, dS and dy/den are rounded to bf16); every
 * other shape, fp32 inputs and REHYAT_FLAG_FORCE_SIMT run fp32 CUDA cores.
 * No atomics, so repeated calls agree bit for bit.
 * Pointers: q, k, v, y, dy, dq, dk, dv, workspace 16-byte aligned; c, den and
 * the parameter gradients 4-byte aligned.  Errors as for
 * rehyat_hybrid_attn_fwd; REHYAT_FLAG_FP8_QK is refused (UNSUPPORTED).
 * REHYAT_FLAG_FWD_STATE as for rehyat_phi_bwd. */
REHYAT_API rehyat_status rehyat_hybrid_attn_bwd(const rehyat_params* p, const void* q,
                                                const void* k, const void* v,
                                                const rehyat_phi* phi, const float* y,
                                                const float* dy, const float* c,
                                                const float* den, float* dq, float* dk,
                                                float* dv, const rehyat_phi_grad* grad,
                                                void* workspace, size_t ws_bytes,
                                                void* stream);

/* ---------------------------------------------------------------------- */
/* Diagnostic: every wait inside the tensor-core kernels is bounded (~2 s);
 * a wait that runs out sets a bit in a device-side error word and the
 * kernel returns early instead of hanging.  This reads that word for the
 * current device into *flags (0 = no timeout since the last reset) and
 * clears it when reset != 0.  Unlike the other entry points it synchronises
 * the device (a blocking copy). */
REHYAT_API rehyat_status rehyat_device_error_flags(unsigned* flags, int reset);

/* Denominator report for the forward with phi given
 * (rehyat_hybrid_attn_fwd_phi).  A general feature map with a degree-1 part
 * (Key design 3 of the ReHyAt note) is signed, so n^L can be negative and
 * the joint denominator n^S + n^L can approach zero or drop below it (n^S
 * >= 1 always holds).  The forward keeps y = (a^S + a^L) / (n^S + n^L) as
 * written, and counts the query rows where n^S + n^L < 2^-10 n^S (a
 * non-positive or NaN denominator, or one cancelled to ~10 bits).  This
 * reads the count for the current device into *rows (summed over every
 * such forward since the last reset) and clears it when reset != 0.  The
 * closed-form phi (a sum of squares) never adds to it.  Synchronises the
 * device (blocking copies). */
REHYAT_API rehyat_status rehyat_denominator_report(unsigned long long* rows, int reset);

/* Which attention kernel these params select: 1 = the tensor-core kernel
 * (bf16 inputs, D = 128, Dp in {64, 128, 256}, no REHYAT_FLAG_FORCE_SIMT),
 * 0 = the fp32 CUDA-core kernel, -1 = invalid params.  Host-only. */
REHYAT_API int rehyat_attn_path(const rehyat_params* p);

REHYAT_API const char* rehyat_status_string(rehyat_status s);

/* Library ABI version (major*10000 + minor*100 + patch). */
REHYAT_API int rehyat_version(void);

#ifdef __cplusplus
}
#endif
#endif /* REHYAT_H */
