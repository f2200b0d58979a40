"""Python binding of librehyat.so: ReHyAt chunked hybrid attention on B200.

Two layers:

* ``lib()`` and the ``rehyat_*`` functions are the C ABI of include/rehyat.h,
  called through ctypes with plain integers for device pointers and streams
  (argument marshalling only).
* ``hybrid_attn``, ``softmax_attn`` and ``StreamingState`` take torch CUDA
  tensors, allocate outputs/workspace with torch and call the C ABI on
  torch's current stream.  torch provides device memory and streams; every
  step of the computation runs in the library's CUDA kernels.

There is no CPU fallback: if librehyat.so is missing, ``lib()`` raises.
Build it with ``python -m linear_attention_video_chunked_b200.build``.

Method: "ReHyAt: Recurrent Hybrid Attention for Video Diffusion
Transformers" (papernotes.org note), Method, Key designs 1-4.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

__all__ = [
    "RehyatParams", "RehyatPhi", "RehyatDebug", "RehyatError", "lib", "lib_path",
    "EXPORTED_SYMBOLS", "F32", "BF16", "FLAG_FORCE_SIMT", "FLAG_FP8_QK", "FLAG_PHI_BF16",
    "FLAG_FWD_STATE",
    "rehyat_workspace_bytes", "rehyat_hybrid_attn_fwd", "rehyat_fwd_state", "rehyat_fwd_attn",
    "rehyat_softmax_attn_fwd", "rehyat_state_bytes", "rehyat_state_init", "rehyat_step_workspace_bytes",
    "rehyat_chunk_step", "rehyat_device_error_flags", "rehyat_attn_path",
    "rehyat_status_string", "rehyat_version", "rehyat_hybrid_attn_fwd_noalloc",
    "RehyatPhiGrad", "rehyat_phi_bwd_workspace_bytes", "rehyat_phi_bwd",
    "RehyatPhiMlp", "rehyat_hybrid_attn_fwd_phi", "rehyat_feature_map_mlp",
    "rehyat_feature_map_mlp_workspace_bytes", "rehyat_host_workspace_bytes",
    "rehyat_hybrid_attn_fwd_host", "hybrid_attn_host",
    "make_params", "hybrid_attn", "hybrid_attn_phi", "feature_map_mlp", "softmax_attn",
    "phi_grad", "bwd_workspace", "StreamingState", "rehyat_hybrid_attn_bwd_workspace_bytes",
    "rehyat_hybrid_attn_bwd", "hybrid_attn_bwd", "rehyat_denominator_report",
    "rehyat_step_key_split",
]

F32, BF16 = 0, 1
FLAG_FORCE_SIMT = 1
FLAG_ONE_TILE = 2
FLAG_FP8_QK = 4
FLAG_PHI_BF16 = 8
FLAG_FWD_STATE = 16

STATUS = {0: "REHYAT_OK", 1: "REHYAT_ERR_INVALID_ARG", 2: "REHYAT_ERR_UNSUPPORTED",
          3: "REHYAT_ERR_MISALIGNED", 4: "REHYAT_ERR_WORKSPACE", 5: "REHYAT_ERR_CUDA",
          6: "REHYAT_ERR_SCRATCH_LIMIT"}

EXPORTED_SYMBOLS = (
    "rehyat_workspace_bytes", "rehyat_hybrid_attn_fwd", "rehyat_fwd_state",
    "rehyat_fwd_attn", "rehyat_softmax_attn_fwd", "rehyat_state_bytes", "rehyat_state_init",
    "rehyat_step_workspace_bytes", "rehyat_chunk_step", "rehyat_device_error_flags",
    "rehyat_attn_path", "rehyat_status_string", "rehyat_version",
    "rehyat_hybrid_attn_fwd_noalloc", "rehyat_phi_bwd_workspace_bytes", "rehyat_phi_bwd",
    "rehyat_hybrid_attn_fwd_phi", "rehyat_feature_map_mlp",
    "rehyat_feature_map_mlp_workspace_bytes", "rehyat_host_workspace_bytes",
    "rehyat_hybrid_attn_fwd_host", "rehyat_hybrid_attn_bwd_workspace_bytes",
    "rehyat_hybrid_attn_bwd", "rehyat_denominator_report", "rehyat_step_key_split",
)


class RehyatParams(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int), ("heads", ctypes.c_int), ("T", ctypes.c_int),
                ("Hs", ctypes.c_int), ("Ws", ctypes.c_int), ("D", ctypes.c_int),
                ("Dp", ctypes.c_int), ("Tc", ctypes.c_int), ("To", ctypes.c_int),
                ("causal", ctypes.c_int), ("in_dtype", ctypes.c_int),
                ("out_dtype", ctypes.c_int), ("scale", ctypes.c_float),
                ("flags", ctypes.c_int)]


class RehyatPhi(ctypes.Structure):
    _fields_ = [("Wq", ctypes.c_void_p), ("bq", ctypes.c_void_p),
                ("Wk", ctypes.c_void_p), ("bk", ctypes.c_void_p)]


class RehyatDebug(ctypes.Structure):
    _fields_ = [("aS", ctypes.c_void_p), ("nS", ctypes.c_void_p), ("c", ctypes.c_void_p),
                ("aL", ctypes.c_void_p), ("nL", ctypes.c_void_p)]


class RehyatPhiGrad(ctypes.Structure):
    _fields_ = [("dWq", ctypes.c_void_p), ("dbq", ctypes.c_void_p),
                ("dWk", ctypes.c_void_p), ("dbk", ctypes.c_void_p)]


class RehyatPhiMlp(ctypes.Structure):
    _fields_ = [("Wa", ctypes.c_void_p), ("ba", ctypes.c_void_p), ("Wb", ctypes.c_void_p),
                ("bb", ctypes.c_void_p), ("Dh", ctypes.c_int), ("parts", ctypes.c_int)]


class RehyatError(RuntimeError):
    def __init__(self, status: int, where: str):
        super().__init__(f"{where}: {STATUS.get(status, status)}")
        self.status = status


_LIB = None


def lib_path() -> str:
    """librehyat.so next to this file, or the file named by REHYAT_LIBRARY."""
    override = os.environ.get("REHYAT_LIBRARY")
    if override:
        return override
    return os.path.join(os.path.dirname(os.path.abspath(__file__)), "librehyat.so")


def lib() -> ctypes.CDLL:
    """Load librehyat.so (raises if it has not been built)."""
    global _LIB
    if _LIB is None:
        path = lib_path()
        if not os.path.exists(path):
            raise ImportError(f"{path} is missing; build it with "
                              "`python -m linear_attention_video_chunked_b200.build`")
        L = ctypes.CDLL(path)
        P = ctypes.POINTER
        vp, sz, i = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int
        L.rehyat_workspace_bytes.argtypes = [P(RehyatParams)]
        L.rehyat_workspace_bytes.restype = sz
        L.rehyat_hybrid_attn_fwd.argtypes = [P(RehyatParams), vp, vp, vp, P(RehyatPhi), vp, vp,
                                             sz, P(RehyatDebug), vp]
        L.rehyat_hybrid_attn_fwd.restype = i
        L.rehyat_fwd_state.argtypes = [P(RehyatParams), vp, vp, P(RehyatPhi), vp, sz, vp]
        L.rehyat_fwd_state.restype = i
        L.rehyat_fwd_attn.argtypes = [P(RehyatParams), vp, vp, vp, P(RehyatPhi), vp, vp, sz,
                                      P(RehyatDebug), vp]
        L.rehyat_fwd_attn.restype = i
        L.rehyat_hybrid_attn_fwd_noalloc.argtypes = [P(RehyatParams), vp, vp, vp, P(RehyatPhi),
                                                     vp, P(RehyatDebug), vp]
        L.rehyat_hybrid_attn_fwd_noalloc.restype = i
        L.rehyat_softmax_attn_fwd.argtypes = [P(RehyatParams), vp, vp, vp, vp, vp]
        L.rehyat_softmax_attn_fwd.restype = i
        L.rehyat_state_bytes.argtypes = [P(RehyatParams)]
        L.rehyat_state_bytes.restype = sz
        L.rehyat_state_init.argtypes = [P(RehyatParams), vp, vp]
        L.rehyat_state_init.restype = i
        L.rehyat_step_workspace_bytes.argtypes = [P(RehyatParams)]
        L.rehyat_step_workspace_bytes.restype = sz
        L.rehyat_step_key_split.argtypes = [P(RehyatParams), ctypes.c_int]
        L.rehyat_step_key_split.restype = ctypes.c_int
        L.rehyat_chunk_step.argtypes = [P(RehyatParams), vp, vp, vp, i, P(RehyatPhi), vp, vp, vp,
                                        sz, P(RehyatDebug), vp]
        L.rehyat_chunk_step.restype = i
        L.rehyat_denominator_report.argtypes = [P(ctypes.c_ulonglong), i]
        L.rehyat_denominator_report.restype = i
        L.rehyat_device_error_flags.argtypes = [P(ctypes.c_uint), i]
        L.rehyat_device_error_flags.restype = i
        L.rehyat_attn_path.argtypes = [P(RehyatParams)]
        L.rehyat_attn_path.restype = i
        L.rehyat_status_string.argtypes = [i]
        L.rehyat_status_string.restype = ctypes.c_char_p
        L.rehyat_version.argtypes = []
        L.rehyat_version.restype = i
        L.rehyat_phi_bwd_workspace_bytes.argtypes = [P(RehyatParams)]
        L.rehyat_phi_bwd_workspace_bytes.restype = sz
        L.rehyat_phi_bwd.argtypes = [P(RehyatParams), vp, vp, vp, vp, vp, vp, P(RehyatPhi),
                                     P(RehyatPhiGrad), vp, sz, vp]
        L.rehyat_phi_bwd.restype = i
        L.rehyat_hybrid_attn_bwd_workspace_bytes.argtypes = [P(RehyatParams)]
        L.rehyat_hybrid_attn_bwd_workspace_bytes.restype = sz
        L.rehyat_hybrid_attn_bwd.argtypes = [P(RehyatParams), vp, vp, vp, P(RehyatPhi), vp, vp,
                                             vp, vp, vp, vp, vp, P(RehyatPhiGrad), vp, sz, vp]
        L.rehyat_hybrid_attn_bwd.restype = i
        L.rehyat_hybrid_attn_fwd_phi.argtypes = [P(RehyatParams), vp, vp, vp, vp, vp, vp, vp, sz,
                                                 vp, vp]
        L.rehyat_hybrid_attn_fwd_phi.restype = i
        L.rehyat_feature_map_mlp.argtypes = [P(RehyatParams), vp, P(RehyatPhiMlp), vp, vp,
                                             ctypes.c_size_t, vp]
        L.rehyat_feature_map_mlp.restype = i
        L.rehyat_feature_map_mlp_workspace_bytes.argtypes = [P(RehyatParams), P(RehyatPhiMlp),
                                                             vp, vp]
        L.rehyat_feature_map_mlp_workspace_bytes.restype = ctypes.c_size_t
        L.rehyat_host_workspace_bytes.argtypes = [P(RehyatParams), i]
        L.rehyat_host_workspace_bytes.restype = ctypes.c_size_t
        L.rehyat_hybrid_attn_fwd_host.argtypes = [P(RehyatParams), vp, vp, vp, P(RehyatPhi), vp,
                                                  i, vp, ctypes.c_size_t, vp]
        L.rehyat_hybrid_attn_fwd_host.restype = i
        _LIB = L
    return _LIB


# ---------------------------------------------------------------- raw C ABI
def rehyat_workspace_bytes(p: RehyatParams) -> int:
    return lib().rehyat_workspace_bytes(ctypes.byref(p))


def rehyat_hybrid_attn_fwd(p, q, k, v, phi, y, workspace, ws_bytes, dbg, stream) -> int:
    return lib().rehyat_hybrid_attn_fwd(ctypes.byref(p), q, k, v, ctypes.byref(phi), y,
                                        workspace, ws_bytes,
                                        None if dbg is None else ctypes.byref(dbg), stream)


def rehyat_fwd_state(p, k, v, phi, workspace, ws_bytes, stream) -> int:
    return lib().rehyat_fwd_state(ctypes.byref(p), k, v, ctypes.byref(phi), workspace, ws_bytes,
                                  stream)


def rehyat_fwd_attn(p, q, k, v, phi, y, workspace, ws_bytes, dbg, stream) -> int:
    return lib().rehyat_fwd_attn(ctypes.byref(p), q, k, v, ctypes.byref(phi), y, workspace,
                                 ws_bytes, None if dbg is None else ctypes.byref(dbg), stream)


def rehyat_hybrid_attn_fwd_noalloc(p, q, k, v, phi, y, dbg, stream) -> int:
    """The full forward on the library's built-in 32 MiB device scratch, for
    callers that cannot allocate a workspace (see include/rehyat.h)."""
    return lib().rehyat_hybrid_attn_fwd_noalloc(ctypes.byref(p), q, k, v, ctypes.byref(phi), y,
                                                None if dbg is None else ctypes.byref(dbg),
                                                stream)


def rehyat_phi_bwd_workspace_bytes(p: RehyatParams) -> int:
    return lib().rehyat_phi_bwd_workspace_bytes(ctypes.byref(p))


def rehyat_denominator_report(reset: bool = False) -> int:
    """Rows with n^S + n^L < 2^-10 n^S in forwards with phi given, since the
    last reset (blocking)."""
    rows = ctypes.c_ulonglong(0)
    _check(lib().rehyat_denominator_report(ctypes.byref(rows), 1 if reset else 0),
           "rehyat_denominator_report")
    return rows.value


def rehyat_hybrid_attn_bwd_workspace_bytes(p: RehyatParams) -> int:
    return lib().rehyat_hybrid_attn_bwd_workspace_bytes(ctypes.byref(p))


def rehyat_hybrid_attn_bwd(p, q, k, v, phi, y, dy, c, den, dq, dk, dv, grad, workspace, ws_bytes,
                           stream) -> int:
    return lib().rehyat_hybrid_attn_bwd(ctypes.byref(p), q, k, v, ctypes.byref(phi), y, dy, c, den,
                                        dq, dk, dv, ctypes.byref(grad), workspace, ws_bytes,
                                        stream)


def rehyat_phi_bwd(p, q, k, v, y, dy, den, phi, grad, workspace, ws_bytes, stream) -> int:
    return lib().rehyat_phi_bwd(ctypes.byref(p), q, k, v, y, dy, den, ctypes.byref(phi),
                                ctypes.byref(grad), workspace, ws_bytes, stream)


def rehyat_hybrid_attn_fwd_phi(p, q, k, v, phi_q, phi_k, y, workspace, ws_bytes, dbg,
                               stream) -> int:
    return lib().rehyat_hybrid_attn_fwd_phi(ctypes.byref(p), q, k, v, phi_q, phi_k, y, workspace,
                                            ws_bytes, None if dbg is None else ctypes.byref(dbg),
                                            stream)


def rehyat_host_workspace_bytes(p, heads_per_slab) -> int:
    return lib().rehyat_host_workspace_bytes(ctypes.byref(p), heads_per_slab)


def rehyat_hybrid_attn_fwd_host(p, q, k, v, phi, y, heads_per_slab, workspace, ws_bytes,
                                stream) -> int:
    return lib().rehyat_hybrid_attn_fwd_host(ctypes.byref(p), q, k, v, ctypes.byref(phi), y,
                                             heads_per_slab, workspace, ws_bytes, stream)


def rehyat_feature_map_mlp_workspace_bytes(p, mlp, x, phi) -> int:
    return lib().rehyat_feature_map_mlp_workspace_bytes(ctypes.byref(p), ctypes.byref(mlp), x,
                                                        phi)


def rehyat_feature_map_mlp(p, x, mlp, phi, workspace, ws_bytes, stream) -> int:
    return lib().rehyat_feature_map_mlp(ctypes.byref(p), x, ctypes.byref(mlp), phi, workspace,
                                        ws_bytes, stream)


def rehyat_softmax_attn_fwd(p, q, k, v, y, stream) -> int:
    return lib().rehyat_softmax_attn_fwd(ctypes.byref(p), q, k, v, y, stream)


def rehyat_state_bytes(p: RehyatParams) -> int:
    return lib().rehyat_state_bytes(ctypes.byref(p))


def rehyat_state_init(p, state, stream) -> int:
    return lib().rehyat_state_init(ctypes.byref(p), state, stream)


def rehyat_step_workspace_bytes(p: RehyatParams) -> int:
    return lib().rehyat_step_workspace_bytes(ctypes.byref(p))


def rehyat_step_key_split(p: RehyatParams, nslices: int) -> int:
    return lib().rehyat_step_key_split(ctypes.byref(p), int(nslices))


def rehyat_chunk_step(p, q, k, v, nslices, phi, state, y, workspace, ws_bytes, dbg,
                      stream) -> int:
    return lib().rehyat_chunk_step(ctypes.byref(p), q, k, v, nslices, ctypes.byref(phi), state,
                                   y, workspace, ws_bytes,
                                   None if dbg is None else ctypes.byref(dbg), stream)


def rehyat_device_error_flags(reset: bool = False) -> int:
    """Timeout bits of the tensor-core kernels' bounded waits (synchronises)."""
    out = ctypes.c_uint(0)
    _check(lib().rehyat_device_error_flags(ctypes.byref(out), int(reset)),
           "rehyat_device_error_flags")
    return out.value


def rehyat_attn_path(p: RehyatParams) -> int:
    """1 = tensor-core attention kernel, 0 = CUDA-core kernel, -1 = invalid."""
    return lib().rehyat_attn_path(ctypes.byref(p))


def rehyat_status_string(status: int) -> str:
    return lib().rehyat_status_string(status).decode()


def rehyat_version() -> int:
    return lib().rehyat_version()


# ------------------------------------------------------------- torch layer
def make_params(*, batch, heads, T, Hs, Ws, D, Dp, Tc, To, causal, in_dtype=BF16,
                out_dtype=F32, scale=0.0, flags=0) -> RehyatParams:
    return RehyatParams(batch, heads, T, Hs, Ws, D, Dp, Tc, To, int(causal), in_dtype,
                        out_dtype, float(scale), flags)


def _torch():
    import torch
    return torch


def _dtype_code(t) -> int:
    torch = _torch()
    if t == torch.bfloat16:
        return BF16
    if t == torch.float32:
        return F32
    raise TypeError(f"unsupported dtype {t}")


def _check(status: int, where: str):
    if status != 0:
        raise RehyatError(status, where)


def _stream_handle(stream=None) -> int:
    torch = _torch()
    s = torch.cuda.current_stream() if stream is None else stream
    return s.cuda_stream


# The C ABI takes bare pointers and sizes: a tensor of the wrong shape,
# strides or device would make the kernels read or write outside it.  The
# torch layer therefore checks every tensor against the sizes it passes
# before anything is launched.
def _need(ok: bool, what: str, exc=ValueError):
    if not ok:
        raise exc(what)


def _check_qkv(q, k, v, *, cuda=True):
    """q, k, v: contiguous [B, h, N, D] tensors of one shape and dtype on one
    device (a CUDA device for the device entry points, host memory for the
    host-buffer forward)."""
    _need(q.dim() == 4, "q must be a [B, h, N, D] tensor")
    where = "CUDA tensors on one device" if cuda else "host (CPU) tensors"
    for name, t in (("q", q), ("k", k), ("v", v)):
        _need(tuple(t.shape) == tuple(q.shape), f"{name} must be shaped like q {tuple(q.shape)}")
        _need(t.dtype == q.dtype, f"{name} must have q's dtype {q.dtype}", TypeError)
        _need(t.is_contiguous(), f"{name} must be contiguous")
        _need(t.is_cuda == cuda and t.device == q.device, f"q, k and v must be {where}")


def _check_current_device(device):
    """The library launches on the current CUDA device: its tensors must live
    there (a pointer into another GPU's memory would fault)."""
    cur = _torch().cuda.current_device()
    _need(device.type == "cuda" and device.index == cur,
          f"tensors are on {device} but the current CUDA device is cuda:{cur}; "
          "call torch.cuda.set_device first")


def _check_tokens(N, T, Hs, Ws):
    _need(N == T * Hs * Ws, f"N = {N} tokens per head must equal T*Hs*Ws = {T * Hs * Ws}")


def _check_out(t, shape, dtype, device, name="out"):
    _need(tuple(t.shape) == tuple(shape), f"{name} must be shaped {tuple(shape)}")
    _need(t.dtype == dtype, f"{name} must be {dtype}", TypeError)
    _need(t.is_contiguous(), f"{name} must be contiguous")
    _need(t.device == device, f"{name} must be on {device}")


def _check_workspace(ws, device):
    _need(ws.is_contiguous() and ws.device == device,
          f"workspace must be a contiguous tensor on {device}")


def _nbytes(t) -> int:
    return t.numel() * t.element_size()


def _check_params(named, sizes, device=None, what="phi parameters"):
    """Each parameter tensor holds exactly its count of fp32 values, in a
    contiguous CUDA tensor (on ``device`` when given)."""
    torch = _torch()
    for (name, t), n in zip(named, sizes):
        _need(t.numel() == n, f"{name} must hold {n} values, not {t.numel()}")
    for name, t in named:
        _need(t.dtype == torch.float32 and t.is_cuda and t.is_contiguous(),
              f"{what} must be contiguous fp32 CUDA tensors", TypeError)
        _need(device is None or t.device == device, f"{name} must be on {device}")


def _phi_struct(Wq, bq, Wk, bk, *, heads=None, D=None, Dp=None, device=None) -> RehyatPhi:
    """phi_q, phi_k parameters: W [heads, 2, D, D'/2] and b [heads, 2, D'/2]
    (heads x D x D' and heads x D' values) when the sizes are given."""
    named = (("Wq", Wq), ("bq", bq), ("Wk", Wk), ("bk", bk))
    if heads is None:
        sizes = [t.numel() for _, t in named]
    else:
        sizes = [heads * D * Dp, heads * Dp, heads * D * Dp, heads * Dp]
    _check_params(named, sizes, device)
    return RehyatPhi(Wq.data_ptr(), bq.data_ptr(), Wk.data_ptr(), bk.data_ptr())


def _debug_tensors(shape4, device):
    torch = _torch()
    B, H, N, D = shape4
    d = dict(aS=torch.empty(B, H, N, D, device=device), nS=torch.empty(B, H, N, device=device),
             c=torch.empty(B, H, N, device=device), aL=torch.empty(B, H, N, D, device=device),
             nL=torch.empty(B, H, N, device=device))
    st = RehyatDebug(*(d[k].data_ptr() for k in ("aS", "nS", "c", "aL", "nL")))
    return d, st


def hybrid_attn(q, k, v, Wq, bq, Wk, bk, *, T, Hs, Ws, Tc, To, causal, out_dtype=None,
                scale=0.0, debug=False, force_simt=False, one_tile=False, fp8_qk=False,
                workspace=None, out=None, stream=None):
    """ReHyAt hybrid attention of torch CUDA tensors q, k, v [B, h, N, D].

    ``fp8_qk``: the softmax logits from E4M3 copies of q and k
    (REHYAT_FLAG_FP8_QK).  Returns y (and a dict of branch partials when
    ``debug``)."""
    torch = _torch()
    _check_qkv(q, k, v)
    _check_current_device(q.device)
    B, H, N, D = q.shape
    _check_tokens(N, T, Hs, Ws)
    Dp = 2 * Wq.shape[-1]
    phi = _phi_struct(Wq, bq, Wk, bk, heads=H, D=D, Dp=Dp, device=q.device)
    out_dtype = torch.float32 if out_dtype is None else out_dtype
    p = make_params(batch=B, heads=H, T=T, Hs=Hs, Ws=Ws, D=D, Dp=Dp, Tc=Tc, To=To,
                    causal=causal, in_dtype=_dtype_code(q.dtype),
                    out_dtype=_dtype_code(out_dtype), scale=scale,
                    flags=(FLAG_FORCE_SIMT if force_simt else 0) |
                    (FLAG_ONE_TILE if one_tile else 0) | (FLAG_FP8_QK if fp8_qk else 0))
    if out is not None:
        _check_out(out, (B, H, N, D), out_dtype, q.device)
    y = torch.empty(B, H, N, D, dtype=out_dtype, device=q.device) if out is None else out
    nbytes = rehyat_workspace_bytes(p)
    if nbytes == 0:
        raise RehyatError(1, "rehyat_workspace_bytes")
    if workspace is not None:
        _check_workspace(workspace, q.device)
    if workspace is None or _nbytes(workspace) < nbytes:
        workspace = torch.empty(nbytes, dtype=torch.uint8, device=q.device)
    dbg_t, dbg_s = _debug_tensors((B, H, N, D), q.device) if debug else (None, None)
    st = rehyat_hybrid_attn_fwd(p, q.data_ptr(), k.data_ptr(), v.data_ptr(), phi, y.data_ptr(),
                                workspace.data_ptr(), _nbytes(workspace), dbg_s,
                                _stream_handle(stream))
    _check(st, "rehyat_hybrid_attn_fwd")
    return (y, dbg_t) if debug else y


def hybrid_attn_host(q, k, v, Wq, bq, Wk, bk, *, T, Hs, Ws, Tc, To, causal, out=None,
                     heads_per_slab=2, fp8_qk=False, workspace=None, stream=None):
    """hybrid_attn on CPU tensors q, k, v [B, h, N, D] (pin them for overlap):
    slabs of heads are uploaded, computed and downloaded concurrently by
    rehyat_hybrid_attn_fwd_host; the phi parameters are CUDA tensors.
    Returns y (fp32, CPU; `out` if given), valid after `stream` syncs (this
    function synchronises it)."""
    torch = _torch()
    _check_qkv(q, k, v, cuda=False)
    B, H, N, D = q.shape
    _check_tokens(N, T, Hs, Ws)
    Dp = 2 * Wq.shape[-1]
    phi = _phi_struct(Wq, bq, Wk, bk, heads=H, D=D, Dp=Dp)
    _check_current_device(Wq.device)
    p = make_params(batch=B, heads=H, T=T, Hs=Hs, Ws=Ws, D=D, Dp=Dp, Tc=Tc, To=To,
                    causal=causal, in_dtype=_dtype_code(q.dtype), out_dtype=F32,
                    flags=FLAG_FP8_QK if fp8_qk else 0)
    if out is not None:
        _check_out(out, (B, H, N, D), torch.float32, q.device)
    y = torch.empty(B, H, N, D, dtype=torch.float32, pin_memory=True) if out is None else out
    nbytes = rehyat_host_workspace_bytes(p, heads_per_slab)
    if nbytes == 0:
        raise RehyatError(1, "rehyat_host_workspace_bytes")
    if workspace is not None:
        _check_workspace(workspace, Wq.device)
    if workspace is None or _nbytes(workspace) < nbytes:
        workspace = torch.empty(nbytes, dtype=torch.uint8, device=Wq.device)
    st = rehyat_hybrid_attn_fwd_host(p, q.data_ptr(), k.data_ptr(), v.data_ptr(), phi,
                                     y.data_ptr(), heads_per_slab, workspace.data_ptr(),
                                     _nbytes(workspace), _stream_handle(stream))
    _check(st, "rehyat_hybrid_attn_fwd_host")
    (stream or torch.cuda.current_stream()).synchronize()
    return y


def feature_map_mlp(x, Wa, ba, Wb, bb, *, parts, T, Hs, Ws, stream=None, force_simt=False,
                    workspace=None, out=None, out_dtype=None):
    """phi = [psi_1^1, ..., psi_P^P], psi = GELU(x Wa + ba) Wb + bb per head,
    of a torch CUDA tensor x [B, h, N, D]; Wa [h, D, Dh], ba [h, Dh],
    Wb [h, Dh, D'], bb [h, D'] fp32.  Returns [B, h, N, D'] in out_dtype
    (fp32 by default, or bf16).  bf16 x with D = 128 runs on the tensor cores
    (bf16 operands) unless force_simt."""
    torch = _torch()
    _need(x.dim() == 4, "x must be a [B, h, N, D] tensor")
    _need(x.is_contiguous() and x.is_cuda, "x must be a contiguous CUDA tensor")
    _check_current_device(x.device)
    B, H, N, D = x.shape
    _check_tokens(N, T, Hs, Ws)
    Dh, Dp = Wa.shape[-1], Wb.shape[-1]
    _check_params((("Wa", Wa), ("ba", ba), ("Wb", Wb), ("bb", bb)),
                  (H * D * Dh, H * Dh, H * Dh * Dp, H * Dp), x.device, "MLP parameters")
    out_dtype = torch.float32 if out_dtype is None else out_dtype
    _need(out_dtype in (torch.float32, torch.bfloat16), "out_dtype must be fp32 or bf16",
          TypeError)
    p = make_params(batch=B, heads=H, T=T, Hs=Hs, Ws=Ws, D=D, Dp=Dp, Tc=1, To=0, causal=0,
                    in_dtype=_dtype_code(x.dtype), out_dtype=F32,
                    flags=(FLAG_FORCE_SIMT if force_simt else 0) |
                    (FLAG_PHI_BF16 if out_dtype == torch.bfloat16 else 0))
    if out is not None:
        _check_out(out, (B, H, N, Dp), out_dtype, x.device)
    phi = out if out is not None else torch.empty(B, H, N, Dp, dtype=out_dtype,
                                                  device=x.device)
    mlp = RehyatPhiMlp(Wa.data_ptr(), ba.data_ptr(), Wb.data_ptr(), bb.data_ptr(), Dh, parts)
    nbytes = rehyat_feature_map_mlp_workspace_bytes(p, mlp, x.data_ptr(), phi.data_ptr())
    if nbytes and workspace is not None:
        _check_workspace(workspace, x.device)
    if nbytes and (workspace is None or _nbytes(workspace) < nbytes):
        workspace = torch.empty(nbytes, dtype=torch.uint8, device=x.device)
    ws_ptr = workspace.data_ptr() if nbytes else None
    _check(rehyat_feature_map_mlp(p, x.data_ptr(), mlp, phi.data_ptr(), ws_ptr, nbytes,
                                  _stream_handle(stream)), "rehyat_feature_map_mlp")
    return phi


def hybrid_attn_phi(q, k, v, phi_q, phi_k, *, T, Hs, Ws, Tc, To, causal, out_dtype=None,
                    scale=0.0, debug=False, force_simt=False, workspace=None, out=None,
                    stream=None):
    """The hybrid forward with the feature maps given: phi_q = phi_q(q) and
    phi_k = phi_k(k), [B, h, N, D'] CUDA tensors, both fp32 or both bf16.
    Returns y (and the branch partials when ``debug``)."""
    torch = _torch()
    _check_qkv(q, k, v)
    _check_current_device(q.device)
    B, H, N, D = q.shape
    _check_tokens(N, T, Hs, Ws)
    Dp = phi_q.shape[-1]
    for t in (phi_q, phi_k):
        if (t.dtype not in (torch.float32, torch.bfloat16) or t.dtype != phi_q.dtype
                or not t.is_contiguous() or t.dim() != 4 or tuple(t.shape) != (B, H, N, Dp)):
            raise TypeError("phi_q, phi_k must be contiguous [B, h, N, D'] tensors, both fp32 "
                            "or both bf16")
        _need(t.device == q.device, "phi_q, phi_k must be on q's device")
    out_dtype = torch.float32 if out_dtype is None else out_dtype
    p = make_params(batch=B, heads=H, T=T, Hs=Hs, Ws=Ws, D=D, Dp=Dp, Tc=Tc, To=To,
                    causal=causal, in_dtype=_dtype_code(q.dtype),
                    out_dtype=_dtype_code(out_dtype), scale=scale,
                    flags=(FLAG_FORCE_SIMT if force_simt else 0) |
                    (FLAG_PHI_BF16 if phi_q.dtype == torch.bfloat16 else 0))
    if out is not None:
        _check_out(out, (B, H, N, D), out_dtype, q.device)
    y = torch.empty(B, H, N, D, dtype=out_dtype, device=q.device) if out is None else out
    nbytes = rehyat_workspace_bytes(p)
    if nbytes == 0:
        raise RehyatError(1, "rehyat_workspace_bytes")
    if workspace is not None:
        _check_workspace(workspace, q.device)
    if workspace is None:
        workspace = torch.empty(nbytes, dtype=torch.uint8, device=q.device)
    dbg_t, dbg_s = _debug_tensors((B, H, N, D), q.device) if debug else (None, None)
    st = rehyat_hybrid_attn_fwd_phi(p, q.data_ptr(), k.data_ptr(), v.data_ptr(),
                                    phi_q.data_ptr(), phi_k.data_ptr(), y.data_ptr(),
                                    workspace.data_ptr(), _nbytes(workspace), dbg_s,
                                    _stream_handle(stream))
    _check(st, "rehyat_hybrid_attn_fwd_phi")
    return (y, dbg_t) if debug else y


def bwd_workspace(q, Wq, *, T, Hs, Ws, Tc, To, causal, full=True, force_simt=False):
    """A device workspace large enough for the forward and for the backward
    (``hybrid_attn_bwd`` if ``full``, else ``phi_grad``) of q's shape: pass it
    to ``hybrid_attn`` and then, with ``state_from_forward=True``, to the
    backward, which reuses the forward's linear-set state."""
    torch = _torch()
    B, H, N, D = q.shape
    _check_tokens(N, T, Hs, Ws)
    p = make_params(batch=B, heads=H, T=T, Hs=Hs, Ws=Ws, D=D, Dp=2 * Wq.shape[-1], Tc=Tc,
                    To=To, causal=causal, in_dtype=_dtype_code(q.dtype), out_dtype=F32,
                    flags=FLAG_FORCE_SIMT if force_simt else 0)
    nbytes = (rehyat_hybrid_attn_bwd_workspace_bytes(p) if full
              else rehyat_phi_bwd_workspace_bytes(p))
    if nbytes == 0:
        raise RehyatError(1, "rehyat_*_bwd_workspace_bytes")
    return torch.empty(max(nbytes, rehyat_workspace_bytes(p)), dtype=torch.uint8,
                       device=q.device)


def phi_grad(q, k, v, y, dy, den, Wq, bq, Wk, bk, *, T, Hs, Ws, Tc, To, causal, scale=0.0,
             force_simt=False, workspace=None, stream=None, state_from_forward=False):
    """Gradients of L with respect to the phi parameters, given the forward's
    q, k, v, its fp32 output y, dy = dL/dy (fp32) and den = n^S + n^L per
    query (``parts["nS"] + parts["nL"]`` of ``hybrid_attn(..., debug=True)``).
    ``state_from_forward`` (REHYAT_FLAG_FWD_STATE): ``workspace`` is the
    buffer the forward ran on (from ``bwd_workspace(..., full=False)``), so
    its linear-set state is reused instead of recomputed.
    Returns dict(dWq, dbq, dWk, dbk) shaped like the parameters."""
    torch = _torch()
    _check_qkv(q, k, v)
    _check_current_device(q.device)
    B, H, N, D = q.shape
    _check_tokens(N, T, Hs, Ws)
    Dp = 2 * Wq.shape[-1]
    for t in (y, dy, den):
        if t.dtype != torch.float32 or not t.is_contiguous():
            raise TypeError("y, dy and den must be contiguous fp32 tensors")
    _check_out(y, (B, H, N, D), torch.float32, q.device, "y")
    _check_out(dy, (B, H, N, D), torch.float32, q.device, "dy")
    _check_out(den, (B, H, N), torch.float32, q.device, "den")
    phi = _phi_struct(Wq, bq, Wk, bk, heads=H, D=D, Dp=Dp, device=q.device)
    _need(not state_from_forward or workspace is not None,
          "state_from_forward needs the forward's workspace")
    p = make_params(batch=B, heads=H, T=T, Hs=Hs, Ws=Ws, D=D, Dp=Dp, Tc=Tc, To=To,
                    causal=causal, in_dtype=_dtype_code(q.dtype), out_dtype=F32, scale=scale,
                    flags=(FLAG_FORCE_SIMT if force_simt else 0) |
                    (FLAG_FWD_STATE if state_from_forward else 0))
    nbytes = rehyat_phi_bwd_workspace_bytes(p)
    if nbytes == 0:
        raise RehyatError(1, "rehyat_phi_bwd_workspace_bytes")
    if workspace is not None:
        _check_workspace(workspace, q.device)
    if workspace is None:
        workspace = torch.empty(nbytes, dtype=torch.uint8, device=q.device)
    g = {name: torch.empty_like(t, memory_format=torch.contiguous_format) for name, t in
         (("dWq", Wq), ("dbq", bq), ("dWk", Wk), ("dbk", bk))}
    grad = RehyatPhiGrad(*(g[n].data_ptr() for n in ("dWq", "dbq", "dWk", "dbk")))
    st = rehyat_phi_bwd(p, q.data_ptr(), k.data_ptr(), v.data_ptr(), y.data_ptr(), dy.data_ptr(),
                        den.data_ptr(), phi, grad, workspace.data_ptr(), _nbytes(workspace),
                        _stream_handle(stream))
    _check(st, "rehyat_phi_bwd")
    return g


def hybrid_attn_bwd(q, k, v, y, dy, c, den, Wq, bq, Wk, bk, *, T, Hs, Ws, Tc, To, causal,
                    scale=0.0, force_simt=False, workspace=None, stream=None,
                    state_from_forward=False):
    """Full backward: gradients of L with respect to q, k, v and the phi
    parameters, given the forward's q, k, v, its fp32 output y, dy = dL/dy
    (fp32), and per query the stabiliser c and den = n^S + n^L
    (``parts["c"]`` and ``parts["nS"] + parts["nL"]`` of
    ``hybrid_attn(..., debug=True)``).  ``state_from_forward`` as for
    ``phi_grad`` (the shared workspace from ``bwd_workspace(...)``).
    Returns dict(dq, dk, dv (fp32, shaped like q), dWq, dbq, dWk, dbk (shaped
    like the parameters))."""
    torch = _torch()
    _check_qkv(q, k, v)
    _check_current_device(q.device)
    B, H, N, D = q.shape
    _check_tokens(N, T, Hs, Ws)
    Dp = 2 * Wq.shape[-1]
    for t in (y, dy, c, den):
        if t.dtype != torch.float32 or not t.is_contiguous():
            raise TypeError("y, dy, c and den must be contiguous fp32 tensors")
    _check_out(y, (B, H, N, D), torch.float32, q.device, "y")
    _check_out(dy, (B, H, N, D), torch.float32, q.device, "dy")
    _check_out(c, (B, H, N), torch.float32, q.device, "c")
    _check_out(den, (B, H, N), torch.float32, q.device, "den")
    phi = _phi_struct(Wq, bq, Wk, bk, heads=H, D=D, Dp=Dp, device=q.device)
    _need(not state_from_forward or workspace is not None,
          "state_from_forward needs the forward's workspace")
    p = make_params(batch=B, heads=H, T=T, Hs=Hs, Ws=Ws, D=D, Dp=Dp, Tc=Tc, To=To,
                    causal=causal, in_dtype=_dtype_code(q.dtype), out_dtype=F32, scale=scale,
                    flags=(FLAG_FORCE_SIMT if force_simt else 0) |
                    (FLAG_FWD_STATE if state_from_forward else 0))
    nbytes = rehyat_hybrid_attn_bwd_workspace_bytes(p)
    if nbytes == 0:
        raise RehyatError(1, "rehyat_hybrid_attn_bwd_workspace_bytes")
    if workspace is not None:
        _check_workspace(workspace, q.device)
    if workspace is None:
        workspace = torch.empty(nbytes, dtype=torch.uint8, device=q.device)
    out = {name: torch.empty(B, H, N, D, dtype=torch.float32, device=q.device)
           for name in ("dq", "dk", "dv")}
    out.update({name: torch.empty_like(t, memory_format=torch.contiguous_format) for name, t in
                (("dWq", Wq), ("dbq", bq), ("dWk", Wk), ("dbk", bk))})
    grad = RehyatPhiGrad(*(out[n].data_ptr() for n in ("dWq", "dbq", "dWk", "dbk")))
    st = rehyat_hybrid_attn_bwd(p, q.data_ptr(), k.data_ptr(), v.data_ptr(), phi, y.data_ptr(),
                                dy.data_ptr(), c.data_ptr(), den.data_ptr(), out["dq"].data_ptr(),
                                out["dk"].data_ptr(), out["dv"].data_ptr(), grad,
                                workspace.data_ptr(), _nbytes(workspace), _stream_handle(stream))
    _check(st, "rehyat_hybrid_attn_bwd")
    return out


def softmax_attn(q, k, v, *, out_dtype=None, scale=0.0, force_simt=False, out=None,
                 stream=None):
    """Plain softmax attention over all keys (the dense comparator)."""
    torch = _torch()
    _check_qkv(q, k, v)
    _check_current_device(q.device)
    B, H, N, D = q.shape
    out_dtype = torch.float32 if out_dtype is None else out_dtype
    p = make_params(batch=B, heads=H, T=1, Hs=1, Ws=N, D=D, Dp=32, Tc=1, To=0, causal=0,
                    in_dtype=_dtype_code(q.dtype), out_dtype=_dtype_code(out_dtype),
                    scale=scale, flags=FLAG_FORCE_SIMT if force_simt else 0)
    if out is not None:
        _check_out(out, (B, H, N, D), out_dtype, q.device)
    y = torch.empty(B, H, N, D, dtype=out_dtype, device=q.device) if out is None else out
    st = rehyat_softmax_attn_fwd(p, q.data_ptr(), k.data_ptr(), v.data_ptr(), y.data_ptr(),
                                 _stream_handle(stream))
    _check(st, "rehyat_softmax_attn_fwd")
    return y


class StreamingState:
    """Caller-owned state of the causal chunk-wise RNN (Key design 4).

    ``step(q, k, v)`` consumes the next chunk ([B, h, n*HW, D], n <= Tc
    slices) and returns its outputs; memory stays constant over any number of
    steps.  ``snapshot()``/``restore()`` copy the opaque state bytes."""

    def __init__(self, *, batch, heads, Hs, Ws, D, Dp, Tc, To, Wq, bq, Wk, bk,
                 in_dtype, out_dtype=None, scale=0.0, force_simt=False, device="cuda"):
        torch = _torch()
        self.out_dtype = torch.float32 if out_dtype is None else out_dtype
        self.HW = Hs * Ws
        self.Tc = Tc
        self.p = make_params(batch=batch, heads=heads, T=Tc, Hs=Hs, Ws=Ws, D=D, Dp=Dp, Tc=Tc,
                             To=To, causal=1, in_dtype=_dtype_code(in_dtype),
                             out_dtype=_dtype_code(self.out_dtype), scale=scale,
                             flags=FLAG_FORCE_SIMT if force_simt else 0)
        self.shape = (batch, heads, D)
        self.in_dtype = in_dtype
        self.phi_tensors = (Wq, bq, Wk, bk)
        self.phi = _phi_struct(Wq, bq, Wk, bk, heads=heads, D=D, Dp=Dp)
        nstate = rehyat_state_bytes(self.p)
        nws = rehyat_step_workspace_bytes(self.p)
        if nstate == 0 or nws == 0:
            raise RehyatError(1, "rehyat_state_bytes")
        self.state = torch.empty(nstate, dtype=torch.uint8, device=device)
        self.workspace = torch.empty(nws, dtype=torch.uint8, device=device)
        self.reset()

    def reset(self, stream=None):
        _check_current_device(self.state.device)
        _check(rehyat_state_init(self.p, self.state.data_ptr(), _stream_handle(stream)),
               "rehyat_state_init")

    def step(self, q, k, v, *, debug=False, out=None, stream=None):
        torch = _torch()
        _check_qkv(q, k, v)
        B, H, rows, D = q.shape
        _need((B, H, D) == self.shape, f"a chunk must be shaped [{self.shape[0]}, "
              f"{self.shape[1]}, rows, {self.shape[2]}]")
        _need(q.dtype == self.in_dtype, f"a chunk must be {self.in_dtype}", TypeError)
        _need(q.device == self.state.device, f"a chunk must be on {self.state.device}")
        _check_current_device(q.device)
        n = rows // self.HW
        if n * self.HW != rows:
            raise ValueError("a chunk must hold whole slices")
        if out is not None:
            _check_out(out, (B, H, rows, D), self.out_dtype, q.device)
        y = torch.empty(B, H, rows, D, dtype=self.out_dtype, device=q.device) if out is None else out
        dbg_t, dbg_s = _debug_tensors((B, H, rows, D), q.device) if debug else (None, None)
        st = rehyat_chunk_step(self.p, q.data_ptr(), k.data_ptr(), v.data_ptr(), n, self.phi,
                               self.state.data_ptr(), y.data_ptr(), self.workspace.data_ptr(),
                               self.workspace.numel(), dbg_s, _stream_handle(stream))
        _check(st, "rehyat_chunk_step")
        return (y, dbg_t) if debug else y

    def snapshot(self):
        return self.state.clone()

    def restore(self, saved):
        self.state.copy_(saved)

    def capture_steps(self, chunks, out):
        """Record consecutive steps, one per (q, k, v) chunk of ``chunks``, as
        one CUDA graph: each step reads its own chunk tensors and writes
        ``out``.  Replaying it runs the whole sequence from the state's
        current slice count with one launch of the graph.  The state is left
        as it was before the call."""
        torch = _torch()
        saved = self.snapshot()
        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):  # warm-up launch outside the capture
            self.step(*chunks[0], out=out)
        torch.cuda.current_stream().wait_stream(side)
        self.restore(saved)
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            for c in chunks:
                self.step(*c, out=out)
        torch.cuda.synchronize()
        self.restore(saved)
        return graph

    def capture_step(self, q, k, v, out):
        """Record one step on fixed buffers q, k, v, out as a CUDA graph.

        The slice counter lives in the state on the device, so the same graph
        advances the recurrence each time it is replayed: copy the next chunk
        into q, k, v, then ``graph.replay()``; the outputs land in ``out``.
        The state is left as it was before the call."""
        torch = _torch()
        saved = self.snapshot()
        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):  # warm-up launch outside the capture
            self.step(q, k, v, out=out)
        torch.cuda.current_stream().wait_stream(side)
        self.restore(saved)
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            self.step(q, k, v, out=out)
        torch.cuda.synchronize()
        self.restore(saved)
        return graph
