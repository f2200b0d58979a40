"""Host-side checks of the torch layer of the binding (no GPU needed).

The C ABI takes bare device pointers and sizes, so the torch layer must
refuse any tensor whose shape, dtype, strides or device disagree with the
sizes it passes: otherwise the kernels would read or write outside the
buffers.  These tests run the wrappers on stand-in tensors that report a
CUDA device, with the library's launching entry points replaced by
recorders (its size queries are the real, host-only ones):

* the call patterns the GPU tests, the bench and smoke() use reach the C ABI
  with the tensors' own pointers and byte counts;
* each malformed call raises before anything reaches the C ABI;
* with the library missing, the binding raises instead of computing.
"""
import math
import os
import subprocess
import sys
import types

import pytest
import torch

import linear_attention_video_chunked_b200 as rh

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


class FakeTensor:
    """Shape, dtype, device and strides of a tensor, with a distinct
    256-byte-aligned address; holds no data."""

    _next_ptr = 1 << 32

    def __init__(self, shape, dtype, device="cuda:0", contiguous=True):
        self.shape = torch.Size(shape)
        self.dtype = dtype
        dev = torch.device(device)
        if dev.type == "cuda" and dev.index is None:  # torch places it on the current device
            dev = torch.device("cuda", 0)
        self.device = dev
        self._contiguous = contiguous
        self._ptr = FakeTensor._next_ptr
        FakeTensor._next_ptr += 1 << 32

    @property
    def is_cuda(self):
        return self.device.type == "cuda"

    def is_contiguous(self):
        return self._contiguous

    def dim(self):
        return len(self.shape)

    def numel(self):
        return math.prod(self.shape)

    def element_size(self):
        return torch.empty((), dtype=self.dtype).element_size()

    def data_ptr(self):
        return self._ptr


def _shim():
    """The parts of torch the wrappers use, allocating FakeTensors."""
    def empty(*shape, dtype=torch.float32, device="cpu", pin_memory=False):
        if len(shape) == 1 and isinstance(shape[0], (tuple, list, torch.Size)):
            shape = shape[0]
        return FakeTensor(shape, dtype, device)

    stream = types.SimpleNamespace(cuda_stream=0, synchronize=lambda: None)
    return types.SimpleNamespace(
        float32=torch.float32, bfloat16=torch.bfloat16, uint8=torch.uint8,
        contiguous_format=torch.contiguous_format, empty=empty,
        empty_like=lambda t, memory_format=None: FakeTensor(t.shape, t.dtype, t.device),
        cuda=types.SimpleNamespace(current_stream=lambda: stream, current_device=lambda: 0))


LAUNCHERS = ("rehyat_hybrid_attn_fwd", "rehyat_hybrid_attn_fwd_host", "rehyat_feature_map_mlp",
             "rehyat_hybrid_attn_fwd_phi", "rehyat_phi_bwd", "rehyat_softmax_attn_fwd",
             "rehyat_state_init", "rehyat_chunk_step", "rehyat_hybrid_attn_bwd")


@pytest.fixture
def calls(monkeypatch):
    """Route the wrappers to the shim; record every launching C call."""
    rh.lib()  # the real library answers the size queries
    log = []
    monkeypatch.setattr(rh, "_torch", _shim)
    for name in LAUNCHERS:
        monkeypatch.setattr(rh, name, lambda *a, _n=name: log.append((_n, a)) or 0)
    monkeypatch.setattr(rh, "rehyat_feature_map_mlp_workspace_bytes", lambda *a: 1 << 20)
    return log


BF, F32 = torch.bfloat16, torch.float32


def qkv(shape=(2, 3, 5 * 7 * 9, 128), dtype=BF, device="cuda:0"):
    return [FakeTensor(shape, dtype, device) for _ in range(3)]


def phi_params(H=3, D=128, Dp=128, device="cuda:0"):
    W = lambda: FakeTensor((H, 2, D, Dp // 2), F32, device)
    b = lambda: FakeTensor((H, 2, Dp // 2), F32, device)
    return [W(), b(), W(), b()]


GEOM = dict(T=5, Hs=7, Ws=9, Tc=2, To=1, causal=False)


# ------------------------------------------------------ accepted patterns
@pytest.mark.parametrize("dtype", [BF, F32])
@pytest.mark.parametrize("extra", [{}, dict(debug=True), dict(fp8_qk=True), dict(force_simt=True),
                                   dict(out_dtype=BF)])
def test_hybrid_attn_reaches_the_abi(calls, dtype, extra):
    if extra.get("fp8_qk") and dtype != BF:
        pytest.skip("fp8 is a bf16 variant")
    q, k, v = qkv(dtype=dtype)
    res = rh.hybrid_attn(q, k, v, *phi_params(), **GEOM, **extra)
    y = res[0] if extra.get("debug") else res
    (name, a), = calls
    assert name == "rehyat_hybrid_attn_fwd"
    assert a[1:4] == (q.data_ptr(), k.data_ptr(), v.data_ptr())
    assert a[5] == y.data_ptr() and tuple(y.shape) == tuple(q.shape)
    assert y.dtype == extra.get("out_dtype", F32)
    assert a[7] >= rh.rehyat_workspace_bytes(a[0])  # bytes of the workspace passed


def test_hybrid_attn_with_caller_out_and_workspace(calls):
    q, k, v = qkv()
    out = FakeTensor(q.shape, F32)
    ws = FakeTensor((64 << 20,), torch.uint8)
    assert rh.hybrid_attn(q, k, v, *phi_params(), **GEOM, out=out, workspace=ws) is out
    (_, a), = calls
    assert a[5] == out.data_ptr() and a[6] == ws.data_ptr() and a[7] == 64 << 20


def test_workspace_size_counts_bytes_not_elements(calls):
    q, k, v = qkv()
    need = rh.rehyat_workspace_bytes(rh.make_params(batch=2, heads=3, T=5, Hs=7, Ws=9, D=128,
                                                    Dp=128, Tc=2, To=1, causal=0))
    ws = FakeTensor(((need + 3) // 4,), F32)  # an fp32 tensor of enough bytes is used as is
    rh.hybrid_attn(q, k, v, *phi_params(), **GEOM, workspace=ws)
    (_, a), = calls
    assert a[6] == ws.data_ptr() and a[7] == 4 * ((need + 3) // 4)


def test_host_forward_reaches_the_abi(calls):
    q, k, v = qkv(device="cpu")
    y = rh.hybrid_attn_host(q, k, v, *phi_params(), **GEOM, heads_per_slab=2)
    (name, a), = calls
    assert name == "rehyat_hybrid_attn_fwd_host"
    assert a[1:4] == (q.data_ptr(), k.data_ptr(), v.data_ptr()) and a[5] == y.data_ptr()
    assert y.device.type == "cpu" and a[6] == 2


def test_phi_given_feature_map_and_gradient_reach_the_abi(calls):
    q, k, v = qkv()
    mlp = [FakeTensor(s, F32) for s in ((3, 128, 384), (3, 384), (3, 384, 128), (3, 128))]
    pq = rh.feature_map_mlp(q, *mlp, parts=2, T=5, Hs=7, Ws=9)
    pk = rh.feature_map_mlp(k, *mlp, parts=2, T=5, Hs=7, Ws=9)
    y, parts = rh.hybrid_attn_phi(q, k, v, pq, pk, **GEOM, debug=True)
    den = FakeTensor(q.shape[:3], F32)
    dy = FakeTensor(q.shape, F32)
    g = rh.phi_grad(q, k, v, y, dy, den, *phi_params(), **GEOM)
    assert [c[0] for c in calls] == ["rehyat_feature_map_mlp"] * 2 + [
        "rehyat_hybrid_attn_fwd_phi", "rehyat_phi_bwd"]
    assert tuple(pq.shape) == (2, 3, 315, 128) and set(g) == {"dWq", "dbq", "dWk", "dbk"}


def test_full_backward_reaches_the_abi(calls):
    q, k, v = qkv()
    y, dy = FakeTensor(q.shape, F32), FakeTensor(q.shape, F32)
    c, den = FakeTensor(q.shape[:3], F32), FakeTensor(q.shape[:3], F32)
    g = rh.hybrid_attn_bwd(q, k, v, y, dy, c, den, *phi_params(), **GEOM)
    (name, a), = calls
    assert name == "rehyat_hybrid_attn_bwd"
    assert a[1:4] == (q.data_ptr(), k.data_ptr(), v.data_ptr())
    assert a[5:9] == (y.data_ptr(), dy.data_ptr(), c.data_ptr(), den.data_ptr())
    assert a[9:12] == (g["dq"].data_ptr(), g["dk"].data_ptr(), g["dv"].data_ptr())
    assert all(tuple(g[n].shape) == tuple(q.shape) and g[n].dtype == F32 for n in ("dq", "dk", "dv"))
    assert a[14] >= rh.rehyat_hybrid_attn_bwd_workspace_bytes(a[0])


@pytest.mark.parametrize("bad", ["c_shape", "den_dtype", "dy_shape", "y_bf16"])
def test_full_backward_refuses_malformed_tensors(calls, bad):
    q, k, v = qkv()
    t = dict(y=FakeTensor(q.shape, F32), dy=FakeTensor(q.shape, F32),
             c=FakeTensor(q.shape[:3], F32), den=FakeTensor(q.shape[:3], F32))
    if bad == "c_shape":
        t["c"] = FakeTensor((2, 3, 314), F32)
    elif bad == "den_dtype":
        t["den"] = FakeTensor(q.shape[:3], BF)
    elif bad == "dy_shape":
        t["dy"] = FakeTensor((2, 3, 315, 64), F32)
    else:
        t["y"] = FakeTensor(q.shape, BF)
    with pytest.raises((ValueError, TypeError)):
        rh.hybrid_attn_bwd(q, k, v, t["y"], t["dy"], t["c"], t["den"], *phi_params(), **GEOM)
    assert calls == []


def test_backward_with_the_forwards_state_shares_one_workspace(calls):
    # forward, then both backward entry points on the same buffer, the
    # backward calls with REHYAT_FLAG_FWD_STATE; the buffer holds both layouts.
    q, k, v = qkv()
    prm = phi_params()
    ws = rh.bwd_workspace(q, prm[0], **GEOM)
    y, parts = rh.hybrid_attn(q, k, v, *prm, **GEOM, debug=True, workspace=ws)
    dy, den = FakeTensor(q.shape, F32), FakeTensor(q.shape[:3], F32)
    rh.phi_grad(q, k, v, y, dy, den, *prm, **GEOM, workspace=ws, state_from_forward=True)
    rh.hybrid_attn_bwd(q, k, v, y, dy, den, den, *prm, **GEOM, workspace=ws,
                       state_from_forward=True)
    (f, af), (g, ag), (b, ab) = calls
    assert (f, g, b) == ("rehyat_hybrid_attn_fwd", "rehyat_phi_bwd", "rehyat_hybrid_attn_bwd")
    assert af[6] == ag[9] == ab[13] == ws.data_ptr()
    assert af[7] == ag[10] == ab[14] == ws.numel()
    assert not af[0].flags & rh.FLAG_FWD_STATE
    assert ag[0].flags & rh.FLAG_FWD_STATE and ab[0].flags & rh.FLAG_FWD_STATE
    assert ws.numel() >= max(rh.rehyat_workspace_bytes(af[0]),
                             rh.rehyat_hybrid_attn_bwd_workspace_bytes(ab[0]),
                             rh.rehyat_phi_bwd_workspace_bytes(ag[0]))


def test_softmax_and_streaming_reach_the_abi(calls):
    q, k, v = qkv(shape=(1, 2, 3 * 10 * 30, 128))
    rh.softmax_attn(q, k, v)
    st = rh.StreamingState(batch=1, heads=2, Hs=6, Ws=11, D=128, Dp=128, Tc=2, To=1,
                           **dict(zip(("Wq", "bq", "Wk", "bk"), phi_params(H=2))),
                           in_dtype=BF)
    out = FakeTensor((1, 2, 2 * 66, 128), F32)
    st.step(*qkv(shape=(1, 2, 2 * 66, 128)), out=out)   # a full chunk
    st.step(*qkv(shape=(1, 2, 66, 128)))                # a last chunk of one slice
    names = [c[0] for c in calls]
    assert names == ["rehyat_softmax_attn_fwd", "rehyat_state_init", "rehyat_chunk_step",
                     "rehyat_chunk_step"]
    assert calls[2][1][4] == 2 and calls[3][1][4] == 1  # slices per step


# ------------------------------------------------------ refused patterns
def _bad_hybrid(**change):
    q, k, v = qkv()
    W = phi_params()
    args = dict(q=q, k=k, v=v, Wq=W[0], bq=W[1], Wk=W[2], bk=W[3])
    args.update(change)
    kw = dict(GEOM)
    kw.update(change.pop("geom", {}))
    args.pop("geom", None)
    return args, kw


BAD_FORWARD = [
    ("cpu q", dict(q=FakeTensor((2, 3, 315, 128), BF, "cpu")), ValueError),
    ("k on another GPU", dict(k=FakeTensor((2, 3, 315, 128), BF, "cuda:1")), ValueError),
    ("short v", dict(v=FakeTensor((2, 3, 314, 128), BF)), ValueError),
    ("fp32 k with bf16 q", dict(k=FakeTensor((2, 3, 315, 128), F32)), TypeError),
    ("strided q", dict(q=FakeTensor((2, 3, 315, 128), BF, contiguous=False)), ValueError),
    ("3-d q", dict(q=FakeTensor((6, 315, 128), BF)), ValueError),
    ("fp16 q", dict(q=FakeTensor((2, 3, 315, 128), torch.float16),
                    k=FakeTensor((2, 3, 315, 128), torch.float16),
                    v=FakeTensor((2, 3, 315, 128), torch.float16)), TypeError),
    ("N != T*Hs*Ws", dict(geom=dict(T=4)), ValueError),
    ("Wq of two heads", dict(Wq=FakeTensor((2, 2, 128, 64), F32)), ValueError),
    ("bk of the wrong width", dict(bk=FakeTensor((3, 2, 32), F32)), ValueError),
    ("bf16 Wk", dict(Wk=FakeTensor((3, 2, 128, 64), BF)), TypeError),
    ("host bq", dict(bq=FakeTensor((3, 2, 64), F32, "cpu")), TypeError),
    ("Wq on another GPU", dict(Wq=FakeTensor((3, 2, 128, 64), F32, "cuda:1")), ValueError),
]


@pytest.mark.parametrize("what,change,exc", BAD_FORWARD, ids=[b[0] for b in BAD_FORWARD])
def test_hybrid_attn_refuses_before_launch(calls, what, change, exc):
    args, kw = _bad_hybrid(**change)
    with pytest.raises(exc):
        rh.hybrid_attn(args["q"], args["k"], args["v"], args["Wq"], args["bq"], args["Wk"],
                       args["bk"], **kw)
    assert calls == []


@pytest.mark.parametrize("out", [
    FakeTensor((2, 3, 315, 64), F32),               # wrong shape
    FakeTensor((2, 3, 315, 128), BF),               # not the requested out_dtype
    FakeTensor((2, 3, 315, 128), F32, contiguous=False),
    FakeTensor((2, 3, 315, 128), F32, "cuda:1"),
    FakeTensor((2, 3, 315, 128), F32, "cpu"),
])
def test_hybrid_attn_refuses_bad_out(calls, out):
    with pytest.raises((ValueError, TypeError)):
        rh.hybrid_attn(*qkv(), *phi_params(), **GEOM, out=out)
    assert calls == []


def test_tensors_off_the_current_device_are_refused(calls):
    """Everything on cuda:1 while cuda:0 is current: the library would launch
    on cuda:0 with cuda:1's pointers."""
    q, k, v = qkv(device="cuda:1")
    W = phi_params(device="cuda:1")
    with pytest.raises(ValueError, match="current CUDA device"):
        rh.hybrid_attn(q, k, v, *W, **GEOM)
    with pytest.raises(ValueError, match="current CUDA device"):
        rh.softmax_attn(q, k, v)
    mlp = [FakeTensor(s, F32, "cuda:1") for s in ((3, 128, 384), (3, 384), (3, 384, 128),
                                                  (3, 128))]
    with pytest.raises(ValueError, match="current CUDA device"):
        rh.feature_map_mlp(q, *mlp, parts=2, T=5, Hs=7, Ws=9)
    with pytest.raises(ValueError, match="current CUDA device"):
        rh.hybrid_attn_host(*qkv(device="cpu"), *W, **GEOM)
    with pytest.raises(ValueError, match="current CUDA device"):
        rh.StreamingState(batch=1, heads=3, Hs=7, Ws=9, D=128, Dp=128, Tc=2, To=1,
                          **dict(zip(("Wq", "bq", "Wk", "bk"), W)), in_dtype=BF,
                          device="cuda:1")
    assert calls == []


def test_hybrid_attn_refuses_workspace_elsewhere(calls):
    for ws in (FakeTensor((64 << 20,), torch.uint8, "cpu"),
               FakeTensor((64 << 20,), torch.uint8, contiguous=False)):
        with pytest.raises(ValueError):
            rh.hybrid_attn(*qkv(), *phi_params(), **GEOM, workspace=ws)
    assert calls == []


def test_host_forward_refusals(calls):
    host = qkv(device="cpu")
    with pytest.raises(ValueError):        # device tensors given to the host-buffer entry
        rh.hybrid_attn_host(*qkv(), *phi_params(), **GEOM)
    with pytest.raises(ValueError):        # a short host k
        rh.hybrid_attn_host(host[0], FakeTensor((2, 3, 300, 128), BF, "cpu"), host[2],
                            *phi_params(), **GEOM)
    with pytest.raises(ValueError):
        rh.hybrid_attn_host(*host, *phi_params(), **dict(GEOM, Hs=8))
    with pytest.raises(TypeError):         # phi parameters must live on the GPU
        rh.hybrid_attn_host(*host, *phi_params(device="cpu"), **GEOM)
    with pytest.raises(TypeError):         # y is fp32
        rh.hybrid_attn_host(*host, *phi_params(), **GEOM,
                            out=FakeTensor((2, 3, 315, 128), BF, "cpu"))
    with pytest.raises(ValueError):        # y is host memory
        rh.hybrid_attn_host(*host, *phi_params(), **GEOM,
                            out=FakeTensor((2, 3, 315, 128), F32))
    assert calls == []


def test_feature_map_and_phi_given_refusals(calls):
    q, k, v = qkv()
    mlp = [FakeTensor(s, F32) for s in ((3, 128, 384), (3, 384), (3, 384, 128), (3, 128))]
    with pytest.raises(ValueError):        # ba sized for another hidden width
        rh.feature_map_mlp(q, mlp[0], FakeTensor((3, 256), F32), mlp[2], mlp[3], parts=2,
                           T=5, Hs=7, Ws=9)
    with pytest.raises(ValueError):
        rh.feature_map_mlp(FakeTensor(q.shape, BF, contiguous=False), *mlp, parts=2, T=5,
                           Hs=7, Ws=9)
    with pytest.raises(ValueError):
        rh.feature_map_mlp(q, *mlp, parts=2, T=5, Hs=7, Ws=9,
                           out=FakeTensor((2, 3, 315, 64), F32))
    pq = FakeTensor((2, 3, 315, 128), F32)
    with pytest.raises(TypeError):         # phi_k of another width than phi_q
        rh.hybrid_attn_phi(q, k, v, pq, FakeTensor((2, 3, 315, 64), F32), **GEOM)
    with pytest.raises(TypeError):         # phi_q of fewer tokens
        rh.hybrid_attn_phi(q, k, v, FakeTensor((2, 3, 300, 128), F32), pq, **GEOM)
    with pytest.raises(ValueError):
        rh.hybrid_attn_phi(q, k, v, pq, FakeTensor((2, 3, 315, 128), F32, "cuda:1"), **GEOM)
    with pytest.raises(TypeError):         # one map bf16, the other fp32
        rh.hybrid_attn_phi(q, k, v, pq, FakeTensor((2, 3, 315, 128), BF), **GEOM)
    with pytest.raises(TypeError):         # an fp16 map
        rh.feature_map_mlp(q, *mlp, parts=2, T=5, Hs=7, Ws=9, out_dtype=torch.float16)
    assert calls == []


def test_bf16_feature_maps_reach_the_abi_with_the_flag(calls):
    q, k, v = qkv()
    mlp = [FakeTensor(s, F32) for s in ((3, 128, 384), (3, 384), (3, 384, 128), (3, 128))]
    pq = rh.feature_map_mlp(q, *mlp, parts=2, T=5, Hs=7, Ws=9, out_dtype=BF)
    pk = rh.feature_map_mlp(k, *mlp, parts=2, T=5, Hs=7, Ws=9, out_dtype=BF)
    rh.hybrid_attn_phi(q, k, v, pq, pk, **GEOM)
    assert [c[0] for c in calls] == ["rehyat_feature_map_mlp"] * 2 + ["rehyat_hybrid_attn_fwd_phi"]
    assert pq.dtype == BF and all(c[1][0].flags & rh.FLAG_PHI_BF16 for c in calls)


def test_gradient_refusals(calls):
    q, k, v = qkv()
    y = FakeTensor(q.shape, F32)
    den = FakeTensor(q.shape[:3], F32)
    with pytest.raises(ValueError):        # den per query, not per element
        rh.phi_grad(q, k, v, y, FakeTensor(q.shape, F32), FakeTensor(q.shape, F32),
                    *phi_params(), **GEOM)
    with pytest.raises(ValueError):        # dy of fewer tokens
        rh.phi_grad(q, k, v, y, FakeTensor((2, 3, 300, 128), F32), den, *phi_params(), **GEOM)
    with pytest.raises(TypeError):
        rh.phi_grad(q, k, v, FakeTensor(q.shape, BF), FakeTensor(q.shape, F32), den,
                    *phi_params(), **GEOM)
    with pytest.raises(ValueError):        # the forward's state lives in its workspace
        rh.phi_grad(q, k, v, y, FakeTensor(q.shape, F32), den, *phi_params(), **GEOM,
                    state_from_forward=True)
    with pytest.raises(ValueError):
        rh.hybrid_attn_bwd(q, k, v, y, FakeTensor(q.shape, F32), den, den, *phi_params(),
                           **GEOM, state_from_forward=True)
    assert calls == []


def test_streaming_refusals(calls):
    W = dict(zip(("Wq", "bq", "Wk", "bk"), phi_params(H=2)))
    with pytest.raises(ValueError):        # phi parameters of three heads for a two-head state
        rh.StreamingState(batch=1, heads=2, Hs=6, Ws=11, D=128, Dp=128, Tc=2, To=1,
                          **dict(zip(("Wq", "bq", "Wk", "bk"), phi_params(H=3))), in_dtype=BF)
    st = rh.StreamingState(batch=1, heads=2, Hs=6, Ws=11, D=128, Dp=128, Tc=2, To=1, **W,
                           in_dtype=BF)
    del calls[:]
    bad = [
        (qkv(shape=(1, 3, 132, 128)), {}, ValueError),          # another head count
        (qkv(shape=(1, 2, 132, 64)), {}, ValueError),           # another head dimension
        (qkv(shape=(1, 2, 130, 128)), {}, ValueError),          # not whole slices
        (qkv(shape=(1, 2, 132, 128), dtype=F32), {}, TypeError),
        (qkv(shape=(1, 2, 132, 128), device="cuda:1"), {}, ValueError),
        (qkv(shape=(1, 2, 132, 128)), dict(out=FakeTensor((1, 2, 66, 128), F32)), ValueError),
    ]
    for chunk, kw, exc in bad:
        with pytest.raises(exc):
            st.step(*chunk, **kw)
    assert calls == []


# ------------------------------------------------------ no fallback
def test_missing_library_raises_instead_of_computing(tmp_path):
    code = (
        "import linear_attention_video_chunked_b200 as rh\n"
        "try:\n"
        "    rh.rehyat_workspace_bytes(rh.make_params(batch=1, heads=1, T=1, Hs=1, Ws=1, D=32,"
        " Dp=32, Tc=1, To=0, causal=0))\n"
        "except ImportError as e:\n"
        "    print('refused:', e)\n"
        "else:\n"
        "    print('computed')\n")
    env = dict(os.environ, REHYAT_LIBRARY=str(tmp_path / "librehyat.so"))
    res = subprocess.run([sys.executable, "-c", code], cwd=ROOT, env=env, capture_output=True,
                         text=True, timeout=120)
    assert res.returncode == 0, res.stderr
    assert res.stdout.startswith("refused:") and "librehyat.so is missing" in res.stdout
