"""GPU parity of the full backward (rehyat_hybrid_attn_bwd, through the C ABI)
against the fp64 backward oracle (oracle/rehyat_grad.py) on the same seeded
inputs: dq, dk, dv and the feature-map parameter gradients.

The GPU backward takes the forward's y, c and den from the GPU forward (as a
caller would).  Bars, per gradient tensor, as the error relative to the
tensor's largest magnitude:
* fp32 CUDA-core forward (force_simt): max <= 1e-4 -- only fp32 rounding
  separates the two sides;
* default tensor-core forward, bf16 inputs: max <= 3e-2 -- the forward rounds
  P and phi_k to bf16 (relative 2^-9 per element) and reads the linear branch
  out in tf32, which reaches y, c and den that the backward is built from.

The maximum's term sends -scale Dc_i q_i to the arg-max key of row i and
-scale Dc_i k_{j*} to dq_i.  Where two window logits tie to within fp32
rounding (a relative 2^-16 here), the kernel's fp32 arg-max and the
oracle's fp64 one may pick different keys, both valid gradients at the
kink: such rows of dq and the keys involved in dk are left out of the
element comparison (the tests also check that they are rare), and dv, which
the term does not touch, is compared everywhere.
"""
import numpy as np
import pytest
import torch

import linear_attention_video_chunked_b200 as rh
from oracle.rehyat_grad import hybrid_grads
from oracle.rehyat_oracle import chunk_table
from rehyat_inputs import config_problem, make_problem
from tests.gpu_util import device_tensors

pytestmark = pytest.mark.gpu

TOKEN = ("dq", "dk", "dv")
PARAM = ("dWq", "dbq", "dWk", "dbk")


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    rh.lib()
    yield


def _gpu(p, dy, force_simt, dev=None):
    dev = device_tensors(p) if dev is None else dev
    kw = dict(T=p.T, Hs=p.Hs, Ws=p.Ws, Tc=p.Tc, To=p.To, causal=p.causal)
    y, parts = rh.hybrid_attn(dev["q"], dev["k"], dev["v"], dev["Wq"], dev["bq"], dev["Wk"],
                              dev["bk"], debug=True, force_simt=force_simt, **kw)
    den = (parts["nS"] + parts["nL"]).contiguous()
    dyt = torch.tensor(dy, dtype=torch.float32, device="cuda")
    g = rh.hybrid_attn_bwd(dev["q"], dev["k"], dev["v"], y, dyt, parts["c"].contiguous(), den,
                           dev["Wq"], dev["bq"], dev["Wk"], dev["bk"], force_simt=force_simt,
                           **kw)
    torch.cuda.synchronize()
    return {n: g[n].double().cpu().numpy() for n in TOKEN + PARAM}


def _ref(p, dy, heads=None):
    if heads is None:
        return hybrid_grads(p.q, p.k, p.v, p.Wq, p.bq, p.Wk, p.bk, dy, T=p.T, HW=p.HW,
                            Tc=p.Tc, To=p.To, causal=p.causal)
    sel = lambda a: np.asarray(a)[:, heads]
    return hybrid_grads(sel(p.q), sel(p.k), sel(p.v), np.asarray(p.Wq)[heads],
                        np.asarray(p.bq)[heads], np.asarray(p.Wk)[heads],
                        np.asarray(p.bk)[heads], np.asarray(dy)[:, heads], T=p.T, HW=p.HW,
                        Tc=p.Tc, To=p.To, causal=p.causal)


def _tie_masks(p, heads):
    """Rows whose window maximum is not unique within 2^-16 (relative), and
    the keys that could be taken as their maximum: masks [B, h, N]."""
    q = np.asarray(p.q, np.float64)[:, heads]
    k = np.asarray(p.k, np.float64)[:, heads]
    B, H, N, D = q.shape
    scale = 1.0 / np.sqrt(D)
    rows = np.zeros((B, H, N), bool)
    keys = np.zeros((B, H, N), bool)
    for b in range(B):
        for h in range(H):
            for first, end, start in chunk_table(p.T, p.Tc, p.To):
                lg = q[b, h, first * p.HW:end * p.HW] @ k[b, h, start * p.HW:end * p.HW].T * scale
                c = lg.max(axis=1)
                near = lg >= (c - 2.0 ** -16 * np.maximum(1.0, np.abs(c)))[:, None]
                amb = near.sum(axis=1) > 1
                rows[b, h, first * p.HW:end * p.HW] |= amb
                if amb.any():
                    keys[b, h, start * p.HW:end * p.HW] |= near[amb].any(axis=0)
    return rows, keys


def _check(got, ref, tol, p, heads=None):
    hs = list(range(p.heads)) if heads is None else heads
    rows, keys = _tie_masks(p, hs)
    assert rows.mean() < 1e-3, f"{rows.sum()} rows with a tied maximum"
    for n in TOKEN + PARAM:
        g = got[n] if heads is None else (got[n][:, heads] if n in TOKEN else got[n][heads])
        r = ref[n]
        scale = np.abs(r).max()
        d = np.abs(g - r)
        if n == "dq":
            d = d[~rows]
        elif n == "dk":
            d = d[~keys]
        err = d.max()
        assert np.all(np.isfinite(g)), f"{n}: non-finite values"
        assert err <= tol * max(scale, 1e-30), f"{n}: max err {err:.3e} vs max |ref| {scale:.3e}"


SHAPES = [
    # B, h, T, Hs, Ws, D, Dp, Tc, To, causal
    (2, 2, 5, 7, 9, 128, 128, 2, 1, False),   # ragged tiles, batch sum
    (1, 2, 7, 10, 13, 128, 128, 3, 2, True),
    (1, 3, 6, 8, 12, 64, 256, 2, 0, False),   # two feature pieces
    (1, 2, 9, 11, 12, 32, 64, 3, 4, True),    # T_o > T_c
    (1, 1, 3, 5, 5, 32, 32, 4, 1, False),     # T_c >= T: no linear set
]


@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: "x".join(map(str, s)))
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_full_bwd_simt_forward_tight(shape, dtype):
    B, h, T, Hs, Ws, D, Dp, Tc, To, causal = shape
    p = make_problem(batch=B, heads=h, T=T, Hs=Hs, Ws=Ws, D=D, Dp=Dp, Tc=Tc, To=To,
                     causal=causal, dtype=dtype, seed=400 + sum(shape[:9]), phi_std=0.1)
    dy = np.random.default_rng(17).standard_normal(np.shape(p.q))
    _check(_gpu(p, dy, force_simt=True), _ref(p, dy), 1e-4, p)


@pytest.mark.parametrize("shape", SHAPES[:2], ids=lambda s: "x".join(map(str, s)))
def test_full_bwd_balanced_branches(shape):
    # phi std 0.01 makes n^L comparable with n^S, so the softmax branch and
    # the maximum's term carry a large share of every gradient.
    B, h, T, Hs, Ws, D, Dp, Tc, To, causal = shape
    p = make_problem(batch=B, heads=h, T=T, Hs=Hs, Ws=Ws, D=D, Dp=Dp, Tc=Tc, To=To,
                     causal=causal, dtype="f32", seed=500 + sum(shape[:9]), phi_std=0.01)
    dy = np.random.default_rng(18).standard_normal(np.shape(p.q))
    _check(_gpu(p, dy, force_simt=True), _ref(p, dy), 1e-4, p)


@pytest.mark.parametrize("shape", SHAPES[:3], ids=lambda s: "x".join(map(str, s)))
def test_full_bwd_tensor_core_forward(shape):
    B, h, T, Hs, Ws, D, Dp, Tc, To, causal = shape
    p = make_problem(batch=B, heads=h, T=T, Hs=Hs, Ws=Ws, D=D, Dp=Dp, Tc=Tc, To=To,
                     causal=causal, dtype="bf16", seed=600 + sum(shape[:9]), phi_std=0.1)
    dy = np.random.default_rng(19).standard_normal(np.shape(p.q))
    _check(_gpu(p, dy, force_simt=False), _ref(p, dy), 3e-2, p)


def test_full_bwd_repeatable_bitwise():
    p = make_problem(batch=1, heads=2, T=6, Hs=8, Ws=9, D=128, Dp=128, Tc=2, To=1, causal=True,
                     dtype="bf16", seed=20)
    dy = np.random.default_rng(20).standard_normal(np.shape(p.q))
    dev = device_tensors(p)
    a = _gpu(p, dy, force_simt=False, dev=dev)
    b = _gpu(p, dy, force_simt=False, dev=dev)
    for n in TOKEN + PARAM:
        assert np.array_equal(a[n], b[n]), n


def test_full_bwd_wan_320x480_causal_sampled_heads():
    """Latent 21x20x30, 12 heads, D = D' = 128, T_c = 3, T_o = 1, causal:
    three sampled heads against the oracle (fp32 forward)."""
    p = config_problem("wan_320x480_causal")
    dy = np.random.default_rng(21).standard_normal(np.shape(p.q)).astype(np.float32)
    heads = [0, 5, 11]
    _check(_gpu(p, dy, force_simt=True), _ref(p, dy, heads), 1e-4, p, heads)


def test_full_bwd_bench_layer_sampled_heads():
    """The bench layer (21x30x52, batch 2, 12 heads, bidirectional), bf16
    through the tensor-core forward: two sampled heads against the oracle."""
    p = config_problem("wan_480x832_bidir")
    dy = np.random.default_rng(22).standard_normal(np.shape(p.q)).astype(np.float32)
    heads = [2, 7]
    _check(_gpu(p, dy, force_simt=False), _ref(p, dy, heads), 3e-2, p, heads)


@pytest.mark.parametrize("force_simt", [False, True], ids=["tc", "simt"])
def test_full_bwd_with_the_forwards_state_is_bitwise_equal(force_simt):
    """REHYAT_FLAG_FWD_STATE: the full backward on the forward's workspace
    equals the one that recomputes the linear-set state, bit for bit."""
    p = make_problem(batch=1, heads=2, T=7, Hs=10, Ws=13, D=128, Dp=128, Tc=3, To=2,
                     causal=True, dtype="bf16", seed=23)
    dy = np.random.default_rng(23).standard_normal(np.shape(p.q))
    dev = device_tensors(p)
    kw = dict(T=p.T, Hs=p.Hs, Ws=p.Ws, Tc=p.Tc, To=p.To, causal=p.causal)
    prm = [dev[n] for n in ("Wq", "bq", "Wk", "bk")]
    ws = rh.bwd_workspace(dev["q"], dev["Wq"], force_simt=force_simt, **kw)
    y, parts = rh.hybrid_attn(dev["q"], dev["k"], dev["v"], *prm, debug=True,
                              force_simt=force_simt, workspace=ws, **kw)
    den = (parts["nS"] + parts["nL"]).contiguous()
    dyt = torch.tensor(dy, dtype=torch.float32, device="cuda")
    args = (dev["q"], dev["k"], dev["v"], y, dyt, parts["c"].contiguous(), den, *prm)
    a = rh.hybrid_attn_bwd(*args, force_simt=force_simt, **kw)
    b = rh.hybrid_attn_bwd(*args, force_simt=force_simt, workspace=ws, state_from_forward=True,
                           **kw)
    torch.cuda.synchronize()
    for n in TOKEN + PARAM:
        assert torch.equal(a[n], b[n]), n
    assert rh.rehyat_device_error_flags() == 0
