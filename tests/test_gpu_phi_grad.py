"""GPU parity of the feature-map backward (rehyat_phi_bwd, through the C ABI)
against the fp64 gradient oracle on the same seeded inputs.

Bar (per gradient tensor, error relative to its largest magnitude):
* fp32 CUDA-core forward and state pass (force_simt): <= 1e-4 -- only fp32
  rounding separates the two;
* default tensor-core path, bf16 inputs: <= 3e-2 -- the forward rounds P and
  phi_k to bf16 (relative 2^-9 per element), which reaches y, the
  denominators and S_L that the gradient is built from; with D = D' = 128
  the backward's q and k passes run on tcgen05 too, with E = g / den, S_L,
  Ghat, phi and du entering the products as bf16 (the same 2^-9 per element,
  averaged over the sums over rows).
"""
import numpy as np
import pytest
import torch

import linear_attention_video_chunked_b200 as rh
from oracle.rehyat_phi_grad import phi_grads
from rehyat_inputs import config_problem, make_problem
from tests.gpu_util import device_tensors

pytestmark = pytest.mark.gpu

NAMES = ("dWq", "dbq", "dWk", "dbk")


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    rh.lib()
    yield


def _gpu_grads(p, dy, force_simt, dev=None):
    dev = device_tensors(p) if dev is None else dev
    kw = dict(T=p.T, Hs=p.Hs, Ws=p.Ws, Tc=p.Tc, To=p.To, causal=p.causal)
    y, parts = rh.hybrid_attn(dev["q"], dev["k"], dev["v"], dev["Wq"], dev["bq"], dev["Wk"],
                              dev["bk"], debug=True, force_simt=force_simt, **kw)
    den = (parts["nS"] + parts["nL"]).contiguous()
    dyt = torch.tensor(dy, dtype=torch.float32, device="cuda")
    g = rh.phi_grad(dev["q"], dev["k"], dev["v"], y, dyt, den, dev["Wq"], dev["bq"], dev["Wk"],
                    dev["bk"], force_simt=force_simt, **kw)
    torch.cuda.synchronize()
    return {n: g[n].double().cpu().numpy() for n in NAMES}


def _ref(p, dy, heads=None):
    if heads is None:
        return phi_grads(p.q, p.k, p.v, p.Wq, p.bq, p.Wk, p.bk, dy, T=p.T, HW=p.HW, Tc=p.Tc,
                         To=p.To, causal=p.causal)
    # Per-head parameters: the gradient of head h only needs head h's data.
    sel = lambda a: np.asarray(a)[:, heads]
    r = phi_grads(sel(p.q), sel(p.k), sel(p.v), np.asarray(p.Wq)[heads],
                  np.asarray(p.bq)[heads], np.asarray(p.Wk)[heads], np.asarray(p.bk)[heads],
                  np.asarray(dy)[:, heads], T=p.T, HW=p.HW, Tc=p.Tc, To=p.To, causal=p.causal)
    return r


def _check(got, ref, tol, heads=None):
    for n in NAMES:
        g = got[n] if heads is None else got[n][heads]
        scale = np.abs(ref[n]).max()
        err = np.abs(g - ref[n]).max()
        assert err <= tol * max(scale, 1e-30), f"{n}: max err {err:.3e} vs max |ref| {scale:.3e}"


SHAPES = [
    # B, h, T, Hs, Ws, D, Dp, Tc, To, causal
    (2, 2, 5, 7, 9, 128, 128, 2, 1, False),   # ragged tiles, batch sum
    (1, 2, 7, 10, 13, 128, 128, 3, 2, True),
    (1, 3, 6, 8, 12, 64, 256, 2, 0, False),   # two feature pieces
    (1, 2, 9, 11, 12, 32, 64, 3, 4, True),    # T_o > T_c
]


@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: "x".join(map(str, s)))
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_phi_grad_simt_forward_tight(shape, dtype):
    B, h, T, Hs, Ws, D, Dp, Tc, To, causal = shape
    p = make_problem(batch=B, heads=h, T=T, Hs=Hs, Ws=Ws, D=D, Dp=Dp, Tc=Tc, To=To,
                     causal=causal, dtype=dtype, seed=200 + sum(shape[:9]), phi_std=0.1)
    dy = np.random.default_rng(7).standard_normal(np.shape(p.q))
    _check(_gpu_grads(p, dy, force_simt=True), _ref(p, dy), 1e-4)


@pytest.mark.parametrize("shape", SHAPES[:3], ids=lambda s: "x".join(map(str, s)))
def test_phi_grad_tensor_core_path(shape):
    B, h, T, Hs, Ws, D, Dp, Tc, To, causal = shape
    p = make_problem(batch=B, heads=h, T=T, Hs=Hs, Ws=Ws, D=D, Dp=Dp, Tc=Tc, To=To,
                     causal=causal, dtype="bf16", seed=300 + sum(shape[:9]), phi_std=0.1)
    dy = np.random.default_rng(8).standard_normal(np.shape(p.q))
    _check(_gpu_grads(p, dy, force_simt=False), _ref(p, dy), 3e-2)


def test_phi_grad_no_linear_set_is_zero():
    p = make_problem(batch=1, heads=2, T=4, Hs=5, Ws=6, D=64, Dp=64, Tc=4, To=1, causal=False,
                     dtype="f32", seed=9)
    dy = np.random.default_rng(9).standard_normal(np.shape(p.q))
    got = _gpu_grads(p, dy, force_simt=True)
    for n in NAMES:
        assert np.all(got[n] == 0.0), n


def test_phi_grad_repeatable_bitwise():
    p = make_problem(batch=1, heads=2, T=6, Hs=8, Ws=9, D=128, Dp=128, Tc=2, To=1, causal=True,
                     dtype="bf16", seed=10)
    dy = np.random.default_rng(10).standard_normal(np.shape(p.q))
    dev = device_tensors(p)
    a = _gpu_grads(p, dy, force_simt=False, dev=dev)
    b = _gpu_grads(p, dy, force_simt=False, dev=dev)
    for n in NAMES:
        assert np.array_equal(a[n], b[n]), n


def test_phi_grad_wan_320x480_causal_sampled_heads():
    """Latent 21x20x30, 12 heads, D = D' = 128, T_c = 3, T_o = 1, causal: the
    gradients of three sampled heads against the oracle (fp32 forward)."""
    p = config_problem("wan_320x480_causal")
    dy = np.random.default_rng(11).standard_normal(np.shape(p.q)).astype(np.float32)
    heads = [0, 5, 11]
    got = _gpu_grads(p, dy, force_simt=True)
    _check(got, _ref(p, dy, heads), 1e-4, heads)


def test_phi_grad_tensor_core_full_size_causal():
    """Latent 21x20x30, 12 heads, D = D' = 128, causal, bf16: the tensor-core
    forward and backward, three sampled heads against the oracle."""
    p = config_problem("wan_320x480_causal")
    dy = np.random.default_rng(12).standard_normal(np.shape(p.q)).astype(np.float32)
    heads = [1, 6, 10]
    got = _gpu_grads(p, dy, force_simt=False)
    _check(got, _ref(p, dy, heads), 3e-2, heads)


def test_phi_grad_tensor_core_bench_layer_sampled_heads():
    """The bench layer (21x30x52, batch 2, 12 heads, bidirectional), bf16,
    tensor-core path: two sampled heads (both batch elements) against the
    oracle."""
    p = config_problem("wan_480x832_bidir")
    dy = np.random.default_rng(13).standard_normal(np.shape(p.q)).astype(np.float32)
    heads = [3, 9]
    got = _gpu_grads(p, dy, force_simt=False)
    _check(got, _ref(p, dy, heads), 3e-2, heads)


@pytest.mark.parametrize("force_simt", [False, True], ids=["tc", "simt"])
def test_phi_grad_with_the_forwards_state_is_bitwise_equal(force_simt):
    """REHYAT_FLAG_FWD_STATE: the backward run on the forward's workspace reads
    the forward's S_L, z_L and weight images and gives the same gradients bit
    for bit as the call that recomputes them; on a zeroed workspace the same
    call gives different gradients (so the state is read, not recomputed)."""
    p = make_problem(batch=2, heads=2, T=5, Hs=7, Ws=9, D=128, Dp=128, Tc=2, To=1,
                     causal=False, dtype="bf16", seed=12)
    dy = np.random.default_rng(12).standard_normal(np.shape(p.q))
    dev = device_tensors(p)
    kw = dict(T=p.T, Hs=p.Hs, Ws=p.Ws, Tc=p.Tc, To=p.To, causal=p.causal)
    prm = [dev[n] for n in ("Wq", "bq", "Wk", "bk")]
    ws = rh.bwd_workspace(dev["q"], dev["Wq"], full=False, force_simt=force_simt, **kw)
    y, parts = rh.hybrid_attn(dev["q"], dev["k"], dev["v"], *prm, debug=True,
                              force_simt=force_simt, workspace=ws, **kw)
    den = (parts["nS"] + parts["nL"]).contiguous()
    dyt = torch.tensor(dy, dtype=torch.float32, device="cuda")
    args = (dev["q"], dev["k"], dev["v"], y, dyt, den, *prm)
    a = rh.phi_grad(*args, force_simt=force_simt, **kw)
    b = rh.phi_grad(*args, force_simt=force_simt, workspace=ws, state_from_forward=True, **kw)
    ws.zero_()
    z = rh.phi_grad(*args, force_simt=force_simt, workspace=ws, state_from_forward=True, **kw)
    torch.cuda.synchronize()
    for n in NAMES:
        assert torch.equal(a[n], b[n]), n
    assert any(not torch.equal(a[n], z[n]) for n in NAMES)
    assert rh.rehyat_device_error_flags() == 0
