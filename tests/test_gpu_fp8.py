"""GPU parity of the fp8 softmax-branch variant (REHYAT_FLAG_FP8_QK: logits
from E4M3 copies of q and k on tcgen05 kind::f8f6f4) against its fp64 oracle
(oracle/rehyat_fp8.py), through the C ABI, on the same seeded inputs.

The oracle rounds q and k to E4M3 exactly as the kernel's conversion does, so
the bar is the bf16 path's (y max abs <= 2e-2, mean <= 2e-3; partials as in
tests/gpu_util.py); what the variant loses against the bf16 forward -- the
E4M3 rounding of q and k, 2^-4 relative per element -- is measured against
the main oracle and reported, not hidden in the bar.
"""
import numpy as np
import pytest
import torch

import linear_attention_video_chunked_b200 as rh
from oracle import rehyat_oracle as orc
from oracle.rehyat_fp8 import e4m3_round, hybrid_fp8_qk
from rehyat_inputs import config_problem, make_problem
from tests.gpu_util import assert_close_partials, assert_close_y, device_tensors

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    rh.lib()
    rh.rehyat_device_error_flags(reset=True)
    yield
    assert rh.rehyat_device_error_flags() == 0


def _run(p, fp8=True):
    dev = device_tensors(p)
    y, parts = rh.hybrid_attn(dev["q"], dev["k"], dev["v"], dev["Wq"], dev["bq"], dev["Wk"],
                              dev["bk"], T=p.T, Hs=p.Hs, Ws=p.Ws, Tc=p.Tc, To=p.To,
                              causal=p.causal, debug=True, fp8_qk=fp8)
    torch.cuda.synchronize()
    return y.double().cpu().numpy(), {k: v.double().cpu().numpy() for k, v in parts.items()}


def _oracle(p, **kw):
    return hybrid_fp8_qk(p.q, p.k, p.v, p.Wq, p.bq, p.Wk, p.bk, T=p.T, HW=p.HW, Tc=p.Tc,
                         To=p.To, causal=p.causal, **kw)


SHAPES = [
    # B, h, T, Hs, Ws, Dp, Tc, To
    (1, 2, 5, 7, 9, 128, 2, 1),     # ragged key and query tiles
    (2, 3, 7, 10, 13, 64, 3, 2),    # T_o > 0, several chunks, D' = 64
    (1, 2, 4, 16, 16, 128, 1, 0),   # exact 256-token slices
]


@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: "x".join(map(str, s)))
@pytest.mark.parametrize("causal", [False, True])
def test_fp8_small_shapes(shape, causal):
    B, h, T, Hs, Ws, Dp, Tc, To = shape
    p = make_problem(batch=B, heads=h, T=T, Hs=Hs, Ws=Ws, D=128, Dp=Dp, Tc=Tc, To=To,
                     causal=causal, dtype="bf16", dist="scaled", seed=700 + sum(shape))
    ref_y, ref_p = _oracle(p)
    y, parts = _run(p)
    assert_close_y(y, ref_y, "bf16")
    assert_close_partials(parts, ref_p, "bf16")


def test_fp8_sharp_softmax_and_cost_against_bf16():
    """Low-rank q, k (logit std ~4), weak feature map: the softmax branch
    dominates y.  Parity against the fp8 oracle; the E4M3 rounding's effect
    on y against the main (bf16-logit) oracle is bounded loosely."""
    p = make_problem(batch=1, heads=2, T=6, Hs=12, Ws=20, D=128, Dp=128, Tc=2, To=1,
                     causal=False, dtype="bf16", dist="lowrank", seed=78, phi_std=0.005)
    ref_y, ref_p = _oracle(p)
    y, parts = _run(p)
    assert_close_y(y, ref_y, "bf16")
    assert_close_partials(parts, ref_p, "bf16")
    full_y, _ = orc.run_problem(p)
    d = np.abs(y - full_y)
    assert d.mean() < 0.05, d.mean()  # the variant's own error, not a parity bar
    assert np.abs(ref_y - full_y).max() > 1e-3  # the rounding is visible


def test_fp8_rounding_ties_and_saturation_seen_in_c():
    """q_i = (t_i, 0, ...), k_j = (8, 0, ...): each row max c is t_i' * 8 * s
    with t_i' the E4M3 value of t_i -- ties (1.0625 -> 1.0, 1.1875 -> 1.25),
    a subnormal, and saturation (600 -> 448) -- visible exactly in c."""
    B, H, T, Hs, Ws, D, Dp = 1, 1, 1, 8, 16, 128, 64
    N = T * Hs * Ws
    p = make_problem(batch=B, heads=H, T=T, Hs=Hs, Ws=Ws, D=D, Dp=Dp, Tc=1, To=0,
                     causal=False, dtype="bf16", seed=79)
    t = np.array([1.0625, 1.1875, 3 * 2 ** -10, 600.0, -2.5, 0.3] * N)[:N]
    q = np.zeros((B, H, N, D))
    q[0, 0, :, 0] = t
    k = np.zeros((B, H, N, D))
    k[0, 0, :, 0] = 8.0
    p.q = q.astype(np.float32)
    p.k = k.astype(np.float32)
    y, parts = _run(p)
    t_bf16 = torch.tensor(t, dtype=torch.float32).to(torch.bfloat16).double().numpy()
    want_c = e4m3_round(t_bf16) * 8.0 / np.sqrt(D)
    assert np.allclose(parts["c"][0, 0], want_c, rtol=1e-6, atol=1e-6)


def test_fp8_full_size_sampled_heads():
    """Latent 21x30x52, batch 2, 12 heads, bidirectional (the bench layer):
    every output of three sampled (batch, head) pairs."""
    p = config_problem("wan_480x832_bidir")
    subset = [2, 11, 20]
    ref_y, ref_p = _oracle(p, heads_subset=subset)
    y, parts = _run(p)
    for idx in subset:
        b, hh = divmod(idx, p.heads)
        assert_close_y(y[b, hh], ref_y[b, hh], "bf16", f"y[{b},{hh}]")
        assert_close_partials({k: v[b, hh] for k, v in parts.items()},
                              {k: v[b, hh] for k, v in ref_p.items()}, "bf16")


def test_fp8_flag_refused_where_unsupported():
    base = dict(batch=1, heads=2, T=3, Hs=4, Ws=4, D=128, Dp=128, Tc=1, To=0, causal=0)
    f = rh.FLAG_FP8_QK
    assert rh.rehyat_workspace_bytes(rh.make_params(**base, in_dtype=rh.F32, flags=f)) == 0
    assert rh.rehyat_workspace_bytes(rh.make_params(**{**base, "Dp": 256}, flags=f)) == 0
    assert rh.rehyat_workspace_bytes(rh.make_params(**base, flags=f | rh.FLAG_FORCE_SIMT)) == 0
    assert rh.rehyat_state_bytes(rh.make_params(**base, flags=f)) == 0
    ok = rh.make_params(**base, flags=f)
    plain = rh.make_params(**base)
    # The workspace grows by the two E4M3 copies (2 * B * h * N * D bytes).
    assert rh.rehyat_workspace_bytes(ok) >= rh.rehyat_workspace_bytes(plain) + 2 * 2 * 48 * 128
