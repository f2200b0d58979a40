"""Pins of the fp8 softmax-branch oracle (oracle/rehyat_fp8.py), CPU only.

* e4m3_round against torch's float8_e4m3fn cast (a library implementation of
  the same format, round to nearest even) on every bf16 value of magnitude
  <= 464 that the cast maps to a finite number, and against hand values for
  ties, subnormals and saturation;
* the variant equals the main oracle when q and k are already E4M3 values,
  and differs from it otherwise only through the logits (the linear-branch
  partials are identical);
* brute force on a tiny case: per query, the masked definition with logits
  from the rounded q, k.
"""
import numpy as np
import pytest
import torch

from oracle import rehyat_oracle as orc
from oracle.rehyat_fp8 import e4m3_round, hybrid_fp8_qk
from rehyat_inputs import make_problem


def test_e4m3_round_matches_torch_on_all_bf16_in_range():
    bits = torch.arange(0, 1 << 16, dtype=torch.int32).to(torch.int16)
    x = bits.view(torch.bfloat16).to(torch.float32)
    x = x[torch.isfinite(x) & (x.abs() <= 464)]
    ref = x.to(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = e4m3_round(x.double().numpy())
    assert np.array_equal(got, ref)


def test_e4m3_round_hand_values():
    cases = {
        448.0: 448.0, 464.0: 448.0,     # the tie above 448 rounds to even (448)
        500.0: 448.0, -1e4: -448.0,     # saturation
        1.0625: 1.0, 1.1875: 1.25,      # ties to even at spacing 1/8
        2 ** -9: 2 ** -9, 2 ** -10: 0.0,  # smallest subnormal; its half ties to 0
        1.5 * 2 ** -9: 2 ** -8, 3 * 2 ** -10: 2 ** -8,
        0.0: 0.0, -0.0: -0.0,
    }
    for x, want in cases.items():
        assert e4m3_round(x) == want, x
    assert np.isnan(e4m3_round(np.nan))


def test_identity_on_e4m3_inputs_and_linear_branch_unchanged():
    p = make_problem(batch=1, heads=2, T=5, Hs=2, Ws=3, D=8, Dp=8, Tc=2, To=1, causal=False,
                     dtype="f32", seed=31)
    kw = dict(T=p.T, HW=p.HW, Tc=p.Tc, To=p.To, causal=p.causal)
    q8, k8 = e4m3_round(p.q), e4m3_round(p.k)
    y_ref, parts_ref = orc.hybrid_factored(q8, k8, p.v, p.Wq, p.bq, p.Wk, p.bk, **kw)
    y, parts = hybrid_fp8_qk(q8, k8, p.v, p.Wq, p.bq, p.Wk, p.bk, **kw)
    assert np.array_equal(y, y_ref)
    y2, parts2 = hybrid_fp8_qk(p.q, p.k, p.v, p.Wq, p.bq, p.Wk, p.bk, **kw)
    _, parts_full = orc.hybrid_factored(p.q, p.k, p.v, p.Wq, p.bq, p.Wk, p.bk, **kw)
    assert np.array_equal(parts2["aL"], parts_full["aL"])
    assert np.array_equal(parts2["nL"], parts_full["nL"])
    assert not np.allclose(parts2["c"], parts_full["c"])


@pytest.mark.parametrize("causal", [False, True])
def test_brute_force_tiny(causal):
    rng = np.random.default_rng(5)
    T, HW, D, Dp, Tc, To = 5, 2, 4, 4, 2, 1
    N = T * HW
    q, k, v = (rng.standard_normal((1, 1, N, D)) * 2 for _ in range(3))
    Wq, Wk = (rng.standard_normal((1, 2, D, Dp // 2)) * 0.3 for _ in range(2))
    bq, bk = (rng.standard_normal((1, 2, Dp // 2)) * 0.3 for _ in range(2))
    y, _ = hybrid_fp8_qk(q, k, v, Wq, bq, Wk, bk, T=T, HW=HW, Tc=Tc, To=To, causal=causal)
    q8, k8 = e4m3_round(q[0, 0]), e4m3_round(k[0, 0])
    fq = orc.feature_map(q[0, 0], Wq[0], bq[0])
    fk = orc.feature_map(k[0, 0], Wk[0], bk[0])
    Np = Tc * HW
    for i in range(N):
        t = i // Np
        lo, hi = max(t * Np - To * HW, 0), min((t + 1) * Np, N)
        c = max(q8[i] @ k8[j] / np.sqrt(D) for j in range(lo, hi))
        num, den = np.zeros(D), 0.0
        for j in range(N):
            if lo <= j < hi:
                w = np.exp(q8[i] @ k8[j] / np.sqrt(D) - c)
            elif j < lo or (not causal and j >= hi):
                w = fq[i] @ fk[j]
            else:
                w = 0.0
            num += w * v[0, 0, j]
            den += w
        assert np.allclose(y[0, 0, i], num / den, rtol=1e-12, atol=1e-14), i
