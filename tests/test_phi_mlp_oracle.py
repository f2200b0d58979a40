"""Pins of the general feature map and of the phi-given forward oracle
(oracle/rehyat_phi_mlp.py), CPU only.

* a hand-worked map (D = 2, D_h = 3, D' = 2) in terms of the normal CDF;
* GELU against scipy.stats.norm.cdf (x * Phi(x)) and its odd part
  gelu(x) - gelu(-x) = x;
* the P-part powers: part i of phi equals the i-th power of part i of the
  P = 1 map (which is psi itself);
* the phi-given forward with phi computed by the degree-2 closed form equals
  the pinned factored forward, and with a general (partly negative) phi it
  equals a brute-force pairwise evaluation of the masked definition.
"""
import numpy as np
import pytest
from scipy.stats import norm

from oracle import rehyat_oracle as orc
from oracle.rehyat_phi_mlp import feature_map_mlp, gelu, hybrid_phi_given
from rehyat_inputs import make_problem


def test_gelu_matches_normal_cdf_and_odd_part():
    x = np.random.default_rng(0).standard_normal(1000) * 3
    assert np.allclose(gelu(x), x * norm.cdf(x), rtol=1e-13, atol=1e-15)
    assert np.allclose(gelu(x) - gelu(-x), x, rtol=1e-13, atol=1e-14)
    assert gelu(0.0) == 0.0


def test_feature_map_mlp_hand_example():
    """psi = GELU(x W_a + b_a) W_b + b_b worked by hand for D = 2, D_h = 3,
    D' = 2 (non-square weights, non-zero biases), GELU(u) = u Phi(u):

      row 1, x = (1, -2):    u = (1 + 0.5, 2, 2 - 1 - 1) = (1.5, 2, 0)
        psi = (1.5 Phi(1.5) + 0.5 * 2 Phi(2) + 0.25,  -1.5 Phi(1.5) + 3 * 0 - 0.5)
      row 2, x = (0.5, 0.25): u = (0.5 + 0.5, -0.25, 1 + 0.125 - 1) = (1, -0.25, 0.125)
        psi = (Phi(1) + 0.5 * (-0.25) Phi(-0.25) + 0.25,
               -Phi(1) + 3 * 0.125 Phi(0.125) - 0.5)

    P = 2 keeps part 1 and squares part 2."""
    x = np.array([[1.0, -2.0], [0.5, 0.25]])
    Wa = np.array([[1.0, 0.0, 2.0], [0.0, -1.0, 0.5]])
    ba = np.array([0.5, 0.0, -1.0])
    Wb = np.array([[1.0, -1.0], [0.5, 0.0], [0.0, 3.0]])
    bb = np.array([0.25, -0.5])
    F = norm.cdf
    psi = np.array([
        [1.5 * F(1.5) + 0.5 * 2.0 * F(2.0) + 0.25, -1.5 * F(1.5) - 0.5],
        [F(1.0) + 0.5 * (-0.25) * F(-0.25) + 0.25, -F(1.0) + 3.0 * 0.125 * F(0.125) - 0.5],
    ])
    np.testing.assert_allclose(feature_map_mlp(x, Wa, ba, Wb, bb, 1), psi, rtol=0, atol=1e-14)
    np.testing.assert_allclose(feature_map_mlp(x, Wa, ba, Wb, bb, 2),
                               np.stack([psi[:, 0], psi[:, 1] ** 2], axis=1), rtol=0, atol=1e-14)


@pytest.mark.parametrize("P", [1, 2, 4])
def test_parts_are_powers_of_psi(P):
    rng = np.random.default_rng(1)
    D, Dh, Dp = 8, 24, 16
    x = rng.standard_normal((5, D))
    Wa, ba = rng.standard_normal((D, Dh)) * 0.3, rng.standard_normal(Dh) * 0.1
    Wb, bb = rng.standard_normal((Dh, Dp)) * 0.3, rng.standard_normal(Dp) * 0.1
    psi = feature_map_mlp(x, Wa, ba, Wb, bb, 1)
    phi = feature_map_mlp(x, Wa, ba, Wb, bb, P)
    w = Dp // P
    for i in range(P):
        assert np.allclose(phi[:, i * w:(i + 1) * w], psi[:, i * w:(i + 1) * w] ** (i + 1),
                           rtol=1e-13)


@pytest.mark.parametrize("causal", [False, True])
def test_phi_given_equals_factored_with_closed_form_phi(causal):
    p = make_problem(batch=1, heads=2, T=5, Hs=2, Ws=3, D=8, Dp=8, Tc=2, To=1, causal=causal,
                     dtype="f32", seed=3, phi_std=0.3)
    fq = np.stack([np.stack([orc.feature_map(p.q[b, h], p.Wq[h], p.bq[h]) for h in range(2)])
                   for b in range(1)])
    fk = np.stack([np.stack([orc.feature_map(p.k[b, h], p.Wk[h], p.bk[h]) for h in range(2)])
                   for b in range(1)])
    y, parts = hybrid_phi_given(p.q, p.k, p.v, fq, fk, T=p.T, HW=p.HW, Tc=p.Tc, To=p.To,
                                causal=causal)
    ref_y, ref_p = orc.run_problem(p)
    assert np.allclose(y, ref_y, rtol=1e-12, atol=1e-14)
    for key in ref_p:
        assert np.allclose(parts[key], ref_p[key], rtol=1e-12, atol=1e-14), key


@pytest.mark.parametrize("causal", [False, True])
def test_phi_given_equals_pairwise_definition(causal):
    """General phi with a degree-1 part (negative values allowed)."""
    rng = np.random.default_rng(4)
    T, HW, D, Dp, Tc, To = 6, 3, 4, 6, 2, 1
    N = T * HW
    q, k, v = (rng.standard_normal((1, 1, N, D)) for _ in range(3))
    fq = rng.standard_normal((1, 1, N, Dp)) * 0.2
    fk = rng.standard_normal((1, 1, N, Dp)) * 0.2
    y, _ = hybrid_phi_given(q, k, v, fq, fk, T=T, HW=HW, Tc=Tc, To=To, causal=causal)
    scale = 1 / np.sqrt(D)
    Np = Tc * HW
    for i in range(N):
        t = i // Np
        lo, hi = max(t * Np - To * HW, 0), min((t + 1) * Np, N)
        num = np.zeros(D)
        den = 0.0
        c = max((q[0, 0, i] @ k[0, 0, j]) * scale for j in range(lo, hi))
        for j in range(N):
            if lo <= j < hi:
                w = np.exp((q[0, 0, i] @ k[0, 0, j]) * scale - c)
            elif (j < lo) or (not causal and j >= hi):
                w = fq[0, 0, i] @ fk[0, 0, j]
            else:
                w = 0.0
            num += w * v[0, 0, j]
            den += w
        assert np.allclose(y[0, 0, i], num / den, rtol=1e-10, atol=1e-12), i


def _bf16(a):
    import torch
    return torch.tensor(np.asarray(a, np.float32)).to(torch.bfloat16).double().numpy()


@pytest.mark.parametrize("P", [1, 2, 4])
def test_bf16_bound_covers_emulated_bf16_map(P):
    """The tolerance used for the tensor-core map (tests/mlp_bound.py) holds
    for an fp64 emulation that rounds W_a, GELU(.) and W_b to bf16 the way
    the kernel does, and is tight enough to catch a dropped bias or a wrong
    power (each exceeds it)."""
    from tests.mlp_bound import bf16_bound
    rng = np.random.default_rng(9)
    D, Dh, Dp = 128, 256, 64
    x = _bf16(rng.standard_normal((200, D)) * 1.5)
    Wa = rng.standard_normal((D, Dh)) / np.sqrt(D)
    ba = rng.standard_normal(Dh) * 0.1
    Wb = rng.standard_normal((Dh, Dp)) / np.sqrt(Dh) * 0.5
    bb = rng.standard_normal(Dp) * 0.05
    ref = feature_map_mlp(x, Wa, ba, Wb, bb, P)
    g = _bf16(gelu(x @ _bf16(Wa) + ba))
    psi = g @ _bf16(Wb) + bb
    w = Dp // P
    emu = np.concatenate([psi[:, i * w:(i + 1) * w] ** (i + 1) for i in range(P)], axis=1)
    bound = bf16_bound(x, Wa, ba, Wb, bb, P)
    assert np.all(np.abs(emu - ref) <= bound)
    no_bias = np.concatenate([(psi - bb)[:, i * w:(i + 1) * w] ** (i + 1) for i in range(P)],
                             axis=1)
    assert np.any(np.abs(no_bias - ref) > bound)
    if P > 1:
        wrong_power = psi ** 2
        assert np.any(np.abs(wrong_power - ref) > bound)


def test_tensor_core_gelu_constants_meet_published_bound():
    """The erf approximation in the tensor-core feature map (Abramowitz &
    Stegun 7.1.28) with the constants as written in its source reproduces
    erf within the handbook's 3e-7, and Phi for negative arguments (r/2,
    r = 1/poly^16) without cancellation."""
    import os
    import re
    from scipy.special import erf
    src = open(os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                            "linear_attention_video_chunked_b200", "csrc",
                            "tc_phi_mlp.cuh")).read()
    c = {k: float(v) for k, v in re.findall(r"\b(kErfA[1-6]) = (-?[0-9.]+)f", src)}
    assert set(c) == {"kErfA1", "kErfA2", "kErfA3", "kErfA4", "kErfA5", "kErfA6"}
    c = {k.replace("Erf", ""): v for k, v in c.items()}
    x = np.linspace(0.0, 8.0, 20001)
    poly = 1.0 + x * (c["kA1"] + x * (c["kA2"] + x * (c["kA3"] + x * (c["kA4"] + x * (
        c["kA5"] + x * c["kA6"])))))
    r = 1.0 / poly ** 16
    assert np.abs((1.0 - r) - erf(x)).max() <= 3e-7
    u = -x * np.sqrt(2.0)
    assert np.abs(0.5 * r - 0.5 * (1.0 + erf(u / np.sqrt(2.0)))).max() <= 1.5e-7
