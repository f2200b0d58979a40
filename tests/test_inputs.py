"""The seeded input generator (rehyat_inputs) draws what its recipe states.

* "scaled" (the named workloads): q, k, v ~ N(0, 1) times a scale
  s ~ U(0.5, 2) drawn per (tensor, head) and shared across the batch;
* "lowrank" (the sweep): q = U_q G + eps, k = U_k G + eps with a per-head
  G in R^{8 x D} of N(0, 1/8) entries and eps ~ N(0, 0.3^2), which puts the
  standard deviation of the scaled logits q.k / sqrt(D) near
  sqrt(8) * (D / 8) / sqrt(D) = 4 at D = 128;
* phi weights and biases ~ N(0, std^2) per head, std 0.1 by default;
* the named workloads have the shapes their names give.
"""
import numpy as np
import pytest

from rehyat_inputs import CONFIGS, make_problem


def _per_head_std(a):
    # a: [B, h, N, D] -> [B, h]
    return a.reshape(a.shape[0], a.shape[1], -1).std(axis=-1)


def test_scaled_inputs_have_one_scale_per_tensor_and_head():
    p = make_problem(batch=2, heads=6, T=4, Hs=10, Ws=10, D=64, Dp=64, Tc=2, To=1,
                     causal=False, dtype="f32", dist="scaled", seed=11)
    for a in (p.q, p.k, p.v):
        s = _per_head_std(a)                        # 25,600 draws per (b, h)
        assert np.all((s > 0.5 * 0.97) & (s < 2.0 * 1.03)), s
        assert np.allclose(s[0], s[1], rtol=0.03)   # shared across the batch
        assert np.ptp(s[0]) > 0.1                   # and different across heads
    # The three tensors draw their own scales.
    assert not np.allclose(_per_head_std(p.q)[0], _per_head_std(p.k)[0], rtol=0.03)


def test_lowrank_inputs_give_logits_of_std_near_four():
    D = 128
    p = make_problem(batch=1, heads=2, T=2, Hs=16, Ws=16, D=D, Dp=32, Tc=1, To=0,
                     causal=False, dtype="f32", dist="lowrank", seed=12)
    for h in range(2):
        logits = (p.q[0, h] @ p.k[0, h].T) / np.sqrt(D)
        assert 3.0 < logits.std() < 5.0, logits.std()
    # q and k of one head share the subspace: far from independent draws.
    q, k = p.q[0, 0], p.k[0, 0]
    cq = np.linalg.svd(q, compute_uv=False)
    assert cq[7] > 5 * cq[8]                        # rank 8 plus the small noise floor
    assert np.all(np.isfinite(k)) and abs(p.v.std() - 1.0) < 0.05


def test_phi_parameters_have_the_stated_std():
    p = make_problem(batch=1, heads=4, T=1, Hs=2, Ws=2, D=128, Dp=128, Tc=1, To=0,
                     causal=False, dtype="f32", seed=13, phi_std=0.1)
    for a in (p.Wq, p.Wk):
        assert a.shape == (4, 2, 128, 64) and abs(a.std() - 0.1) < 0.005
    for b in (p.bq, p.bk):
        assert b.shape == (4, 2, 64) and abs(b.std() - 0.1) < 0.02


@pytest.mark.parametrize("name,shape", [
    ("tiny_f32", (1, 2, 4 * 4 * 4, 32)),
    ("wan_320x480_causal", (1, 12, 21 * 20 * 30, 128)),
    ("wan_480x832_bidir", (2, 12, 21 * 30 * 52, 128)),
    ("stream_81x30x52", (1, 12, 81 * 30 * 52, 128)),
])
def test_named_workloads_have_the_shapes_their_names_give(name, shape):
    c = CONFIGS[name]
    B, h, N, D = shape
    assert (c["batch"], c["heads"], c["T"] * c["Hs"] * c["Ws"], c["D"]) == (B, h, N, D)
    assert c["Tc"] >= 1 and c["To"] >= 0
