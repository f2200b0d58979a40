"""Pins for the fp64 oracle: it is checked against things other than itself.

* hand-worked values of the formulas (tests/golden/hand_examples.json);
* special cases that reduce to a library routine (torch's fp64
  scaled_dot_product_attention): T_c >= T is full softmax, a zero feature map
  is windowed softmax, T_c = 1 with T_o = 0 is per-slice spatial softmax;
* the three independently written forms agree (masked pairwise, factored,
  chunk-wise RNN), as the page states for the causal form;
* invariants: convex hull, affine equivariance in V, permutation within a
  slice, and the last chunk being identical in the causal and bidirectional
  forms.

Source: "ReHyAt: Recurrent Hybrid Attention for Video Diffusion Transformers"
(papernotes.org note), Method, Key designs 1-4.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

from oracle import rehyat_oracle as orc

pytestmark = pytest.mark.filterwarnings("ignore::UserWarning")

GOLDEN = json.load(open(os.path.join(os.path.dirname(__file__), "golden",
                                     "hand_examples.json")))


def _rand_case(seed, *, T, HW, D, Dp, B=1, H=2, phi_std=0.3, zero_phi=False):
    g = np.random.default_rng(seed)
    q = g.standard_normal((B, H, T * HW, D))
    k = g.standard_normal((B, H, T * HW, D))
    v = g.standard_normal((B, H, T * HW, D))
    Wq = g.standard_normal((H, 2, D, Dp // 2)) * phi_std
    bq = g.standard_normal((H, 2, Dp // 2)) * phi_std
    Wk = g.standard_normal((H, 2, D, Dp // 2)) * phi_std
    bk = g.standard_normal((H, 2, Dp // 2)) * phi_std
    if zero_phi:
        Wq[:] = bq[:] = Wk[:] = bk[:] = 0.0
    return q, k, v, Wq, bq, Wk, bk


def _sdpa(q, k, v, mask=None):
    """torch's fp64 CPU attention, scale 1/sqrt(D), boolean mask = allowed."""
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a, np.float64))
    m = None if mask is None else torch.from_numpy(mask)
    with torch.no_grad():
        out = torch.nn.functional.scaled_dot_product_attention(t(q), t(k), t(v), attn_mask=m)
    return out.numpy()


# ---------------------------------------------------------------- hand values
def test_phi_hand_example():
    ex = GOLDEN["phi"]
    got = orc.feature_map(np.array(ex["x"], float), np.array(ex["W"], float),
                          np.array(ex["b"], float))
    np.testing.assert_allclose(got, np.array(ex["phi"], float), rtol=0, atol=1e-12)


@pytest.mark.parametrize("case", GOLDEN["chunks"]["cases"], ids=lambda c: f"T{c['T']}Tc{c['Tc']}To{c['To']}")
def test_chunk_table_golden(case):
    assert [list(r) for r in orc.chunk_table(case["T"], case["Tc"], case["To"])] == case["rows"]


def _hand_cases():
    for c in GOLDEN["hybrid"]:
        for form_key in ("bidir", "causal"):
            if form_key in c:
                yield pytest.param(c, form_key, id=f"{c['name']}-{form_key}")


@pytest.mark.parametrize("case,form_key", list(_hand_cases()))
@pytest.mark.parametrize("form", ["pairwise", "factored", "rnn"])
def test_hand_worked_examples(case, form_key, form):
    causal = form_key == "causal"
    if form == "rnn" and not causal:
        pytest.skip("the RNN form is causal")
    arr = lambda key: np.array(case[key], float)[None, None]
    q, k, v = arr("q"), arr("k"), arr("v")
    W = lambda key: np.array(case[key], float)[None]
    kw = dict(T=case["T"], HW=case["HW"], Tc=case["Tc"], To=case["To"])
    args = (q, k, v, W("Wq"), W("bq"), W("Wk"), W("bk"))
    if form == "pairwise":
        y, p = orc.hybrid_pairwise(*args, causal=causal, **kw)
    elif form == "factored":
        y, p = orc.hybrid_factored(*args, causal=causal, **kw)
    else:
        y, p = orc.hybrid_rnn(*args, **kw)
    exp = case[form_key]
    np.testing.assert_allclose(y[0, 0], np.array(exp["y"]), rtol=0, atol=1e-12)
    np.testing.assert_allclose(p["c"][0, 0], exp["c"], rtol=0, atol=1e-12)
    np.testing.assert_allclose(p["nS"][0, 0], exp["nS"], rtol=0, atol=1e-12)
    np.testing.assert_allclose(p["nL"][0, 0], exp["nL"], rtol=0, atol=1e-12)


# ----------------------------------------------------- cross-form agreement
TINY_SHAPES = [
    # (T, HW, Tc, To)
    (1, 3, 1, 0), (2, 1, 1, 0), (4, 4, 2, 1), (5, 3, 2, 1), (6, 2, 4, 3),
    (5, 2, 1, 2), (3, 5, 3, 0), (6, 1, 2, 3), (7, 2, 3, 1), (4, 9, 1, 1),
]


@pytest.mark.parametrize("shape", TINY_SHAPES, ids=str)
@pytest.mark.parametrize("causal", [False, True])
def test_pairwise_equals_factored(shape, causal):
    T, HW, Tc, To = shape
    args = _rand_case(hash(shape) % 1000 + causal, T=T, HW=HW, D=4, Dp=6)
    kw = dict(T=T, HW=HW, Tc=Tc, To=To, causal=causal)
    y1, p1 = orc.hybrid_pairwise(*args, **kw)
    y2, p2 = orc.hybrid_factored(*args, **kw)
    np.testing.assert_allclose(y1, y2, rtol=1e-12, atol=1e-12)
    for key in p1:
        np.testing.assert_allclose(p1[key], p2[key], rtol=1e-11, atol=1e-11)


@pytest.mark.parametrize("shape", TINY_SHAPES, ids=str)
def test_rnn_equals_causal_forms(shape):
    """The page states the non-recursive causal form equals the RNN."""
    T, HW, Tc, To = shape
    args = _rand_case(7 + hash(shape) % 1000, T=T, HW=HW, D=4, Dp=6)
    kw = dict(T=T, HW=HW, Tc=Tc, To=To)
    y_rnn, p_rnn = orc.hybrid_rnn(*args, **kw)
    y_fac, p_fac = orc.hybrid_factored(*args, causal=True, **kw)
    y_pw, _ = orc.hybrid_pairwise(*args, causal=True, **kw)
    np.testing.assert_allclose(y_rnn, y_fac, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(y_rnn, y_pw, rtol=1e-12, atol=1e-12)
    for key in p_rnn:
        np.testing.assert_allclose(p_rnn[key], p_fac[key], rtol=1e-11, atol=1e-11)


def test_rnn_state_constant_size():
    """Key design 4: the recurrent state has a fixed size however long the video."""
    q, k, v, Wq, bq, Wk, bk = _rand_case(3, T=9, HW=2, D=4, Dp=6, H=1)
    rnn = orc.ChunkRNN(4, 6, 2, 1, Wq[0], bq[0], Wk[0], bk[0], 0.5)
    sizes = set()
    for first in range(0, 9, 2):
        rows = slice(first * 2, min(9, first + 2) * 2)
        rnn.step(q[0, 0, rows], k[0, 0, rows], v[0, 0, rows])
        sizes.add((rnn.s.shape, rnn.z.shape, rnn.ring_k.shape))
    assert len({s[:2] for s in sizes}) == 1
    assert all(r[0] <= 2 for _, _, r in sizes)


# ------------------------------------------------ library special cases
@pytest.mark.parametrize("causal", [False, True])
def test_whole_video_chunk_is_full_softmax(causal):
    """T_c >= T: the softmax set is every token, the linear set is empty."""
    T, HW = 3, 5
    args = _rand_case(11, T=T, HW=HW, D=8, Dp=8)
    y, p = orc.hybrid_factored(*args, T=T, HW=HW, Tc=4, To=2, causal=causal)
    np.testing.assert_allclose(y, _sdpa(*args[:3]), rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(y, orc.full_softmax(*args[:3]), rtol=1e-12, atol=1e-12)
    assert np.all(p["nL"] == 0)
    y_pw, _ = orc.hybrid_pairwise(*args, T=T, HW=HW, Tc=T, To=0, causal=causal)
    np.testing.assert_allclose(y_pw, _sdpa(*args[:3]), rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("shape", [(5, 3, 2, 1), (6, 2, 1, 2), (4, 4, 3, 0)], ids=str)
@pytest.mark.parametrize("form", ["pairwise", "factored", "rnn"])
def test_zero_feature_map_is_windowed_softmax(shape, form):
    """phi == 0 removes the linear branch: y is softmax over the window."""
    T, HW, Tc, To = shape
    args = _rand_case(5, T=T, HW=HW, D=8, Dp=8, zero_phi=True)
    kw = dict(T=T, HW=HW, Tc=Tc, To=To)
    if form == "rnn":
        y, _ = orc.hybrid_rnn(*args, **kw)
    else:
        y, _ = getattr(orc, f"hybrid_{form}")(*args, causal=False, **kw)
    # allowed[i, j]: key j is in query i's softmax window (Key design 2).
    N = T * HW
    allowed = np.zeros((N, N), bool)
    for i in range(N):
        t = (i // HW) // Tc
        lo = max(t * Tc - To, 0) * HW
        hi = min((t + 1) * Tc, T) * HW
        allowed[i, lo:hi] = True
    np.testing.assert_allclose(y, _sdpa(*args[:3], mask=allowed), rtol=1e-12, atol=1e-12)


def test_single_slice_chunks_are_spatial_softmax():
    """T_c = 1, T_o = 0 with phi == 0: softmax over each slice alone."""
    T, HW, D = 4, 6, 8
    q, k, v, *phi = _rand_case(9, T=T, HW=HW, D=D, Dp=8, zero_phi=True)
    y, _ = orc.hybrid_factored(q, k, v, *phi, T=T, HW=HW, Tc=1, To=0, causal=False)
    per_slice = lambda a: a.reshape(1, 2, T, HW, D)
    ref = _sdpa(per_slice(q), per_slice(k), per_slice(v)).reshape(1, 2, T * HW, D)
    np.testing.assert_allclose(y, ref, rtol=1e-12, atol=1e-12)


# ---------------------------------------------------------------- invariants
@pytest.mark.parametrize("causal", [False, True])
def test_last_chunk_same_in_both_forms(causal):
    T, HW, Tc, To = 7, 3, 3, 1
    args = _rand_case(13, T=T, HW=HW, D=4, Dp=6)
    kw = dict(T=T, HW=HW, Tc=Tc, To=To)
    yb, _ = orc.hybrid_factored(*args, causal=False, **kw)
    yc, _ = orc.hybrid_factored(*args, causal=True, **kw)
    last = slice(6 * HW, 7 * HW)
    np.testing.assert_allclose(yb[..., last, :], yc[..., last, :], rtol=1e-12, atol=1e-12)
    assert not np.allclose(yb[..., :HW, :], yc[..., :HW, :])


@pytest.mark.parametrize("causal", [False, True])
def test_output_in_convex_hull_of_values(causal):
    """phi >= 0 (squares) and exp > 0: every weight is non-negative."""
    T, HW, Tc, To = 5, 4, 2, 1
    q, k, v, *phi = _rand_case(17, T=T, HW=HW, D=4, Dp=6)
    y, _ = orc.hybrid_factored(q, k, v, *phi, T=T, HW=HW, Tc=Tc, To=To, causal=causal)
    N = T * HW
    for i in range(N):
        # every key a query can reach: window plus linear set
        if causal:
            t = (i // HW) // Tc
            hi = min((t + 1) * Tc, T) * HW
        else:
            hi = N
        vmin = v[..., :hi, :].min(axis=-2)
        vmax = v[..., :hi, :].max(axis=-2)
        assert np.all(y[..., i, :] >= vmin - 1e-12)
        assert np.all(y[..., i, :] <= vmax + 1e-12)


@pytest.mark.parametrize("form", ["pairwise", "factored", "rnn"])
def test_affine_in_values(form):
    T, HW, Tc, To = 5, 3, 2, 1
    q, k, v, *phi = _rand_case(19, T=T, HW=HW, D=4, Dp=6)
    kw = dict(T=T, HW=HW, Tc=Tc, To=To)
    run = {"pairwise": lambda vv: orc.hybrid_pairwise(q, k, vv, *phi, causal=True, **kw),
           "factored": lambda vv: orc.hybrid_factored(q, k, vv, *phi, causal=False, **kw),
           "rnn": lambda vv: orc.hybrid_rnn(q, k, vv, *phi, **kw)}[form]
    y0, _ = run(v)
    y1, _ = run(2.5 * v - 0.75)
    np.testing.assert_allclose(y1, 2.5 * y0 - 0.75, rtol=1e-11, atol=1e-11)


@pytest.mark.parametrize("causal", [False, True])
def test_permutation_within_a_slice(causal):
    T, HW, Tc, To = 4, 5, 2, 1
    q, k, v, *phi = _rand_case(23, T=T, HW=HW, D=4, Dp=6)
    kw = dict(T=T, HW=HW, Tc=Tc, To=To, causal=causal)
    perm = np.arange(T * HW)
    g = np.random.default_rng(0)
    for s in range(T):
        perm[s * HW:(s + 1) * HW] = s * HW + g.permutation(HW)
    y, _ = orc.hybrid_factored(q, k, v, *phi, **kw)
    yp, _ = orc.hybrid_factored(q[..., perm, :], k[..., perm, :], v[..., perm, :], *phi, **kw)
    np.testing.assert_allclose(yp, y[..., perm, :], rtol=1e-12, atol=1e-12)


def test_softmax_denominator_at_least_one():
    """With c the window maximum, the largest softmax weight is exactly 1."""
    args = _rand_case(29, T=5, HW=3, D=4, Dp=6)
    _, p = orc.hybrid_factored(*args, T=5, HW=3, Tc=2, To=1, causal=False)
    assert np.all(p["nS"] >= 1.0)


def test_stabiliser_changes_output():
    """c_t is not a pure stabiliser: the linear branch is not scaled by it,
    so a shift of all logits (scaling q) changes the mix of the branches."""
    args = list(_rand_case(31, T=4, HW=3, D=4, Dp=6))
    y, p = orc.hybrid_factored(*args, T=4, HW=3, Tc=2, To=1, causal=False)
    # Reconstruct y from the partials: the joint normalisation.
    yy = (p["aS"] + p["aL"]) / (p["nS"] + p["nL"])[..., None]
    np.testing.assert_allclose(y, yy, rtol=1e-13, atol=1e-13)
    # A version that also divided the linear branch by exp(c) differs.
    ec = np.exp(p["c"])[..., None]
    y_alt = (p["aS"] * ec + p["aL"]) / (p["nS"] * ec[..., 0] + p["nL"])[..., None]
    assert not np.allclose(y, y_alt, rtol=1e-6, atol=1e-6)


def test_input_generator_is_deterministic_and_bf16_exact():
    from rehyat_inputs import make_problem
    p1 = make_problem(batch=1, heads=2, T=3, Hs=2, Ws=3, D=16, Dp=16, Tc=2, To=1,
                      causal=False, dtype="bf16", seed=5)
    p2 = make_problem(batch=1, heads=2, T=3, Hs=2, Ws=3, D=16, Dp=16, Tc=2, To=1,
                      causal=False, dtype="bf16", seed=5)
    assert np.array_equal(p1.q, p2.q) and np.array_equal(p1.Wk, p2.Wk)
    for a in (p1.q, p1.k, p1.v, p1.Wq, p1.Wk):
        assert np.all((a.view(np.uint32) & 0xFFFF) == 0)
