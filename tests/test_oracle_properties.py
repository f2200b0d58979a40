"""Property-based cross-checks of the oracle's three forms (hypothesis, CPU):
on random small geometries (T, H*W, T_c, T_o, D, D'), including ragged last
chunks and windows that reach back over several chunks (T_o > T_c), the
masked pairwise definition equals the factored form in both forms, and the
chunk-wise RNN equals both in the causal form.  The fixed-shape versions of
these pins are in test_oracle.py; here the shapes are drawn."""
import numpy as np
from hypothesis import given, settings, strategies as st

from oracle import rehyat_oracle as orc

GEOMETRY = st.tuples(
    st.integers(1, 6),                 # T slices
    st.integers(1, 5),                 # H*W tokens per slice
    st.integers(1, 4),                 # T_c
    st.integers(0, 4),                 # T_o
    st.sampled_from([2, 4, 8]),        # D
    st.sampled_from([2, 4, 6]),        # D' (two parts of D'/2)
    st.integers(0, 2 ** 31 - 1),       # seed
)


def _case(T, HW, D, Dp, seed):
    g = np.random.default_rng(seed)
    N = T * HW
    q, k, v = (g.standard_normal((1, 1, N, D)) for _ in range(3))
    W = lambda: g.standard_normal((1, 2, D, Dp // 2)) * 0.4
    b = lambda: g.standard_normal((1, 2, Dp // 2)) * 0.4
    return q, k, v, W(), b(), W(), b()


@settings(max_examples=40, deadline=None, derandomize=True)
@given(GEOMETRY, st.booleans())
def test_pairwise_equals_factored_on_random_geometries(geom, causal):
    T, HW, Tc, To, D, Dp, seed = geom
    args = _case(T, HW, D, Dp, seed)
    kw = dict(T=T, HW=HW, Tc=Tc, To=To, causal=causal)
    y1, p1 = orc.hybrid_pairwise(*args, **kw)
    y2, p2 = orc.hybrid_factored(*args, **kw)
    np.testing.assert_allclose(y1, y2, rtol=1e-11, atol=1e-12)
    for key in ("nS", "c", "nL"):
        np.testing.assert_allclose(p1[key], p2[key], rtol=1e-11, atol=1e-12)


@settings(max_examples=40, deadline=None, derandomize=True)
@given(GEOMETRY)
def test_rnn_equals_causal_forms_on_random_geometries(geom):
    T, HW, Tc, To, D, Dp, seed = geom
    args = _case(T, HW, D, Dp, seed)
    y_rnn, p_rnn = orc.hybrid_rnn(*args, T=T, HW=HW, Tc=Tc, To=To)
    y_fac, p_fac = orc.hybrid_factored(*args, T=T, HW=HW, Tc=Tc, To=To, causal=True)
    np.testing.assert_allclose(y_rnn, y_fac, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(p_rnn["nL"], p_fac["nL"], rtol=1e-11, atol=1e-12)


@settings(max_examples=15, deadline=None, derandomize=True)
@given(GEOMETRY, st.booleans())
def test_phi_gradients_match_central_differences_on_random_geometries(geom, causal):
    """The feature-map gradient oracle against central differences of the
    masked pairwise forward, on a few entries of each parameter tensor."""
    from oracle.rehyat_phi_grad import phi_grads
    T, HW, Tc, To, D, Dp, seed = geom
    q, k, v, Wq, bq, Wk, bk = _case(T, HW, D, Dp, seed)
    dy = np.random.default_rng(seed ^ 0x5A5A).standard_normal(q.shape)
    kw = dict(T=T, HW=HW, Tc=Tc, To=To, causal=causal)
    g = phi_grads(q, k, v, Wq, bq, Wk, bk, dy, **kw)
    params = dict(Wq=Wq, bq=bq, Wk=Wk, bk=bk)

    def loss(name, value):
        a = dict(params, **{name: value})
        y, _ = orc.hybrid_pairwise(q, k, v, a["Wq"], a["bq"], a["Wk"], a["bk"], **kw)
        return float((dy * y).sum())

    eps = 1e-6
    rng = np.random.default_rng(seed)
    for name, base in params.items():
        for idx in rng.choice(base.size, size=min(3, base.size), replace=False):
            plus, minus = base.copy(), base.copy()
            plus.flat[idx] += eps
            minus.flat[idx] -= eps
            fd = (loss(name, plus) - loss(name, minus)) / (2 * eps)
            an = g["d" + name].flat[idx]
            assert abs(fd - an) <= 1e-5 * max(1.0, abs(an)), (name, idx, fd, an)
