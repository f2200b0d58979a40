"""Pins of the full-backward oracle (oracle/rehyat_grad.py), CPU only.

* central finite differences of L = sum(dy * y) through the pairwise masked
  forward (a separate implementation that never forms the factored sums the
  gradient oracle uses), for q, k, v and the feature-map parameters;
* torch autograd (fp64) of the masked definition restated in torch;
* torch's own softmax-attention backward where the linear branch is absent
  (T_c >= T: full softmax; phi = 0: window softmax through a mask);
* identities of the forward: y(V + 1 beta^T) = y(V) + beta, so
  sum_j dv_j = sum_i g_i; y(alpha V) = alpha y(V), so sum_j v_j.dv_j =
  sum_i g_i.y_i;
* the feature-map parameter gradients equal those of the (separately pinned)
  phi-gradient oracle.
"""
import numpy as np
import pytest

from oracle import rehyat_oracle as orc
from oracle.rehyat_grad import forward_aux_head, hybrid_grads
from oracle.rehyat_phi_grad import phi_grads
from rehyat_inputs import make_problem

torch = pytest.importorskip("torch")

CASES = [
    # T, Hs, Ws, D, Dp, Tc, To, causal
    (5, 2, 3, 8, 8, 2, 1, False),
    (5, 2, 3, 8, 8, 2, 1, True),
    (6, 1, 4, 8, 12, 1, 2, True),     # T_o > T_c
    (7, 2, 2, 4, 8, 3, 0, False),     # no overlap, T % T_c != 0
    (4, 3, 3, 8, 8, 2, 1, False),
]


def _problem(case, seed, phi_std=0.3):
    T, Hs, Ws, D, Dp, Tc, To, causal = case
    return make_problem(batch=2, heads=2, T=T, Hs=Hs, Ws=Ws, D=D, Dp=Dp, Tc=Tc, To=To,
                        causal=causal, dtype="f32", seed=seed, phi_std=phi_std)


def _dy(p, seed):
    return np.random.default_rng(seed).standard_normal(p.q.shape)


def _grads(p, dy):
    return hybrid_grads(p.q, p.k, p.v, p.Wq, p.bq, p.Wk, p.bk, dy, T=p.T, HW=p.HW, Tc=p.Tc,
                        To=p.To, causal=p.causal)


def _loss(p, dy, **over):
    args = dict(q=p.q, k=p.k, v=p.v, Wq=p.Wq, bq=p.bq, Wk=p.Wk, bk=p.bk)
    args.update(over)
    y, _ = orc.hybrid_pairwise(args["q"], args["k"], args["v"], args["Wq"], args["bq"],
                               args["Wk"], args["bk"], T=p.T, HW=p.HW, Tc=p.Tc, To=p.To,
                               causal=p.causal)
    return float((dy * y).sum())


def _min_top2_gap(p):
    """Smallest gap between the two largest window logits over all queries
    (a finite difference must not cross the kink of the maximum)."""
    gap = np.inf
    scale = 1.0 / np.sqrt(p.D)
    for b in range(p.batch):
        for h in range(p.heads):
            q = np.asarray(p.q[b, h], np.float64)
            k = np.asarray(p.k[b, h], np.float64)
            for first, end, start in orc.chunk_table(p.T, p.Tc, p.To):
                lg = q[first * p.HW:end * p.HW] @ k[start * p.HW:end * p.HW].T * scale
                if lg.shape[1] < 2:
                    continue
                top = np.sort(lg, axis=1)[:, -2:]
                gap = min(gap, float((top[:, 1] - top[:, 0]).min()))
    return gap


@pytest.mark.parametrize("case", CASES, ids=lambda c: "x".join(map(str, c)))
def test_matches_central_differences(case):
    p = _problem(case, 41)
    assert _min_top2_gap(p) > 1e-4
    dy = _dy(p, 42)
    g = _grads(p, dy)
    rng = np.random.default_rng(43)
    eps = 1e-6
    for name in ("q", "k", "v", "Wq", "bq", "Wk", "bk"):
        base = np.asarray(getattr(p, name), np.float64)
        for idx in rng.choice(base.size, size=min(10, base.size), replace=False):
            plus, minus = base.copy(), base.copy()
            plus.flat[idx] += eps
            minus.flat[idx] -= eps
            fd = (_loss(p, dy, **{name: plus}) - _loss(p, dy, **{name: minus})) / (2 * eps)
            an = g["d" + name].flat[idx]
            assert abs(fd - an) <= 2e-6 * max(1.0, abs(an)), (name, idx, fd, an)


def test_central_differences_balanced_branches():
    # A smaller phi makes n^L comparable with n^S, so the maximum's gradient
    # (which scales with the linear branch's share) is large relative to the
    # rest; the finite differences would see it missing.
    p = _problem(CASES[0], 51, phi_std=0.05)
    nL_over_nS = []
    for b in range(p.batch):
        for h in range(p.heads):
            aux = forward_aux_head(p.q[b, h], p.k[b, h], p.v[b, h], p.Wq[h], p.bq[h], p.Wk[h],
                                   p.bk[h], T=p.T, HW=p.HW, Tc=p.Tc, To=p.To, causal=p.causal,
                                   scale=1.0 / np.sqrt(p.D))
            nL_over_nS.append(np.median(aux["nL"] / aux["nS"]))
    assert 0.05 < np.median(nL_over_nS) < 20
    dy = _dy(p, 52)
    g = _grads(p, dy)
    eps = 1e-6
    for name in ("q", "k"):
        base = np.asarray(getattr(p, name), np.float64)
        for idx in range(0, base.size, 7):
            plus, minus = base.copy(), base.copy()
            plus.flat[idx] += eps
            minus.flat[idx] -= eps
            fd = (_loss(p, dy, **{name: plus}) - _loss(p, dy, **{name: minus})) / (2 * eps)
            an = g["d" + name].flat[idx]
            assert abs(fd - an) <= 2e-6 * max(1.0, abs(an)), (name, idx, fd, an)


def _torch_loss(p, dy, q, k, v, Wq, bq, Wk, bk):
    """The masked pairwise definition of the forward in torch (fp64); the
    stabiliser is the window maximum, differentiated through (torch.max)."""
    dyt = torch.tensor(dy)
    B, H, N, D = q.shape
    scale = 1.0 / np.sqrt(D)
    Np = p.Tc * p.HW
    i = torch.arange(N)[:, None]
    j = torch.arange(N)[None, :]
    t = i // Np
    lo = torch.clamp(t * Np - p.To * p.HW, min=0)
    hi = torch.clamp((t + 1) * Np, max=N)
    soft = (j >= lo) & (j < hi)
    lin = (j < lo) if p.causal else ~soft
    total = 0.0

    def phi(x, W, b):
        return torch.cat([(x @ W[0] + b[0]) ** 2, (x @ W[1] + b[1]) ** 2], dim=-1)

    for h in range(H):
        for b_ in range(B):
            logits = (q[b_, h] @ k[b_, h].T) * scale
            masked = torch.where(soft, logits, torch.tensor(-np.inf, dtype=torch.float64))
            c = masked.max(dim=1).values
            w_soft = torch.where(soft, torch.exp(logits - c[:, None]), torch.zeros(()))
            w_lin = torch.where(lin, phi(q[b_, h], Wq[h], bq[h]) @ phi(k[b_, h], Wk[h], bk[h]).T,
                                torch.zeros(()))
            w = w_soft + w_lin
            y = (w @ v[b_, h]) / w.sum(1, keepdim=True)
            total = total + (dyt[b_, h] * y).sum()
    return total


@pytest.mark.parametrize("case", CASES[:3], ids=lambda c: "x".join(map(str, c)))
def test_matches_torch_autograd(case):
    p = _problem(case, 61)
    dy = _dy(p, 62)
    g = _grads(p, dy)
    names = ("q", "k", "v", "Wq", "bq", "Wk", "bk")
    leaves = [torch.tensor(np.asarray(getattr(p, n), np.float64), requires_grad=True)
              for n in names]
    _torch_loss(p, dy, *leaves).backward()
    for name, t in zip(names, leaves):
        ref = t.grad.numpy()
        assert np.allclose(g["d" + name], ref, rtol=1e-10, atol=1e-12 * np.abs(ref).max()), name


def _sdpa_grads(q, k, v, dy, mask=None):
    qt, kt, vt = (torch.tensor(np.asarray(a, np.float64), requires_grad=True) for a in (q, k, v))
    y = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, attn_mask=mask)
    (torch.tensor(dy) * y).sum().backward()
    return qt.grad.numpy(), kt.grad.numpy(), vt.grad.numpy()


def test_no_linear_set_is_softmax_backward():
    # T_c >= T: every key is in the window of every query; phi is non-zero but
    # has no linear set to act on.
    p = make_problem(batch=1, heads=2, T=4, Hs=2, Ws=3, D=8, Dp=8, Tc=4, To=1, causal=False,
                     dtype="f32", seed=71, phi_std=0.3)
    dy = _dy(p, 72)
    g = _grads(p, dy)
    dq, dk, dv = _sdpa_grads(p.q, p.k, p.v, dy)
    for name, ref in (("dq", dq), ("dk", dk), ("dv", dv)):
        assert np.allclose(g[name], ref, rtol=1e-10, atol=1e-13), name
    for name in ("dWq", "dbq", "dWk", "dbk"):
        assert np.all(g[name] == 0.0), name


@pytest.mark.parametrize("causal", [False, True])
def test_zero_feature_map_is_window_softmax_backward(causal):
    p = make_problem(batch=1, heads=2, T=5, Hs=2, Ws=2, D=8, Dp=8, Tc=2, To=1, causal=causal,
                     dtype="f32", seed=81)
    for name in ("Wq", "bq", "Wk", "bk"):
        setattr(p, name, np.zeros_like(np.asarray(getattr(p, name))))
    dy = _dy(p, 82)
    g = _grads(p, dy)
    # Window mask from the set definition (Key designs 1, 2).
    N, Np = p.N, p.Tc * p.HW
    i = np.arange(N)[:, None]
    j = np.arange(N)[None, :]
    lo = np.maximum((i // Np) * Np - p.To * p.HW, 0)
    hi = np.minimum((i // Np + 1) * Np, N)
    mask = torch.tensor((j >= lo) & (j < hi))
    dq, dk, dv = _sdpa_grads(p.q, p.k, p.v, dy, mask)
    for name, ref in (("dq", dq), ("dk", dk), ("dv", dv)):
        assert np.allclose(g[name], ref, rtol=1e-10, atol=1e-13), name


@pytest.mark.parametrize("case", CASES, ids=lambda c: "x".join(map(str, c)))
def test_value_identities(case):
    p = _problem(case, 91)
    dy = _dy(p, 92)
    g = _grads(p, dy)
    y, _ = orc.run_problem(p, form="pairwise")
    # sum_j dv_j = sum_i g_i per (b, h): a constant shift of every value row
    # shifts every output row by the same amount.
    assert np.allclose(g["dv"].sum(axis=2), dy.sum(axis=2), rtol=1e-10, atol=1e-11)
    # sum_j v_j.dv_j = sum_i g_i.y_i per (b, h): y is linear in V.
    lhs = (np.asarray(p.v, np.float64) * g["dv"]).sum(axis=(2, 3))
    rhs = (dy * y).sum(axis=(2, 3))
    assert np.allclose(lhs, rhs, rtol=1e-10, atol=1e-11)


@pytest.mark.parametrize("case", CASES[:4], ids=lambda c: "x".join(map(str, c)))
def test_parameter_gradients_match_phi_gradient_oracle(case):
    p = _problem(case, 101)
    dy = _dy(p, 102)
    g = _grads(p, dy)
    ref = phi_grads(p.q, p.k, p.v, p.Wq, p.bq, p.Wk, p.bk, dy, T=p.T, HW=p.HW, Tc=p.Tc,
                    To=p.To, causal=p.causal)
    for name in ("dWq", "dbq", "dWk", "dbk"):
        assert np.allclose(g[name], ref[name], rtol=1e-11, atol=1e-13), name


def test_forward_aux_matches_forward_oracle():
    p = _problem(CASES[2], 111)
    y, part = orc.run_problem(p, form="factored")
    for b in range(p.batch):
        for h in range(p.heads):
            aux = forward_aux_head(p.q[b, h], p.k[b, h], p.v[b, h], p.Wq[h], p.bq[h], p.Wk[h],
                                   p.bk[h], T=p.T, HW=p.HW, Tc=p.Tc, To=p.To, causal=p.causal,
                                   scale=1.0 / np.sqrt(p.D))
            assert np.allclose(aux["y"], y[b, h], rtol=1e-12, atol=1e-13)
            assert np.allclose(aux["den"], aux["nS"] + aux["nL"], rtol=1e-14)
            assert np.allclose(aux["y"] * aux["den"][:, None], aux["aS"] + aux["aL"], rtol=1e-11,
                               atol=1e-13)
