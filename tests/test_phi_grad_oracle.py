"""Pins of the phi-gradient oracle (oracle/rehyat_phi_grad.py), CPU only.

* central finite differences of L = sum(dy * y) through the forward oracle
  (pairwise masked form, independent of the factored structure the gradient
  oracle uses);
* torch autograd (fp64) of the masked pairwise definition restated in torch;
* special cases: no linear set (T_c >= T) gives zero gradients; phi = 0
  (W = b = 0) gives zero gradients.
"""
import numpy as np
import pytest

from oracle import rehyat_oracle as orc
from oracle.rehyat_phi_grad import phi_grads
from rehyat_inputs import make_problem

torch = pytest.importorskip("torch")

CASES = [
    # T, Hs, Ws, D, Dp, Tc, To, causal
    (5, 2, 3, 8, 8, 2, 1, False),
    (5, 2, 3, 8, 8, 2, 1, True),
    (6, 1, 4, 8, 12, 1, 2, True),     # T_o > T_c
    (7, 2, 2, 4, 8, 3, 0, False),     # no overlap, T % T_c != 0
]


def _problem(case, seed):
    T, Hs, Ws, D, Dp, Tc, To, causal = case
    return make_problem(batch=2, heads=2, T=T, Hs=Hs, Ws=Ws, D=D, Dp=Dp, Tc=Tc, To=To,
                        causal=causal, dtype="f32", seed=seed, phi_std=0.3)


def _dy(p, seed):
    return np.random.default_rng(seed).standard_normal(p.q.shape)


def _loss(p, dy, **params):
    args = dict(Wq=p.Wq, bq=p.bq, Wk=p.Wk, bk=p.bk)
    args.update(params)
    y, _ = orc.hybrid_pairwise(p.q, p.k, p.v, args["Wq"], args["bq"], args["Wk"], args["bk"],
                               T=p.T, HW=p.HW, Tc=p.Tc, To=p.To, causal=p.causal)
    return float((dy * y).sum())


def _grads(p, dy):
    return phi_grads(p.q, p.k, p.v, p.Wq, p.bq, p.Wk, p.bk, dy, T=p.T, HW=p.HW, Tc=p.Tc,
                     To=p.To, causal=p.causal)


@pytest.mark.parametrize("case", CASES, ids=lambda c: "x".join(map(str, c)))
def test_matches_central_differences(case):
    p = _problem(case, 11)
    dy = _dy(p, 12)
    g = _grads(p, dy)
    rng = np.random.default_rng(13)
    eps = 1e-6
    for name in ("Wq", "bq", "Wk", "bk"):
        base = np.asarray(getattr(p, name), np.float64)
        flat = rng.choice(base.size, size=min(6, base.size), replace=False)
        for idx in flat:
            plus, minus = base.copy(), base.copy()
            plus.flat[idx] += eps
            minus.flat[idx] -= eps
            fd = (_loss(p, dy, **{name: plus}) - _loss(p, dy, **{name: minus})) / (2 * eps)
            an = g["d" + name].flat[idx]
            assert abs(fd - an) <= 1e-6 * max(1.0, abs(an)), (name, idx, fd, an)


def _torch_pairwise_loss(p, dy, Wq, bq, Wk, bk):
    """The masked pairwise definition of the forward, in torch (fp64)."""
    q, k, v = (torch.tensor(np.asarray(a, np.float64)) for a in (p.q, p.k, p.v))
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
    for h in range(H):
        def phi(x, W, b):
            return torch.cat([(x @ W[0] + b[0]) ** 2, (x @ W[1] + b[1]) ** 2], dim=-1)
        for b_ in range(B):
            logits = (q[b_, h] @ k[b_, h].T) * scale
            c = torch.where(soft, logits, torch.tensor(-np.inf, dtype=torch.float64)).amax(1)
            w_soft = torch.where(soft, torch.exp(logits - c[:, None]), torch.zeros(()))
            w_lin = torch.where(lin, phi(q[b_, h], Wq[h], bq[h]) @ phi(k[b_, h], Wk[h], bk[h]).T,
                                torch.zeros(()))
            w = w_soft + w_lin
            y = (w @ v[b_, h]) / w.sum(1, keepdim=True)
            total = total + (dyt[b_, h] * y).sum()
    return total


@pytest.mark.parametrize("case", CASES[:3], ids=lambda c: "x".join(map(str, c)))
def test_matches_torch_autograd(case):
    p = _problem(case, 21)
    dy = _dy(p, 22)
    g = _grads(p, dy)
    params = [torch.tensor(np.asarray(a, np.float64), requires_grad=True)
              for a in (p.Wq, p.bq, p.Wk, p.bk)]
    _torch_pairwise_loss(p, dy, *params).backward()
    for name, t in zip(("dWq", "dbq", "dWk", "dbk"), params):
        ref = t.grad.numpy()
        assert np.allclose(g[name], ref, rtol=1e-10, atol=1e-12 * np.abs(ref).max()), name


def test_no_linear_set_gives_zero_gradients():
    p = make_problem(batch=1, heads=2, T=4, Hs=2, Ws=2, D=8, Dp=8, Tc=4, To=1, causal=False,
                     dtype="f32", seed=5)
    g = _grads(p, _dy(p, 6))
    for name in g:
        assert np.all(g[name] == 0.0), name


def test_zero_feature_map_gives_zero_gradients():
    p = _problem(CASES[0], 31)
    for name in ("Wq", "bq", "Wk", "bk"):
        setattr(p, name, np.zeros_like(np.asarray(getattr(p, name))))
    g = _grads(p, _dy(p, 32))
    for name in g:
        assert np.all(g[name] == 0.0), name
