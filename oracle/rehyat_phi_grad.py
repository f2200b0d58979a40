"""fp64 CPU oracle for the gradient of ReHyAt's hybrid attention with respect
to the feature-map parameters (W_q, b_q, W_k, b_k).

TEST INFRASTRUCTURE, NOT PRODUCT CODE.  Only the tests and the CPU-baseline
leg of ``bench.py`` may import this module.  It shares no code with the CUDA
path (numpy only, plus the forward oracle of this package).

Source: "ReHyAt: Recurrent Hybrid Attention for Video Diffusion Transformers"
(papernotes.org note of the CVPR 2026 paper).  Section "Method / Key designs"
defines the forward (joint normalisation y = (a^S + a^L) / (n^S + n^L) with
a^L = phi_q(q) S_L, n^L = phi_q(q) z_L, S_L = sum over the linear set of
phi_k(k) v^T, z_L = sum of phi_k(k)).  Key design 5 (two-stage training):
its first stage, block-wise attention distillation, updates only phi_q and
phi_k by gradient steps on the distance between the hybrid output and the
teacher's softmax output, so the gradient of phi's parameters is the useful
first slice of a backward pass.

Nothing on the page writes the gradient out.  It follows from the forward by
the chain rule; for a loss L with upstream gradient g_i = dL/dy_i:

* only a^L and n^L depend on phi, so with den_i = n^S_i + n^L_i,
  dL/dphi_q(q_i) = (S_L g_i - z_L (g_i . y_i)) / den_i      (chunk t of i);
* S_L and z_L of chunk t collect the keys of its linear set, so a key j gets
  dL/dphi_k(k_j) = sum over chunks t whose linear set holds j of
                   (G_t v_j + h_t),
  G_t = sum_{i in t} phi_q(q_i) g_i^T / den_i  ([D', D]),
  h_t = -sum_{i in t} phi_q(q_i) (g_i . y_i) / den_i  ([D']);
* through phi(x) = [(x W_1 + b_1)^2, (x W_2 + b_2)^2] with u_p = x W_p + b_p:
  dL/du_p = 2 u_p * dL/dphi_p, dL/dW_p = sum_x x^T dL/du_p, dL/db_p = sum dL/du_p,
  summed over every token and, since W and b are per head, over the batch.

The tests pin this against central finite differences of the forward oracle
and against torch autograd of the masked pairwise definition.
"""
from __future__ import annotations

import numpy as np

from oracle.rehyat_oracle import _scale_of, chunk_table

__all__ = ["phi_grads_head", "phi_grads", "run_problem_grads"]


def phi_grads_head(q, k, v, Wq, bq, Wk, bk, dy, *, T, HW, Tc, To, causal, scale):
    """One (batch, head): returns dWq [2, D, D'/2], dbq [2, D'/2], dWk, dbk."""
    q, k, v, dy = (np.asarray(a, np.float64) for a in (q, k, v, dy))
    Wq, bq, Wk, bk = (np.asarray(a, np.float64) for a in (Wq, bq, Wk, bk))
    N, D = q.shape
    half = Wq.shape[2]
    uq = [q @ Wq[p] + bq[p] for p in range(2)]
    uk = [k @ Wk[p] + bk[p] for p in range(2)]
    fq = np.concatenate([u ** 2 for u in uq], axis=1)   # phi_q(q)  [N, D']
    fk = np.concatenate([u ** 2 for u in uk], axis=1)   # phi_k(k)  [N, D']
    dfq = np.zeros_like(fq)
    dfk = np.zeros_like(fk)
    for first, end, start in chunk_table(T, Tc, To):
        rows = slice(first * HW, end * HW)
        # Forward of this chunk (as in the factored form of the forward).
        logits = (q[rows] @ k[start * HW:end * HW].T) * scale
        E = np.exp(logits - logits.max(axis=1, keepdims=True))
        aS = E @ v[start * HW:end * HW]
        nS = E.sum(axis=1)
        before = np.arange(0, start * HW)
        after = np.arange(end * HW, N)
        lin = before if causal else np.concatenate([before, after])
        S_L = fk[lin].T @ v[lin]          # [D', D]
        z_L = fk[lin].sum(axis=0)         # [D']
        den = nS + fq[rows] @ z_L
        y = (aS + fq[rows] @ S_L) / den[:, None]
        # Backward.
        g = dy[rows]
        e = g / den[:, None]                      # g_i / den_i
        r = (g * y).sum(axis=1) / den             # (g_i . y_i) / den_i
        dfq[rows] += e @ S_L.T - r[:, None] * z_L[None, :]
        G = fq[rows].T @ e                        # dL/dS_L  [D', D]
        h = -(fq[rows] * r[:, None]).sum(axis=0)  # dL/dz_L  [D']
        dfk[lin] += v[lin] @ G.T + h[None, :]
    dWq = np.zeros_like(Wq)
    dbq = np.zeros_like(bq)
    dWk = np.zeros_like(Wk)
    dbk = np.zeros_like(bk)
    for p in range(2):
        cols = slice(p * half, (p + 1) * half)
        duq = 2.0 * uq[p] * dfq[:, cols]
        duk = 2.0 * uk[p] * dfk[:, cols]
        dWq[p] = q.T @ duq
        dbq[p] = duq.sum(axis=0)
        dWk[p] = k.T @ duk
        dbk[p] = duk.sum(axis=0)
    return dWq, dbq, dWk, dbk


def phi_grads(q, k, v, Wq, bq, Wk, bk, dy, *, T, HW, Tc, To, causal, scale=None):
    """[B, heads, N, D] inputs; per-head parameters [heads, 2, D, D'/2] and
    [heads, 2, D'/2].  Returns dict(dWq, dbq, dWk, dbk) summed over the batch."""
    q = np.asarray(q, np.float64)
    B, H, N, D = q.shape
    sc = _scale_of(D, scale)
    out = dict(dWq=np.zeros(np.shape(Wq)), dbq=np.zeros(np.shape(bq)),
               dWk=np.zeros(np.shape(Wk)), dbk=np.zeros(np.shape(bk)))
    for b in range(B):
        for h in range(H):
            g = phi_grads_head(q[b, h], k[b, h], v[b, h], Wq[h], bq[h], Wk[h], bk[h], dy[b, h],
                               T=T, HW=HW, Tc=Tc, To=To, causal=causal, scale=sc)
            for key, val in zip(("dWq", "dbq", "dWk", "dbk"), g):
                out[key][h] += val
    return out


def run_problem_grads(p, dy):
    """Gradients for one ``rehyat_inputs.Problem`` and upstream gradient dy."""
    return phi_grads(p.q, p.k, p.v, p.Wq, p.bq, p.Wk, p.bk, dy, T=p.T, HW=p.HW, Tc=p.Tc,
                     To=p.To, causal=p.causal)
