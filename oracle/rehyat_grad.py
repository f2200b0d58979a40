"""fp64 CPU oracle for the full backward of ReHyAt's chunked hybrid attention:
the gradients with respect to q, k, v and the feature-map parameters.

TEST INFRASTRUCTURE, NOT PRODUCT CODE.  Only the tests and the CPU-baseline
leg of ``bench.py`` may import this module.  It shares no code with the CUDA
path (numpy only, plus the forward oracle of this package for the chunk
table).

Source: "ReHyAt: Recurrent Hybrid Attention for Video Diffusion Transformers"
(papernotes.org note of the CVPR 2026 paper), section "Method / Key designs".
Key designs 1-4 define the forward; Key design 5 (two-stage training) says the
second stage fine-tunes the whole converted model, so the gradient flows
through q, k and v of every hybrid block, not only through phi.

The page does not write the backward out.  It is the chain rule applied to
the forward as defined there (and as the forward oracle computes it).  For
a query i of chunk t, with window W_t (its softmax keys) and linear set L_t:

  s_ij = scale q_i.k_j (j in W_t),  c_i = max_j s_ij,  e_ij = exp(s_ij - c_i)
  aS_i = sum_j e_ij v_j,  nS_i = sum_j e_ij
  aL_i = phi_q(q_i) S_L,  nL_i = phi_q(q_i).z_L,  S_L = sum_{L_t} phi_k(k) v^T,
  z_L = sum_{L_t} phi_k(k)
  den_i = nS_i + nL_i,  y_i = (aS_i + aL_i) / den_i

With g_i = dL/dy_i, write gh_i = g_i / den_i and r_i = (g_i.y_i) / den_i:

* dL/daS_i = dL/daL_i = gh_i,  dL/dnS_i = dL/dnL_i = -r_i.
* Softmax branch: dL/de_ij = gh_i.v_j - r_i.  c_i is not a free stabiliser
  here (the linear branch is not multiplied by exp(-c_i)), so the gradient
  also flows through the maximum: dL/dc_i = -sum_j e_ij (gh_i.v_j - r_i)
  = -(gh_i.aS_i - r_i nS_i) =: -Dc_i, and c_i moves with the logit of its
  arg-max key j*_i.  Hence
      dL/ds_ij = e_ij (gh_i.v_j - r_i) - [j = j*_i] Dc_i,
      dq_i += scale sum_j dL/ds_ij k_j,  dk_j += scale sum_i dL/ds_ij q_i,
      dv_j += sum_i e_ij gh_i.
  (With no linear branch, Dc_i = 0 and this is the usual softmax backward.)
  Where two window keys tie for the maximum the function has a kink; this
  oracle sends the maximum's gradient to the first of them (lowest index).
* Linear branch: dL/dphi_q(q_i) = S_L gh_i - r_i z_L; the chunk's state
  receives G_t = sum_{i in t} phi_q(q_i) gh_i^T and h_t = -sum_{i in t}
  phi_q(q_i) r_i, so a key j of L_t gets dL/dphi_k(k_j) += G_t v_j + h_t and
  dv_j += G_t^T phi_k(k_j).
* Through phi(x) = [(x W_1 + b_1)^2, (x W_2 + b_2)^2], u_p = x W_p + b_p:
  dL/du_p = 2 u_p * dL/dphi_p; dx += sum_p dL/du_p W_p^T;
  dW_p = sum_x x^T dL/du_p, db_p = sum dL/du_p (summed over the batch too,
  since W and b are per head).

The tests pin this against central finite differences of the pairwise
forward (a separate implementation that never forms the factored sums),
torch fp64 autograd of the masked definition, torch's softmax attention
backward for the no-linear-branch case, and two exact identities of the
forward: y(V + 1 beta^T) = y(V) + beta gives sum_j dv_j = sum_i g_i, and
y(alpha V) = alpha y(V) gives sum_j v_j.dv_j = sum_i g_i.y_i.
"""
from __future__ import annotations

import numpy as np

from oracle.rehyat_oracle import _scale_of, chunk_table

__all__ = ["grads_head", "hybrid_grads", "run_problem_full_grads", "forward_aux_head"]


def forward_aux_head(q, k, v, Wq, bq, Wk, bk, *, T, HW, Tc, To, causal, scale):
    """Forward of one (batch, head) with the per-query quantities the backward
    uses: y [N, D], c [N] (row max of the scaled logits over the window),
    nS, nL, den [N], aS, aL [N, D], and the window arg-max key index [N]."""
    q, k, v = (np.asarray(a, np.float64) for a in (q, k, v))
    Wq, bq, Wk, bk = (np.asarray(a, np.float64) for a in (Wq, bq, Wk, bk))
    N, D = q.shape
    fq = np.concatenate([(q @ Wq[p] + bq[p]) ** 2 for p in range(2)], axis=1)
    fk = np.concatenate([(k @ Wk[p] + bk[p]) ** 2 for p in range(2)], axis=1)
    out = dict(y=np.zeros((N, D)), c=np.zeros(N), nS=np.zeros(N), nL=np.zeros(N),
               den=np.zeros(N), aS=np.zeros((N, D)), aL=np.zeros((N, D)),
               jstar=np.zeros(N, np.int64))
    for first, end, start in chunk_table(T, Tc, To):
        rows = slice(first * HW, end * HW)
        win = slice(start * HW, end * HW)
        logits = (q[rows] @ k[win].T) * scale
        c = logits.max(axis=1)
        E = np.exp(logits - c[:, None])
        lin = np.arange(0, start * HW) if causal else \
            np.concatenate([np.arange(0, start * HW), np.arange(end * HW, N)])
        S_L = fk[lin].T @ v[lin]
        z_L = fk[lin].sum(axis=0)
        aS = E @ v[win]
        nS = E.sum(axis=1)
        aL = fq[rows] @ S_L
        nL = fq[rows] @ z_L
        den = nS + nL
        out["y"][rows] = (aS + aL) / den[:, None]
        out["c"][rows] = c
        out["nS"][rows] = nS
        out["nL"][rows] = nL
        out["den"][rows] = den
        out["aS"][rows] = aS
        out["aL"][rows] = aL
        out["jstar"][rows] = start * HW + np.argmax(logits, axis=1)  # first of any ties
    return out


def grads_head(q, k, v, Wq, bq, Wk, bk, dy, *, T, HW, Tc, To, causal, scale):
    """One (batch, head): returns dict(dq, dk, dv [N, D], dWq, dWk [2, D, D'/2],
    dbq, dbk [2, D'/2])."""
    q, k, v, dy = (np.asarray(a, np.float64) for a in (q, k, v, dy))
    Wq, bq, Wk, bk = (np.asarray(a, np.float64) for a in (Wq, bq, Wk, bk))
    N, D = q.shape
    half = Wq.shape[2]
    uq = [q @ Wq[p] + bq[p] for p in range(2)]
    uk = [k @ Wk[p] + bk[p] for p in range(2)]
    fq = np.concatenate([u ** 2 for u in uq], axis=1)   # phi_q(q)  [N, D']
    fk = np.concatenate([u ** 2 for u in uk], axis=1)   # phi_k(k)  [N, D']
    dq = np.zeros_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    dfq = np.zeros_like(fq)
    dfk = np.zeros_like(fk)
    for first, end, start in chunk_table(T, Tc, To):
        rows = slice(first * HW, end * HW)
        win = slice(start * HW, end * HW)
        lin = np.arange(0, start * HW) if causal else \
            np.concatenate([np.arange(0, start * HW), np.arange(end * HW, N)])
        # Forward of this chunk.
        logits = (q[rows] @ k[win].T) * scale            # s_ij
        jmax = np.argmax(logits, axis=1)                  # j*_i (first of any ties)
        c = logits[np.arange(logits.shape[0]), jmax]
        E = np.exp(logits - c[:, None])                   # e_ij
        aS = E @ v[win]
        nS = E.sum(axis=1)
        S_L = fk[lin].T @ v[lin]                          # [D', D]
        z_L = fk[lin].sum(axis=0)                         # [D']
        den = nS + fq[rows] @ z_L
        y = (aS + fq[rows] @ S_L) / den[:, None]
        # Backward: the joint normalisation.
        g = dy[rows]
        gh = g / den[:, None]                             # dL/daS = dL/daL
        r = (g * y).sum(axis=1) / den                     # -dL/dnS = -dL/dnL
        # Softmax branch, through e_ij and through the maximum c_i.
        dE = gh @ v[win].T - r[:, None]                   # dL/de_ij
        Dc = (gh * aS).sum(axis=1) - r * nS               # -dL/dc_i
        dS = E * dE
        dS[np.arange(dS.shape[0]), jmax] -= Dc
        dq[rows] += scale * (dS @ k[win])
        dk[win] += scale * (dS.T @ q[rows])
        dv[win] += E.T @ gh
        # Linear branch.
        dfq[rows] += gh @ S_L.T - r[:, None] * z_L[None, :]
        G = fq[rows].T @ gh                               # dL/dS_L  [D', D]
        h = -(fq[rows] * r[:, None]).sum(axis=0)          # dL/dz_L  [D']
        dfk[lin] += v[lin] @ G.T + h[None, :]
        dv[lin] += fk[lin] @ G
    # Through the feature maps.
    out = dict(dq=dq, dk=dk, dv=dv, dWq=np.zeros_like(Wq), dbq=np.zeros_like(bq),
               dWk=np.zeros_like(Wk), dbk=np.zeros_like(bk))
    for p in range(2):
        cols = slice(p * half, (p + 1) * half)
        duq = 2.0 * uq[p] * dfq[:, cols]
        duk = 2.0 * uk[p] * dfk[:, cols]
        out["dq"] += duq @ Wq[p].T
        out["dk"] += duk @ Wk[p].T
        out["dWq"][p] = q.T @ duq
        out["dbq"][p] = duq.sum(axis=0)
        out["dWk"][p] = k.T @ duk
        out["dbk"][p] = duk.sum(axis=0)
    return out


def hybrid_grads(q, k, v, Wq, bq, Wk, bk, dy, *, T, HW, Tc, To, causal, scale=None):
    """[B, heads, N, D] inputs, per-head parameters [heads, 2, D, D'/2] and
    [heads, 2, D'/2].  Returns dict(dq, dk, dv [B, heads, N, D], dWq, dbq, dWk,
    dbk summed over the batch)."""
    q = np.asarray(q, np.float64)
    B, H, N, D = q.shape
    sc = _scale_of(D, scale)
    out = dict(dq=np.zeros((B, H, N, D)), dk=np.zeros((B, H, N, D)), dv=np.zeros((B, H, N, D)),
               dWq=np.zeros(np.shape(Wq)), dbq=np.zeros(np.shape(bq)),
               dWk=np.zeros(np.shape(Wk)), dbk=np.zeros(np.shape(bk)))
    for b in range(B):
        for h in range(H):
            g = grads_head(q[b, h], k[b, h], v[b, h], Wq[h], bq[h], Wk[h], bk[h], dy[b, h],
                           T=T, HW=HW, Tc=Tc, To=To, causal=causal, scale=sc)
            for key in ("dq", "dk", "dv"):
                out[key][b, h] = g[key]
            for key in ("dWq", "dbq", "dWk", "dbk"):
                out[key][h] += g[key]
    return out


def run_problem_full_grads(p, dy):
    """Gradients for one ``rehyat_inputs.Problem`` and upstream gradient dy."""
    return hybrid_grads(p.q, p.k, p.v, p.Wq, p.bq, p.Wk, p.bk, dy, T=p.T, HW=p.HW, Tc=p.Tc,
                        To=p.To, causal=p.causal)
