"""fp64 CPU oracle for ReHyAt's general feature map and for the hybrid
forward with the feature maps given as arrays.

TEST INFRASTRUCTURE, NOT PRODUCT CODE.  Only the tests and the CPU-baseline
leg of ``bench.py`` may import this module.  It shares no code with the CUDA
path (numpy and scipy's erf only, plus this package's forward oracle).

Source: "ReHyAt: Recurrent Hybrid Attention for Video Diffusion Transformers"
(papernotes.org note), Method, Key design 3: phi_q, phi_k map R^D to R^D'
through a light per-head embedding network (a grouped 1x1 convolution, i.e. a
per-head linear map, with a nonlinearity); its output psi is cut into P equal
parts and part i is raised to the i-th power, phi = [psi_1^1, ..., psi_P^P];
the note's experiments use a 2-layer MLP with degree 2 (P = 2).  Key design 1
gives the hybrid forward that consumes phi_q(q) and phi_k(k).

Readings where the page is silent (each stated in the design notes):
* the nonlinearity is GELU in its exact form, x * Phi(x) with Phi the
  standard normal CDF;
* the two layers are psi = GELU(x W_a + b_a) W_b + b_b with a hidden width
  D_h (the caller's choice; D_h = 3 D matches the note's ~2.4M extra
  parameters per converted block for 12 heads, D = D' = 128);
* a degree-1 part can be negative, so n^L can be negative; the joint
  normalisation is applied as written (no clamping).
"""
from __future__ import annotations

import math

import numpy as np
from scipy.special import erf

from oracle.rehyat_oracle import _empty_partials, _scale_of, chunk_table

__all__ = ["gelu", "feature_map_mlp", "hybrid_phi_given"]


def gelu(x):
    """GELU, exact form: x * Phi(x) = x/2 (1 + erf(x / sqrt(2)))."""
    x = np.asarray(x, np.float64)
    return 0.5 * x * (1.0 + erf(x / math.sqrt(2.0)))


def feature_map_mlp(x, Wa, ba, Wb, bb, P):
    """phi(x) = [psi_1^1, ..., psi_P^P], psi = GELU(x W_a + b_a) W_b + b_b
    (Key design 3).  x [n, D], W_a [D, D_h], b_a [D_h], W_b [D_h, D'], b_b [D'];
    D' a multiple of P.  Returns [n, D']."""
    x = np.asarray(x, np.float64)
    psi = gelu(x @ np.asarray(Wa, np.float64) + np.asarray(ba, np.float64))
    psi = psi @ np.asarray(Wb, np.float64) + np.asarray(bb, np.float64)
    width = psi.shape[1] // P
    return np.concatenate([psi[:, i * width:(i + 1) * width] ** (i + 1) for i in range(P)],
                          axis=1)


def _phi_given_head(q, k, v, fq, fk, T, HW, Tc, To, causal, scale):
    """One (batch, head), factored form (Key designs 1, 2, 4): per chunk, the
    window softmax and the linear state summed over the linear set, with the
    feature maps given as arrays fq = phi_q(q), fk = phi_k(k)."""
    N, D = q.shape
    y = np.zeros((N, D))
    parts = _empty_partials(N, D)
    for first, end, start in chunk_table(T, Tc, To):
        rows = slice(first * HW, end * HW)
        logits = (q[rows] @ k[start * HW:end * HW].T) * scale
        c = logits.max(axis=1)
        E = np.exp(logits - c[:, None])
        aS = E @ v[start * HW:end * HW]
        nS = E.sum(axis=1)
        before = np.arange(0, start * HW)
        after = np.arange(end * HW, N)
        lin = before if causal else np.concatenate([before, after])
        S_L = fk[lin].T @ v[lin]
        z_L = fk[lin].sum(axis=0)
        aL = fq[rows] @ S_L
        nL = fq[rows] @ z_L
        y[rows] = (aS + aL) / (nS + nL)[:, None]
        parts["aS"][rows], parts["nS"][rows], parts["c"][rows] = aS, nS, c
        parts["aL"][rows], parts["nL"][rows] = aL, nL
    return y, parts


def hybrid_phi_given(q, k, v, fq, fk, *, T, HW, Tc, To, causal, scale=None):
    """[B, heads, N, D] q, k, v and [B, heads, N, D'] feature maps.  Returns
    (y [B,h,N,D], partials dict)."""
    q, k, v, fq, fk = (np.asarray(a, np.float64) for a in (q, k, v, fq, fk))
    B, H, N, D = q.shape
    sc = _scale_of(D, scale)
    y = np.zeros((B, H, N, D))
    parts = dict(aS=np.zeros((B, H, N, D)), nS=np.zeros((B, H, N)), c=np.zeros((B, H, N)),
                 aL=np.zeros((B, H, N, D)), nL=np.zeros((B, H, N)))
    for b in range(B):
        for h in range(H):
            yy, pp = _phi_given_head(q[b, h], k[b, h], v[b, h], fq[b, h], fk[b, h], T, HW, Tc,
                                     To, causal, sc)
            y[b, h] = yy
            for key in parts:
                parts[key][b, h] = pp[key]
    return y, parts
