"""fp64 CPU oracle for the fp8 softmax-branch variant of ReHyAt's hybrid
attention.

TEST INFRASTRUCTURE, NOT PRODUCT CODE.  Only the tests and the CPU-baseline
leg of ``bench.py`` may import this module.  It shares no code with the CUDA
path (numpy only, plus this package's forward oracle).

The variant: the softmax branch's logits q.k^T (Key designs 1 and 2 of "ReHyAt:
Recurrent Hybrid Attention for Video Diffusion Transformers", papernotes.org
note) are formed from q and k rounded to the 8-bit float format E4M3 (1 sign,
4 exponent bits with bias 7, 3 fraction bits; no infinities; largest finite
value 448; subnormals down to 2^-9), round to nearest even, values beyond
+-448 saturating to +-448 and NaN kept.  Everything else -- the exponentials,
the P.V product with the bf16 values, the feature maps of q and k, the linear
state and the joint normalisation -- is the forward of the main oracle.

Readings (the pages give no fp8 variant; the scope table asks for an fp8
q.k^T / P.V variant of the softmax branch checked at a looser stated bar):
* no scaling before the cast (unit scale): the heads' q and k are O(1);
* only q.k^T is in fp8; P.V keeps bf16 P and V (see the design notes).
"""
from __future__ import annotations

import numpy as np

from oracle.rehyat_oracle import _f64, _factored_head, _scale_of

__all__ = ["e4m3_round", "hybrid_fp8_qk"]

E4M3_MAX = 448.0
E4M3_MIN_NORMAL_EXP = -6   # smallest normal: 2^-6
E4M3_FRACTION_BITS = 3


def e4m3_round(x):
    """Nearest E4M3 value (ties to even), saturating at +-448, as float64."""
    x = np.asarray(x, np.float64)
    a = np.abs(x)
    with np.errstate(divide="ignore", invalid="ignore"):
        e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    e = np.maximum(e, E4M3_MIN_NORMAL_EXP)          # subnormal range shares 2^-6's spacing
    spacing = np.exp2(e - E4M3_FRACTION_BITS)       # distance between neighbours
    r = np.round(a / spacing) * spacing             # numpy rounds halves to even
    r = np.minimum(r, E4M3_MAX)
    r = np.copysign(r, x)
    return np.where(np.isnan(x), np.nan, r)


def hybrid_fp8_qk(q, k, v, Wq, bq, Wk, bk, *, T, HW, Tc, To, causal, scale=None,
                  heads_subset=None, chunks_subset=None):
    """The factored forward with the softmax logits formed from
    e4m3_round(q) and e4m3_round(k) (the feature maps keep q and k).
    ``heads_subset`` / ``chunks_subset`` restrict the work to a sample as in
    ``hybrid_factored``.  Returns (y [B,h,N,D], partials dict)."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    Wq, bq, Wk, bk = _f64(Wq), _f64(bq), _f64(Wk), _f64(bk)
    q8, k8 = e4m3_round(q), e4m3_round(k)
    sc = _scale_of(q.shape[-1], scale)
    B, H, N, D = q.shape
    y = np.zeros((B, H, N, D))
    parts = dict(aS=np.zeros((B, H, N, D)), nS=np.zeros((B, H, N)), c=np.zeros((B, H, N)),
                 aL=np.zeros((B, H, N, D)), nL=np.zeros((B, H, N)))
    pairs = [(b, h) for b in range(B) for h in range(H)]
    if heads_subset is not None:
        pairs = [pairs[i] for i in heads_subset]
    for b, h in pairs:
        yy, pp = _factored_head(q[b, h], k[b, h], v[b, h], Wq[h], bq[h], Wk[h], bk[h], T, HW,
                                Tc, To, causal, sc, chunks_subset, q8[b, h], k8[b, h])
        y[b, h] = yy
        for key in parts:
            parts[key][b, h] = pp[key]
    return y, parts
