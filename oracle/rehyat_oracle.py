"""fp64 CPU oracle for ReHyAt's temporally chunked hybrid attention (forward).

TEST INFRASTRUCTURE, NOT PRODUCT CODE.  Only the tests, the package's
``smoke()`` check and the CPU-baseline leg of ``bench.py`` may import this
module.  It shares no code with the CUDA path (it imports numpy only) and is
written for a reader checking it against the pages by eye, not for speed.

Source: "ReHyAt: Recurrent Hybrid Attention for Video Diffusion Transformers"
(papernotes.org note of the CVPR 2026 paper), section "Method / Key designs":

* Key design 1: the N = T*H*W tokens are put in time-major order and cut into
  chunks of N' = T_c*H*W tokens.  Queries of chunk t use softmax over a set
  T^S_t and linear attention over the rest T^L_t; the two branches keep their
  own numerators a and denominators n and are normalised jointly,
  y = (a^S + a^L) / (n^S + n^L).  a^S sums exp(q k^T / sqrt(D) - c_t) v over
  T^S_t; a^L = phi_q(q) (sum over T^L_t of phi_k(k) v^T).
* Key design 2: the softmax set also covers the T_o slices before the chunk:
  T^S_t = { j : max(t N' - T_o H W, 0) <= j < (t+1) N' }.
* Key design 3: phi is a learnable polynomial map; here in the closed form
  phi(x) = [(x W_1 + b_1)^2, (x W_2 + b_2)^2] with total width D'.
* Key design 4: the causal form keeps only earlier tokens in the linear set,
  T^L_t = { j : j < max(t N' - T_o H W, 0) }, and unrolls into a chunk-wise
  RNN whose state (s_t, z_t) accumulates phi_k(k) v^T and phi_k(k); the
  non-recursive causal form and the RNN are stated to be equivalent.

Readings where the page is silent or inconsistent (each is tested):

* c_t is the per-query maximum of the scaled logits over T^S_t.  The linear
  branch is not multiplied by exp(-c_t), so this choice changes y.
* n^S and n^L are a^S and a^L with v replaced by 1.
* phi_q sees the raw q (no 1/sqrt(D)); the softmax logits are scaled.
* The printed RNN update adds the whole softmax set T^S_t into the state,
  which would count the T_o overlap slices twice when T_o > 0.  This oracle
  follows the set definition instead: after a chunk, the state absorbs exactly
  the slices that leave the softmax window.  For T_o = 0 both agree.
* When T is not a multiple of T_c the last chunk is shorter.  When T_o > T_c
  the window reaches back over several earlier chunks (clipped at slice 0).

Three independent forms of the same function are given:

* ``hybrid_pairwise``: per query, the explicit masked weights over all keys
  (O(N^2); tiny inputs only).
* ``hybrid_factored``: per chunk, window softmax plus the linear state summed
  directly over the linear set (no total-minus-window subtraction).
* ``hybrid_rnn`` / ``ChunkRNN``: chunk by chunk with a running (s, z) and a
  ring of the last T_o slices, exactly as streamed.

All arithmetic is float64.  Inputs are taken as exact values (bf16 inputs
arrive already rounded by the input generator).
"""
from __future__ import annotations

import math

import numpy as np

__all__ = [
    "feature_map", "chunk_table", "hybrid_pairwise", "hybrid_factored",
    "hybrid_rnn", "ChunkRNN", "full_softmax", "run_problem",
]


def feature_map(x, W, b):
    """phi(x) = [(x W_1 + b_1)^2, (x W_2 + b_2)^2] (Key design 3 of the
    papernotes.org ReHyAt note, in its degree-2, two-part closed form).

    x: [n, D]; W: [2, D, D'/2]; b: [2, D'/2]  ->  [n, D'].
    """
    x = np.asarray(x, np.float64)
    W = np.asarray(W, np.float64)
    b = np.asarray(b, np.float64)
    psi_1 = x @ W[0] + b[0]
    psi_2 = x @ W[1] + b[1]
    return np.concatenate([psi_1 ** 2, psi_2 ** 2], axis=1)


def chunk_table(T, Tc, To):
    """Per chunk t: (first slice, end slice (exclusive), softmax window start).

    Chunk t holds slices [t*Tc, min(T, (t+1)*Tc)); its softmax keys start
    T_o slices earlier, clipped at 0 (Key designs 1 and 2).
    """
    rows = []
    for t in range(-(-T // Tc)):
        first = t * Tc
        end = min(T, first + Tc)
        rows.append((first, end, max(first - To, 0)))
    return rows


def _empty_partials(N, D):
    return dict(aS=np.zeros((N, D)), nS=np.zeros(N), c=np.zeros(N),
                aL=np.zeros((N, D)), nL=np.zeros(N))


# --------------------------------------------------------------------------
# Form (i): explicit masked weights, one query at a time.
# --------------------------------------------------------------------------
def _pairwise_head(q, k, v, Wq, bq, Wk, bk, HW, Tc, To, causal, scale):
    N, D = q.shape
    Np = Tc * HW                      # tokens per chunk, N'
    fq = feature_map(q, Wq, bq)
    fk = feature_map(k, Wk, bk)
    y = np.zeros((N, D))
    parts = _empty_partials(N, D)
    j = np.arange(N)
    for i in range(N):
        t = i // Np                   # chunk of query i
        lo = max(t * Np - To * HW, 0)
        hi = min((t + 1) * Np, N)
        soft = (j >= lo) & (j < hi)
        lin = (j < lo) if causal else ~soft
        logits = (k @ q[i]) * scale
        c = logits[soft].max()
        w_soft = np.where(soft, np.exp(np.where(soft, logits - c, 0.0)), 0.0)
        w_lin = np.where(lin, fk @ fq[i], 0.0)
        w = w_soft + w_lin
        y[i] = (w @ v) / w.sum()
        parts["aS"][i] = w_soft @ v
        parts["nS"][i] = w_soft.sum()
        parts["c"][i] = c
        parts["aL"][i] = w_lin @ v
        parts["nL"][i] = w_lin.sum()
    return y, parts


# --------------------------------------------------------------------------
# Form (ii): per chunk, window softmax + linear state over the linear set.
# --------------------------------------------------------------------------
def _factored_head(q, k, v, Wq, bq, Wk, bk, T, HW, Tc, To, causal, scale, chunks=None,
                   q_logit=None, k_logit=None):
    # q_logit, k_logit: the vectors the softmax logits are formed from when
    # they differ from q, k (the fp8 softmax variant); phi always sees q, k.
    N, D = q.shape
    ql = q if q_logit is None else q_logit
    kl = k if k_logit is None else k_logit
    y = np.zeros((N, D))
    parts = _empty_partials(N, D)
    for t, (first, end, start) in enumerate(chunk_table(T, Tc, To)):
        if chunks is not None and t not in chunks:
            continue
        rows = slice(first * HW, end * HW)
        Qc = q[rows]
        Kw, Vw = k[start * HW:end * HW], v[start * HW:end * HW]
        logits = (ql[rows] @ kl[start * HW:end * HW].T) * scale
        c = logits.max(axis=1)
        E = np.exp(logits - c[:, None])
        aS = E @ Vw
        nS = E.sum(axis=1)
        before = np.arange(0, start * HW)
        after = np.arange(end * HW, N)
        lin = before if causal else np.concatenate([before, after])
        fk = feature_map(k[lin], Wk, bk)
        S_L = fk.T @ v[lin]              # [D', D]
        z_L = fk.sum(axis=0)             # [D']
        fq = feature_map(Qc, Wq, bq)
        aL = fq @ S_L
        nL = fq @ z_L
        y[rows] = (aS + aL) / (nS + nL)[:, None]
        parts["aS"][rows], parts["nS"][rows], parts["c"][rows] = aS, nS, c
        parts["aL"][rows], parts["nL"][rows] = aL, nL
    return y, parts


# --------------------------------------------------------------------------
# Form (iii): chunk-wise RNN with constant-size state.
# --------------------------------------------------------------------------
class ChunkRNN:
    """Causal chunk-wise recurrence of Key design 4, one head.

    State: s [D', D], z [D'], the keys/values of the last <= T_o slices
    (``ring``) and the count of slices consumed so far.  ``step`` takes the
    q, k, v rows of the next chunk (whole slices, time-major) and returns
    y and the branch partials for those rows.
    """

    def __init__(self, D, Dp, HW, To, Wq, bq, Wk, bk, scale):
        self.HW, self.To, self.scale = HW, To, scale
        self.Wq, self.bq, self.Wk, self.bk = Wq, bq, Wk, bk
        self.s = np.zeros((Dp, D))
        self.z = np.zeros(Dp)
        self.ring_k = np.zeros((0, D))
        self.ring_v = np.zeros((0, D))
        self.seen = 0

    def step(self, qc, kc, vc):
        HW = self.HW
        n_slices = qc.shape[0] // HW
        Kw = np.concatenate([self.ring_k, np.asarray(kc, np.float64)])
        Vw = np.concatenate([self.ring_v, np.asarray(vc, np.float64)])
        logits = (np.asarray(qc, np.float64) @ Kw.T) * self.scale
        c = logits.max(axis=1)
        E = np.exp(logits - c[:, None])
        aS, nS = E @ Vw, E.sum(axis=1)
        fq = feature_map(qc, self.Wq, self.bq)
        aL, nL = fq @ self.s, fq @ self.z
        y = (aS + aL) / (nS + nL)[:, None]
        # Slices that leave the softmax window are folded into the state;
        # the last min(T_o, seen) slices stay in the ring.
        self.seen += n_slices
        keep = min(self.To, self.seen)
        leave = Kw.shape[0] // HW - keep
        fk = feature_map(Kw[:leave * HW], self.Wk, self.bk)
        self.s = self.s + fk.T @ Vw[:leave * HW]
        self.z = self.z + fk.sum(axis=0)
        self.ring_k, self.ring_v = Kw[leave * HW:], Vw[leave * HW:]
        return y, dict(aS=aS, nS=nS, c=c, aL=aL, nL=nL)


def _rnn_head(q, k, v, Wq, bq, Wk, bk, T, HW, Tc, To, scale):
    N, D = q.shape
    Dp = 2 * np.asarray(Wq).shape[-1]
    rnn = ChunkRNN(D, Dp, HW, To, Wq, bq, Wk, bk, scale)
    ys, parts = [], {key: [] for key in ("aS", "nS", "c", "aL", "nL")}
    for first in range(0, T, Tc):
        rows = slice(first * HW, min(T, first + Tc) * HW)
        y, p = rnn.step(q[rows], k[rows], v[rows])
        ys.append(y)
        for key in parts:
            parts[key].append(p[key])
    return np.concatenate(ys), {key: np.concatenate(val) for key, val in parts.items()}


# --------------------------------------------------------------------------
# Whole-tensor drivers ([B, heads, N, D] inputs).
# --------------------------------------------------------------------------
def _f64(a):
    return np.asarray(a, np.float64)


def _over_heads(fn, q, k, v, Wq, bq, Wk, bk, heads_subset=None):
    q, k, v = _f64(q), _f64(k), _f64(v)
    Wq, bq, Wk, bk = _f64(Wq), _f64(bq), _f64(Wk), _f64(bk)
    B, H, N, D = q.shape
    y = np.zeros((B, H, N, D))
    parts = dict(aS=np.zeros((B, H, N, D)), nS=np.zeros((B, H, N)),
                 c=np.zeros((B, H, N)), aL=np.zeros((B, H, N, D)),
                 nL=np.zeros((B, H, N)))
    pairs = [(b, h) for b in range(B) for h in range(H)]
    if heads_subset is not None:
        pairs = [pairs[i] for i in heads_subset]
    for b, h in pairs:
        yy, pp = fn(q[b, h], k[b, h], v[b, h], Wq[h], bq[h], Wk[h], bk[h])
        y[b, h] = yy
        for key in parts:
            parts[key][b, h] = pp[key]
    return y, parts


def _scale_of(D, scale):
    return 1.0 / math.sqrt(D) if scale is None else float(scale)


def hybrid_pairwise(q, k, v, Wq, bq, Wk, bk, *, T, HW, Tc, To, causal, scale=None):
    """Form (i).  Returns (y [B,h,N,D], partials dict)."""
    sc = _scale_of(q.shape[-1], scale)
    fn = lambda *a: _pairwise_head(*a, HW, Tc, To, causal, sc)
    return _over_heads(fn, q, k, v, Wq, bq, Wk, bk)


def hybrid_factored(q, k, v, Wq, bq, Wk, bk, *, T, HW, Tc, To, causal, scale=None,
                    heads_subset=None, chunks_subset=None):
    """Form (ii).  ``heads_subset`` (flattened (b, h) indices) and
    ``chunks_subset`` (chunk indices) restrict the work to a sample; rows
    outside it are left zero.  Returns (y, partials)."""
    sc = _scale_of(q.shape[-1], scale)
    fn = lambda *a: _factored_head(*a, T, HW, Tc, To, causal, sc, chunks_subset)
    return _over_heads(fn, q, k, v, Wq, bq, Wk, bk, heads_subset)


def hybrid_rnn(q, k, v, Wq, bq, Wk, bk, *, T, HW, Tc, To, scale=None):
    """Form (iii), causal only.  Returns (y, partials)."""
    sc = _scale_of(q.shape[-1], scale)
    fn = lambda *a: _rnn_head(*a, T, HW, Tc, To, sc)
    return _over_heads(fn, q, k, v, Wq, bq, Wk, bk)


def full_softmax(q, k, v, scale=None):
    """Plain softmax attention over all keys (the dense comparator)."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    sc = _scale_of(q.shape[-1], scale)
    logits = np.einsum("bhnd,bhmd->bhnm", q, k) * sc
    logits -= logits.max(axis=-1, keepdims=True)
    E = np.exp(logits)
    return np.einsum("bhnm,bhmd->bhnd", E, v) / E.sum(axis=-1)[..., None]


def run_problem(p, form="factored", heads_subset=None, chunks_subset=None):
    """Run one ``rehyat_inputs.Problem`` through the chosen form."""
    kw = dict(T=p.T, HW=p.HW, Tc=p.Tc, To=p.To)
    args = (p.q, p.k, p.v, p.Wq, p.bq, p.Wk, p.bk)
    if form == "pairwise":
        return hybrid_pairwise(*args, causal=p.causal, **kw)
    if form == "factored":
        return hybrid_factored(*args, causal=p.causal, heads_subset=heads_subset,
                               chunks_subset=chunks_subset, **kw)
    if form == "rnn":
        if not p.causal:
            raise ValueError("the RNN form is causal")
        return hybrid_rnn(*args, **kw)
    raise ValueError(form)
