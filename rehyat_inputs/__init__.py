"""Seeded synthetic inputs for ReHyAt's chunked hybrid attention.

This module only draws random numbers and lays them out. It holds none of the
method's arithmetic: both the fp64 CPU oracle and the CUDA path consume the
arrays it returns, so the two sides always see bit-identical inputs.

Workload shapes follow the ReHyAt pages: a 21-slice latent of 20x30 or 30x52
tokens (a 5 s Wan2.1 clip at 320x480 / 480x832, papernotes.org "ReHyAt" page,
Experiments; sciencestack.ai page, Figure 4 caption), 12 heads of width 128,
chunks of T_c slices with T_o overlap slices (papernotes.org page, Key designs
1 and 2), and a polynomial feature map phi(x) = [(x W_1 + b_1)^2,
(x W_2 + b_2)^2] (same page, Key design 3).

Recipe (all draws are float32 from numpy ``Generator(Philox(seed))``):

* ``dist="scaled"``: Q, K, V ~ N(0, 1) times a per-(tensor, head) factor
  s ~ U(0.5, 2) that is shared across the batch.
* ``dist="normal"``: Q, K, V ~ N(0, 1).
* ``dist="lowrank"``: per head a shared G in R^{8 x D} with entries
  N(0, 1/8); Q = U_q G + eps, K = U_k G + eps with U ~ N(0, 1) and
  eps ~ N(0, 0.3^2); V ~ N(0, 1).  This sharpens the softmax.
* phi weights, per head in the fixed order Wq1, Wq2, bq1, bq2, Wk1, Wk2,
  bk1, bk2, each ~ N(0, phi_std^2) (phi_std = 0.1 by default).

In bf16 mode Q, K, V and the W matrices are rounded to bf16 (round to
nearest even) and handed to both sides as those exact values; b stays fp32.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import numpy as np

__all__ = ["Problem", "make_problem", "round_to_bf16", "bf16_bits", "CONFIGS",
           "config_problem"]


def round_to_bf16(x: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest bf16 value (ties to even).

    Returns float32 values that are exactly representable in bf16.
    """
    x = np.ascontiguousarray(x, dtype=np.float32)
    bits = x.view(np.uint32).astype(np.uint64)
    rounding = ((bits >> 16) & 1) + 0x7FFF
    out = (((bits + rounding) >> 16) << 16).astype(np.uint32)
    return out.view(np.float32).reshape(x.shape)


def bf16_bits(x: np.ndarray) -> np.ndarray:
    """The upper 16 bits of float32 values that are already bf16-exact."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    return (x.view(np.uint32) >> 16).astype(np.uint16).reshape(x.shape)


@dataclasses.dataclass
class Problem:
    """One seeded problem instance.

    Tensors are float32 numpy arrays; in bf16 mode their values are
    bf16-exact.  Layout: q, k, v are [B, heads, N, D] with N = T*Hs*Ws in
    time-major order (slice, row, column).  Wq, Wk are [heads, 2, D, Dp/2];
    bq, bk are [heads, 2, Dp/2].
    """
    batch: int
    heads: int
    T: int
    Hs: int
    Ws: int
    D: int
    Dp: int
    Tc: int
    To: int
    causal: bool
    dtype: str  # "f32" or "bf16"
    q: np.ndarray
    k: np.ndarray
    v: np.ndarray
    Wq: np.ndarray
    bq: np.ndarray
    Wk: np.ndarray
    bk: np.ndarray
    seed: int = 0
    name: str = ""

    @property
    def HW(self) -> int:
        return self.Hs * self.Ws

    @property
    def N(self) -> int:
        return self.T * self.Hs * self.Ws

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.D)


def _draw_qkv(g: np.random.Generator, shape, dist: str, heads: int, D: int):
    B, h, N, _ = shape
    if dist == "normal":
        q = g.standard_normal(shape, dtype=np.float32)
        k = g.standard_normal(shape, dtype=np.float32)
        v = g.standard_normal(shape, dtype=np.float32)
    elif dist == "scaled":
        q = g.standard_normal(shape, dtype=np.float32)
        k = g.standard_normal(shape, dtype=np.float32)
        v = g.standard_normal(shape, dtype=np.float32)
        s = g.uniform(0.5, 2.0, size=(3, heads)).astype(np.float32)
        q *= s[0][None, :, None, None]
        k *= s[1][None, :, None, None]
        v *= s[2][None, :, None, None]
    elif dist == "lowrank":
        rank = 8
        G = (g.standard_normal((heads, rank, D), dtype=np.float32)
             * np.float32(1.0 / math.sqrt(rank)))
        uq = g.standard_normal((B, h, N, rank), dtype=np.float32)
        uk = g.standard_normal((B, h, N, rank), dtype=np.float32)
        q = np.einsum("bhnr,hrd->bhnd", uq, G, optimize=True).astype(np.float32)
        k = np.einsum("bhnr,hrd->bhnd", uk, G, optimize=True).astype(np.float32)
        q += g.standard_normal(shape, dtype=np.float32) * np.float32(0.3)
        k += g.standard_normal(shape, dtype=np.float32) * np.float32(0.3)
        v = g.standard_normal(shape, dtype=np.float32)
    else:
        raise ValueError(f"unknown dist {dist!r}")
    return q, k, v


def _draw_phi(g: np.random.Generator, heads: int, D: int, Dp: int, std: float):
    half = Dp // 2
    Wq = np.empty((heads, 2, D, half), np.float32)
    bq = np.empty((heads, 2, half), np.float32)
    Wk = np.empty((heads, 2, D, half), np.float32)
    bk = np.empty((heads, 2, half), np.float32)
    for hh in range(heads):
        for dst in (Wq[hh, 0], Wq[hh, 1], bq[hh, 0], bq[hh, 1],
                    Wk[hh, 0], Wk[hh, 1], bk[hh, 0], bk[hh, 1]):
            dst[...] = g.standard_normal(dst.shape, dtype=np.float32) * np.float32(std)
    return Wq, bq, Wk, bk


def make_problem(*, batch: int, heads: int, T: int, Hs: int, Ws: int, D: int,
                 Dp: int, Tc: int, To: int, causal: bool, dtype: str = "bf16",
                 dist: str = "scaled", seed: int = 0, phi_std: float = 0.1,
                 name: str = "") -> Problem:
    """Draw one problem instance (see the module docstring for the recipe)."""
    if dtype not in ("f32", "bf16"):
        raise ValueError("dtype must be 'f32' or 'bf16'")
    g = np.random.Generator(np.random.Philox(seed))
    N = T * Hs * Ws
    q, k, v = _draw_qkv(g, (batch, heads, N, D), dist, heads, D)
    Wq, bq, Wk, bk = _draw_phi(g, heads, D, Dp, phi_std)
    if dtype == "bf16":
        q, k, v = round_to_bf16(q), round_to_bf16(k), round_to_bf16(v)
        Wq, Wk = round_to_bf16(Wq), round_to_bf16(Wk)
    return Problem(batch, heads, T, Hs, Ws, D, Dp, Tc, To, bool(causal), dtype,
                   q, k, v, Wq, bq, Wk, bk, seed, name)


# The five workloads, named by what they are.
CONFIGS = {
    # tiny fp32 check: 4 slices of 4x4 tokens, 2 heads of width 32
    "tiny_f32": dict(batch=1, heads=2, T=4, Hs=4, Ws=4, D=32, Dp=32, Tc=2, To=1,
                     dtype="f32", dist="normal", seed=0),
    # one Wan2.1-1.3B-shaped layer at 320x480: latent 21x20x30, causal
    "wan_320x480_causal": dict(batch=1, heads=12, T=21, Hs=20, Ws=30, D=128,
                               Dp=128, Tc=3, To=1, causal=True, dtype="bf16",
                               dist="scaled", seed=1),
    # 5 s at 480x832: latent 21x30x52, batch 2, bidirectional
    "wan_480x832_bidir": dict(batch=2, heads=12, T=21, Hs=30, Ws=52, D=128,
                              Dp=128, Tc=3, To=1, causal=False, dtype="bf16",
                              dist="scaled", seed=2),
    # ~20 s streaming: 81 slices of 30x52, causal chunk-wise RNN
    "stream_81x30x52": dict(batch=1, heads=12, T=81, Hs=30, Ws=52, D=128,
                            Dp=128, Tc=3, To=1, causal=True, dtype="bf16",
                            dist="scaled", seed=3),
}


def config_problem(name: str, *, causal: Optional[bool] = None, **overrides) -> Problem:
    """Draw a named workload; keyword arguments override its fields."""
    cfg = dict(CONFIGS[name])
    if causal is not None:
        cfg["causal"] = causal
    cfg.setdefault("causal", False)
    cfg.update(overrides)
    return make_problem(name=name, **cfg)
