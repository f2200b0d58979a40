"""Tolerance for the general feature map computed with bf16 operands (test
infrastructure).

The tensor-core map rounds W_a, GELU(x W_a + b_a) and W_b to bf16 (x is
already bf16; accumulation, b_a, b_b and the powers stay fp32).  A worst-case
bound (every rounding error aligned) is ~sqrt(D * D_h) times the typical error
and would hide a dropped bias, so the bar is a probabilistic one: each
rounding is an independent relative error of at most u = 2^-8 (variance
u^2/3 for round-to-nearest), so to first order psi_f's error has standard
deviation
  sigma_f = u/sqrt(3) * sqrt(sum_j W_b[j,f]^2 (GELU'(a_j)^2 sum_d (x_d W_a[d,j])^2
                                                + 2 g_j^2)),
a_j = x W_a[:, j] + b_a[j], g_j = GELU(a_j); the bar is |d psi| <= 6 sigma
(a sum of hundreds of independent terms; a 6-sigma excursion has probability
~2e-9 per element), and for part i, phi = psi^i,
  |d phi| <= (|psi| + 6 sigma)^i - |psi|^i.
fp32 accumulation (relative ~sqrt(n) 2^-24) is covered by a 1e-6 relative
absolute term in the tests.
"""
import math

import numpy as np
from scipy.special import erf

U_BF16 = 2.0 ** -8
SIGMAS = 6.0


def bf16_bound(x, Wa, ba, Wb, bb, parts):
    """Element-wise bar [n, D'] for x [n, D] and one head's parameters."""
    x = np.asarray(x, np.float64)
    Wa, ba, Wb, bb = (np.asarray(t, np.float64) for t in (Wa, ba, Wb, bb))
    a = x @ Wa + ba
    cdf = 0.5 * (1.0 + erf(a / math.sqrt(2.0)))
    g = a * cdf
    dgelu = cdf + a * np.exp(-0.5 * a * a) / math.sqrt(2.0 * math.pi)
    var_j = dgelu ** 2 * ((x * x) @ (Wa * Wa)) + 2.0 * g * g
    sigma = U_BF16 / math.sqrt(3.0) * np.sqrt(var_j @ (Wb * Wb))
    psi = g @ Wb + bb
    width = psi.shape[1] // parts
    power = np.arange(psi.shape[1]) // width + 1
    return (np.abs(psi) + SIGMAS * sigma) ** power - np.abs(psi) ** power
