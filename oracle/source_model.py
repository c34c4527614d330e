"""Gaussian source model of the Qift level sets -- TEST INFRASTRUCTURE ONLY.

The Qift abstract models Hadamard-rotated weights as a zero-centred, Gaussian-like source and
compares 2-bit level sets through a scale-invariant inner/outer centroid ratio: sets whose
ratio lies in 0.25..0.33 (mirror no-zero, Lloyd, NF2, PoT-MNZ) work, {+-1, +-2} (ratio 0.5)
does not.  ("Qift: Shift-Friendly No-Zero W2 Post-Training Quantization for Rotated W2A4/KV4
LLM Inference", Abstract.)

This module computes, for a unit Gaussian source X ~ N(0, 1):
  * the mean squared error of nearest-level quantization to ``scale * levels`` in closed form
    (truncated Gaussian moments), D(scale);
  * the best scale for a fixed level shape (Brent's method on the bounded interval);
  * the Lloyd-Max 4-level quantizer by the classical centroid/midpoint iteration;
  * the inner/outer ratio of a symmetric 4-level set.
No value is hard-coded: the tests compare these numbers with the classical tables and with a
Monte Carlo brute force.
"""
from __future__ import annotations

import math

import numpy as np
from scipy.optimize import minimize_scalar
from scipy.special import ndtr


def _pdf(x: float) -> float:
    if math.isinf(x):
        return 0.0
    return math.exp(-0.5 * x * x) / math.sqrt(2.0 * math.pi)


def _cdf(x: float) -> float:
    return float(ndtr(x))


def _xpdf(x: float) -> float:
    return 0.0 if math.isinf(x) else x * _pdf(x)


def region_moments(a: float, b: float):
    """M0, M1, M2 = E[X^j ; a < X <= b] for j = 0, 1, 2 (X ~ N(0,1))."""
    m0 = _cdf(b) - _cdf(a)
    m1 = _pdf(a) - _pdf(b)
    m2 = m0 + _xpdf(a) - _xpdf(b)
    return m0, m1, m2


def gaussian_quant_mse(levels, scale: float) -> float:
    """E[(X - Q(X))^2] for nearest-level quantization to ``scale * levels``."""
    c = np.sort(np.asarray(levels, dtype=np.float64)) * scale
    edges = [-math.inf] + [0.5 * (c[i] + c[i + 1]) for i in range(len(c) - 1)] + [math.inf]
    d = 0.0
    for i, ci in enumerate(c):
        m0, m1, m2 = region_moments(edges[i], edges[i + 1])
        d += m2 - 2.0 * ci * m1 + ci * ci * m0
    return d


def best_scale(levels):
    """(scale*, D(scale*)) minimising the Gaussian MSE over the scale of a fixed level shape."""
    top = float(np.max(np.abs(levels)))
    res = minimize_scalar(lambda s: gaussian_quant_mse(levels, s), bounds=(0.05 / top, 4.0 / top),
                          method="bounded", options={"xatol": 1e-12})
    return float(res.x), float(res.fun)


def lloyd_max(n_levels: int = 4, iters: int = 2000, tol: float = 1e-14):
    """Lloyd-Max quantizer of N(0,1): centroids of the cells, cells bounded by midpoints."""
    c = np.linspace(-1.5, 1.5, n_levels)
    for _ in range(iters):
        edges = [-math.inf] + [0.5 * (c[i] + c[i + 1]) for i in range(n_levels - 1)] + [math.inf]
        new = np.empty_like(c)
        for i in range(n_levels):
            m0, m1, _ = region_moments(edges[i], edges[i + 1])
            new[i] = m1 / m0
        if np.max(np.abs(new - c)) < tol:
            c = new
            break
        c = new
    return c, gaussian_quant_mse(c, 1.0)


def inner_outer_ratio(levels) -> float:
    """|inner| / |outer| of a 4-level set symmetric about zero (the abstract's ratio)."""
    a = np.sort(np.abs(np.asarray(levels, dtype=np.float64)))
    if not np.allclose(np.sort(levels), -np.sort(levels)[::-1]):
        raise ValueError("ratio is defined for sets symmetric about zero")
    return float(a[0] / a[-1])


def optimal_mse_for_ratio(r: float) -> float:
    """Best-scale Gaussian MSE of the mirror no-zero family {-1, -r, +r, +1}."""
    return best_scale(np.array([-1.0, -r, r, 1.0]))[1]
