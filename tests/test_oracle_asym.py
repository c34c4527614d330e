"""Pins of the oracle's conventional asymmetric W2 baseline (per-channel scale and integer zero
point, weight (c - z) * s, min-max range shrunk over the candidate grid).

"Qift: Shift-Friendly No-Zero W2 Post-Training Quantization for Rotated W2A4/KV4 LLM
Inference", Abstract: the no-zero sets are compared against "conventional asymmetric W2" and
the page gives no formula for it.  These tests pin the oracle's reading to constructed rows
whose answer is known exactly, to exact rational nearest-level search, to the grid optimum, to
integer matrix products, and to the page's claim that the no-zero sets do better.
"""
from fractions import Fraction

import numpy as np
import pytest

import oracle
from w2a4_gemm_b200 import synth


def _one_candidate(w, f):
    # lo == hi == f leaves a single candidate: the range [f min, f max] (0 included)
    codes, scales, zeros, mse, _ = oracle.quantize_weights_asym(w, grid_points=2, lo=f, hi=f)
    return oracle.unpack_codes(codes, w.shape[1]).astype(np.int64), scales, zeros, mse


def test_lossless_row_on_the_grid():
    # levels (c - 1) * 0.25 = -0.25, 0, 0.25, 0.5; the row reaches both ends, so at f = 1 the
    # range is 0.75, s = 0.25 and z = 0.25 / 0.25 = 1 exactly, and every weight is a level.
    rng = np.random.default_rng(5)
    c = rng.integers(0, 4, size=(1, 64))
    c[0, 0], c[0, 1] = 0, 3
    w = ((c - 1) * 0.25).astype(np.float32)
    got, s, z, mse = _one_candidate(w, 1.0)
    assert s[0] == np.float32(0.25) and z[0] == 1 and mse[0] == 0.0
    assert np.array_equal(got, c)
    codes, scales, zeros, mse, best = oracle.quantize_weights_asym(w)   # the full grid finds it too
    assert best[0] == 99 and mse[0] == 0.0 and scales[0] == np.float32(0.25) and zeros[0] == 1


@pytest.mark.parametrize("lo_w,hi_w,z_expected", [(-1.0, 2.0, 1), (-2.0, 1.0, 2), (0.5, 3.0, 0), (-3.0, -0.5, 3),
                                                  (-1.5, 1.5, 2)])
def test_zero_point_from_the_range(lo_w, hi_w, z_expected):
    # f = 1: s = (max(hi, 0) - min(lo, 0)) / 3 and z = round(-min(lo, 0) / s), ties to even
    # (-1.5 .. 1.5: s = 1, -lo / s = 1.5 -> 2).  A row entirely on one side of 0 still has 0
    # in its range, at z = 0 or z = 3.
    w = np.linspace(lo_w, hi_w, 32, dtype=np.float32)[None, :]
    _, s, z, _ = _one_candidate(w, 1.0)
    rng_lo, rng_hi = min(lo_w, 0.0), max(hi_w, 0.0)
    assert s[0] == np.float32((rng_hi - rng_lo) / 3)
    assert z[0] == z_expected


def test_zero_weights_reconstruct_exactly():
    w = oracle.rotate_f32(synth.weights(6, 256, (8,)), 128)
    w[:, ::5] = 0.0
    codes, scales, zeros, _, _ = oracle.quantize_weights_asym(w)
    c = oracle.unpack_codes(codes, 256).astype(np.int64)
    # code z is level 0, and every zero weight takes it
    assert np.all(c[:, ::5] == zeros[:, None])


def test_codes_are_exact_nearest_levels():
    w = oracle.rotate_f32(synth.weights(4, 128, (9,)), 128)
    for f in (0.3, 0.7, 1.0):
        c, s, z, _ = _one_candidate(w, f)
        for n in range(w.shape[0]):
            sq, zq = Fraction(float(s[n])), int(z[n])
            for k in range(w.shape[1]):
                wq = Fraction(float(w[n, k]))
                dists = [abs(wq - (j - zq) * sq) for j in range(4)]
                assert dists[c[n, k]] == min(dists), (f, n, k)


def test_scale_search_is_grid_optimal():
    w = oracle.rotate_f32(synth.weights(5, 256, (33,)), 128)
    _, _, _, mse, best = oracle.quantize_weights_asym(w)
    fs = 0.2 + (0.8 * np.arange(100)) / 99
    for n in range(w.shape[0]):
        errs = []
        for f in fs:  # each candidate's (s, z) alone, and its error by an independent nearest search
            _, s, z, _ = _one_candidate(w[n:n + 1], float(f))
            lv = (np.arange(4) - int(z[0])) * float(s[0])
            rec = lv[np.argmin(np.abs(w[n].astype(np.float64)[:, None] - lv[None, :]), axis=1)]
            errs.append(float(np.sum((w[n].astype(np.float64) - rec) ** 2)))
        assert errs[best[n]] <= min(errs) * (1 + 1e-6)
        assert abs(mse[n] * 256 - errs[best[n]]) <= 1e-6 * errs[best[n]]


@pytest.mark.parametrize("T,N,K", [(1, 5, 16), (3, 7, 64), (4, 33, 256)])
def test_linear_asym_is_integer_matmul(T, N, K):
    rng = np.random.default_rng(T * N + K)
    q = rng.integers(-7, 8, size=(T, K)).astype(np.int8)
    c = rng.integers(0, 4, size=(N, K)).astype(np.uint32)
    codes = np.zeros((N, K // 16), np.uint32)
    for k in range(K):
        codes[:, k // 16] |= c[:, k] << np.uint32(2 * (k % 16))
    z = rng.integers(0, 4, size=N).astype(np.int32)
    s_w = rng.uniform(1e-3, 1e-2, N).astype(np.float32)
    s_a = rng.uniform(0.1, 2.0, T).astype(np.float32)
    y, acc = oracle.linear_asym(q, s_a, codes, s_w, z)
    ref = q.astype(np.int64) @ (c.astype(np.int64) - z[:, None]).T
    assert np.array_equal(acc.astype(np.int64), ref)
    yr = ((acc.astype(np.float32) * s_w[None, :]).astype(np.float32) * s_a[:, None]).astype(np.float32)
    assert np.array_equal(y, yr)


def test_no_zero_sets_beat_conventional_asymmetric_w2():
    # The Abstract reports that the no-zero sets improve over conventional asymmetric W2; on
    # rotated heavy-tailed rows their reconstruction error is lower.
    w = oracle.rotate_f32(synth.weights(32, 2048, (44,)), 128)
    asym = oracle.quantize_weights_asym(w)[3].mean()
    assert oracle.quantize_weights(w, "qift")[2].mean() < 0.9 * asym
    assert oracle.quantize_weights(w, "pot")[2].mean() < 0.9 * asym
