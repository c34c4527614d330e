"""Pins of the oracle's INT4 activation quantizer and W2A4 linear.

Qift abstract: W2A4 -- 2-bit weights applied to 4-bit activations ("sign-and-shift decoded
weight application" for the power-of-two set).  Symmetric per-token INT4 with range [-7, 7],
round half to even, and the int32-accumulate / binary32-epilogue linear are the readings taken
where the abstract is silent.
"""
from fractions import Fraction

import numpy as np
import pytest

import oracle
from conftest import golden_lines

GOLD_INTS = {r[0]: [int(v) for v in r[5:9]] for r in golden_lines("level_sets.txt")}


def _acts(T, K, seed, outliers=0):
    rng = np.random.default_rng(seed)
    x = rng.normal(size=(T, K))
    if outliers:
        x[:, rng.choice(K, outliers, replace=False)] *= 20
    return x.astype(np.float16)


def test_int4_range_and_per_token_max():
    x = _acts(16, 512, 0, outliers=4)
    q, s, _ = oracle.quantize_acts(x, 128)
    assert q.dtype == np.int8 and q.shape == x.shape
    assert np.all(np.abs(q.astype(np.int32)) <= 7)
    assert np.all(np.max(np.abs(q.astype(np.int32)), axis=1) == 7)


def test_int4_is_nearest_integer_within_half_step():
    # |x/s_a - q| <= 1/2 up to the rounding of the binary32 scale, checked in exact rationals.
    x = _acts(4, 256, 1)
    q, s, xr = oracle.quantize_acts(x, 64)
    for t in range(4):
        st = Fraction(float(s[t]))
        for k in range(256):
            d = abs(Fraction(float(xr[t, k])) / st - q[t, k])
            assert d <= Fraction(1, 2) + Fraction(1, 10 ** 5)


def test_int4_exact_grid_points_and_half_even():
    # A token whose values are exact multiples m*j/7 reproduces j; values exactly on a half
    # step go to the even integer (R11).  m = 7 makes every product exact in binary32.
    row = np.array([7, -7, 3, -3, 0, 1, 2.5, -2.5, 3.5, -0.5, 0.5, 6.5] + [0] * 4, np.float16)
    q, s, _ = oracle.quantize_acts(row[None, :], 0)
    assert s[0] == np.float32(1.0)
    assert q[0, :12].tolist() == [7, -7, 3, -3, 0, 1, 2, -2, 4, 0, 0, 6]


def test_zero_token():
    x = np.zeros((2, 64), np.float16)
    x[1, 5] = np.float16(-0.0)
    q, s, _ = oracle.quantize_acts(x, 16)
    assert np.all(q == 0) and np.all(s == 0)


def test_acts_rotation_then_quant_composes():
    x = _acts(3, 4096, 2, outliers=41)
    q, s, xr = oracle.quantize_acts(x, 4096)
    assert np.array_equal(xr, oracle.rotate_f16(x, 4096))
    q2, s2, _ = oracle.quantize_acts(xr, 0)
    assert np.array_equal(q, q2) and np.array_equal(s, s2)


@pytest.mark.parametrize("name", ["qift", "pot", "std"])
@pytest.mark.parametrize("T,N,K", [(1, 3, 16), (5, 7, 48), (3, 33, 160)])
def test_linear_accumulators_brute_force(name, T, N, K):
    rng = np.random.default_rng(T * 100 + N)
    q = rng.integers(-7, 8, size=(T, K)).astype(np.int8)
    codes = rng.integers(0, 2 ** 32, size=(N, K // 16), dtype=np.uint64).astype(np.uint32)
    s_w = rng.uniform(0.001, 0.01, N).astype(np.float32)
    s_a = rng.uniform(0.1, 2.0, T).astype(np.float32)
    y, acc = oracle.linear(q, s_a, codes, s_w, name)
    # Brute force: unpack each code by hand, look up the level table copied from the
    # abstract, integer matmul with numpy.
    lv = np.array(GOLD_INTS[name], dtype=np.int64)
    c = np.zeros((N, K), np.int64)
    for k in range(K):
        c[:, k] = (codes[:, k // 16].astype(np.int64) >> (2 * (k % 16))) & 3
    ref = q.astype(np.int64) @ lv[c].T
    assert np.array_equal(acc.astype(np.int64), ref)
    # Epilogue: within one binary32 rounding of each of the two products of the exact value.
    exact = ref.astype(np.float64) * s_w.astype(np.float64)[None, :] * s_a.astype(np.float64)[:, None]
    assert np.all(np.abs(y.astype(np.float64) - exact) <= np.abs(exact) * 2 * 2.0 ** -24 * 1.001)


def test_linear_qift_affine_identity():
    # sum q*L = 2*sum q*c - 3*sum q for the Qift table L(c) = 2c - 3.
    rng = np.random.default_rng(9)
    q = rng.integers(-7, 8, size=(4, 64)).astype(np.int8)
    codes = rng.integers(0, 2 ** 32, size=(5, 4), dtype=np.uint64).astype(np.uint32)
    _, acc = oracle.linear(q, np.ones(4, np.float32), codes, np.ones(5, np.float32), "qift")
    c = oracle.unpack_codes(codes, 64).astype(np.int64)
    lhs = 2 * (q.astype(np.int64) @ c.T) - 3 * q.astype(np.int64).sum(1, keepdims=True)
    assert np.array_equal(acc.astype(np.int64), lhs)


def test_linear_end_to_end_tracks_float_product():
    # Diagnostic for the whole path: y approximates W x and the no-zero set does better than
    # the standard set (abstract: the standard set "often collapses" under W2A4).
    rng = np.random.default_rng(10)
    W = (rng.standard_t(4, size=(128, 1024)) * 0.02).astype(np.float32)
    x = rng.normal(size=(8, 1024)).astype(np.float16)
    ref = x.astype(np.float64) @ W.astype(np.float64).T
    err = {}
    for name in ("qift", "std"):
        out = oracle.pipeline(W, x, name, 128, 128, out_dtype=np.float32)
        err[name] = np.linalg.norm(out["y"] - ref) / np.linalg.norm(ref)
    assert err["qift"] < 0.6
    assert err["qift"] < err["std"]
