"""Pins of the oracle's Hadamard rotation against mathematics and a library routine.

Qift abstract: weights and activations pass through a "Hadamard-rotated quantization
pipeline"; rotating W by H^T and x by H leaves W x unchanged because H is orthogonal.
"""
import numpy as np
import pytest
import scipy.linalg

import oracle
from conftest import golden_lines

POW2 = [2, 4, 8, 16, 32, 64]


@pytest.mark.parametrize("n", POW2)
def test_fwht_equals_sylvester_matrix(n):
    # scipy.linalg.hadamard builds the Sylvester matrix independently of the oracle.
    H = scipy.linalg.hadamard(n).astype(np.float64) / np.sqrt(n)
    rng = np.random.default_rng(n)
    x = rng.normal(size=(5, n))
    y = oracle.fwht_f64(x, n)
    np.testing.assert_allclose(y, x @ H.T, rtol=0, atol=1e-12)


@pytest.mark.parametrize("n", POW2)
def test_fwht_matrix_is_integer_orthogonal(n):
    # Rows of the oracle applied to the identity, unnormalised, must be +-1 with H H^T = n I
    # in exact integer arithmetic.
    F = oracle.fwht_f64(np.eye(n), n) * np.sqrt(n)
    M = np.rint(F).astype(np.int64)
    assert np.max(np.abs(F - M)) < 1e-9
    assert set(np.unique(M)) <= {-1, 1}
    assert np.array_equal(M @ M.T, n * np.eye(n, dtype=np.int64))


@pytest.mark.parametrize("n", [2, 16, 128, 4096])
def test_fwht_involution_and_parseval(n):
    rng = np.random.default_rng(7)
    x = rng.normal(size=(3, n))
    y = oracle.fwht_f64(x, n)
    np.testing.assert_allclose(np.linalg.norm(y, axis=1), np.linalg.norm(x, axis=1), rtol=1e-13)
    np.testing.assert_allclose(oracle.fwht_f64(y, n), x, rtol=0, atol=1e-12)


@pytest.mark.parametrize("block,K", [(128, 512), (512, 512), (16, 64), (4096, 4096)])
def test_rotation_preserves_linear(block, K):
    # (W H_b^T)(H_b x) = W x, block-diagonal along the input dimension.
    rng = np.random.default_rng(block)
    W = rng.standard_t(4, size=(24, K)) * 0.02
    x = rng.normal(size=(3, K))
    Wr = oracle.fwht_f64(W, block)
    xr = oracle.fwht_f64(x, block)
    np.testing.assert_allclose(xr @ Wr.T, x @ W.T, rtol=1e-10, atol=1e-12)


def test_block_diagonal_segments_are_independent():
    rng = np.random.default_rng(3)
    x = rng.normal(size=(2, 256))
    y = oracle.fwht_f64(x, 64)
    for s in range(4):
        seg = x[:, 64 * s:64 * (s + 1)]
        H = scipy.linalg.hadamard(64) / 8.0
        np.testing.assert_allclose(y[:, 64 * s:64 * (s + 1)], seg @ H.T, atol=1e-12)


@pytest.mark.parametrize("block", [2, 32, 128, 512, 4096])
def test_rotate_f32_within_fp32_error_of_exact(block):
    rng = np.random.default_rng(block + 1)
    x = (rng.standard_t(4, size=(8, 4096)) * 0.02).astype(np.float32)
    y32 = oracle.rotate_f32(x, block).astype(np.float64)
    y64 = oracle.fwht_f64(x.astype(np.float64), block)
    # Each of the log2(b) stages contributes at most 2^-24 * (l1 norm of the segment) to any
    # output (the partial sums feeding one output cover disjoint inputs); the rounded
    # constant and the final multiply add two more units; normalisation divides by sqrt(b).
    stages = int(np.log2(block)) + 2
    seg = x.astype(np.float64).reshape(8, -1, block)
    bound = stages * 2.0 ** -24 * np.abs(seg).sum(-1, keepdims=True) / np.sqrt(block) * 1.01
    err = np.abs(y32 - y64).reshape(8, -1, block)
    assert np.all(err <= bound)


def test_rotate_f32_stage_order_worked_example():
    (_, *inp), (_, *exp) = golden_lines("fwht_stage_order.txt")
    x = np.array([float(v) for v in inp], dtype=np.float32)[None, :]
    y = oracle.rotate_f32(x, 4)[0]
    assert y.tolist() == [float(v) for v in exp]


def test_rotate_f16_rounds_once():
    # fp16 in, fp32 stages, one round-to-nearest-even to fp16: equals rounding the fp32 result.
    rng = np.random.default_rng(11)
    x = rng.normal(size=(4, 512)).astype(np.float16)
    y16 = oracle.rotate_f16(x, 128)
    y32 = oracle.rotate_f32(x.astype(np.float32), 128)
    assert y16.dtype == np.float16
    assert np.array_equal(y16, y32.astype(np.float16))
    np.testing.assert_allclose(y16.astype(np.float64), oracle.fwht_f64(x.astype(np.float64), 128),
                               rtol=2e-3, atol=2e-3)


def test_rotation_gaussianizes_heavy_tails():
    # Abstract: Hadamard rotation "primarily Gaussianizes" weight shape -- excess kurtosis
    # drops by orders of magnitude.  Student-t(4) rows have large sample kurtosis; after a
    # 128-block rotation each rotated coordinate is a normalised sum of 128 t(4) draws.
    rng = np.random.default_rng(5)
    w = (rng.standard_t(4, size=(256, 4096)) * 0.02).astype(np.float32)
    wr = oracle.rotate_f32(w, 128).astype(np.float64)

    def excess_kurtosis(a):
        a = a - a.mean()
        return float(np.mean(a ** 4) / np.mean(a ** 2) ** 2 - 3.0)

    k0, k1 = excess_kurtosis(w.astype(np.float64)), excess_kurtosis(wr)
    assert k0 > 3.0
    assert abs(k1) < 0.1 * k0
