"""Pins of the oracle's W4 path (4-bit weights {-7..7} * s, per-channel MSE scale, W4A4 linear).

"Qift: Shift-Friendly No-Zero W2 Post-Training Quantization for Rotated W2A4/KV4 LLM
Inference", Abstract: the evaluation mixes W2 and W4 layers ("L-layer mixed W2/W4") and gives no
W4 scheme.  The oracle reads it with this method's own rules (one scale per output channel, no
zero point, the MSE-searched candidate grid) and symmetric 4-bit levels.  These tests pin the
encoding to exact brute force, the packing to a hand-derived word, the scale to the grid optimum
and the linear to integer matrix products.
"""
from fractions import Fraction

import numpy as np
import pytest

import oracle
from w2a4_gemm_b200 import synth


def _encode_exact(w: float, s: float) -> int:
    """Nearest level of {-7..7} * s in exact rational arithmetic; ties to the smaller magnitude,
    w >= 0 (and -0.0) on the positive side."""
    wq, sq = Fraction(float(w)), Fraction(float(s))
    a = abs(wq)
    best = None
    for j in range(8):
        d = abs(a - j * sq)
        if best is None or d < best[0]:
            best = (d, j)
    j = best[1]
    return j if (w > 0 or (w == 0)) else -j


def _codes_for_scale(w: np.ndarray, f: float):
    # lo == hi == f pins every candidate to s = fp32((f * max|w|) / 7)
    codes, scales, _, _ = oracle.quantize_weights_w4(w, grid_points=2, lo=f, hi=f)
    return oracle.unpack_w4(codes, w.shape[1]), scales


def test_encoding_is_exact_nearest_level():
    rng = np.random.default_rng(21)
    w = (rng.standard_t(4, size=(6, 64)) * 0.02).astype(np.float32)
    for f in (0.2, 0.55, 1.0):
        levels, scales = _codes_for_scale(w, f)
        for n in range(w.shape[0]):
            for k in range(w.shape[1]):
                assert levels[n, k] == _encode_exact(w[n, k], scales[n]), (n, k, f)


def test_midpoint_ties_and_signed_zero():
    s = np.float32(0.25)                       # m = 1.75 -> s = 1.75 / 7 = 0.25 exactly
    mids = [(j + 0.5) * 0.25 for j in range(7)]
    row = np.array([1.75] + mids + [-x for x in mids] + [-0.0, 0.0], dtype=np.float32)
    row = np.concatenate([row, np.zeros(32 - len(row), np.float32)])[None, :]
    levels, scales = _codes_for_scale(row, 1.0)
    assert scales[0] == s
    assert levels[0, 1:8].tolist() == list(range(7))          # a tie keeps the smaller magnitude
    assert levels[0, 8:15].tolist() == [-j for j in range(7)]
    assert levels[0, 15] == 0 and levels[0, 16] == 0          # -0.0 and +0.0


def test_packing_hand_word():
    # levels -7, 0, 7, 1 (inputs 0..3) and -1, 3, -3, 6 (inputs 4..7) as two's-complement
    # nibbles 9, 0, 7, 1 and F, 3, D, 6; byte j = input j | input j+4 << 4:
    #   0xF9, 0x30, 0xD7, 0x61 -> 0x61D730F9.
    levels = np.array([-7, 0, 7, 1, -1, 3, -3, 6], dtype=np.float32)
    w = np.concatenate([levels * np.float32(0.25)] * 2)[None, :]    # max |w| = 1.75 -> s = 0.25
    codes, scales, _, _ = oracle.quantize_weights_w4(w, grid_points=2, lo=1.0, hi=1.0)
    assert scales[0] == np.float32(0.25)
    assert codes.tolist() == [[0x61D730F9, 0x61D730F9]]
    assert oracle.unpack_w4(codes, 16).tolist() == [levels.astype(int).tolist() * 2]
    assert oracle.pack_w4(levels.astype(int)[None, :]).tolist() == [[0x61D730F9]]


def _pack_by_hand(lv: np.ndarray) -> np.ndarray:
    """Bit by bit: input k of a row goes to word k // 8, byte k % 4, high nibble when k % 8 >= 4."""
    N, K = lv.shape
    out = np.zeros((N, K // 8), np.uint32)
    for n in range(N):
        for k in range(K):
            nib = int(lv[n, k]) % 16
            out[n, k // 8] |= np.uint32(nib << (8 * (k % 4) + (4 if k % 8 >= 4 else 0)))
    return out


def test_nibble_sign_and_byte_scaling():
    # Every nibble reads as its two's-complement level, and the nibble moved to the top of a
    # byte reads, as a signed byte, 16 times that level (the form a signed dp4a consumes).
    for nib in range(16):
        level = nib - 16 if nib >= 8 else nib
        word = np.array([[nib << 4 | nib]], np.uint32)            # inputs 0 (low) and 4 (high)
        assert oracle.unpack_w4(np.array([[word[0, 0]]], np.uint32), 8)[0, [0, 4]].tolist() == [level, level]
        assert int(np.uint8(nib << 4).view(np.int8)) == 16 * level


def test_scale_search_is_grid_optimal():
    w = oracle.rotate_f32(synth.weights(5, 256, (31,)), 128)
    codes, scales, mse, best = oracle.quantize_weights_w4(w)
    m = np.abs(w).max(axis=1)
    for n in range(w.shape[0]):
        cands = [np.float32((f * float(m[n])) / 7.0) for f in 0.2 + (0.8 * np.arange(100)) / 99]
        errs = []
        for s in cands:
            lv = np.clip(np.floor(np.abs(w[n]).astype(np.float64) / float(s) + 0.5), 0, 7) if s > 0 else np.zeros(256)
            errs.append(float(np.sum((np.abs(w[n]).astype(np.float64) - lv * float(s)) ** 2)))
        assert scales[n] == cands[best[n]]
        assert errs[best[n]] <= min(errs) * (1 + 1e-6)  # the chosen candidate is the grid optimum
        assert abs(mse[n] * 256 - errs[best[n]]) <= 1e-6 * errs[best[n]]


@pytest.mark.parametrize("T,N,K", [(1, 5, 16), (3, 7, 64), (4, 33, 256)])
def test_linear_w4_is_integer_matmul(T, N, K):
    rng = np.random.default_rng(T + N + K)
    q = rng.integers(-7, 8, size=(T, K)).astype(np.int8)
    lv = rng.integers(-8, 8, size=(N, K)).astype(np.int64)       # every nibble, -8 included
    codes = _pack_by_hand(lv)
    assert np.array_equal(oracle.pack_w4(lv), codes)
    s_w = rng.uniform(1e-3, 1e-2, N).astype(np.float32)
    s_a = rng.uniform(0.1, 2.0, T).astype(np.float32)
    y, acc = oracle.linear_w4(q, s_a, codes, s_w)
    ref = q.astype(np.int64) @ lv.T
    assert np.array_equal(acc.astype(np.int64), ref)
    yr = ((acc.astype(np.float32) * s_w[None, :]).astype(np.float32) * s_a[:, None]).astype(np.float32)
    assert np.array_equal(y, yr)


def test_w4_error_is_far_below_w2_on_rotated_heavy_tails():
    w = oracle.rotate_f32(synth.weights(16, 1024, (41,)), 128)
    _, _, mse4, _ = oracle.quantize_weights_w4(w)
    _, _, mse2, _ = oracle.quantize_weights(w, "qift")
    assert mse4.mean() < 0.15 * mse2.mean()
