"""Pins of the oracle's KV4 path (rotated per-token INT4 keys/values, two codes per byte).

"Qift: Shift-Friendly No-Zero W2 Post-Training Quantization for Rotated W2A4/KV4 LLM
Inference" names KV4 in its title and gives no scheme; the oracle reads it as the activation
path (rotation by head-dimension blocks, symmetric per-token INT4) with the codes packed as
two's-complement nibbles.  These tests pin the packing to its definition and the dequantization
to the mathematics of an orthogonal rotation, independently of the GPU path.
"""
import numpy as np
import pytest

import oracle
from w2a4_gemm_b200 import synth


def test_pack_int4_hand_example():
    # Two's-complement nibbles, lower index in the low nibble:
    #   (1, -1)  -> 0x1 | 0xF << 4 = 0xF1      (7, -7) -> 0x7 | 0x9 << 4 = 0x97
    #   (0, -8)  -> 0x0 | 0x8 << 4 = 0x80      (3, 4)  -> 0x3 | 0x4 << 4 = 0x43
    q = np.array([[1, -1, 7, -7, 0, -8, 3, 4]], dtype=np.int8)
    assert oracle.pack_int4(q).tolist() == [[0xF1, 0x97, 0x80, 0x43]]


def test_unpack_inverts_pack_for_every_nibble_pair():
    lo, hi = np.meshgrid(np.arange(-8, 8), np.arange(-8, 8), indexing="ij")
    q = np.stack([lo.ravel(), hi.ravel()], axis=1).reshape(1, -1).astype(np.int8)
    p = oracle.pack_int4(q)
    assert len(np.unique(p)) == 256  # every byte value, once
    assert np.array_equal(oracle.unpack_int4(p), q)


def test_lossless_token_round_trips_exactly():
    # Without rotation, a token whose values are k * 0.5 with integer k in [-7, 7] and max |k| = 7
    # quantizes to q = k, s = 0.5 exactly, so the dequantized token is the token itself.
    rng = np.random.default_rng(3)
    k = rng.integers(-7, 8, size=(4, 64))
    k[:, 5] = 7
    x = (k * 0.5).astype(np.float16)
    packed, s = oracle.quantize_kv(x, 0)
    assert np.array_equal(s, np.full(4, 0.5, np.float32))
    assert np.array_equal(oracle.dequantize_kv(packed, s, 0), x)


@pytest.mark.parametrize("block,n", [(64, 256), (128, 1024), (128, 4096)])
def test_round_trip_error_equals_rotated_domain_error(block, n):
    # H_b / sqrt(b) is orthogonal and its own inverse, so the error of the round trip, measured in
    # the original domain, has the norm of the quantization error in the rotated domain (Parseval).
    # A missing, doubled or transposed inverse rotation breaks the equality by a wide margin.
    x = synth.activations(6, n, (block, n), n_outliers=synth.outlier_count(n))
    packed, s = oracle.quantize_kv(x, block)
    q, s2, x_rot = oracle.quantize_acts(x, block)
    assert np.array_equal(s, s2) and np.array_equal(oracle.unpack_int4(packed), q)
    xh = oracle.dequantize_kv(packed, s, block).astype(np.float64)
    e_rot = q.astype(np.float64) * s[:, None].astype(np.float64) - x_rot.astype(np.float64)
    e = xh - x.astype(np.float64)
    for t in range(x.shape[0]):
        ne, nr = np.linalg.norm(e[t]), np.linalg.norm(e_rot[t])
        fp16_slack = 2e-3 * np.linalg.norm(x[t].astype(np.float64))  # two binary16 roundings
        assert abs(ne - nr) <= 0.01 * nr + fp16_slack, (t, ne, nr)
        # ... and each rotated-domain error is at most half a quantization step.
        assert np.abs(e_rot[t]).max() <= s[t] / 2 * (1 + 1e-6) + 1e-12


def test_zero_token_dequantizes_to_zero():
    x = np.zeros((2, 128), np.float16)
    packed, s = oracle.quantize_kv(x, 128)
    assert np.all(packed == 0) and np.all(s == 0)
    assert np.all(oracle.dequantize_kv(packed, s, 128) == 0)
