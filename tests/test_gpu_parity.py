"""GPU-vs-oracle parity of every stage of the Qift W2A4 path, called through the C ABI.

Integer outputs (packed codes, INT4 activations, the int32 accumulators behind y) must match
bit for bit.  Floating-point outputs are checked against the tolerances of the contract --
fp32 epilogue |g - r| <= 1e-5 |r| + 1e-5 rms(r), fp16 rotation <= 2e-3 |r| + 2e-3 rms(r) --
and, because both sides run the same IEEE operations in the same order, also for exact
equality.  Inputs come from the seeded generators both sides share; expected values come from
the CPU oracle only.
"""
import numpy as np
import pytest
import torch

import oracle
import w2a4_gemm_b200 as qg
from w2a4_gemm_b200 import build, synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _setup():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    build.build()
    qg.lib()


def dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def host(t):
    torch.cuda.synchronize()
    return t.cpu().numpy()


def tol_check(got, ref, rel):
    got = got.astype(np.float64)
    ref = ref.astype(np.float64)
    rms = np.sqrt(np.mean(ref ** 2)) if ref.size else 0.0
    bad = np.abs(got - ref) > rel * np.abs(ref) + rel * rms
    assert not bad.any(), f"{bad.sum()} of {bad.size} outside tolerance; max err {np.abs(got - ref).max()}"


def codes_u32(t):
    return host(t).view(np.uint32)


# ------------------------------------------------------------------------------ rotation
@pytest.mark.parametrize("block", [2, 4, 8, 16, 32, 64, 128, 256, 512, 1024, 2048, 4096])
def test_rotate_f32_parity(block):
    rows = 37
    n = max(block, 4096) if block >= 1024 else block * 24
    w = synth.weights(rows, n, (block, 1))
    ref = oracle.rotate_f32(w, block)
    got = host(qg.qift_rotate(dev(w), block))
    tol_check(got, ref, 2e-3)
    assert np.array_equal(got.view(np.uint32), ref.view(np.uint32))


@pytest.mark.parametrize("block", [2, 16, 128, 512, 2048, 4096])
def test_rotate_f16_parity(block):
    x = synth.activations(19, max(block, 256) * 3, (block, 2), n_outliers=5)
    ref = oracle.rotate_f16(x, block)
    got = host(qg.qift_rotate(dev(x), block))
    tol_check(got, ref, 2e-3)
    assert np.array_equal(got.view(np.uint16), ref.view(np.uint16))


def test_rotate_in_place():
    w = synth.weights(8, 4096, (5,))
    t = dev(w)
    qg.qift_rotate(t, 4096, out=t)
    assert np.array_equal(host(t).view(np.uint32), oracle.rotate_f32(w, 4096).view(np.uint32))


# ------------------------------------------------------------------------ weight quantizer
@pytest.mark.parametrize("name", ["qift", "pot", "std"])
@pytest.mark.parametrize("n_out,n_in,block", [(5, 16, 16), (33, 48, 16), (64, 512, 128), (40, 4096, 4096),
                                               (9, 11008, 128)])
def test_quantize_weights_parity(name, n_out, n_in, block):
    w = oracle.rotate_f32(synth.weights(n_out, n_in, (n_in, 3)), block)
    codes, scales, mse, best = oracle.quantize_weights(w, name)
    gc, gs, gm = qg.qift_quantize_weights(dev(w), name)
    assert np.array_equal(codes_u32(gc), codes)
    assert np.array_equal(host(gs).view(np.uint32), scales.view(np.uint32))
    assert np.array_equal(host(gm).view(np.uint64), mse.view(np.uint64))


@pytest.mark.parametrize("n_in", [2560, 2816, 3072])
def test_quantize_weights_static_plus_dynamic_smem_past_48k(n_in):
    # Four rows of 2560..3072 inputs ask for 40..48 KB of dynamic shared memory; with the
    # kernel's static buffers the total passes the default 48 KB limit.
    w = oracle.rotate_f32(synth.weights(9, n_in, (n_in, 11)), 128)
    codes, scales, mse, _ = oracle.quantize_weights(w, "qift")
    gc, gs, gm = qg.qift_quantize_weights(dev(w), "qift")
    assert np.array_equal(codes_u32(gc), codes)
    assert np.array_equal(host(gs).view(np.uint32), scales.view(np.uint32))


def test_quantize_weights_edge_rows():
    # all-zero row, a single huge outlier, -0.0 entries, exact midpoints, constant row
    K = 64
    w = np.zeros((6, K), np.float32)
    w[1, 7] = 1e3
    w[1, 8:] = 1e-3
    w[2, :] = -0.0
    w[2, 3] = 0.5
    w[3, :] = np.float32(0.25)
    w[4, ::2] = np.float32(0.75)
    w[4, 1::2] = np.float32(-0.25)
    w[5] = synth.weights(1, K, (99,))[0]
    for name in ("qift", "pot", "std"):
        for grid, lo, hi in ((100, 0.2, 1.0), (2, 1.0, 1.0), (256, 0.05, 4.0)):
            codes, scales, mse, _ = oracle.quantize_weights(w, name, grid, lo, hi)
            gc, gs, gm = qg.qift_quantize_weights(dev(w), name, grid, lo, hi)
            assert np.array_equal(codes_u32(gc), codes), (name, grid)
            assert np.array_equal(host(gs).view(np.uint32), scales.view(np.uint32))
            assert np.array_equal(host(gm).view(np.uint64), mse.view(np.uint64))


def test_quantize_weights_tiny_rows():
    # Rows small enough that squared errors are subnormal or zero (exact widening fallback),
    # beside ordinary rows in the same launch.
    K = 256
    w = synth.weights(8, K, (77,)) * np.float32(1e-22)
    w[0] = synth.weights(1, K, (78,))[0]
    w[1] = 0
    w[2, ::3] = np.float32(1e-30)
    w = w.astype(np.float32)
    for name in ("qift", "pot", "std"):
        codes, scales, mse, _ = oracle.quantize_weights(w, name)
        gc, gs, gm = qg.qift_quantize_weights(dev(w), name)
        assert np.array_equal(codes_u32(gc), codes), name
        assert np.array_equal(host(gs).view(np.uint32), scales.view(np.uint32))
        assert np.array_equal(host(gm).view(np.uint64), mse.view(np.uint64))


# ------------------------------------------- fused offline pass: rotation + quantization
@pytest.mark.parametrize("name", ["qift", "pot", "std"])
@pytest.mark.parametrize("n_out,n_in,block", [(256, 512, 512), (300, 4096, 128), (37, 14336, 128), (9, 4096, 4096),
                                              (5, 64, 16), (130, 1024, 2), (3, 32768, 4096)])
def test_rotate_quantize_weights_fused(name, n_out, n_in, block):
    # Same bits as the oracle's rotate-then-quantize and as the two library calls, for R = 4, 2
    # and 1 rows per CTA, every block size class, and the largest row.
    w = synth.weights(n_out, n_in, (n_in, block, 5))
    codes, scales, mse, _ = oracle.quantize_weights(oracle.rotate_f32(w, block), name)
    gw = dev(w)
    gc, gs, gm = qg.qift_rotate_quantize_weights(gw, block, name)
    assert np.array_equal(codes_u32(gc), codes)
    assert np.array_equal(host(gs).view(np.uint32), scales.view(np.uint32))
    assert np.array_equal(host(gm).view(np.uint64), mse.view(np.uint64))
    c2, s2, m2 = qg.qift_quantize_weights(qg.qift_rotate(gw, block), name)
    assert torch.equal(gc, c2) and torch.equal(gs, s2) and torch.equal(gm, m2)
    assert np.array_equal(host(gw), w)  # the raw weights are left as they were


def test_rotate_quantize_weights_block0_and_bad_block():
    w = synth.weights(4, 256, (6,))
    gc, gs, gm = qg.qift_rotate_quantize_weights(dev(w), 0, "qift")
    codes, scales, mse, _ = oracle.quantize_weights(w, "qift")
    assert np.array_equal(codes_u32(gc), codes) and np.array_equal(host(gs), scales)
    for bad in (3, 512, 8192):
        with pytest.raises(qg.QiftError):
            qg.qift_rotate_quantize_weights(dev(w), bad, "qift")


# ------------------------------------------------------- conventional asymmetric W2 baseline
@pytest.mark.parametrize("n_out,n_in,block", [(5, 16, 16), (33, 48, 16), (64, 512, 128), (40, 4096, 4096),
                                               (9, 11008, 128), (7, 3072, 128)])
def test_quantize_weights_asym_parity(n_out, n_in, block):
    w = oracle.rotate_f32(synth.weights(n_out, n_in, (n_in, 29)), block)
    codes, scales, zeros, mse, _ = oracle.quantize_weights_asym(w)
    gc, gs, gz, gm = qg.qift_quantize_weights_asym(dev(w))
    assert np.array_equal(codes_u32(gc), codes)
    assert np.array_equal(host(gs).view(np.uint32), scales.view(np.uint32))
    assert np.array_equal(host(gz), zeros)
    assert np.array_equal(host(gm).view(np.uint64), mse.view(np.uint64))


def test_quantize_weights_asym_edge_rows():
    # zero row, rows on one side of 0, a lossless grid row, a tie of the zero point, signed zeros
    K = 64
    w = np.zeros((7, K), np.float32)
    w[1] = np.linspace(0.5, 3.0, K, dtype=np.float32)
    w[2] = np.linspace(-3.0, -0.5, K, dtype=np.float32)
    rng = np.random.default_rng(5)
    c = rng.integers(0, 4, size=K)
    c[0], c[1] = 0, 3
    w[3] = ((c - 1) * 0.25).astype(np.float32)
    w[4] = np.linspace(-1.5, 1.5, K, dtype=np.float32)
    w[5, :] = -0.0
    w[5, 3] = 0.5
    w[6] = synth.weights(1, K, (97,))[0]
    for grid, lo, hi in ((100, 0.2, 1.0), (2, 1.0, 1.0), (256, 0.05, 4.0)):
        codes, scales, zeros, mse, _ = oracle.quantize_weights_asym(w, grid, lo, hi)
        gc, gs, gz, gm = qg.qift_quantize_weights_asym(dev(w), grid, lo, hi)
        assert np.array_equal(codes_u32(gc), codes), grid
        assert np.array_equal(host(gs).view(np.uint32), scales.view(np.uint32))
        assert np.array_equal(host(gz), zeros)
        assert np.array_equal(host(gm).view(np.uint64), mse.view(np.uint64))


# ----------------------------------------------------------------- W4A4 (4-bit weights)
@pytest.mark.parametrize("n_out,n_in,block", [(5, 16, 16), (33, 48, 16), (64, 512, 128), (40, 4096, 4096),
                                               (9, 11008, 128), (7, 3072, 128)])
def test_quantize_weights_w4_parity(n_out, n_in, block):
    w = oracle.rotate_f32(synth.weights(n_out, n_in, (n_in, 13)), block)
    codes, scales, mse, _ = oracle.quantize_weights_w4(w)
    gc, gs, gm = qg.qift_quantize_weights(dev(w), "int4")
    assert gc.shape == (n_out, n_in // 8)
    assert np.array_equal(codes_u32(gc), codes)
    assert np.array_equal(host(gs).view(np.uint32), scales.view(np.uint32))
    assert np.array_equal(host(gm).view(np.uint64), mse.view(np.uint64))
    raw = synth.weights(n_out, n_in, (n_in, 13))
    fc, fs, fm = qg.qift_rotate_quantize_weights(dev(raw), block, "int4")
    assert torch.equal(fc, gc) and torch.equal(fs, gs) and torch.equal(fm, gm)


def test_quantize_weights_w4_edge_rows():
    # zero row, one outlier, signed zeros, exact midpoints (j + 0.5) s, a constant row
    K = 64
    w = np.zeros((6, K), np.float32)
    w[1, 7] = 1e3
    w[1, 8:] = 1e-3
    w[2, :] = -0.0
    w[2, 3] = 0.5
    w[3, :] = np.float32(0.25)
    w[4, 0] = np.float32(1.75)                                  # s = 0.25 at f = 1
    w[4, 1:8] = [(j + 0.5) * 0.25 for j in range(7)]
    w[4, 8:15] = [-(j + 0.5) * 0.25 for j in range(7)]
    w[5] = synth.weights(1, K, (98,))[0]
    for grid, lo, hi in ((100, 0.2, 1.0), (2, 1.0, 1.0), (256, 0.05, 4.0)):
        codes, scales, mse, _ = oracle.quantize_weights_w4(w, grid, lo, hi)
        gc, gs, gm = qg.qift_quantize_weights(dev(w), "int4", grid, lo, hi)
        assert np.array_equal(codes_u32(gc), codes), grid
        assert np.array_equal(host(gs).view(np.uint32), scales.view(np.uint32))
        assert np.array_equal(host(gm).view(np.uint64), mse.view(np.uint64))


def _linear_w4_case(T, N, K, seed, out_dtype):
    rng = np.random.default_rng(seed)
    q = rng.integers(-7, 8, size=(T, K)).astype(np.int8)
    codes = rng.integers(0, 2 ** 32, size=(N, K // 8), dtype=np.uint64).astype(np.uint32)
    s_w = rng.uniform(1e-3, 1e-2, N).astype(np.float32)
    s_a = rng.uniform(0.1, 2.0, T).astype(np.float32)
    npdt = np.float16 if out_dtype == torch.float16 else np.float32
    y, _ = oracle.linear_w4(q, s_a, codes, s_w, npdt)
    gy = qg.qift_linear(dev(q), dev(s_a), dev(codes.view(np.int32)), dev(s_w), "int4", out_dtype)
    return host(gy), y


@pytest.mark.parametrize("pin", ["auto", "skinny", "gemv"])   # auto: tensor cores from 2 tokens
@pytest.mark.parametrize("T", [1, 2, 3, 4, 5, 8, 9, 16])
@pytest.mark.parametrize("N,K", [(1, 64), (37, 64), (129, 4096), (4096, 4096), (17, 14336), (300, 11008),
                                 (9, 32768), (130, 192)])
def test_linear_w4_parity(pin, T, N, K):
    qg.qift_debug_set_linear_path(pin)
    try:
        for out_dtype in (torch.float32, torch.float16):
            got, ref = _linear_w4_case(T, N, K, T * 7919 + N + K, out_dtype)
            tol_check(got, ref, 1e-5 if out_dtype == torch.float32 else 2e-3)
            u = np.uint16 if out_dtype == torch.float16 else np.uint32
            assert np.array_equal(got.view(u), ref.view(u)), (pin, T, N, K)
    finally:
        qg.qift_debug_set_linear_path("auto")
    assert qg.qift_device_error() == (qg.QIFT_OK, 0)


def test_linear_w4_extreme_accumulators():
    # activations +-7 against the outer levels +7 (nibble 7) and -7 (nibble 9): |acc| = 49 K at
    # K = 32768
    T, N, K = 3, 8, 32768
    q = np.full((T, K), 7, np.int8)
    q[1] = -7
    q[2, ::2] = -7
    codes = np.full((N, K // 8), 0x77777777, np.uint32)
    codes[1::2] = 0x99999999
    s_w = np.ones(N, np.float32)
    s_a = np.ones(T, np.float32)
    y, acc = oracle.linear_w4(q, s_a, codes, s_w, np.float32)
    assert np.abs(acc).max() == 49 * K
    for pin in ("skinny", "gemv", "gemm_pair"):
        qg.qift_debug_set_linear_path(pin)
        try:
            gy = qg.qift_linear(dev(q), dev(s_a), dev(codes.view(np.int32)), dev(s_w), "int4", torch.float32)
        finally:
            qg.qift_debug_set_linear_path("auto")
        assert np.array_equal(host(gy), y), pin
    # one token (the one-token kernel splits every code of its chunk before the wait)
    for t in range(T):
        y1, acc1 = oracle.linear_w4(q[t:t + 1], s_a[t:t + 1], codes, s_w, np.float32)
        assert np.abs(acc1).max() == (49 * K if t < 2 else 0)  # token 2 alternates +-7: zero sum
        gy = qg.qift_linear(dev(q[t:t + 1]), dev(s_a[t:t + 1]), dev(codes.view(np.int32)), dev(s_w), "int4",
                            torch.float32)
        assert np.array_equal(host(gy), y1), t


@pytest.mark.parametrize("pin", ["auto", "gemm_pair"])
@pytest.mark.parametrize("T,N,K", [(17, 256, 64), (128, 256, 128), (129, 257, 192), (300, 600, 4096), (256, 40, 640),
                                   (2048, 512, 11008), (64, 1000, 4160), (513, 130, 1024), (33, 64, 32768)])
def test_linear_w4_gemm_parity(pin, T, N, K):
    # 4-bit weights at prefill sizes on the tcgen05 pair GEMM: ragged token and row tiles, K not a
    # multiple of the 128-input ring stage (4160, 192), the largest n_in.
    qg.qift_debug_set_linear_path(pin)
    try:
        for out_dtype in (torch.float32, torch.float16):
            got, ref = _linear_w4_case(T, N, K, 7 * T + N + K, out_dtype)
            u = np.uint16 if out_dtype == torch.float16 else np.uint32
            assert np.array_equal(got.view(u), ref.view(u)), (pin, T, N, K)
    finally:
        qg.qift_debug_set_linear_path("auto")
    assert qg.qift_device_error() == (qg.QIFT_OK, 0)


def test_linear_w4_unsupported_shapes_and_decode():
    rng = np.random.default_rng(1)
    K, N = 128, 16
    codes = dev(rng.integers(0, 2 ** 32, size=(N, K // 8), dtype=np.uint64).astype(np.uint32).view(np.int32))
    s_w = dev(np.ones(N, np.float32))
    q48 = dev(np.zeros((2, 48), np.int8))                      # n_in not a multiple of 64
    with pytest.raises(qg.QiftError):
        qg.qift_linear(q48, dev(np.ones(2, np.float32)), dev(np.zeros((N, 6), np.int32)), s_w, "int4")
    q20 = dev(np.zeros((20, K), np.int8))                      # the CUDA-core GEMV takes at most 16 tokens
    qg.qift_debug_set_linear_path("gemv")
    try:
        with pytest.raises(qg.QiftError):
            qg.qift_linear(q20, dev(np.ones(20, np.float32)), codes, s_w, "int4")
    finally:
        qg.qift_debug_set_linear_path("auto")
    y = qg.qift_linear(dev(np.zeros((0, K), np.int8)), dev(np.ones(0, np.float32)), codes, s_w, "int4")
    assert y.shape == (0, N)


@pytest.mark.parametrize("T,N,K,block", [(1, 256, 512, 128), (4, 1000, 4096, 128), (16, 64, 16384, 4096),
                                         (5, 96, 14336, 1024)])
def test_w4a4_path_end_to_end(T, N, K, block):
    # raw weights and fp16 tokens through rotation, 4-bit weights, INT4 tokens and the W4A4 linear
    W = synth.weights(N, K, (N, K, 17))
    x = synth.activations(T, K, (T, K, 17), n_outliers=synth.outlier_count(K))
    codes, scales, _, _ = oracle.quantize_weights_w4(oracle.rotate_f32(W, block))
    q, s_a, _ = oracle.quantize_acts(x, block)
    ref, _ = oracle.linear_w4(q, s_a, codes, scales, np.float32)
    gc, gs, _ = qg.qift_rotate_quantize_weights(dev(W), block, "int4")
    gq, gsa = qg.qift_quantize_acts(dev(x), block)
    gy = qg.qift_linear(gq, gsa, gc, gs, "int4", torch.float32)
    assert np.array_equal(codes_u32(gc), codes)
    assert np.array_equal(host(gq), q)
    assert np.array_equal(host(gy), ref)


# ------------------------------------------------------------------- KV4 (packed INT4 K/V)
@pytest.mark.parametrize("T,n,block", [(1, 128, 128), (7, 1024, 128), (300, 4096, 128), (16, 4096, 4096),
                                       (5, 64, 0), (33, 8192, 64), (2, 16384, 128), (3, 1024, 1024)])
def test_kv4_quantize_dequantize_match_oracle(T, n, block):
    x = synth.activations(T, n, (T, n, block), n_outliers=synth.outlier_count(n))
    x[0, : n // 2] = 0  # a half-zero token beside ordinary ones
    packed, s = oracle.quantize_kv(x, block)
    gp, gs = qg.qift_quantize_kv(dev(x), block)
    assert np.array_equal(host(gp), packed)
    assert np.array_equal(host(gs).view(np.uint32), s.view(np.uint32))
    ref = oracle.dequantize_kv(packed, s, block)
    gx = qg.qift_dequantize_kv(gp, gs, block)
    assert np.array_equal(host(gx).view(np.uint16), ref.view(np.uint16))


def test_kv4_zero_token_and_bad_arguments():
    x = np.zeros((2, 256), np.float16)
    gp, gs = qg.qift_quantize_kv(dev(x), 128)
    assert int(gp.abs().sum() if gp.dtype != torch.uint8 else gp.sum()) == 0 and float(gs.abs().sum()) == 0.0
    assert float(qg.qift_dequantize_kv(gp, gs, 128).abs().sum()) == 0.0
    with pytest.raises(qg.QiftError):
        qg.qift_quantize_kv(dev(np.zeros((2, 200), np.float16)), 0)      # n % 16
    with pytest.raises(qg.QiftError):
        qg.qift_quantize_kv(dev(x), 96)                                   # not a power of two
    with pytest.raises(qg.QiftError):
        qg.qift_dequantize_kv(torch.zeros((1, 16384), dtype=torch.uint8, device="cuda"),
                              torch.ones(1, device="cuda"), 128)          # n = 32768 > 16384


# -------------------------------------------------------------------- activation quantizer
@pytest.mark.parametrize("block", [0, 16, 128, 512, 4096])
@pytest.mark.parametrize("T,K", [(1, 4096), (3, 512), (16, 11008), (33, 4096)])
def test_quantize_acts_parity(block, T, K):
    if block and K % block:
        pytest.skip("block must divide K")
    x = synth.activations(T, K, (T, K), n_outliers=synth.outlier_count(K))
    q, s, _ = oracle.quantize_acts(x, block)
    gq, gs = qg.qift_quantize_acts(dev(x), block)
    assert np.array_equal(host(gq), q)
    assert np.array_equal(host(gs).view(np.uint32), s.view(np.uint32))


def test_quantize_acts_zero_and_tiny_tokens():
    x = np.zeros((4, 256), np.float16)
    x[1, 5] = np.float16(-0.0)
    x[2, 17] = np.float16(6e-8)          # subnormal fp16
    x[3] = synth.activations(1, 256, (7,))[0]
    for block in (0, 256, 64):
        q, s, _ = oracle.quantize_acts(x, block)
        gq, gs = qg.qift_quantize_acts(dev(x), block)
        assert np.array_equal(host(gq), q)
        assert np.array_equal(host(gs).view(np.uint32), s.view(np.uint32))


# Batches of many tokens take the streaming quantizer (persistent CTAs, registers only): blocks
# 16..512, widths of one to four 4096-element passes with ragged last passes, zero tokens.
@pytest.mark.parametrize("block,K", [(16, 1024), (32, 4160), (128, 4096), (128, 11008), (256, 12288),
                                      (512, 16384), (64, 8256)])
def test_quantize_acts_many_tokens(block, K):
    T = 700
    x = synth.activations(T, K, (T, K, block), n_outliers=synth.outlier_count(K))
    x[3] = 0
    x[T - 1] = 0
    q, s, _ = oracle.quantize_acts(x, block)
    gq, gs = qg.qift_quantize_acts(dev(x), block)
    assert np.array_equal(host(gq), q)
    assert np.array_equal(host(gs).view(np.uint32), s.view(np.uint32))


# ---------------------------------------------------------------------------------- linear
def _linear_case(name, T, N, K, seed, out_dtype):
    rng = np.random.default_rng(seed)
    q = rng.integers(-7, 8, size=(T, K)).astype(np.int8)
    codes = rng.integers(0, 2 ** 32, size=(N, K // 16), dtype=np.uint64).astype(np.uint32)
    s_w = rng.uniform(1e-3, 1e-2, N).astype(np.float32)
    s_a = rng.uniform(0.1, 2.0, T).astype(np.float32)
    npdt = np.float16 if out_dtype == torch.float16 else np.float32
    y, _ = oracle.linear(q, s_a, codes, s_w, name, npdt)
    gy = qg.qift_linear(dev(q), dev(s_a), dev(codes.view(np.int32)), dev(s_w), name, out_dtype)
    return host(gy), y


@pytest.mark.parametrize("name", ["qift", "pot"])
@pytest.mark.parametrize("T,N,K", [(1, 1, 16), (1, 4096, 4096), (1, 37, 48), (2, 33, 528), (3, 70, 1024),
                                    (5, 17, 4096), (16, 129, 4096), (16, 64, 14336), (33, 40, 64)])
def test_linear_parity(name, T, N, K):
    for out_dtype in (torch.float32, torch.float16):
        got, ref = _linear_case(name, T, N, K, T * 1000 + N + K, out_dtype)
        tol_check(got, ref, 1e-5 if out_dtype == torch.float32 else 2e-3)
        assert np.array_equal(got.view(np.uint16 if out_dtype == torch.float16 else np.uint32),
                              ref.view(np.uint16 if out_dtype == torch.float16 else np.uint32))


def test_linear_extreme_accumulators():
    # Every activation +-7 and every weight at the outer level: |acc| = 7 * 4 * K at K = 32768.
    T, N, K = 2, 8, 32768
    q = np.full((T, K), 7, np.int8)
    q[1] = -7
    codes = np.full((N, K // 16), 0xFFFFFFFF, np.uint32)   # code 3 everywhere
    codes[1::2] = 0                                         # code 0 everywhere
    s_w = np.full(N, 1.0, np.float32)
    s_a = np.full(T, 1.0, np.float32)
    for name, top in (("qift", 3), ("pot", 4)):
        y, acc = oracle.linear(q, s_a, codes, s_w, name, np.float32)
        assert np.abs(acc).max() == 7 * top * K
        gy = qg.qift_linear(dev(q), dev(s_a), dev(codes.view(np.int32)), dev(s_w), name, torch.float32)
        assert np.array_equal(host(gy), y)


# ---------------------------------------------------------------------- whole path, small
def test_single_linear_256x512_end_to_end():
    wl = synth.SINGLE_256x512
    lin = wl.linears[0]
    W, x = wl.w(lin), wl.x(lin)
    ref = oracle.pipeline(W, x, wl.levelset, wl.w_block, wl.a_block, out_dtype=np.float32)
    w_rot = qg.qift_rotate(dev(W), wl.w_block)
    gc, gs, gm = qg.qift_quantize_weights(w_rot, wl.levelset)
    gq, gsa = qg.qift_quantize_acts(dev(x), wl.a_block)
    gy = qg.qift_linear(gq, gsa, gc, gs, wl.levelset, torch.float32)
    assert np.array_equal(host(w_rot).view(np.uint32), ref["w_rot"].view(np.uint32))
    assert np.array_equal(codes_u32(gc), ref["codes"])
    assert np.array_equal(host(gq), ref["q"])
    tol_check(host(gy), ref["y"], 1e-5)
    assert np.array_equal(host(gy), ref["y"])


# ------------------------------------------------- one token (codes bulk-copied on chip)
@pytest.mark.parametrize("pin", ["auto", "one_token"])
@pytest.mark.parametrize("name", ["qift", "pot"])
@pytest.mark.parametrize("N,K", [(1, 64), (37, 64), (147, 128), (149, 640), (300, 4096), (4096, 4096), (1000, 11008),
                                 (257, 14336), (14336, 4096), (4096, 14336), (5, 16384), (28000, 4096)])
def test_linear_one_token_parity(pin, name, N, K):
    # N < SMs (one row per CTA), ragged rows per CTA, slices of 32 groups that do not divide a
    # row (K = 11008, 14336, 640), and a matrix tall enough to take two CTAs per SM (28000).
    qg.qift_debug_set_linear_path(pin)
    try:
        for out_dtype in (torch.float16, torch.float32):
            got, ref = _linear_case(name, 1, N, K, 3 * N + K, out_dtype)
            assert np.array_equal(got.view(np.uint16 if out_dtype == torch.float16 else np.uint32),
                                  ref.view(np.uint16 if out_dtype == torch.float16 else np.uint32)), (N, K)
    finally:
        qg.qift_debug_set_linear_path("auto")
    assert qg.qift_device_error() == (qg.QIFT_OK, 0)


def test_linear_one_token_extreme_accumulators():
    # |acc| = 7 * 4 * 16384 (PoT) with every code value, and activations of both signs: the
    # Qift path applies the codes through masks (bytes up to 0xC0, unsigned) and 2 sum qc - 3 sum q.
    N, K = 8, 16384
    codes = np.zeros((N, K // 16), np.uint32)
    codes[0], codes[1], codes[2], codes[3] = 0xFFFFFFFF, 0, 0xAAAAAAAA, 0x55555555
    codes[4], codes[5] = 0x1B1B1B1B, 0xE4E4E4E4   # codes 3,2,1,0 / 0,1,2,3 in every byte
    codes[6] = np.random.default_rng(1).integers(0, 2 ** 32, K // 16, dtype=np.uint64).astype(np.uint32)
    s_w = np.full(N, 1.0, np.float32)
    s_a = np.full(1, 1.0, np.float32)
    for qv in (7, -7, None):
        q = np.full((1, K), 7 if qv is None else qv, np.int8)
        if qv is None:
            q[0, 1::2] = -7
        for name, top in (("qift", 3), ("pot", 4)):
            y, acc = oracle.linear(q, s_a, codes, s_w, name, np.float32)
            if qv is not None:
                assert np.abs(acc).max() == 7 * top * K
            gy = qg.qift_linear(dev(q), dev(s_a), dev(codes.view(np.int32)), dev(s_w), name, torch.float32)
            assert np.array_equal(host(gy), y), (qv, name)


# ------------------------------------------------------------- tensor-core GEMM (prefill)
@pytest.mark.parametrize("path", ["auto", "gemm_pair"])
@pytest.mark.parametrize("name", ["qift", "pot"])
@pytest.mark.parametrize("T,N,K", [(17, 256, 64), (128, 256, 128), (129, 257, 192), (300, 600, 4096),
                                    (256, 40, 640), (2048, 512, 11008), (64, 1000, 4160), (513, 130, 1024)])
def test_linear_gemm_parity(path, name, T, N, K):
    qg.qift_debug_set_linear_path(path)
    try:
        for out_dtype in (torch.float16, torch.float32):
            got, ref = _linear_case(name, T, N, K, T + 7 * N + K, out_dtype)
            tol_check(got, ref, 1e-5 if out_dtype == torch.float32 else 2e-3)
            assert np.array_equal(got.view(np.uint16 if out_dtype == torch.float16 else np.uint32),
                                  ref.view(np.uint16 if out_dtype == torch.float16 else np.uint32))
    finally:
        qg.qift_debug_set_linear_path("auto")
    assert qg.qift_device_error() == (qg.QIFT_OK, 0)


# ------------------------------------------------------- every kernel family, same inputs
@pytest.mark.parametrize("path", ["gemv", "skinny", "gemm_pair"])
@pytest.mark.parametrize("name", ["qift", "pot"])
@pytest.mark.parametrize("T,N,K", [(1, 300, 4096), (2, 129, 512), (7, 64, 1024), (9, 257, 14336), (16, 4096, 4096),
                                    (16, 130, 64), (5, 1000, 11008)])
def test_linear_each_kernel_family(path, name, T, N, K):
    qg.qift_debug_set_linear_path(path)
    try:
        for out_dtype in (torch.float16, torch.float32):
            got, ref = _linear_case(name, T, N, K, 31 * T + N + K, out_dtype)
            assert np.array_equal(got.view(np.uint16 if out_dtype == torch.float16 else np.uint32),
                                  ref.view(np.uint16 if out_dtype == torch.float16 else np.uint32)), (path, T, N, K)
    finally:
        qg.qift_debug_set_linear_path("auto")
    assert qg.qift_device_error() == (qg.QIFT_OK, 0)


@pytest.mark.parametrize("name", ["qift", "pot", "int4"])
@pytest.mark.parametrize("T,N,K", [(16, 16000, 4096),   # 125 row blocks: no K split, two warps per row group
                                   (16, 16000, 256),    # no K split, one chunk: one warp per row group
                                   (8, 14336, 4096),    # clusters of 2, two CTAs per SM
                                   (16, 4096, 4096),    # clusters of 4, one CTA per SM
                                   (16, 1024, 4096),    # clusters of 8, two chunks per CTA
                                   (3, 300, 14336)])    # clusters of 8, seven chunks per CTA
def test_skinny_cluster_plans(name, T, N, K):
    # The skinny kernel picks its cluster size (the K split) and its warps per row group from
    # the grid it would launch; these shapes reach every cluster size and both warp splits.
    qg.qift_debug_set_linear_path("skinny")
    try:
        for out_dtype in (torch.float16, torch.float32):
            seed = 13 * T + N + K
            got, ref = (_linear_w4_case(T, N, K, seed, out_dtype) if name == "int4"
                        else _linear_case(name, T, N, K, seed, out_dtype))
            u = np.uint16 if out_dtype == torch.float16 else np.uint32
            assert np.array_equal(got.view(u), ref.view(u)), (name, T, N, K)
    finally:
        qg.qift_debug_set_linear_path("auto")
    assert qg.qift_device_error() == (qg.QIFT_OK, 0)


@pytest.mark.parametrize("name", ["qift", "pot"])
@pytest.mark.parametrize("N,K", [(5, 64), (37, 1088), (300, 2112), (130, 4160), (64, 6208), (257, 11008), (3, 32768)])
def test_linear_one_token_gemv_partial_chunks(name, N, K):
    # the warp-per-row GEMV stages the token in 2048-input chunks: rows of one partial chunk,
    # and of several chunks with a partial last one, on the pinned family
    qg.qift_debug_set_linear_path("gemv")
    try:
        for out_dtype in (torch.float16, torch.float32):
            got, ref = _linear_case(name, 1, N, K, 5 * N + K, out_dtype)
            u = np.uint16 if out_dtype == torch.float16 else np.uint32
            assert np.array_equal(got.view(u), ref.view(u)), (name, N, K)
    finally:
        qg.qift_debug_set_linear_path("auto")


def test_prefill_with_unaligned_inputs_is_refused_not_slow():
    """Seventeen or more tokens run on the tensor cores only; an n_in they cannot take (not a
    multiple of 64) is refused, not sent to the CUDA-core GEMV.  Pinned to the GEMV the same call
    still runs, and matches the oracle."""
    T, N, K = 64, 96, 4112
    q = torch.zeros((T, K), dtype=torch.int8, device="cuda")
    codes = torch.zeros((N, K // 16), dtype=torch.int32, device="cuda")
    with pytest.raises(qg.QiftError) as e:
        qg.qift_linear(q, torch.ones(T, device="cuda"), codes, torch.ones(N, device="cuda"), "qift")
    assert e.value.status == qg.QIFT_ERR_UNSUPPORTED
    qg.qift_debug_set_linear_path("gemv")
    try:
        got, ref = _linear_case("qift", T, N, K, 4112, torch.float32)
    finally:
        qg.qift_debug_set_linear_path("auto")
    assert np.array_equal(got.view(np.uint32), ref.view(np.uint32))
    # 16 tokens with the same n_in stay on the decode-size GEMV
    got, ref = _linear_case("pot", 16, N, K, 4113, torch.float16)
    assert np.array_equal(got.view(np.uint16), ref.view(np.uint16))


def test_removed_gemm_pins_are_invalid():
    for p in (3, 4, 5, 8, -1):
        with pytest.raises(qg.QiftError) as e:
            qg.qift_debug_set_linear_path(p)
        assert e.value.status == qg.QIFT_ERR_INVALID_ARG
    qg.qift_debug_set_linear_path("auto")


def test_pinned_family_rejects_unsupported_shape():
    qg.qift_debug_set_linear_path("skinny")
    try:
        q = torch.zeros((17, 64), dtype=torch.int8, device="cuda")
        with pytest.raises(qg.QiftError):
            qg.qift_linear(q, torch.ones(17, device="cuda"), torch.zeros((8, 4), dtype=torch.int32, device="cuda"),
                           torch.ones(8, device="cuda"), "qift")
    finally:
        qg.qift_debug_set_linear_path("auto")


# ---------------------------------------------------------- one-launch decode (fused a3-a5)
@pytest.mark.parametrize("name", ["qift", "pot"])
@pytest.mark.parametrize("T,N,K,block", [(1, 4096, 4096, 4096), (1, 37, 64, 16), (2, 300, 512, 128), (3, 129, 11008, 128),
                                          (4, 64, 14336, 128), (1, 1, 1024, 0), (4, 200, 2048, 2048), (1, 5000, 512, 512),
                                          (1, 14336, 4096, 4096), (1, 300, 11008, 128), (1, 4096, 14336, 128),
                                          (1, 149, 8192, 2048), (1, 28000, 4096, 128)])
def test_decode_linear_matches_oracle(name, T, N, K, block):
    rng = np.random.default_rng(T * 7 + N + K)
    x = synth.activations(T, K, (T, N, K), n_outliers=synth.outlier_count(K))
    codes = rng.integers(0, 2 ** 32, size=(N, K // 16), dtype=np.uint64).astype(np.uint32)
    s_w = rng.uniform(1e-3, 1e-2, N).astype(np.float32)
    q, s_a, _ = oracle.quantize_acts(x, block)
    for out_dtype, npdt in ((torch.float16, np.float16), (torch.float32, np.float32)):
        ref, _ = oracle.linear(q, s_a, codes, s_w, name, npdt)
        gq = torch.empty((T, K), dtype=torch.int8, device="cuda")
        gsa = torch.empty(T, dtype=torch.float32, device="cuda")
        gy = qg.qift_decode_linear(dev(x), block, dev(codes.view(np.int32)), dev(s_w), name, out_dtype,
                                   q_out=gq, act_scale_out=gsa)
        assert np.array_equal(host(gy).view(np.uint16 if npdt == np.float16 else np.uint32),
                              ref.view(np.uint16 if npdt == np.float16 else np.uint32))
        assert np.array_equal(host(gq), q)
        assert np.array_equal(host(gsa).view(np.uint32), s_a.view(np.uint32))


@pytest.mark.parametrize("pin", ["auto", "gemv"])   # gemv: one token on the warp-per-row kernel
@pytest.mark.parametrize("T,N,K,block", [(1, 4096, 4096, 4096), (1, 37, 64, 16), (2, 300, 512, 128),
                                          (3, 129, 11008, 128), (4, 64, 14336, 128), (1, 1, 1024, 0),
                                          (1, 14336, 4096, 128), (1, 4096, 14336, 128), (1, 149, 16384, 2048),
                                          (1, 28000, 4096, 128), (4, 200, 2048, 2048)])
def test_decode_linear_w4_matches_oracle(pin, T, N, K, block):
    # 4-bit weights through the one-launch decode: rotation + INT4 + W4A4 linear, bit-exact
    rng = np.random.default_rng(T * 11 + N + K)
    x = synth.activations(T, K, (T, N, K, 4), n_outliers=synth.outlier_count(K))
    codes = rng.integers(0, 2 ** 32, size=(N, K // 8), dtype=np.uint64).astype(np.uint32)
    s_w = rng.uniform(1e-3, 1e-2, N).astype(np.float32)
    q, s_a, _ = oracle.quantize_acts(x, block)
    qg.qift_debug_set_linear_path(pin)
    try:
        for out_dtype, npdt in ((torch.float16, np.float16), (torch.float32, np.float32)):
            ref, _ = oracle.linear_w4(q, s_a, codes, s_w, npdt)
            gq = torch.empty((T, K), dtype=torch.int8, device="cuda")
            gsa = torch.empty(T, dtype=torch.float32, device="cuda")
            gy = qg.qift_decode_linear(dev(x), block, dev(codes.view(np.int32)), dev(s_w), "int4", out_dtype,
                                       q_out=gq, act_scale_out=gsa)
            u = np.uint16 if npdt == np.float16 else np.uint32
            assert np.array_equal(host(gy).view(u), ref.view(u)), (pin, T, N, K, block)
            assert np.array_equal(host(gq), q)
            assert np.array_equal(host(gsa).view(np.uint32), s_a.view(np.uint32))
    finally:
        qg.qift_debug_set_linear_path("auto")
    assert qg.qift_device_error() == (qg.QIFT_OK, 0)


def test_decode_linear_w4_extreme_accumulators():
    # every activation at +7 (a token of equal entries, no rotation) against the outer levels
    # +-7: |acc| = 49 K at the largest n_in the one-launch decode takes
    T, N, K = 1, 8, 16384
    x = np.full((T, K), 3.0, np.float16)
    codes = np.full((N, K // 8), 0x77777777, np.uint32)
    codes[1::2] = 0x99999999
    codes[2] = 0x79797979
    s_w = np.ones(N, np.float32)
    q, s_a, _ = oracle.quantize_acts(x, 0)
    assert q.min() == 7
    ref, acc = oracle.linear_w4(q, s_a, codes, s_w, np.float32)
    assert acc.max() == 49 * K and acc.min() == -49 * K
    gy = qg.qift_decode_linear(dev(x), 0, dev(codes.view(np.int32)), dev(s_w), "int4", torch.float32)
    assert np.array_equal(host(gy).view(np.uint32), ref.view(np.uint32))


@pytest.mark.parametrize("name", ["qift", "pot"])
@pytest.mark.parametrize("N,K,block", [(4096, 4096, 4096), (300, 512, 128)])
def test_decode_linear_one_token_pinned_to_warp_per_row(name, N, K, block):
    # Any pin other than auto / one_token sends a one-token decode to the warp-per-row kernel.
    rng = np.random.default_rng(N + K)
    x = synth.activations(1, K, (N, K), n_outliers=synth.outlier_count(K))
    codes = rng.integers(0, 2 ** 32, size=(N, K // 16), dtype=np.uint64).astype(np.uint32)
    s_w = rng.uniform(1e-3, 1e-2, N).astype(np.float32)
    q, s_a, _ = oracle.quantize_acts(x, block)
    ref, _ = oracle.linear(q, s_a, codes, s_w, name, np.float16)
    qg.qift_debug_set_linear_path("gemv")
    try:
        gy = qg.qift_decode_linear(dev(x), block, dev(codes.view(np.int32)), dev(s_w), name, torch.float16)
    finally:
        qg.qift_debug_set_linear_path("auto")
    assert np.array_equal(host(gy).view(np.uint16), ref.view(np.uint16))


def test_decode_linear_zero_token_and_unsupported():
    K, N = 256, 40
    x = np.zeros((2, K), np.float16)
    x[1] = synth.activations(1, K, (3,))[0]
    rng = np.random.default_rng(0)
    codes = rng.integers(0, 2 ** 32, size=(N, K // 16), dtype=np.uint64).astype(np.uint32)
    s_w = rng.uniform(1e-3, 1e-2, N).astype(np.float32)
    q, s_a, _ = oracle.quantize_acts(x, 64)
    ref, _ = oracle.linear(q, s_a, codes, s_w, "qift", np.float32)
    gy = qg.qift_decode_linear(dev(x), 64, dev(codes.view(np.int32)), dev(s_w), "qift", torch.float32)
    assert np.array_equal(host(gy), ref)
    with pytest.raises(qg.QiftError):
        qg.qift_decode_linear(dev(np.zeros((5, K), np.float16)), 64, dev(codes.view(np.int32)), dev(s_w))
