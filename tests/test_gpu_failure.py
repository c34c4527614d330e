"""Failure paths on a real GPU, driven without any fault: a test hook makes the tensor-core
GEMM's MMA thread, or every CTA of a one-token launch, wait on a barrier that nothing arrives
on.  The bounded wait must run out, the kernel must exit cleanly, qift_device_error() must
report QIFT_ERR_TIMEOUT once, and the same context must then compute correct results again."""
import numpy as np
import pytest
import torch

import oracle
import w2a4_gemm_b200 as qg
from w2a4_gemm_b200 import build

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _setup():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    build.build()
    qg.lib()
    yield
    qg.qift_debug_set_wait_limit(0)


def _case(T=128, N=256, K=512, seed=5):
    rng = np.random.default_rng(seed)
    q = rng.integers(-7, 8, size=(T, K)).astype(np.int8)
    codes = rng.integers(0, 2 ** 32, size=(N, K // 16), dtype=np.uint64).astype(np.uint32)
    s_w = rng.uniform(1e-3, 1e-2, N).astype(np.float32)
    s_a = rng.uniform(0.1, 2.0, T).astype(np.float32)
    ref, _ = oracle.linear(q, s_a, codes, s_w, "qift", np.float32)
    args = [torch.from_numpy(a).cuda() for a in (q, s_a, codes.view(np.int32), s_w)]
    return args, ref


@pytest.mark.parametrize("path", ["gemm_pair"])
def test_gemm_wait_timeout_is_reported_and_context_survives(path):
    args, ref = _case()
    qg.qift_debug_set_linear_path(path)
    assert qg.qift_device_error() == (qg.QIFT_OK, 0)
    qg.qift_debug_set_wait_limit(20_000_000)          # ~10 ms per wait
    qg.qift_debug_stall_next_gemm()
    qg.qift_linear(*args, "qift", torch.float32)
    status, word = qg.qift_device_error()
    assert status == qg.QIFT_ERR_TIMEOUT and word != 0
    assert qg.qift_device_error() == (qg.QIFT_OK, 0)  # read-and-clear
    qg.qift_debug_set_wait_limit(0)
    y = qg.qift_linear(*args, "qift", torch.float32)
    torch.cuda.synchronize()
    assert np.array_equal(y.cpu().numpy(), ref)
    assert qg.qift_device_error() == (qg.QIFT_OK, 0)
    qg.qift_debug_set_linear_path("auto")


@pytest.mark.parametrize("entry", ["linear", "decode"])
def test_one_token_wait_timeout_is_reported_and_context_survives(entry):
    rng = np.random.default_rng(11)
    N, K, block = 300, 4096, 128
    codes = rng.integers(0, 2 ** 32, size=(N, K // 16), dtype=np.uint64).astype(np.uint32)
    s_w = rng.uniform(1e-3, 1e-2, N).astype(np.float32)
    x = rng.standard_normal((1, K)).astype(np.float16)
    q, s_a, _ = oracle.quantize_acts(x, block)
    ref, _ = oracle.linear(q, s_a, codes, s_w, "qift", np.float32)
    gc, gw = torch.from_numpy(codes.view(np.int32)).cuda(), torch.from_numpy(s_w).cuda()
    if entry == "linear":
        gq, gsa = torch.from_numpy(q).cuda(), torch.from_numpy(s_a).cuda()
        call = lambda: qg.qift_linear(gq, gsa, gc, gw, "qift", torch.float32)
    else:
        gx = torch.from_numpy(x).cuda()
        call = lambda: qg.qift_decode_linear(gx, block, gc, gw, "qift", torch.float32)
    qg.qift_debug_set_linear_path("one_token")        # this shape would go to the warp-per-row GEMV
    try:
        assert qg.qift_device_error() == (qg.QIFT_OK, 0)
        qg.qift_debug_set_wait_limit(20_000_000)      # ~10 ms per wait
        qg.qift_debug_stall_next_one_token()
        call()
        status, word = qg.qift_device_error()
        assert status == qg.QIFT_ERR_TIMEOUT and word != 0
        assert qg.qift_device_error() == (qg.QIFT_OK, 0)  # read-and-clear
        qg.qift_debug_set_wait_limit(0)
        y = call()
        torch.cuda.synchronize()
        assert np.array_equal(y.cpu().numpy(), ref)
        assert qg.qift_device_error() == (qg.QIFT_OK, 0)
    finally:
        qg.qift_debug_set_linear_path("auto")
        qg.qift_debug_set_wait_limit(0)
