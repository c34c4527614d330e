"""Host-side tests of the C ABI: the library loads without a GPU, exports every entry point
that include/qift.h declares, and rejects invalid arguments on the host before it launches
anything (no call here reaches a kernel)."""
import ctypes as C
import os
import re

import pytest

import w2a4_gemm_b200 as q
from w2a4_gemm_b200 import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    build.build()
    return q.lib()


def declared_functions():
    names = []
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            src = open(os.path.join(ROOT, "include", fn)).read()
            src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
            names += re.findall(r"\b(qift_[a-z0-9_]+)\s*\(", src)
    return sorted(set(names))


def test_header_declares_the_four_calls():
    d = declared_functions()
    for name in ("qift_rotate", "qift_quantize_weights", "qift_quantize_acts", "qift_linear"):
        assert name in d


def test_every_declared_symbol_is_exported(L):
    for name in declared_functions():
        assert hasattr(L, name), name


def test_status_strings(L):
    for s in range(5):
        assert q.qift_status_string(s).startswith("QIFT_")
    assert "UNKNOWN" in q.qift_status_string(99)


FAKE = C.c_void_p(0x10000)          # 16-byte aligned, never dereferenced: validation fails first
MIS = C.c_void_p(0x10004)           # misaligned


def test_rotate_validation(L):
    bad = q.QIFT_ERR_INVALID_ARG
    assert L.qift_rotate(FAKE, FAKE, 0, 4, 96, 64, None) == bad        # n % block
    assert L.qift_rotate(FAKE, FAKE, 0, 4, 96, 3, None) == bad         # not a power of two
    assert L.qift_rotate(FAKE, FAKE, 0, 4, 8192, 8192, None) == bad    # block > 4096
    assert L.qift_rotate(FAKE, FAKE, 7, 4, 64, 64, None) == bad        # dtype
    assert L.qift_rotate(None, FAKE, 0, 4, 64, 64, None) == bad        # null
    assert L.qift_rotate(MIS, FAKE, 0, 4, 64, 64, None) == bad         # alignment
    assert L.qift_rotate(FAKE, C.c_void_p(0x10010), 0, 4, 64, 64, None) == bad  # partial overlap
    assert L.qift_rotate(FAKE, FAKE, 0, 0, 64, 64, None) == q.QIFT_OK  # empty: no-op
    assert L.qift_rotate(None, None, 1, 5, 0, 64, None) == q.QIFT_OK


def test_quantize_weights_validation(L):
    bad = q.QIFT_ERR_INVALID_ARG
    f = L.qift_quantize_weights
    assert f(FAKE, 4, 40, 0, 100, 0.2, 1.0, FAKE, FAKE, None, None) == bad    # n_in % 16
    assert f(FAKE, 4, 64, 4, 100, 0.2, 1.0, FAKE, FAKE, None, None) == bad    # set
    assert f(FAKE, 4, 64, 0, 1, 0.2, 1.0, FAKE, FAKE, None, None) == bad      # grid
    assert f(FAKE, 4, 64, 0, 257, 0.2, 1.0, FAKE, FAKE, None, None) == bad
    assert f(FAKE, 4, 64, 0, 100, 0.0, 1.0, FAKE, FAKE, None, None) == bad    # lo
    assert f(FAKE, 4, 64, 0, 100, 0.5, 0.4, FAKE, FAKE, None, None) == bad    # hi < lo
    assert f(FAKE, 4, 64, 0, 100, 0.2, float("nan"), FAKE, FAKE, None, None) == bad
    assert f(FAKE, 4, 64, 0, 100, 0.2, 1.0, None, FAKE, None, None) == bad    # null codes
    assert f(FAKE, 4, 64, 0, 100, 0.2, 1.0, FAKE, FAKE, C.c_void_p(0x10004), None) == bad
    assert f(FAKE, 4, 65536, 0, 100, 0.2, 1.0, FAKE, FAKE, None, None) == q.QIFT_ERR_UNSUPPORTED
    assert f(None, 0, 64, 0, 100, 0.2, 1.0, None, None, None, None) == q.QIFT_OK


def test_quantize_weights_asym_validation(L):
    bad = q.QIFT_ERR_INVALID_ARG
    f = L.qift_quantize_weights_asym
    assert f(FAKE, 4, 40, 100, 0.2, 1.0, FAKE, FAKE, FAKE, None, None) == bad    # n_in % 16
    assert f(FAKE, 4, 64, 1, 0.2, 1.0, FAKE, FAKE, FAKE, None, None) == bad      # grid
    assert f(FAKE, 4, 64, 100, 0.5, 0.4, FAKE, FAKE, FAKE, None, None) == bad    # hi < lo
    assert f(FAKE, 4, 64, 100, 0.2, 1.0, FAKE, FAKE, None, None, None) == bad    # null zeros
    assert f(FAKE, 4, 64, 100, 0.2, 1.0, FAKE, FAKE, C.c_void_p(0x10002), None, None) == bad  # zeros alignment
    assert f(FAKE, 4, 65536, 100, 0.2, 1.0, FAKE, FAKE, FAKE, None, None) == q.QIFT_ERR_UNSUPPORTED
    assert f(None, 0, 64, 100, 0.2, 1.0, None, None, None, None, None) == q.QIFT_OK


def test_quantize_acts_validation(L):
    bad = q.QIFT_ERR_INVALID_ARG
    f = L.qift_quantize_acts
    assert f(FAKE, 2, 40, 0, FAKE, FAKE, None) == bad          # n_in % 16
    assert f(FAKE, 2, 64, 3, FAKE, FAKE, None) == bad          # block
    assert f(FAKE, 2, 96, 64, FAKE, FAKE, None) == bad         # n_in % block
    assert f(FAKE, -1, 64, 0, FAKE, FAKE, None) == bad
    assert f(MIS, 2, 64, 0, FAKE, FAKE, None) == bad
    assert f(FAKE, 2, 65536, 0, FAKE, FAKE, None) == q.QIFT_ERR_UNSUPPORTED
    assert f(None, 0, 64, 0, None, None, None) == q.QIFT_OK


def test_linear_validation(L):
    bad = q.QIFT_ERR_INVALID_ARG
    f = L.qift_linear
    assert f(FAKE, FAKE, FAKE, FAKE, 2, 1, 8, 64, FAKE, 1, None) == q.QIFT_ERR_UNSUPPORTED   # std set
    assert f(FAKE, FAKE, FAKE, FAKE, 5, 1, 8, 64, FAKE, 1, None) == bad
    assert f(FAKE, FAKE, FAKE, FAKE, 0, 1, 8, 40, FAKE, 1, None) == bad                      # n_in % 16
    assert f(FAKE, FAKE, FAKE, FAKE, 0, 1, 8, 64, FAKE, 3, None) == bad                      # out dtype
    assert f(FAKE, FAKE, None, FAKE, 0, 1, 8, 64, FAKE, 1, None) == bad
    assert f(FAKE, FAKE, FAKE, FAKE, 0, 1, 8, 64, MIS, 1, None) == bad
    assert f(FAKE, FAKE, FAKE, FAKE, 0, 1, 8, 65536, FAKE, 1, None) == q.QIFT_ERR_UNSUPPORTED
    assert f(None, None, None, None, 0, 0, 8, 64, None, 1, None) == q.QIFT_OK                # no tokens
    assert f(None, None, None, None, 1, 3, 0, 64, None, 0, None) == q.QIFT_OK                # no outputs
    # prefill sizes (>= 17 tokens) need n_in % 64 == 0 for the tensor cores: refused, not run on
    # the CUDA-core GEMV
    assert f(FAKE, FAKE, FAKE, FAKE, 0, 17, 8, 80, FAKE, 1, None) == q.QIFT_ERR_UNSUPPORTED
    assert f(FAKE, FAKE, FAKE, FAKE, 1, 2048, 8, 4112, FAKE, 0, None) == q.QIFT_ERR_UNSUPPORTED
    # 4-bit weights (set 3): any batch, n_in a multiple of 64; zero tokens is still a no-op
    assert f(FAKE, FAKE, FAKE, FAKE, 4, 1, 8, 64, FAKE, 1, None) == bad                      # set
    assert f(FAKE, FAKE, FAKE, FAKE, 3, 17, 8, 48, FAKE, 1, None) == q.QIFT_ERR_UNSUPPORTED
    assert f(FAKE, FAKE, FAKE, FAKE, 3, 2, 8, 48, FAKE, 1, None) == q.QIFT_ERR_UNSUPPORTED
    assert f(None, None, None, None, 3, 0, 8, 64, None, 1, None) == q.QIFT_OK


def test_python_binding_refuses_cpu_tensors():
    import torch
    with pytest.raises(ValueError):
        q.qift_quantize_acts(torch.zeros(2, 64, dtype=torch.float16), 16)
    with pytest.raises(ValueError):
        q.qift_rotate(torch.zeros(2, 64), 16)
