"""Shared pytest set-up: the ``gpu`` marker and the repository root on ``sys.path``."""
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

GOLDEN = os.path.join(ROOT, "tests", "golden")


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")


@pytest.fixture(autouse=True)
def _bounds_checked_run(request):
    """When the bounds-checked library is loaded (QIFT_LIB_PATH names libqift_check.so), every
    GPU test must leave the device error word clear: no kernel computed an index, copy range,
    tensor-map coordinate or tensor-memory address outside the extents its arguments imply."""
    if os.environ.get("QIFT_LIB_PATH") and request.node.get_closest_marker("gpu") is not None:
        import w2a4_gemm_b200 as qg
        qg.qift_device_error()  # start from a clear word
        qg.qift_debug_check_line()
    yield
    if not os.environ.get("QIFT_LIB_PATH") or request.node.get_closest_marker("gpu") is None:
        return
    import w2a4_gemm_b200 as qg
    status, word = qg.qift_device_error()
    site = qg.qift_debug_check_line()
    assert word & 0x100 == 0 and site == 0, f"bounds check failed at {check_site_name(site)} (word {word:#x})"


def check_site_name(site: int) -> str:
    """'file:line' of a bounds-check site recorded as file_tag * 100000 + line, the tag being the
    FNV-1a hash of the source file's base name modulo 1000 (as the library computes it)."""
    tag, line = divmod(site, 100000)
    csrc = os.path.join(ROOT, "w2a4_gemm_b200", "csrc")
    for name in sorted(os.listdir(csrc)):
        h = 2166136261
        for b in name.encode():
            h = ((h ^ b) * 16777619) & 0xFFFFFFFF
        if h % 1000 == tag:
            return f"{name}:{line}"
    return f"tag {tag}, line {line}"


def golden_lines(name):
    """Non-comment, non-empty lines of a golden fixture, split on whitespace."""
    with open(os.path.join(GOLDEN, name)) as f:
        return [ln.split() for ln in f if ln.strip() and not ln.lstrip().startswith("#")]
