"""The parity suite run against the bounds-checked build of the library.

`python -m w2a4_gemm_b200.build --check` compiles every kernel with QIFT_CHECK: each global index,
bulk-copy range, tensor-map coordinate and tensor-memory address a kernel computes is tested
against the extent its own arguments imply, and a failure is recorded in the device error word
(the access is skipped; nothing traps).  This test builds that library and runs
tests/test_gpu_parity.py against it in a child process; the suite's autouse fixture asserts,
after every test, that no check failed.  The tests that drive the bounded-wait failure paths are
not part of that file, so a clear error word is the expected state throughout.
"""
import os
import subprocess
import sys

import pytest
import torch

from w2a4_gemm_b200 import build

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_parity_suite_under_bounds_checks():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    lib = build.build(check=True)
    env = dict(os.environ, QIFT_LIB_PATH=lib)
    cmd = [sys.executable, "-m", "pytest", os.path.join(ROOT, "tests", "test_gpu_parity.py"), "-m", "gpu", "-x", "-q",
           "-p", "no:cacheprovider"]
    r = subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=1800)
    tail = (r.stdout + r.stderr)[-3000:]
    assert r.returncode == 0, tail
    assert " passed" in r.stdout, tail


def test_checked_library_reports_itself():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    lib = build.build(check=True)
    code = ("import w2a4_gemm_b200 as qg; import torch; torch.cuda.init(); "
            "assert qg.qift_debug_checked_build(); assert qg.qift_debug_check_line() == 0; print('ok')")
    r = subprocess.run([sys.executable, "-c", code], cwd=ROOT, env=dict(os.environ, QIFT_LIB_PATH=lib),
                       capture_output=True, text=True, timeout=600)
    assert r.returncode == 0 and "ok" in r.stdout, (r.stdout + r.stderr)[-2000:]
