"""Build ``libqift.so`` (the CUDA kernels and the C ABI) in-tree for sm_100a.

    python -m w2a4_gemm_b200.build [--force] [--verbose-ptxas] [--check]

``--check`` builds ``libqift_check.so`` instead: the same sources with ``-DQIFT_CHECK`` (every
global index, bulk-copy range, tensor-map coordinate and tensor-memory address a kernel computes
is tested against its arguments' extents; a failure is recorded in the device error word and the
access skipped) and relocatable device code, so that every kernel file reports into one device
word.  It is a test build: the binding loads it when ``QIFT_LIB_PATH`` names it.

Each ``csrc/*.cu`` is compiled to an object under ``_build/`` (in parallel), then linked with
the static CUDA runtime into ``w2a4_gemm_b200/libqift.so``.  Flags: ``-gencode
arch=compute_100a,code=sm_100a`` (B200 only), ``-O3 -lineinfo``, and ``--fmad=false`` so that
no multiply-add pair is contracted: every floating-point step is the single IEEE operation the
source writes, which keeps the quantization decisions reproducible.
"""
from __future__ import annotations

import concurrent.futures as cf
import glob
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
BUILD = os.path.join(ROOT, "_build")
LIB = os.path.join(PKG, "libqift.so")
LIB_CHECK = os.path.join(PKG, "libqift_check.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
CFLAGS = ARCH + ["-O3", "-lineinfo", "--fmad=false", "-std=c++17", "-Xcompiler", "-fPIC,-O2",
                 "--expt-relaxed-constexpr", "-I" + os.path.join(ROOT, "include")]


def _sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _deps():
    return _sources() + glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.h")) + \
        glob.glob(os.path.join(ROOT, "include", "*.h"))


def _stale(target, deps):
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    return any(os.path.getmtime(d) > t for d in deps)


CHECK_FLAGS = ["-DQIFT_CHECK", "-rdc=true"]


def _compile(src, ptxas_verbose, check=False):
    obj = os.path.join(BUILD, ("check_" if check else "") + os.path.basename(src) + ".o")
    headers = glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.h")) + \
        glob.glob(os.path.join(ROOT, "include", "*.h"))
    if not _stale(obj, [src] + headers) and not ptxas_verbose:
        return obj, ""
    cmd = [NVCC, *CFLAGS, *(CHECK_FLAGS if check else []), "-c", src, "-o", obj]
    if ptxas_verbose:
        cmd.insert(1, "-Xptxas=-v")
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"nvcc failed for {src}:\n{r.stdout}\n{r.stderr}")
    return obj, r.stderr


def build(force: bool = False, ptxas_verbose: bool = False, check: bool = False) -> str:
    """Compile and link libqift.so (libqift_check.so with check=True) if any source is newer
    than it; return the library path."""
    lib = LIB_CHECK if check else LIB
    if not force and not ptxas_verbose and not _stale(lib, _deps()):
        return lib
    os.makedirs(BUILD, exist_ok=True)
    srcs = _sources()
    with cf.ThreadPoolExecutor(max_workers=min(8, len(srcs))) as ex:
        results = list(ex.map(lambda s: _compile(s, ptxas_verbose, check), srcs))
    if ptxas_verbose:
        for obj, log in results:
            sys.stderr.write(log)
    tmp = lib + f".tmp{os.getpid()}"
    cmd = [NVCC, *ARCH, *(["-rdc=true"] if check else []), "-shared", "-cudart", "static", "-o", tmp] + \
        [o for o, _ in results]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"link failed:\n{r.stdout}\n{r.stderr}")
    os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, ptxas_verbose="--verbose-ptxas" in sys.argv,
                check="--check" in sys.argv))
