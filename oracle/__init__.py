"""CPU oracle for the Qift W2A4 linear path -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` / reference leg of
``bench.py`` may import this package.  The product path (``w2a4_gemm_b200``) never imports it
and must fail loudly if its CUDA library is missing; there is no CPU fallback.

The arithmetic lives in ``qift_oracle.c`` (plain C loops in IEEE binary32/binary64); this
module only marshals numpy arrays.  The one step done here in numpy is the single rounding of
the rotated activations to binary16 (``astype(np.float16)``, round-to-nearest-even), which the
C code cannot express portably.  ``source_model`` holds the Gaussian level-set analysis.

Paper: "Qift: Shift-Friendly No-Zero W2 Post-Training Quantization for Rotated W2A4/KV4 LLM
Inference" (Huang, Tsai), Abstract.
"""
from __future__ import annotations

import ctypes as C

import numpy as np

from . import build as _build

SET_QIFT, SET_POT, SET_STD = 0, 1, 2
SET_NAMES = {"qift": SET_QIFT, "pot": SET_POT, "std": SET_STD}

_lib = None


def lib():
    global _lib
    if _lib is None:
        path = _build.build()
        L = C.CDLL(path)
        i64, i32, f32, f64, vp = C.c_int64, C.c_int32, C.c_float, C.c_double, C.c_void_p
        L.qo_fwht_f64.argtypes = [vp, i64, i64, i32]
        L.qo_rotate_f32.argtypes = [vp, i64, i64, i32]
        L.qo_level.argtypes = [i32, i32]
        L.qo_level.restype = i32
        L.qo_candidate_scales.argtypes = [f32, i32, i32, f64, f64, vp]
        L.qo_quantize_weights.argtypes = [vp, i64, i64, i32, i32, f64, f64, vp, vp, vp, vp]
        L.qo_unpack_codes.argtypes = [vp, i64, i64, vp]
        L.qo_quantize_acts.argtypes = [vp, i64, i64, vp, vp]
        L.qo_linear.argtypes = [vp, vp, vp, vp, i32, i64, i64, i64, vp, vp]
        L.qo_quantize_weights_w4.argtypes = [vp, i64, i64, i32, f64, f64, vp, vp, vp, vp]
        L.qo_linear_w4.argtypes = [vp, vp, vp, vp, i64, i64, i64, vp, vp]
        L.qo_pack_int4.argtypes = [vp, i64, vp]
        L.qo_unpack_int4.argtypes = [vp, i64, vp]
        L.qo_dequantize_kv.argtypes = [vp, vp, i64, i64, i32, vp]
        L.qo_quantize_weights_asym.argtypes = [vp, i64, i64, i32, f64, f64, vp, vp, vp, vp, vp]
        L.qo_linear_asym.argtypes = [vp, vp, vp, vp, vp, i64, i64, i64, vp, vp]
        L.qo_set_threads.argtypes = [C.c_int]
        L.qo_set_threads.restype = C.c_int
        for name in ("qo_fwht_f64", "qo_rotate_f32", "qo_candidate_scales", "qo_quantize_weights",
                     "qo_unpack_codes", "qo_quantize_acts", "qo_linear", "qo_pack_int4", "qo_unpack_int4",
                     "qo_dequantize_kv", "qo_quantize_weights_w4", "qo_linear_w4", "qo_quantize_weights_asym",
                     "qo_linear_asym"):
            getattr(L, name).restype = C.c_int
        _lib = L
    return _lib


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(C.c_void_p) if a is not None else None


def _check(rc: int, what: str):
    if rc != 0:
        raise ValueError(f"oracle {what} failed with code {rc}")


def set_id(levelset) -> int:
    return SET_NAMES[levelset] if isinstance(levelset, str) else int(levelset)


# --------------------------------------------------------------------------------- rotation
def fwht_f64(x: np.ndarray, block: int) -> np.ndarray:
    """Block-diagonal normalised Sylvester Hadamard along the last axis, binary64 (R1, R2)."""
    y = np.ascontiguousarray(x, dtype=np.float64).copy()
    n = y.shape[-1]
    _check(lib().qo_fwht_f64(_ptr(y), y.size // max(n, 1), n, block), "fwht_f64")
    return y


def rotate_f32(x: np.ndarray, block: int) -> np.ndarray:
    """Same transform in binary32 with the canonical stage order (the weight rotation)."""
    y = np.ascontiguousarray(x, dtype=np.float32).copy()
    n = y.shape[-1]
    _check(lib().qo_rotate_f32(_ptr(y), y.size // max(n, 1), n, block), "rotate_f32")
    return y


def rotate_f16(x: np.ndarray, block: int) -> np.ndarray:
    """Activation rotation: binary16 in, binary32 stages, one rounding to binary16 out."""
    assert x.dtype == np.float16
    return rotate_f32(x.astype(np.float32), block).astype(np.float16)


# ------------------------------------------------------------------------- weight quantizer
def levels(levelset) -> np.ndarray:
    s = set_id(levelset)
    return np.array([lib().qo_level(s, c) for c in range(4)], dtype=np.int64)


def candidate_scales(m: float, levelset, grid_points: int = 100, lo: float = 0.2, hi: float = 1.0):
    out = np.zeros(grid_points, dtype=np.float32)
    _check(lib().qo_candidate_scales(C.c_float(m), set_id(levelset), grid_points, lo, hi, _ptr(out)),
           "candidate_scales")
    return out


def quantize_weights(w_rot: np.ndarray, levelset, grid_points: int = 100, lo: float = 0.2, hi: float = 1.0):
    """Per-row MSE scale search + nearest-level encode + 2-bit pack.

    Returns ``(codes u32 [N, K/16], scales f32 [N], row_mse f64 [N], best_k i32 [N])``.
    """
    w = np.ascontiguousarray(w_rot, dtype=np.float32)
    n_out, n_in = w.shape
    codes = np.zeros((n_out, n_in // 16), dtype=np.uint32)
    scales = np.zeros(n_out, dtype=np.float32)
    mse = np.zeros(n_out, dtype=np.float64)
    best = np.zeros(n_out, dtype=np.int32)
    _check(lib().qo_quantize_weights(_ptr(w), n_out, n_in, set_id(levelset), grid_points, lo, hi,
                                      _ptr(codes), _ptr(scales), _ptr(mse), _ptr(best)), "quantize_weights")
    return codes, scales, mse, best


def unpack_codes(codes: np.ndarray, n_in: int) -> np.ndarray:
    codes = np.ascontiguousarray(codes, dtype=np.uint32)
    out = np.zeros((codes.shape[0], n_in), dtype=np.uint8)
    _check(lib().qo_unpack_codes(_ptr(codes), codes.shape[0], n_in, _ptr(out)), "unpack_codes")
    return out


# --------------------------------------------------------------------- activation quantizer
def quantize_acts(x: np.ndarray, block: int = 0):
    """Rotate (if ``block``) and quantize activations to symmetric per-token INT4.

    ``x`` is binary16 ``[T, K]``.  Returns ``(q int8 [T, K], s_a f32 [T], x_rot f16 [T, K])``.
    """
    assert x.dtype == np.float16
    xr = rotate_f16(x, block) if block else x.copy()
    xf = np.ascontiguousarray(xr.astype(np.float32))
    T, K = xf.shape
    q = np.zeros((T, K), dtype=np.int8)
    s = np.zeros(T, dtype=np.float32)
    _check(lib().qo_quantize_acts(_ptr(xf), T, K, _ptr(q), _ptr(s)), "quantize_acts")
    return q, s, xr


# --------------------------------------------------------------------------------------- W4
W4_LEVELS = np.arange(-7, 8, dtype=np.int32)


def quantize_weights_w4(w_rot: np.ndarray, grid_points: int = 100, lo: float = 0.2, hi: float = 1.0):
    """W4 per-channel scale search + nearest-level encode + pack (levels {-7..7} * s).

    Returns ``(codes uint32 [N, K/8], scales f32 [N], row_mse f64 [N], best_k int32 [N])``;
    the code of input k is the level's two's-complement nibble, at bits
    ``8*(k%4) + 4*((k%8)//4)`` of word ``k/8`` (byte j: input j low, input j+4 high).
    """
    w = np.ascontiguousarray(w_rot, dtype=np.float32)
    n_out, n_in = w.shape
    codes = np.zeros((n_out, n_in // 8), dtype=np.uint32)
    scales = np.zeros(n_out, dtype=np.float32)
    mse = np.zeros(n_out, dtype=np.float64)
    best = np.zeros(n_out, dtype=np.int32)
    _check(lib().qo_quantize_weights_w4(_ptr(w), n_out, n_in, grid_points, lo, hi, _ptr(codes), _ptr(scales),
                                        _ptr(mse), _ptr(best)), "quantize_weights_w4")
    return codes, scales, mse, best


W4_SHIFTS = np.array([8 * (p % 4) + 4 * (p // 4) for p in range(8)], dtype=np.uint32)


def pack_w4(levels: np.ndarray) -> np.ndarray:
    """int levels [N, K] in [-8, 7] -> uint32 [N, K/8] in the W4 word layout."""
    lv = np.ascontiguousarray(levels).astype(np.int64)
    nib = (lv & 0xF).astype(np.uint32).reshape(lv.shape[0], -1, 8)
    return np.bitwise_or.reduce(nib << W4_SHIFTS[None, None, :], axis=2).astype(np.uint32)


def unpack_w4(codes: np.ndarray, n_in: int) -> np.ndarray:
    """uint32 [N, K/8] -> int8 levels [N, K] (two's-complement nibbles, -8..7)."""
    c = np.ascontiguousarray(codes, dtype=np.uint32)
    u = (c[:, :, None] >> W4_SHIFTS[None, None, :]) & np.uint32(0xF)
    u = u.reshape(c.shape[0], n_in).astype(np.int16)
    return np.where(u >= 8, u - 16, u).astype(np.int8)


def linear_w4(q: np.ndarray, s_a: np.ndarray, codes: np.ndarray, s_w: np.ndarray, out_dtype=np.float32):
    """W4A4 linear: int32 accumulators and the binary32 epilogue.  Returns ``(y, acc)``."""
    q = np.ascontiguousarray(q, dtype=np.int8)
    codes = np.ascontiguousarray(codes, dtype=np.uint32)
    s_a = np.ascontiguousarray(s_a, dtype=np.float32)
    s_w = np.ascontiguousarray(s_w, dtype=np.float32)
    T, K = q.shape
    N = codes.shape[0]
    assert codes.shape[1] * 8 == K
    acc = np.zeros((T, N), dtype=np.int32)
    y = np.zeros((T, N), dtype=np.float32)
    _check(lib().qo_linear_w4(_ptr(q), _ptr(s_a), _ptr(codes), _ptr(s_w), T, N, K, _ptr(acc), _ptr(y)), "linear_w4")
    return y.astype(out_dtype), acc


# ------------------------------------------------------------------- conventional asymmetric W2
def quantize_weights_asym(w_rot: np.ndarray, grid_points: int = 100, lo: float = 0.2, hi: float = 1.0):
    """Asymmetric 2-bit baseline: per channel scale s and integer zero point z in [0, 3], weight
    (c - z) * s, range shrunk over the candidate grid.  Returns
    ``(codes uint32 [N, K/16], scales f32 [N], zeros int32 [N], row_mse f64 [N], best_k int32 [N])``."""
    w = np.ascontiguousarray(w_rot, dtype=np.float32)
    n_out, n_in = w.shape
    codes = np.zeros((n_out, n_in // 16), dtype=np.uint32)
    scales = np.zeros(n_out, dtype=np.float32)
    zeros = np.zeros(n_out, dtype=np.int32)
    mse = np.zeros(n_out, dtype=np.float64)
    best = np.zeros(n_out, dtype=np.int32)
    _check(lib().qo_quantize_weights_asym(_ptr(w), n_out, n_in, grid_points, lo, hi, _ptr(codes), _ptr(scales),
                                          _ptr(zeros), _ptr(mse), _ptr(best)), "quantize_weights_asym")
    return codes, scales, zeros, mse, best


def linear_asym(q: np.ndarray, s_a: np.ndarray, codes: np.ndarray, s_w: np.ndarray, zeros: np.ndarray,
                out_dtype=np.float32):
    """Asymmetric W2A4 linear: levels c - z per row, int32 accumulators, binary32 epilogue."""
    q = np.ascontiguousarray(q, dtype=np.int8)
    codes = np.ascontiguousarray(codes, dtype=np.uint32)
    s_a = np.ascontiguousarray(s_a, dtype=np.float32)
    s_w = np.ascontiguousarray(s_w, dtype=np.float32)
    zeros = np.ascontiguousarray(zeros, dtype=np.int32)
    T, K = q.shape
    N = codes.shape[0]
    assert codes.shape[1] * 16 == K
    acc = np.zeros((T, N), dtype=np.int32)
    y = np.zeros((T, N), dtype=np.float32)
    _check(lib().qo_linear_asym(_ptr(q), _ptr(s_a), _ptr(codes), _ptr(s_w), _ptr(zeros), T, N, K, _ptr(acc),
                                _ptr(y)), "linear_asym")
    return y.astype(out_dtype), acc


# -------------------------------------------------------------------------------------- KV4
def pack_int4(q: np.ndarray) -> np.ndarray:
    """int8 [..., n] in [-8, 7] -> uint8 [..., n/2]: two's-complement nibbles, lower index low."""
    q = np.ascontiguousarray(q, dtype=np.int8)
    out = np.zeros(q.shape[:-1] + (q.shape[-1] // 2,), dtype=np.uint8)
    _check(lib().qo_pack_int4(_ptr(q), q.size, _ptr(out)), "pack_int4")
    return out


def unpack_int4(p: np.ndarray) -> np.ndarray:
    p = np.ascontiguousarray(p, dtype=np.uint8)
    out = np.zeros(p.shape[:-1] + (p.shape[-1] * 2,), dtype=np.int8)
    _check(lib().qo_unpack_int4(_ptr(p), out.size, _ptr(out)), "unpack_int4")
    return out


def quantize_kv(x: np.ndarray, block: int):
    """KV4: rotate by ``block`` (0 = none), per-token INT4, two codes per byte.

    ``x`` is binary16 ``[T, n]``.  Returns ``(packed uint8 [T, n/2], s f32 [T])``.
    """
    q, s, _ = quantize_acts(x, block)
    return pack_int4(q), s


def dequantize_kv(packed: np.ndarray, scales: np.ndarray, block: int) -> np.ndarray:
    """Inverse of ``quantize_kv`` up to the quantization error: (float)q * s in binary32, the
    inverse rotation in binary32, one rounding to binary16.  Returns float16 ``[T, n]``."""
    packed = np.ascontiguousarray(packed, dtype=np.uint8)
    scales = np.ascontiguousarray(scales, dtype=np.float32)
    T, n = packed.shape[0], packed.shape[1] * 2
    out = np.zeros((T, n), dtype=np.float32)
    _check(lib().qo_dequantize_kv(_ptr(packed), _ptr(scales), T, n, block, _ptr(out)), "dequantize_kv")
    return out.astype(np.float16)


# ---------------------------------------------------------------------------------- linear
def linear(q: np.ndarray, s_a: np.ndarray, codes: np.ndarray, s_w: np.ndarray, levelset,
           out_dtype=np.float32):
    """W2A4 linear: int32 accumulators and the binary32 epilogue (cast to ``out_dtype``).

    Returns ``(y [T, N], acc int32 [T, N])``.
    """
    q = np.ascontiguousarray(q, dtype=np.int8)
    codes = np.ascontiguousarray(codes, dtype=np.uint32)
    s_a = np.ascontiguousarray(s_a, dtype=np.float32)
    s_w = np.ascontiguousarray(s_w, dtype=np.float32)
    T, K = q.shape
    N = codes.shape[0]
    assert codes.shape[1] * 16 == K
    acc = np.zeros((T, N), dtype=np.int32)
    y = np.zeros((T, N), dtype=np.float32)
    _check(lib().qo_linear(_ptr(q), _ptr(s_a), _ptr(codes), _ptr(s_w), set_id(levelset), T, N, K,
                           _ptr(acc), _ptr(y)), "linear")
    return y.astype(out_dtype), acc


def pipeline(w: np.ndarray, x: np.ndarray, levelset, w_block: int, a_block: int, out_dtype=np.float16):
    """Whole path: rotate W (binary32), quantize W, rotate+quantize x, W2A4 linear."""
    w_rot = rotate_f32(w, w_block)
    codes, s_w, mse, best = quantize_weights(w_rot, levelset)
    q, s_a, _ = quantize_acts(x, a_block)
    y, acc = linear(q, s_a, codes, s_w, levelset, out_dtype)
    return dict(w_rot=w_rot, codes=codes, s_w=s_w, row_mse=mse, best_k=best, q=q, s_a=s_a, y=y, acc=acc)


def threads() -> int:
    """Host threads the oracle's OpenMP loops use."""
    return int(lib().qo_set_threads(0))


def set_threads(n: int) -> int:
    """Run the oracle's loops on n host threads from now on; returns the count in force."""
    return int(lib().qo_set_threads(int(n)))
