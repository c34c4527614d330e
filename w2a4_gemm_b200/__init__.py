"""Python binding of libqift.so -- the B200 (sm_100a) hot path of Qift W2A4 linear layers.

"Qift: Shift-Friendly No-Zero W2 Post-Training Quantization for Rotated W2A4/KV4 LLM
Inference" (Huang, Tsai), Abstract: Hadamard-rotated weights and activations, fixed no-zero
2-bit level sets with one scale per output channel, 4-bit activations.

The functions here carry the C ABI's names (``include/qift.h``) and only marshal arguments:
they check devices, dtypes and shapes, allocate outputs with torch, and pass raw device
pointers plus the current CUDA stream to the library.  Every step of the path runs in the
library's kernels.  There is no CPU fallback: without the built library or a CUDA device
these functions raise.
"""
from __future__ import annotations

import ctypes as C
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
# QIFT_LIB_PATH selects another build of the same library -- the bounds-checked test build
# (libqift_check.so, `python -m w2a4_gemm_b200.build --check`); by default the normal one.
LIB_PATH = os.environ.get("QIFT_LIB_PATH") or os.path.join(_HERE, "libqift.so")

QIFT_OK, QIFT_ERR_INVALID_ARG, QIFT_ERR_UNSUPPORTED, QIFT_ERR_CUDA, QIFT_ERR_TIMEOUT = range(5)
QIFT_SET_QIFT, QIFT_SET_POT, QIFT_SET_STD, QIFT_SET_INT4 = 0, 1, 2, 3
QIFT_F32, QIFT_F16 = 0, 1
LEVELSETS = {"qift": QIFT_SET_QIFT, "pot": QIFT_SET_POT, "std": QIFT_SET_STD, "int4": QIFT_SET_INT4}

_lib = None


class QiftError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {qift_status_string(status)}")


def lib() -> C.CDLL:
    """Load libqift.so from the package directory; raise if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with `python -m w2a4_gemm_b200.build`")
        L = C.CDLL(LIB_PATH)
        i64, i32, f64, vp = C.c_int64, C.c_int32, C.c_double, C.c_void_p
        L.qift_rotate.argtypes = [vp, vp, i32, i64, i64, i32, vp]
        L.qift_quantize_weights.argtypes = [vp, i64, i64, i32, i32, f64, f64, vp, vp, vp, vp]
        L.qift_rotate_quantize_weights.argtypes = [vp, i64, i64, i32, i32, i32, f64, f64, vp, vp, vp, vp]
        L.qift_quantize_weights_asym.argtypes = [vp, i64, i64, i32, f64, f64, vp, vp, vp, vp, vp]
        L.qift_quantize_acts.argtypes = [vp, i64, i64, i32, vp, vp, vp]
        L.qift_quantize_kv.argtypes = [vp, i64, i64, i32, vp, vp, vp]
        L.qift_dequantize_kv.argtypes = [vp, vp, i64, i64, i32, vp, vp]
        L.qift_linear.argtypes = [vp, vp, vp, vp, i32, i64, i64, i64, vp, i32, vp]
        L.qift_decode_linear.argtypes = [vp, i64, i64, i32, vp, vp, i32, i64, vp, i32, vp, vp, vp]
        L.qift_device_error.argtypes = [vp, C.POINTER(i32)]
        L.qift_debug_set_wait_limit.argtypes = [i64]
        L.qift_debug_stall_next_gemm.argtypes = []
        L.qift_debug_stall_next_one_token.argtypes = []
        L.qift_debug_set_linear_path.argtypes = [i32]
        L.qift_debug_set_pdl.argtypes = [i32]
        L.qift_debug_check_line.argtypes = [C.POINTER(i32)]
        L.qift_debug_checked_build.argtypes = []
        L.qift_debug_checked_build.restype = i32
        L.qift_status_string.argtypes = [i32]
        L.qift_status_string.restype = C.c_char_p
        for name in ("qift_rotate", "qift_quantize_weights", "qift_rotate_quantize_weights",
                     "qift_quantize_weights_asym", "qift_quantize_acts",
                     "qift_quantize_kv", "qift_dequantize_kv",
                     "qift_linear", "qift_decode_linear",
                     "qift_device_error", "qift_debug_set_wait_limit", "qift_debug_stall_next_gemm",
                     "qift_debug_stall_next_one_token",
                     "qift_debug_set_linear_path", "qift_debug_set_pdl", "qift_debug_check_line"):
            getattr(L, name).restype = C.c_int
        _lib = L
    return _lib


def qift_status_string(status: int) -> str:
    return lib().qift_status_string(int(status)).decode()


def _stream(stream, device=None):
    """The stream to launch on: `stream`, else the current stream of `device` (the device the
    call's tensors live on)."""
    if stream is None:
        stream = torch.cuda.current_stream(device)
    elif device is not None and stream.device != device:
        raise ValueError(f"stream is on {stream.device}, the tensors on {device}")
    return C.c_void_p(stream.cuda_stream)


def _ptr(t):
    return C.c_void_p(t.data_ptr()) if t is not None else None


def _cuda(t: torch.Tensor, name: str, dtype=None):
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor (the library has no CPU path)")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t


def _same_device(*named):
    """All given (name, tensor) pairs (None tensors skipped) on one CUDA device; returns it."""
    dev = None
    for name, t in named:
        if t is None:
            continue
        if dev is None:
            dev, first = t.device, name
        elif t.device != dev:
            raise ValueError(f"{name} is on {t.device}, {first} on {dev}: every tensor of a call must be on one device")
    return dev


def _shape(t: torch.Tensor, name: str, shape: tuple):
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    return t


def _at_least(t: torch.Tensor, name: str, n: int):
    if t.numel() < n:
        raise ValueError(f"{name} must hold at least {n} elements, got {t.numel()}")
    return t


def _2d(t: torch.Tensor, name: str):
    if t.dim() != 2:
        raise ValueError(f"{name} must be 2-D, got shape {tuple(t.shape)}")
    return t


def _check(status: int, what: str):
    if status != QIFT_OK:
        raise QiftError(status, what)


def _set(levelset) -> int:
    return LEVELSETS[levelset] if isinstance(levelset, str) else int(levelset)


def _codes_per_word(levelset) -> int:
    """Codes per 32-bit word: 16 two-bit codes, or 8 four-bit codes for the INT4 set."""
    return 8 if _set(levelset) == QIFT_SET_INT4 else 16


def qift_rotate(x: torch.Tensor, block: int, out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """Block-diagonal normalised Walsh-Hadamard rotation along the last axis (fp32 or fp16)."""
    _cuda(x, "x")
    if x.dtype not in (torch.float32, torch.float16):
        raise ValueError("x must be float32 or float16")
    if x.dim() == 0:
        raise ValueError("x must have at least one dimension")
    if out is not None:
        _shape(_cuda(out, "out", x.dtype), "out", x.shape)
    dev = _same_device(("x", x), ("out", out))
    y = torch.empty_like(x) if out is None else out
    n = x.shape[-1]
    rows = x.numel() // n if n else 0
    dt = QIFT_F32 if x.dtype == torch.float32 else QIFT_F16
    with torch.cuda.device(dev):
        _check(lib().qift_rotate(_ptr(x), _ptr(y), dt, rows, n, block, _stream(stream, dev)), "qift_rotate")
    return y


def qift_quantize_weights(w_rot: torch.Tensor, levelset="qift", grid_points: int = 100, lo: float = 0.2,
                          hi: float = 1.0, with_mse: bool = True, stream=None):
    """Per-row scale search + nearest-level encode + 2-bit pack (4-bit for ``"int4"``).

    Returns ``(codes int32-viewed-as-u32 [N, K/16] ([N, K/8] for "int4"), scales f32 [N],
    row_mse f64 [N] or None)``.
    """
    _2d(_cuda(w_rot, "w_rot", torch.float32), "w_rot")
    n_out, n_in = w_rot.shape
    dev = w_rot.device
    codes = torch.empty((n_out, n_in // _codes_per_word(levelset)), dtype=torch.int32, device=dev)
    scales = torch.empty(n_out, dtype=torch.float32, device=dev)
    mse = torch.empty(n_out, dtype=torch.float64, device=dev) if with_mse else None
    with torch.cuda.device(dev):
        _check(lib().qift_quantize_weights(_ptr(w_rot), n_out, n_in, _set(levelset), grid_points, lo, hi,
                                           _ptr(codes), _ptr(scales), _ptr(mse), _stream(stream, dev)),
               "qift_quantize_weights")
    return codes, scales, mse


def qift_quantize_weights_asym(w_rot: torch.Tensor, grid_points: int = 100, lo: float = 0.2, hi: float = 1.0,
                               with_mse: bool = True, stream=None):
    """Conventional asymmetric W2 baseline: per-row scale and integer zero point, weight (c - z) * s.

    Returns ``(codes int32-viewed-as-u32 [N, K/16], scales f32 [N], zeros int32 [N],
    row_mse f64 [N] or None)``.
    """
    _2d(_cuda(w_rot, "w_rot", torch.float32), "w_rot")
    n_out, n_in = w_rot.shape
    dev = w_rot.device
    codes = torch.empty((n_out, n_in // 16), dtype=torch.int32, device=dev)
    scales = torch.empty(n_out, dtype=torch.float32, device=dev)
    zeros = torch.empty(n_out, dtype=torch.int32, device=dev)
    mse = torch.empty(n_out, dtype=torch.float64, device=dev) if with_mse else None
    with torch.cuda.device(dev):
        _check(lib().qift_quantize_weights_asym(_ptr(w_rot), n_out, n_in, grid_points, lo, hi, _ptr(codes),
                                                _ptr(scales), _ptr(zeros), _ptr(mse), _stream(stream, dev)),
               "qift_quantize_weights_asym")
    return codes, scales, zeros, mse


def qift_rotate_quantize_weights(w: torch.Tensor, block: int, levelset="qift", grid_points: int = 100,
                                 lo: float = 0.2, hi: float = 1.0, with_mse: bool = True, stream=None):
    """Rotation (block b; 0 = none) + scale search + encode + pack in one pass over the raw
    weights.  Same outputs, bit for bit, as ``qift_quantize_weights(qift_rotate(w, b))``."""
    _2d(_cuda(w, "w", torch.float32), "w")
    n_out, n_in = w.shape
    dev = w.device
    codes = torch.empty((n_out, n_in // _codes_per_word(levelset)), dtype=torch.int32, device=dev)
    scales = torch.empty(n_out, dtype=torch.float32, device=dev)
    mse = torch.empty(n_out, dtype=torch.float64, device=dev) if with_mse else None
    with torch.cuda.device(dev):
        _check(lib().qift_rotate_quantize_weights(_ptr(w), n_out, n_in, block, _set(levelset), grid_points, lo,
                                                  hi, _ptr(codes), _ptr(scales), _ptr(mse), _stream(stream, dev)),
               "qift_rotate_quantize_weights")
    return codes, scales, mse


def qift_quantize_acts(x: torch.Tensor, block: int = 0, out_q: torch.Tensor | None = None,
                       out_scales: torch.Tensor | None = None, stream=None):
    """Optional rotation + symmetric per-token INT4.  Returns ``(q int8 [T, K], s_a f32 [T])``."""
    _2d(_cuda(x, "x", torch.float16), "x")
    T, K = x.shape
    if out_q is not None:
        _shape(_cuda(out_q, "out_q", torch.int8), "out_q", (T, K))
    if out_scales is not None:
        _at_least(_cuda(out_scales, "out_scales", torch.float32), "out_scales", T)
    dev = _same_device(("x", x), ("out_q", out_q), ("out_scales", out_scales))
    q = torch.empty((T, K), dtype=torch.int8, device=dev) if out_q is None else out_q
    s = torch.empty(T, dtype=torch.float32, device=dev) if out_scales is None else out_scales
    with torch.cuda.device(dev):
        _check(lib().qift_quantize_acts(_ptr(x), T, K, block, _ptr(q), _ptr(s), _stream(stream, dev)),
               "qift_quantize_acts")
    return q, s


def qift_quantize_kv(x: torch.Tensor, block: int, stream=None):
    """KV4: rotation by ``block`` + per-token INT4, two codes per byte.
    Returns ``(packed uint8 [T, n/2], scales f32 [T])``."""
    _2d(_cuda(x, "x", torch.float16), "x")
    T, n = x.shape
    dev = x.device
    packed = torch.empty((T, n // 2), dtype=torch.uint8, device=dev)
    scales = torch.empty(T, dtype=torch.float32, device=dev)
    with torch.cuda.device(dev):
        _check(lib().qift_quantize_kv(_ptr(x), T, n, block, _ptr(packed), _ptr(scales), _stream(stream, dev)),
               "qift_quantize_kv")
    return packed, scales


def qift_dequantize_kv(packed: torch.Tensor, scales: torch.Tensor, block: int, stream=None) -> torch.Tensor:
    """Inverse of ``qift_quantize_kv`` up to the quantization error: fp16 [T, n]."""
    _2d(_cuda(packed, "packed", torch.uint8), "packed")
    _cuda(scales, "scales", torch.float32)
    T, n2 = packed.shape
    _at_least(scales, "scales", T)
    dev = _same_device(("packed", packed), ("scales", scales))
    out = torch.empty((T, 2 * n2), dtype=torch.float16, device=dev)
    with torch.cuda.device(dev):
        _check(lib().qift_dequantize_kv(_ptr(packed), _ptr(scales), T, 2 * n2, block, _ptr(out),
                                        _stream(stream, dev)), "qift_dequantize_kv")
    return out


def qift_linear(q: torch.Tensor, act_scale: torch.Tensor, codes: torch.Tensor, w_scale: torch.Tensor,
                levelset="qift", out_dtype=torch.float16, out: torch.Tensor | None = None, stream=None):
    """Fused W2A4 linear (W4A4 for ``"int4"``, 1..16 tokens):
    ``y[t, n] = ((float)acc * w_scale[n]) * act_scale[t]``."""
    _cuda(q, "q", torch.int8)
    _cuda(act_scale, "act_scale", torch.float32)
    _cuda(codes, "codes")
    _cuda(w_scale, "w_scale", torch.float32)
    if codes.dtype not in (torch.int32, torch.uint32):
        raise ValueError("codes must be 32-bit words")
    if out_dtype not in (torch.float16, torch.float32):
        raise ValueError("out_dtype must be torch.float16 or torch.float32")
    _2d(q, "q")
    _2d(codes, "codes")
    T, K = q.shape
    N = codes.shape[0]
    cpw = _codes_per_word(levelset)
    if codes.shape[1] * cpw != K:
        raise ValueError(f"codes must be [n_out, n_in/{cpw}]")
    _at_least(act_scale, "act_scale", T)
    _at_least(w_scale, "w_scale", N)
    if out is not None:
        _shape(_cuda(out, "out", out_dtype), "out", (T, N))
    dev = _same_device(("q", q), ("act_scale", act_scale), ("codes", codes), ("w_scale", w_scale), ("out", out))
    y = torch.empty((T, N), dtype=out_dtype, device=dev) if out is None else out
    dt = QIFT_F16 if out_dtype == torch.float16 else QIFT_F32
    with torch.cuda.device(dev):
        _check(lib().qift_linear(_ptr(q), _ptr(act_scale), _ptr(codes), _ptr(w_scale), _set(levelset), T, N, K,
                                 _ptr(y), dt, _stream(stream, dev)), "qift_linear")
    return y


def qift_decode_linear(x: torch.Tensor, block: int, codes: torch.Tensor, w_scale: torch.Tensor, levelset="qift",
                       out_dtype=torch.float16, out: torch.Tensor | None = None, q_out: torch.Tensor | None = None,
                       act_scale_out: torch.Tensor | None = None, stream=None):
    """One-launch decode step (1..4 tokens): rotation + INT4 + W2A4 linear.  Returns y."""
    _cuda(x, "x", torch.float16)
    _cuda(codes, "codes")
    _cuda(w_scale, "w_scale", torch.float32)
    if codes.dtype not in (torch.int32, torch.uint32):
        raise ValueError("codes must be 32-bit words")
    if out_dtype not in (torch.float16, torch.float32):
        raise ValueError("out_dtype must be torch.float16 or torch.float32")
    _2d(x, "x")
    _2d(codes, "codes")
    T, K = x.shape
    N = codes.shape[0]
    cpw = _codes_per_word(levelset)
    if codes.shape[1] * cpw != K:
        raise ValueError(f"codes must be [n_out, n_in/{cpw}]")
    _at_least(w_scale, "w_scale", N)
    if out is not None:
        _shape(_cuda(out, "out", out_dtype), "out", (T, N))
    if q_out is not None:
        _shape(_cuda(q_out, "q_out", torch.int8), "q_out", (T, K))
    if act_scale_out is not None:
        _at_least(_cuda(act_scale_out, "act_scale_out", torch.float32), "act_scale_out", T)
    dev = _same_device(("x", x), ("codes", codes), ("w_scale", w_scale), ("out", out), ("q_out", q_out),
                       ("act_scale_out", act_scale_out))
    y = torch.empty((T, N), dtype=out_dtype, device=dev) if out is None else out
    dt = QIFT_F16 if out_dtype == torch.float16 else QIFT_F32
    with torch.cuda.device(dev):
        _check(lib().qift_decode_linear(_ptr(x), T, K, block, _ptr(codes), _ptr(w_scale), _set(levelset), N, _ptr(y),
                                        dt, _ptr(q_out), _ptr(act_scale_out), _stream(stream, dev)),
               "qift_decode_linear")
    return y


def qift_device_error(stream=None) -> tuple[int, int]:
    """Synchronise the stream, read and clear the device error word: ``(status, raw word)``."""
    detail = C.c_int32(0)
    st = lib().qift_device_error(_stream(stream), C.byref(detail))
    return st, detail.value


def qift_debug_checked_build() -> bool:
    """True when the loaded library is the bounds-checked test build."""
    return bool(lib().qift_debug_checked_build())


def qift_debug_check_line() -> int:
    """Source line of the first failed bounds check since the last call (0: none; always 0 in
    the normal build).  Read after qift_device_error(), which synchronises."""
    line = C.c_int32(0)
    _check(lib().qift_debug_check_line(C.byref(line)), "qift_debug_check_line")
    return line.value


def qift_debug_set_wait_limit(cycles: int) -> None:
    """Test hook: SM-cycle limit of every on-chip wait in later tensor-core GEMM and one-token
    launches (<= 0: default)."""
    _check(lib().qift_debug_set_wait_limit(int(cycles)), "qift_debug_set_wait_limit")


def qift_debug_stall_next_gemm() -> None:
    """Test hook: the next tensor-core GEMM waits on a barrier nothing arrives on and times out."""
    _check(lib().qift_debug_stall_next_gemm(), "qift_debug_stall_next_gemm")


def qift_debug_stall_next_one_token() -> None:
    """Test hook: the next one-token launch waits on a barrier nothing arrives on and times out."""
    _check(lib().qift_debug_stall_next_one_token(), "qift_debug_stall_next_one_token")


LINEAR_PATHS = {"auto": 0, "gemv": 1, "skinny": 2, "gemm_pair": 6, "one_token": 7}


def qift_debug_set_linear_path(path) -> None:
    """Test hook: pin qift_linear's kernel family in this thread ("auto", "gemv", "skinny",
    "gemm_pair", "one_token")."""
    p = LINEAR_PATHS[path] if isinstance(path, str) else int(path)
    _check(lib().qift_debug_set_linear_path(p), "qift_debug_set_linear_path")


def qift_debug_set_pdl(enable: bool) -> None:
    """Test hook: programmatic dependent launch of the decode kernels on (default) or off."""
    _check(lib().qift_debug_set_pdl(1 if enable else 0), "qift_debug_set_pdl")
