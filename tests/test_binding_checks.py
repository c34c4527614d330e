"""The Python binding rejects, before anything is launched, tensors whose sizes or devices do not
fit the call: an undersized output or scale buffer would make a kernel write or read past its
end, and a tensor on another device would hand the library a pointer the launching device
cannot use.  Each case must raise ValueError and leave every buffer as it was."""
import pytest
import torch

import w2a4_gemm_b200 as qg
from w2a4_gemm_b200 import build

pytestmark = pytest.mark.gpu

T, K, N = 4, 256, 96


@pytest.fixture(scope="module", autouse=True)
def _setup():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    build.build()
    qg.lib()


@pytest.fixture()
def io():
    g = torch.Generator(device="cuda")
    g.manual_seed(5)
    x = torch.randn(T, K, device="cuda", generator=g).half()
    q, sa = qg.qift_quantize_acts(x, 128)
    w = torch.randn(N, K, device="cuda", generator=g) * 0.02
    codes, sw, _ = qg.qift_quantize_weights(qg.qift_rotate(w, 128), "qift")
    torch.cuda.synchronize()
    return dict(x=x, q=q, sa=sa, codes=codes, sw=sw)


def _sentinel(shape, dtype):
    t = torch.full(shape, 7, dtype=dtype, device="cuda")
    return t, t.clone()


def _untouched(pairs):
    torch.cuda.synchronize()
    for t, ref in pairs:
        assert torch.equal(t, ref), "a rejected call wrote to a buffer"


def test_linear_rejects_wrong_out_shape(io):
    for shape in [(T, N - 1), (T - 1, N), (T * N,)]:
        out, ref = _sentinel(shape, torch.float16)
        with pytest.raises(ValueError):
            qg.qift_linear(io["q"], io["sa"], io["codes"], io["sw"], "qift", torch.float16, out=out)
        _untouched([(out, ref)])


def test_linear_rejects_short_scales(io):
    out, ref = _sentinel((T, N), torch.float16)
    with pytest.raises(ValueError):
        qg.qift_linear(io["q"], io["sa"][: T - 1], io["codes"], io["sw"], "qift", torch.float16, out=out)
    with pytest.raises(ValueError):
        qg.qift_linear(io["q"], io["sa"], io["codes"], io["sw"][: N - 1], "qift", torch.float16, out=out)
    _untouched([(out, ref)])


def test_linear_rejects_wrong_dtype_and_rank(io):
    out, ref = _sentinel((T, N), torch.float32)
    with pytest.raises(ValueError):  # out's dtype must be the requested one
        qg.qift_linear(io["q"], io["sa"], io["codes"], io["sw"], "qift", torch.float16, out=out)
    with pytest.raises(ValueError):
        qg.qift_linear(io["q"].view(-1), io["sa"], io["codes"], io["sw"], "qift", torch.float32, out=out)
    with pytest.raises(ValueError):
        qg.qift_linear(io["q"], io["sa"], io["codes"], io["sw"], "qift", torch.bfloat16)
    _untouched([(out, ref)])


def test_quantize_acts_rejects_wrong_outputs(io):
    q, qref = _sentinel((T, K - 16), torch.int8)
    s, sref = _sentinel((T,), torch.float32)
    with pytest.raises(ValueError):
        qg.qift_quantize_acts(io["x"], 128, out_q=q, out_scales=s)
    q2, q2ref = _sentinel((T, K), torch.int8)
    s2, s2ref = _sentinel((T - 1,), torch.float32)
    with pytest.raises(ValueError):
        qg.qift_quantize_acts(io["x"], 128, out_q=q2, out_scales=s2)
    _untouched([(q, qref), (s, sref), (q2, q2ref), (s2, s2ref)])


def test_rotate_rejects_wrong_out_shape(io):
    out, ref = _sentinel((T, K // 2), torch.float16)
    with pytest.raises(ValueError):
        qg.qift_rotate(io["x"], 128, out=out)
    _untouched([(out, ref)])


def test_decode_linear_rejects_wrong_outputs(io):
    x1 = io["x"][:1].contiguous()
    out, oref = _sentinel((1, N), torch.float16)
    bad_out, bref = _sentinel((1, N + 1), torch.float16)
    with pytest.raises(ValueError):
        qg.qift_decode_linear(x1, 128, io["codes"], io["sw"], "qift", torch.float16, out=bad_out)
    q_bad, qref = _sentinel((1, K - 16), torch.int8)
    with pytest.raises(ValueError):
        qg.qift_decode_linear(x1, 128, io["codes"], io["sw"], "qift", torch.float16, out=out, q_out=q_bad)
    s_bad, sref = _sentinel((0,), torch.float32)
    with pytest.raises(ValueError):
        qg.qift_decode_linear(x1, 128, io["codes"], io["sw"], "qift", torch.float16, out=out, act_scale_out=s_bad)
    with pytest.raises(ValueError):
        qg.qift_decode_linear(x1, 128, io["codes"], io["sw"][: N - 1], "qift", torch.float16, out=out)
    _untouched([(out, oref), (bad_out, bref), (q_bad, qref), (s_bad, sref)])


def test_dequantize_kv_rejects_short_scales(io):
    packed, scales = qg.qift_quantize_kv(io["x"], 128)
    with pytest.raises(ValueError):
        qg.qift_dequantize_kv(packed, scales[: T - 1], 128)


def test_tensor_on_another_device_is_rejected(io):
    if torch.cuda.device_count() < 2:
        pytest.skip("needs two CUDA devices")
    other = torch.device("cuda", 1)
    out, ref = _sentinel((T, N), torch.float16)
    with pytest.raises(ValueError):
        qg.qift_linear(io["q"], io["sa"], io["codes"], io["sw"].to(other), "qift", torch.float16, out=out)
    _untouched([(out, ref)])


def test_stream_of_another_device_is_rejected(io):
    if torch.cuda.device_count() < 2:
        pytest.skip("needs two CUDA devices")
    s = torch.cuda.Stream(device=torch.device("cuda", 1))
    with pytest.raises(ValueError):
        qg.qift_linear(io["q"], io["sa"], io["codes"], io["sw"], "qift", torch.float16, stream=s)


def test_valid_calls_still_run(io):
    """The checks accept what the path produces: a whole linear, and scales longer than needed."""
    y = qg.qift_linear(io["q"], io["sa"], io["codes"], io["sw"], "qift", torch.float32)
    long_sa = torch.cat([io["sa"], torch.ones(3, device="cuda")])
    y2 = torch.empty((T, N), dtype=torch.float32, device="cuda")
    qg.qift_linear(io["q"], long_sa, io["codes"], io["sw"], "qift", torch.float32, out=y2)
    torch.cuda.synchronize()
    assert torch.equal(y, y2)
