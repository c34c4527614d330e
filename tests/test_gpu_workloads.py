"""Full-size parity on the LLaMA-shaped workloads, in the launch configuration the benchmark
times: the GPU runs every stage on the whole matrices; the CPU oracle recomputes sampled rows
and tokens on its own (from the same seeded inputs, never from GPU results) and the two must
agree bit for bit on codes, scales, INT4 activations and outputs."""
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


CASES = [(wl.name, i) for wl in (synth.SINGLE_256x512, synth.LLAMA7B_QPROJ_DECODE, synth.LLAMA7B_MLP_PREFILL,
                                 synth.LLAMA31_8B_MLP_DECODE16, synth.LLAMA7B_QPROJ_DECODE_W4,
                                 synth.LLAMA31_8B_MLP_DECODE16_W4, synth.LLAMA7B_MLP_PREFILL_W4)
         for i in range(len(wl.linears))]


@pytest.mark.parametrize("wname,idx", CASES)
def test_workload_linear_parity(wname, idx):
    wl = synth.WORKLOADS[wname]
    lin = wl.linears[idx]
    W, x = wl.w(lin), wl.x(lin)
    N, K, T = lin.n_out, lin.n_in, wl.tokens
    out_dt = torch.float16 if wl.out_dtype == "f16" else torch.float32
    np_dt = np.float16 if wl.out_dtype == "f16" else np.float32

    # GPU: the whole path on the whole matrices.
    w_rot = qg.qift_rotate(dev(W), wl.w_block)
    gc, gs, _ = qg.qift_quantize_weights(w_rot, wl.levelset)
    gq, gsa = qg.qift_quantize_acts(dev(x), wl.a_block)
    gy = qg.qift_linear(gq, gsa, gc, gs, wl.levelset, out_dt)
    w_rot, gc, gs, gq, gsa, gy = map(host, (w_rot, gc, gs, gq, gsa, gy))
    gc = gc.view(np.uint32)

    # Oracle: sampled rows and tokens, recomputed from the seeded inputs.
    rng = np.random.default_rng(12345 + idx)
    rows = np.sort(rng.choice(N, size=min(N, 96), replace=False))
    toks = np.sort(rng.choice(T, size=min(T, 24), replace=False))
    o_wrot = oracle.rotate_f32(W[rows], wl.w_block)
    o_q, o_sa, _ = oracle.quantize_acts(x[toks], wl.a_block)
    if wl.levelset == "int4":
        o_codes, o_scales, _, _ = oracle.quantize_weights_w4(o_wrot)
        o_y, _ = oracle.linear_w4(o_q, o_sa, o_codes, o_scales, np_dt)
    else:
        o_codes, o_scales, _, _ = oracle.quantize_weights(o_wrot, wl.levelset)
        o_y, _ = oracle.linear(o_q, o_sa, o_codes, o_scales, wl.levelset, np_dt)

    assert np.array_equal(w_rot[rows].view(np.uint32), o_wrot.view(np.uint32))
    assert np.array_equal(gc[rows], o_codes)
    assert np.array_equal(gs[rows].view(np.uint32), o_scales.view(np.uint32))
    assert np.array_equal(gq[toks], o_q)
    assert np.array_equal(gsa[toks].view(np.uint32), o_sa.view(np.uint32))
    g_sub = gy[np.ix_(toks, rows)]
    rel = 1e-5 if np_dt == np.float32 else 2e-3
    ref = o_y.astype(np.float64)
    rms = np.sqrt(np.mean(ref ** 2))
    assert np.all(np.abs(g_sub.astype(np.float64) - ref) <= rel * np.abs(ref) + rel * rms)
    assert np.array_equal(g_sub, o_y)


@pytest.mark.parametrize("layer,proj", [(0, 1), (17, 6), (31, 4)])
def test_offline_model_quantization_sampled(layer, proj):
    # One module of the 224-module 8B-shaped model, all three level sets, sampled rows.
    mods = synth.model_8b_modules()
    _, name, n_out, n_in, seed = mods[7 * layer + proj]
    W = synth.weights(n_out, n_in, (seed,))
    w_rot = qg.qift_rotate(dev(W), synth.MODEL_8B_BLOCK)
    rng = np.random.default_rng(seed)
    rows = np.sort(rng.choice(n_out, size=32, replace=False))
    o_wrot = oracle.rotate_f32(W[rows], synth.MODEL_8B_BLOCK)
    assert np.array_equal(host(w_rot)[rows].view(np.uint32), o_wrot.view(np.uint32))
    mse = {}
    for ls in ("qift", "pot", "std"):
        gc, gs, gm = qg.qift_quantize_weights(w_rot, ls)
        oc, os_, om, _ = oracle.quantize_weights(o_wrot, ls)
        assert np.array_equal(host(gc).view(np.uint32)[rows], oc)
        assert np.array_equal(host(gs)[rows].view(np.uint32), os_.view(np.uint32))
        assert np.array_equal(host(gm)[rows].view(np.uint64), om.view(np.uint64))
        mse[ls] = host(gm).mean()
    assert mse["qift"] < mse["std"] and mse["pot"] < mse["std"]


def test_offline_device_generated_module_parity():
    # The offline benchmark draws the 8B-shaped model's weights on the device; the quantizer
    # must match the oracle on those inputs too (sampled rows copied back to the host).
    _, name, n_out, n_in, seed = synth.model_8b_modules()[7 * 5 + 6]   # layer 5 down_proj
    W = synth.weights_t4_device(n_out, n_in, seed, "cuda")
    w_rot = qg.qift_rotate(W, synth.MODEL_8B_BLOCK)
    rows = np.sort(np.random.default_rng(seed).choice(n_out, size=24, replace=False))
    Wh = host(W)[rows]
    o_wrot = oracle.rotate_f32(Wh, synth.MODEL_8B_BLOCK)
    assert np.array_equal(host(w_rot)[rows].view(np.uint32), o_wrot.view(np.uint32))
    for ls in ("qift", "pot", "std"):
        gc, gs, gm = qg.qift_quantize_weights(w_rot, ls)
        oc, os_, om, _ = oracle.quantize_weights(o_wrot, ls)
        assert np.array_equal(host(gc).view(np.uint32)[rows], oc)
        assert np.array_equal(host(gm)[rows].view(np.uint64), om.view(np.uint64))
