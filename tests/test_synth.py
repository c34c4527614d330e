"""The seeded input generators keep the recipe the benchmark and the parity tests state:
Student-t(4) * 0.02 weights, N(0, 1) fp16 activations with round(1% K) fixed outlier channels
scaled by 20 before the cast, the LLaMA-shaped workloads and the 224 modules of the 8B-shaped
model.  (Inputs only: this module holds none of the method's arithmetic.)"""
import numpy as np
import pytest
import torch

from w2a4_gemm_b200 import synth

T4_Q975 = 2.7764451  # 97.5% quantile of Student's t with 4 degrees of freedom


def test_weights_are_student_t4_times_0_02():
    w = synth.weights(512, 1024, (7,))
    assert w.dtype == np.float32 and w.shape == (512, 1024)
    q = np.quantile(np.abs(w.astype(np.float64)) / 0.02, 0.95)   # |t| quantile 0.95 = t quantile 0.975
    assert abs(q - T4_Q975) < 0.03
    assert abs(float(w.mean())) < 1e-3
    n = synth.weights(512, 1024, (7,), dist="normal")
    assert abs(float(n.std()) - 0.02) < 2e-4


def test_weights_are_seeded():
    assert np.array_equal(synth.weights(4, 64, (3, 1)), synth.weights(4, 64, (3, 1)))
    assert not np.array_equal(synth.weights(4, 64, (3, 1)), synth.weights(4, 64, (3, 2)))


def test_activation_outliers_are_fixed_channels_scaled_by_20():
    K, T = 4096, 64
    n = synth.outlier_count(K)
    assert n == 41 and synth.outlier_count(11008) == 110 and synth.outlier_count(512) == 5
    x = synth.activations(T, K, (9,), n_outliers=n).astype(np.float64)
    col_std = x.std(axis=0)
    big = np.flatnonzero(col_std > 8)
    assert len(big) == n                                     # the same n columns for every token
    assert abs(float(np.median(col_std[big])) - 20) < 3
    assert abs(float(np.median(np.delete(col_std, big))) - 1) < 0.1
    assert synth.activations(T, K, (9,), n_outliers=n).dtype == np.float16


def test_workload_shapes():
    wl = synth.WORKLOADS
    q = wl["llama7b_q_proj_decode_T1"]
    assert (q.tokens, q.w_block, q.levelset, q.out_dtype) == (1, 4096, "qift", "f16")
    assert [(l.n_out, l.n_in) for l in q.linears] == [(4096, 4096)]
    p = wl["llama7b_mlp_prefill_T2048"]
    assert (p.tokens, p.w_block, p.levelset) == (2048, 128, "qift")
    assert [(l.n_out, l.n_in) for l in p.linears] == [(11008, 4096), (11008, 4096), (4096, 11008)]
    d = wl["llama31_8b_mlp_decode_T16_pot"]
    assert (d.tokens, d.w_block, d.levelset) == (16, 128, "pot")
    assert [(l.n_out, l.n_in) for l in d.linears] == [(14336, 4096), (14336, 4096), (4096, 14336)]
    s = wl["single_linear_256x512"]
    assert (s.tokens, s.w_block, s.out_dtype, s.w_dist) == (8, 512, "f32", "normal")
    assert wl["llama7b_q_proj_decode_T1_w4"].levelset == "int4"
    assert wl["llama31_8b_mlp_decode_T16_w4"].levelset == "int4"
    pw = wl["llama7b_mlp_prefill_T2048_w4"]
    assert (pw.tokens, pw.w_block, pw.levelset) == (2048, 128, "int4")
    assert [(l.n_out, l.n_in) for l in pw.linears] == [(l.n_out, l.n_in) for l in p.linears]
    # gate and up read the same input, down its own
    assert d.linears[0].x_seed == d.linears[1].x_seed != d.linears[2].x_seed


def test_model_8b_modules():
    mods = synth.model_8b_modules()
    assert len(mods) == 224
    assert sum(n_out * n_in for _, _, n_out, n_in, _ in mods) == 6_979_321_856
    assert mods[0] == (0, "q_proj", 4096, 4096, 1000) and mods[-1] == (31, "down_proj", 4096, 14336, 1000 + 7 * 31 + 6)
    assert len({m[4] for m in mods}) == 224


def test_device_generator_is_student_t4():
    w = synth.weights_t4_device(512, 2048, 11, torch.device("cpu")).double().numpy()
    q = np.quantile(np.abs(w) / 0.02, 0.95)
    assert abs(q - T4_Q975) < 0.03
    assert abs(float(w.mean())) < 1e-3
    assert np.array_equal(w, synth.weights_t4_device(512, 2048, 11, torch.device("cpu")).double().numpy())
