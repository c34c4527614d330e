"""Pins of the oracle's scale search, nearest-level encoder and 2-bit packing.

Qift abstract: fixed 2-bit level sets -- {+-0.5, +-1.5} (= {+-1, +-3} at half scale), the
power-of-two {+-1, +-4}, the standard {-2,-1,0,+1} -- with one per-channel scale, no zero point
and no group grid.  The scale rule (argmin of MSE over a 100-point grid of
[0.2, 1.0] * max|w| / outer level) and the bit layout are readings the abstract leaves open.
"""
from fractions import Fraction

import numpy as np
import pytest

import oracle
from conftest import golden_lines
from oracle import source_model

SETS = ["qift", "pot", "std"]
# s-form levels (times the searched scale s) and the stored-scale factor t/s, from the golden
# fixture copied from the abstract.
GOLD = {r[0]: dict(s_levels=[Fraction(v) for v in r[1:5]], ints=[int(v) for v in r[5:9]],
                   t_over_s=Fraction(r[9])) for r in golden_lines("level_sets.txt")}


def test_level_tables_match_the_abstract():
    for name in SETS:
        assert oracle.levels(name).tolist() == GOLD[name]["ints"]
        # integer levels * (t/s) are the s-form levels
        assert [Fraction(i) * GOLD[name]["t_over_s"] for i in GOLD[name]["ints"]] == GOLD[name]["s_levels"]


def test_qift_affine_and_pot_sign_and_shift():
    # Qift: L(c) = 2c - 3.  PoT: sign from the high bit, magnitude 1 << (2 * outer) where the
    # outer codes are 0 and 3 -- the abstract's "sign-and-shift" application.
    for c in range(4):
        assert oracle.levels("qift")[c] == 2 * c - 3
        sign = 1 if c >= 2 else -1
        outer = 1 if c in (0, 3) else 0
        assert oracle.levels("pot")[c] == sign * (1 << (2 * outer))


@pytest.mark.parametrize("name", SETS)
def test_candidate_grid_endpoints_and_monotone(name):
    lam = {"qift": 1.5, "pot": 4.0, "std": 2.0}[name]   # largest |level| in s units
    m = np.float32(0.123456)
    s = oracle.candidate_scales(float(m), name)
    assert s.shape == (100,)
    assert s[0] == np.float32(0.2 * float(m) / lam)
    assert s[-1] == np.float32(float(m) / lam)
    assert np.all(np.diff(s.astype(np.float64)) > 0)


def _exact_nearest(w: np.float32, s: np.float32, name):
    """All codes whose level is at minimal exact distance from w (rational arithmetic)."""
    wf, sf = Fraction(float(w)), Fraction(float(s))
    d = [abs(wf - lv * sf) for lv in GOLD[name]["s_levels"]]
    best = min(d)
    return [c for c in range(4) if d[c] == best]


def _codes_for_scale(w_row: np.ndarray, name, s_best):
    """Quantize a row whose grid is forced to a single scale (lo = hi), return codes."""
    m = float(np.max(np.abs(w_row)))
    lam = {"qift": 1.5, "pot": 4.0, "std": 2.0}[name]
    f = float(s_best) * lam / m
    codes, scales, _, _ = oracle.quantize_weights(w_row[None, :], name, grid_points=2, lo=f, hi=f)
    return oracle.unpack_codes(codes, w_row.size)[0], scales[0]


@pytest.mark.parametrize("name", SETS)
def test_encoding_is_exact_nearest_level(name):
    rng = np.random.default_rng(1)
    w = (rng.normal(size=4096) * 0.02).astype(np.float32)
    codes, scales, _, _ = oracle.quantize_weights(w[None, :], name)
    c = oracle.unpack_codes(codes, 4096)[0]
    s = np.float32(float(scales[0]) / float(GOLD[name]["t_over_s"]))  # s-form scale (exact)
    for k in range(4096):
        near = _exact_nearest(w[k], s, name)
        assert c[k] in near, (k, w[k], s, c[k], near)


@pytest.mark.parametrize("name", SETS)
def test_ties_and_signed_zero(name):
    # Constructed ties: a weight exactly on a midpoint takes the smaller-magnitude level (R8);
    # +0.0 and -0.0 both take the positive side / zero level (R7).
    s = np.float32(0.25)
    mids = {"qift": [0.25, -0.25], "pot": [0.625, -0.625], "std": [-0.375, -0.125, 0.125]}[name]
    row = np.array(mids + [0.0, -0.0], dtype=np.float32)
    row = np.concatenate([row, np.full(16 - row.size, 0.001, np.float32)])
    row[-1] = np.float32({"qift": 0.375, "pot": 1.0, "std": 0.5}[name])   # max|w| = outer * s
    c, _ = _codes_for_scale(row, name, s)
    ints = oracle.levels(name)
    for k, v in enumerate(mids):
        near = _exact_nearest(row[k], s, name)
        assert len(near) == 2, "fixture is meant to be a tie"
        mags = [abs(GOLD[name]["s_levels"][q]) for q in near]
        assert c[k] == near[int(np.argmin(mags))]
    zero_code = {"qift": 2, "pot": 2, "std": 2}[name]
    assert c[len(mids)] == zero_code and c[len(mids) + 1] == zero_code
    assert ints[zero_code] >= 0


def test_packing_golden_words():
    for row in golden_lines("pack_examples.txt"):
        codes_in, word = [int(v) for v in row[:16]], int(row[16], 16)
        # weights whose codes are fixed by sign and class alone: outer magnitude 10, inner 1
        # (every grid scale lies in [1.33, 6.67], so |1| is inner and |10| outer for Qift)
        mag = {0: -10.0, 1: -1.0, 2: 1.0, 3: 10.0}
        w = np.array([mag[c] for c in codes_in], dtype=np.float32)
        codes, _, _, _ = oracle.quantize_weights(w[None, :], "qift")
        if all(c == 2 for c in codes_in):
            w = np.zeros(16, np.float32)   # all-zero row: every code 2 by the general rule
            codes, scales, _, _ = oracle.quantize_weights(w[None, :], "qift")
            assert scales[0] == 0.0
        assert int(codes[0, 0]) == word, (codes_in, hex(int(codes[0, 0])))


def test_unpack_roundtrip():
    rng = np.random.default_rng(2)
    w = (rng.standard_t(4, size=(7, 48)) * 0.02).astype(np.float32)
    codes, _, _, _ = oracle.quantize_weights(w, "pot")
    c = oracle.unpack_codes(codes, 48)
    repacked = np.zeros_like(codes)
    for k in range(48):
        repacked[:, k // 16] |= c[:, k].astype(np.uint32) << np.uint32(2 * (k % 16))
    assert np.array_equal(repacked, codes)


@pytest.mark.parametrize("name", SETS)
def test_scale_search_is_grid_optimal(name):
    # The chosen candidate's MSE, recomputed in exact-ish binary64 from the exact nearest
    # levels, is within the binary32 rounding of the sum of the best MSE over the whole grid.
    rng = np.random.default_rng(3)
    K = 512
    w = oracle.rotate_f32((rng.standard_t(4, size=(6, K)) * 0.02).astype(np.float32), 128)
    codes, scales, mse, best = oracle.quantize_weights(w, name)
    lv = np.array([float(v) for v in GOLD[name]["s_levels"]])
    for r in range(w.shape[0]):
        m = float(np.max(np.abs(w[r])))
        cands = oracle.candidate_scales(m, name).astype(np.float64)
        wr = w[r].astype(np.float64)
        true = np.array([np.min((wr[:, None] - s * lv[None, :]) ** 2, axis=1).sum() for s in cands])
        # The oracle rounds levels, errors and squares to binary32 (relative error of the sum a
        # few tens of units of 2^-24 at most for these rows); the reference here is binary64.
        assert true[best[r]] <= true.min() * (1 + 64 * 2.0 ** -24)
        assert abs(mse[r] * K - true[best[r]]) <= true[best[r]] * 64 * 2.0 ** -24
        assert np.float32(float(scales[r]) / float(GOLD[name]["t_over_s"])) == np.float32(cands[best[r]])


def test_zero_row_and_scale_zero():
    w = np.zeros((2, 32), np.float32)
    for name in SETS:
        codes, scales, mse, best = oracle.quantize_weights(w, name)
        assert np.all(scales == 0) and np.all(mse == 0) and np.all(best == 0)
        assert np.all(codes == 0xAAAAAAAA)


def test_no_zero_sets_beat_standard_on_rotated_heavy_tails():
    # Abstract: the no-zero level sets improve over the standard W2 set.  On Student-t(4)
    # rows after a 128-block rotation the per-row reconstruction MSE must order that way.
    rng = np.random.default_rng(4)
    w = oracle.rotate_f32((rng.standard_t(4, size=(64, 1024)) * 0.02).astype(np.float32), 128)
    res = {n: oracle.quantize_weights(w, n)[2].mean() for n in SETS}
    assert res["qift"] < res["std"] and res["pot"] < res["std"]


def test_gaussian_rows_reach_the_closed_form_optimum():
    # Unit-variance Gaussian rows: the grid search's mean MSE matches the closed-form
    # best-scale Gaussian MSE of each set (computed independently in the source model)
    # within sampling error and the grid's resolution.
    rng = np.random.default_rng(6)
    w = rng.normal(size=(64, 4096)).astype(np.float32)
    for name in SETS:
        lv = np.array([float(v) for v in GOLD[name]["s_levels"]])
        _, d_star = source_model.best_scale(lv)
        got = oracle.quantize_weights(w, name)[2].mean()
        assert abs(got - d_star) < 0.004 * d_star + 0.0015, (name, got, d_star)
