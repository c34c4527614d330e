"""Pins of the Gaussian level-set analysis (Qift abstract: "A scale-invariant ratio analysis
identifies an effective inner/outer centroid ratio range" for 2-bit sets under an
"approximate zero-centered Gaussian-like source model")."""
import numpy as np
import pytest

from conftest import golden_lines
from oracle import source_model as sm

GOLD = {r[0]: r[1:] for r in golden_lines("lloyd_max_n01_4level.txt")}
RATIO = golden_lines("ratio_range.txt")
LOW, HIGH = float(RATIO[0][1]), float(RATIO[1][1])

SETS = {"qift": [-1.5, -0.5, 0.5, 1.5], "pot": [-4.0, -1.0, 1.0, 4.0], "std": [-2.0, -1.0, 0.0, 1.0],
        "pm1pm2": [-2.0, -1.0, 1.0, 2.0]}


def test_lloyd_max_matches_classical_table():
    c, mse = sm.lloyd_max(4)
    inner, tol_i = map(float, GOLD["inner"])
    outer, tol_o = map(float, GOLD["outer"])
    m, tol_m = map(float, GOLD["mse"])
    assert abs(c[2] - inner) <= tol_i and abs(-c[1] - inner) <= tol_i
    assert abs(c[3] - outer) <= tol_o and abs(-c[0] - outer) <= tol_o
    assert abs(mse - m) <= tol_m


def test_lloyd_centroid_condition():
    # At the Lloyd-Max optimum, D = 1 - sum_i P_i c_i^2 (centroid condition, unit variance).
    c, mse = sm.lloyd_max(4)
    edges = [-np.inf, 0.5 * (c[0] + c[1]), 0.5 * (c[1] + c[2]), 0.5 * (c[2] + c[3]), np.inf]
    p = [sm.region_moments(edges[i], edges[i + 1])[0] for i in range(4)]
    assert abs(mse - (1.0 - sum(pi * ci * ci for pi, ci in zip(p, c)))) < 1e-12


@pytest.mark.parametrize("name", list(SETS))
def test_closed_form_mse_matches_monte_carlo(name):
    lv = np.array(SETS[name])
    s, d = sm.best_scale(lv)
    rng = np.random.default_rng(123)
    x = rng.normal(size=2_000_000)
    lev = np.sort(lv) * s
    idx = np.argmin(np.abs(x[:, None] - lev[None, :]), axis=1)
    e2 = (x - lev[idx]) ** 2
    assert abs(e2.mean() - d) < 5 * e2.std() / np.sqrt(x.size)


def test_ratio_range_members_and_outsider():
    c, _ = sm.lloyd_max(4)
    r_lloyd = sm.inner_outer_ratio(c)
    r_qift = sm.inner_outer_ratio(SETS["qift"])
    r_pot = sm.inner_outer_ratio(SETS["pot"])
    r_pm2 = sm.inner_outer_ratio(SETS["pm1pm2"])
    for name, val in [(r[1], float(r[2])) for r in RATIO if r[0] in ("inside", "outside")]:
        got = {"qift": r_qift, "pot": r_pot, "pm1pm2": r_pm2}[name]
        assert abs(got - val) < 1e-15
    assert LOW <= r_lloyd <= HIGH
    assert LOW <= r_qift <= HIGH and LOW <= r_pot <= HIGH
    assert not (LOW <= r_pm2 <= HIGH)


def test_optimal_mse_is_flat_inside_the_range_and_poor_outside():
    _, d_lloyd = sm.lloyd_max(4)
    inside = [sm.optimal_mse_for_ratio(r) for r in np.linspace(LOW, HIGH, 9)]
    assert max(inside) < 1.03 * d_lloyd
    assert min(inside) >= d_lloyd - 1e-9        # Lloyd is the optimum of every 4-level set
    assert sm.optimal_mse_for_ratio(0.5) > 1.3 * d_lloyd


def test_no_zero_sets_beat_standard_gaussian():
    d = {n: sm.best_scale(np.array(v))[1] for n, v in SETS.items()}
    assert d["qift"] < d["std"] and d["pot"] < d["std"]
    assert d["qift"] < d["pm1pm2"]
