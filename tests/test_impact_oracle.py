"""Pins of the oracle's impact-weighted dual-axis fit (STEPQuant summary, "Method" para 4;
the blog's offline vs per-step split): row factor r_i = sqrt(max_j |S_ij| / w_i) from the
row's magnitude and its normalized impact w_i; clip-free column scales c0 for those rows;
one impact-weighted least-squares refit c1 of the codes Q0; nearest levels under c1,
clipped."""
import json
import os

import numpy as np
import pytest

from oracle import oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
f32 = np.float32


def weighted_error(S, Q, r, c, w):
    R = Q.astype(np.float64) * r.astype(np.float64)[:, None] * c.astype(np.float64)[None, :]
    return float(np.sum(w.astype(np.float64)[:, None] * (S.astype(np.float64) - R) ** 2))


@pytest.mark.parametrize("case", json.load(open(os.path.join(GOLDEN, "impact_rank1_case.json")))["cases"],
                         ids=lambda c: "%d-bit" % c["bits"])
def test_rank1_hand_derived(case):
    g = json.load(open(os.path.join(GOLDEN, "impact_rank1_case.json")))
    S = np.zeros((128, 128), f32)
    S[:3, :3] = np.outer(g["a"], g["b"])
    Q, r, c, clipped = O.quantize_impact(S, case["bits"], np.ones(128, f32))
    assert list(r[:3]) == g["r"] and not r[3:].any()
    assert clipped == 0
    for j, bj in enumerate(g["b"]):
        assert list(Q[:3, j]) == case["codes_col0"]
        assert c[j] == f32(case["num_over_b"] * bj / case["den"])
    assert not Q[3:].any() and not Q[:, 3:].any() and not c[3:].any()


def random_state(rng, heavy_rows=True):
    S = rng.standard_normal((128, 128))
    if heavy_rows:
        S *= np.exp(rng.normal(0, 1.0, 128))[:, None] * np.exp(rng.normal(0, 0.7, 128))[None, :]
    return S.astype(f32)


@pytest.mark.parametrize("bits", [4, 6, 8])
def test_refit_never_raises_the_weighted_error(bits):
    """Against the clip-free start (c0, Q0) of the same rows, the refit's weighted error is
    never larger: the least-squares step is optimal for Q0, the requantization optimal per
    element.  Catches a wrong weight, a wrong row factor or a wrong normal equation."""
    rng = np.random.default_rng(bits)
    qm = (1 << (bits - 1)) - 1
    for trial in range(6):
        S = random_state(rng)
        w = O.impact_normalize(np.exp(rng.normal(0, 1, 128)).astype(f32))
        Q, r, c, _ = O.quantize_impact(S, bits, w)
        P = np.abs(S.astype(np.float64)) / np.where(r > 0, r, np.inf).astype(np.float64)[:, None]
        c0 = (P.max(axis=0) / qm).astype(f32)
        Q0 = np.clip(np.rint(S / (r.astype(np.float64)[:, None] * c0.astype(np.float64)[None, :])), -qm, qm)
        assert weighted_error(S, Q, r, c, w) <= weighted_error(S, Q0, r, c0, w) * (1 + 1e-9)


@pytest.mark.parametrize("bits", [4, 8])
def test_column_scale_is_the_weighted_least_squares_optimum(bits):
    """For the first codes Q0, moving any column scale away from c1 raises that column's
    weighted error (checked at +-1e-3 relative)."""
    rng = np.random.default_rng(10 + bits)
    qm = (1 << (bits - 1)) - 1
    S = random_state(rng)
    w = O.impact_normalize(np.exp(rng.normal(0, 1, 128)).astype(f32))
    Q, r, c, _ = O.quantize_impact(S, bits, w)
    rd = r.astype(np.float64)
    c0 = ((np.abs(S.astype(np.float64)) / rd[:, None]).max(axis=0) / qm).astype(f32)
    Q0 = np.clip(np.rint(S / (rd[:, None] * c0.astype(np.float64)[None, :])), -qm, qm)
    for j in range(0, 128, 7):
        def err(cj):
            return float(np.sum(w * (S[:, j].astype(np.float64) - rd * cj * Q0[:, j]) ** 2))
        e = err(float(c[j]))
        assert e <= err(float(c[j]) * (1 + 1e-3)) and e <= err(float(c[j]) * (1 - 1e-3))


def test_higher_impact_gets_finer_resolution():
    """Raising one row's impact lowers its row factor (finer levels) and its error."""
    rng = np.random.default_rng(21)
    S = random_state(rng, heavy_rows=False)
    base = np.ones(128, f32)
    hi = base.copy()
    hi[5] = 16.0
    Qa, ra, ca, _ = O.quantize_impact(S, 4, O.impact_normalize(base))
    Qb, rb, cb, _ = O.quantize_impact(S, 4, O.impact_normalize(hi))
    assert rb[5] < ra[5]
    ea = np.sum((S[5] - Qa[5] * ra[5] * ca) ** 2)
    eb = np.sum((S[5] - Qb[5] * rb[5] * cb) ** 2)
    assert eb < ea


def test_impact_normalization_and_pool_plumbing():
    rng = np.random.default_rng(22)
    omega = np.exp(rng.normal(0, 1, (2, 128))).astype(f32)
    w = O.impact_normalize(omega[0])
    assert abs(float(np.mean(w.astype(np.float64))) - 1.0) < 1e-6
    S = np.stack([random_state(rng), random_state(rng)])[None]
    pool = O.OraclePool(2, [6, 8], 2, impact=omega)
    pool.load_fp32([1], S)
    for h, b in enumerate([6, 8]):
        Q, r, c = pool.state(1, h)
        Qe, re, ce, _ = O.quantize_impact(S[0, h], b, O.impact_normalize(omega[h]))
        assert np.array_equal(Q, Qe) and np.array_equal(r, re) and np.array_equal(c, ce)
