"""Pins of the oracle's lifetime-aware bit allocation (STEPQuant summary, 'Method',
second paragraph; ONTLE blog, lifetime-aware bit allocation): the dynamic programme
must equal an exhaustive search, spend the budget, and favour long-lived units."""
import itertools
import math

import numpy as np
import pytest

from oracle import oracle as O

CAND = [4, 6, 8]


@pytest.mark.parametrize("N", [1, 2, 3, 5, 7, 8])
def test_dp_equals_exhaustive_search(N):
    rng = np.random.default_rng(N)
    for trial in range(6):
        hl = np.exp(rng.uniform(0, math.log(4096), N))
        dist = None if trial % 2 == 0 else np.sort(rng.lognormal(0, 1, (N, 3)))[:, ::-1] * \
            np.array([1.0, 0.1, 0.01])
        avg = [5.0, 6.0, 7.0][trial % 3]
        bf, of = O.allocate_bits_bruteforce(hl, dist, CAND, avg)
        bd, od = O.allocate_bits_dp(hl, dist, CAND, avg)
        assert od == pytest.approx(of, rel=1e-12)
        assert bd == bf        # random inputs: the optimum is unique


def test_exhaustive_search_is_the_definition():
    """Brute force over 3^N really scans every feasible assignment (independent recount)."""
    hl = [3.0, 700.0, 40.0, 2000.0]
    best = min((sum(O.lifetime_weight(h) * 2.0 ** (-2 * b) for h, b in zip(hl, combo)), combo)
               for combo in itertools.product(CAND, repeat=4) if sum(combo) <= 24)
    bits, obj = O.allocate_bits_bruteforce(hl, None, CAND, 6.0)
    assert tuple(bits) == best[1] and obj == pytest.approx(best[0])


def test_lifetime_weight_is_geometric_retention_sum():
    # sum_j rho^j with rho = 2^(-1/h): h = 1 gives rho = 1/2 and weight 2
    assert O.lifetime_weight(1.0) == pytest.approx(2.0)
    rho = 2 ** (-1 / 37.0)
    assert O.lifetime_weight(37.0) == pytest.approx(sum(rho ** j for j in range(20000)), rel=1e-9)
    # long half-lives: weight ~ h / ln 2
    assert O.lifetime_weight(4096.0) == pytest.approx(4096 / math.log(2), rel=1e-3)


def test_budget_and_monotonicity():
    rng = np.random.default_rng(9)
    for N in (16, 32, 48):
        hl = np.sort(np.exp(rng.uniform(0, math.log(4096), N)))
        bits, _ = O.allocate_bits_dp(hl, None, CAND, 6.0)
        assert sum(bits) == 6 * N                                   # budget spent exactly
        assert all(a <= b for a, b in zip(bits, bits[1:]))          # longer-lived, more bits
        assert set(bits) <= set(CAND) and len(set(bits)) > 1        # a real mix


# The vectorised programme (one unit per key row, thousands of units) must be the same
# optimisation as the plain dictionary DP above, which is itself pinned to exhaustive search.

@pytest.mark.parametrize("N", [1, 2, 5, 8, 13, 24, 40])
def test_vectorised_dp_equals_dict_dp(N):
    rng = np.random.default_rng(700 + N)
    for trial in range(4):
        hl = np.exp(rng.uniform(0, math.log(4096), N))
        dist = None if trial % 2 == 0 else np.sort(rng.lognormal(0, 1, (N, 3)))[:, ::-1] * \
            np.array([1.0, 0.1, 0.01])
        avg = [6.0, 5.0, 7.0, 4.5][trial]
        bd, od = O.allocate_bits_dp(list(hl), dist, CAND, avg)
        bv, ov = O.allocate_bits_dp_vec(list(hl), dist, CAND, avg)
        assert ov == pytest.approx(od, rel=1e-12)
        assert bv == bd                                   # random inputs: unique optimum
        assert sum(bv) <= math.floor(N * avg + 1e-9)


@pytest.mark.parametrize("N", [1, 3, 6, 8])
def test_vectorised_dp_equals_exhaustive_search(N):
    rng = np.random.default_rng(800 + N)
    for trial in range(5):
        hl = np.exp(rng.uniform(0, math.log(4096), N))
        dist = None if trial % 2 else rng.lognormal(0, 1, (N, 3)) * np.array([1.0, 0.1, 0.01])
        avg = [5.0, 6.0, 7.0, 4.5, 6.5][trial]
        bf, of = O.allocate_bits_bruteforce(list(hl), dist, CAND, avg)
        bv, ov = O.allocate_bits_dp_vec(list(hl), dist, CAND, avg)
        assert bv == bf and ov == pytest.approx(of, rel=1e-12)


def test_vectorised_dp_budget_edges():
    """The budget is floor(N * avg): at exactly 4 bits per unit every unit gets 4; one bit
    below that nothing fits; candidate order in the argument does not matter."""
    hl = [2.0, 40.0, 900.0, 3000.0]
    assert O.allocate_bits_dp_vec(hl, None, CAND, 4.0)[0] == [4, 4, 4, 4]
    with pytest.raises(ValueError):
        O.allocate_bits_dp_vec(hl, None, CAND, 3.9)
    assert O.allocate_bits_dp_vec(hl, None, [8, 4, 6], 6.0)[0] == O.allocate_bits_dp(hl, None, CAND, 6.0)[0]
