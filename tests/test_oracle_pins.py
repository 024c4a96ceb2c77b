"""Pins of the CPU oracle against facts the STEPQuant pages and the mathematics fix.

None of these checks re-types the oracle's own formulas: each uses a hand
derivation, an algebraic identity, an invariant, a special case, or a brute-force
search, chosen so that a dropped term, a wrong sign or index, or a transposed
operand in the oracle fails at least one of them.
"""
import json
import os

import numpy as np
import pytest

from oracle import oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
F32_EPS = 2.0 ** -24
f32 = np.float32


def unit(rng, n):
    x = rng.standard_normal(n)
    return (x / np.linalg.norm(x)).astype(f32)


def random_fp32_state(rng, dk=128, dv=128, steps=24, alpha=0.97):
    """A realistic fp32 state: a few unquantized gated Delta steps from zero."""
    S = np.zeros((dk, dv))
    for _ in range(steps):
        S, _ = O.delta_step(S, unit(rng, dk), unit(rng, dk), rng.standard_normal(dv).astype(f32),
                            f32(alpha), f32(1 / (1 + np.exp(-rng.standard_normal()))))
        S = S.astype(f32).astype(np.float64)
    return S.astype(f32)


# --------------------------------------------------------------------------- packing

def test_packing_golden_bytes():
    g = json.load(open(os.path.join(GOLDEN, "packing_bytes.json")))
    for case in g["cases"]:
        bits = case["bits"]
        Q = np.zeros((128, 128), dtype=np.int32)
        for i, j, code in case["codes"]:
            Q[i, j] = code
        buf = O.pack_codes(Q, bits)
        assert len(buf) == 128 * 128 * bits // 8
        for off, expect in case["bytes_at"].items():
            off = int(off)
            assert list(buf[off:off + len(expect)]) == expect, (bits, off)
        assert np.array_equal(O.unpack_codes(buf, bits), Q)


@pytest.mark.parametrize("bits", [4, 6, 8])
def test_packing_round_trip_every_code(bits):
    qm = (1 << (bits - 1)) - 1
    rng = np.random.default_rng(bits)
    Q = rng.integers(-qm, qm + 1, size=(128, 128)).astype(np.int32)
    Q.flat[: 2 * qm + 1] = np.arange(-qm, qm + 1)       # every representable code at least once
    buf = O.pack_codes(Q, bits)
    assert np.array_equal(O.unpack_codes(buf, bits), Q)
    # the stream is dense: every byte is touched by exactly bits/8 of a code on average
    assert buf.nbytes * 8 == Q.size * bits


def test_block_sizes_and_offsets():
    assert [O.block_bytes(b) for b in (4, 6, 8)] == [9216, 13312, 17408]
    off, stride = O.head_offsets([4, 6, 8, 8])
    assert list(off) == [0, 9216, 9216 + 13312, 9216 + 13312 + 17408]
    assert stride == 9216 + 13312 + 2 * 17408
    assert all(int(o) % 128 == 0 for o in off)


# --------------------------------------------------------------------------- hand-computed steps

@pytest.mark.parametrize("bits", [4, 6, 8])
def test_rank1_worked_case(bits):
    g = json.load(open(os.path.join(GOLDEN, "rank1_worked_case.json")))["step1"]
    rng = np.random.default_rng(0)
    Q0 = np.zeros((128, 128), np.int32)
    z = np.zeros(128, f32)
    k = np.zeros(128, f32)
    k[g["key_index"]] = 1
    v = np.zeros(128, f32)
    v[:4] = g["v_head"]
    q = unit(rng, 128)
    o = O.step_state(Q0, z, z, bits, q, k, v, g["alpha"], g["beta"])
    assert list(o["Q"][0, :4]) == g["codes_row0_head"][str(bits)]
    assert not o["Q"][1:].any() and not o["Q"][0, 4:].any()
    np.testing.assert_allclose(o["c"][:4], g["c_head"], rtol=1e-6)
    assert o["r"][0] == pytest.approx(g["r0"][str(bits)], rel=1e-6)
    assert not o["r"][1:].any()
    # readout from the updated state e_1 v^T
    np.testing.assert_allclose(o["y"], q[0] * v, rtol=1e-6, atol=1e-12)


def test_rank1_second_step():
    g = json.load(open(os.path.join(GOLDEN, "rank1_worked_case.json")))
    s1, s2 = g["step1"], g["step2_4bit"]
    z = np.zeros(128, f32)
    k = np.zeros(128, f32)
    k[0] = 1
    v = np.zeros(128, f32)
    v[:4] = s1["v_head"]
    q = np.zeros(128, f32)
    o = O.step_state(np.zeros((128, 128), np.int32), z, z, 4, q, k, v, s1["alpha"], 1.0)
    k2 = np.zeros(128, f32)
    k2[s2["key_index"]] = 1
    v2 = np.zeros(128, f32)
    v2[:4] = s2["v_head"]
    o2 = O.step_state(o["Q"], o["r"], o["c"], 4, q, k2, v2, 1.0, 1.0)
    assert list(o2["Q"][0, :4]) == s2["codes_row0_head"]
    assert list(o2["Q"][1, :4]) == s2["codes_row1_head"]
    np.testing.assert_allclose(o2["c"][:4], s2["c_head"], rtol=1e-6)
    np.testing.assert_allclose(o2["r"][:2], s2["r01"], rtol=1e-6)


@pytest.mark.parametrize("bits", [4, 6, 8])
def test_zero_state_rank1_closed_form(bits):
    """From the zero state the update is S = beta k v^T, so the codes are
    RHE(qmax sgn(k_i v_j) sqrt(|v_j| / max|v|)) for every row with k_i != 0,
    independent of |k_i| and beta, and y = beta (k.q) v."""
    rng = np.random.default_rng(100 + bits)
    qm = (1 << (bits - 1)) - 1
    for _ in range(5):
        k, q = unit(rng, 128), unit(rng, 128)
        v = rng.standard_normal(128).astype(f32)
        beta = f32(0.3 + 0.6 * rng.random())
        z = np.zeros(128, f32)
        o = O.step_state(np.zeros((128, 128), np.int32), z, z, bits, q, k, v, 0.9, beta)
        x = qm * np.sign(np.outer(k, v)) * np.sqrt(np.abs(v.astype(np.float64)) / np.abs(v).max())
        x = np.broadcast_to(x, (128, 128))
        safe = np.abs(np.abs(x - np.floor(x)) - 0.5) > 1e-4       # away from ties
        assert np.array_equal(o["Q"][safe], np.rint(x)[safe])
        assert safe.mean() > 0.99
        np.testing.assert_allclose(o["y"], float(beta) * float(np.dot(k.astype(np.float64), q)) * v,
                                   rtol=2e-6, atol=1e-7)


# --------------------------------------------------------------------------- delta rule identities

def test_delta_write_retrieves_target():
    """'Write in only the difference': after a step with unit key k, looking the
    key up returns (1 - beta) * (faded prediction) + beta * v; with beta = 1, exactly v."""
    rng = np.random.default_rng(7)
    S0 = random_fp32_state(rng).astype(np.float64)
    for beta, alpha in ((1.0, 0.9), (0.4, 0.75), (0.8, 1.0)):
        beta, alpha = float(f32(beta)), float(f32(alpha))     # the oracle reads fp32 inputs
        k = unit(rng, 128).astype(np.float64)
        k /= np.linalg.norm(k)                       # exactly unit in double
        v = rng.standard_normal(128)
        S1, y = O.delta_step(S0, k, k, v, alpha, beta)    # q = k reads the key back
        kf = k.astype(f32).astype(np.float64)
        u = (alpha * S0).T @ kf
        nk = float(kf @ kf)
        expect = u + beta * nk * (v.astype(f32) - u)
        np.testing.assert_allclose(y, expect, rtol=1e-9, atol=1e-12)
        if beta == 1.0:
            np.testing.assert_allclose(y, v.astype(f32), rtol=0, atol=1e-6)


def test_kda_equal_gates_is_gdn():
    rng = np.random.default_rng(8)
    S = random_fp32_state(rng)
    for bits in (4, 6, 8):
        Q, r, c, _ = O.quantize(S, bits)
        q, k = unit(rng, 128), unit(rng, 128)
        v = rng.standard_normal(128).astype(f32)
        a = f32(0.93)
        g = O.step_state(Q, r, c, bits, q, k, v, a, 0.6)
        d = O.step_state(Q, r, c, bits, q, k, v, np.full(128, a, f32), 0.6)
        for key in ("Q", "r", "c", "y"):
            assert np.array_equal(g[key], d[key])


def test_kda_gate_is_per_key_row():
    """A KDA gate that zeroes key channel i (with beta = 0) clears exactly row i."""
    rng = np.random.default_rng(9)
    S = random_fp32_state(rng)
    Q, r, c, _ = O.quantize(S, 8)
    al = np.ones(128, f32)
    al[5] = 0.0
    z = np.zeros(128, f32)
    o = O.step_state(Q, r, c, 8, z, z, z, al, 0.0)
    deq = O.dequantize(o["Q"], o["r"], o["c"])
    assert not deq[5].any()
    assert np.count_nonzero(deq[6]) > 0


def test_gqa_equals_repeated_key_heads():
    """Value head h reads key head h // (H / Hk): a pool with Hk = 2, H = 4 gives the
    same result as H = Hk = 4 with the key heads repeated consecutively."""
    rng = np.random.default_rng(10)
    n, H, Hk = 3, 4, 2
    bits = [4, 6, 8, 6]
    S = np.stack([np.stack([random_fp32_state(rng, steps=8) for _ in range(H)]) for _ in range(n)])
    slots = np.array([2, 0, 1], np.int32)
    pa = O.OraclePool(3, bits, Hk)
    pb = O.OraclePool(3, bits, H)
    pa.load_fp32(slots, S)
    pb.load_fp32(slots, S)
    q = np.stack([np.stack([unit(rng, 128) for _ in range(Hk)]) for _ in range(n)])
    k = np.stack([np.stack([unit(rng, 128) for _ in range(Hk)]) for _ in range(n)])
    v = rng.standard_normal((n, H, 128)).astype(f32)
    al = np.full((n, H), 0.95, f32)
    be = np.full((n, H), 0.5, f32)
    ya = pa.decode_step(slots, q, k, v, al, be)
    yb = pb.decode_step(slots, np.repeat(q, 2, axis=1), np.repeat(k, 2, axis=1), v, al, be)
    assert np.array_equal(ya, yb)
    assert np.array_equal(pa.data, pb.data)


def test_pool_driver_matches_single_state_steps():
    rng = np.random.default_rng(11)
    n, H, Hk = 2, 2, 1
    bits = [6, 8]
    pool = O.OraclePool(4, bits, Hk, gate_mode=1)
    slots = np.array([3, 1], np.int32)
    S = np.stack([np.stack([random_fp32_state(rng, steps=6) for _ in range(H)]) for _ in range(n)])
    pool.load_fp32(slots, S)
    q = rng.standard_normal((n, Hk, 128)).astype(f32)
    k = np.stack([[unit(rng, 128)] for _ in range(n)])
    v = rng.standard_normal((n, H, 128)).astype(f32)
    al = rng.uniform(0.5, 1.0, (n, H, 128)).astype(f32)
    be = rng.uniform(0, 1, (n, H)).astype(f32)
    before = [[pool.state(s, h) for h in range(H)] for s in slots]
    y = pool.decode_step(slots, q, k, v, al, be)
    for b, s in enumerate(slots):
        for h in range(H):
            Q, r, c = before[b][h]
            o = O.step_state(Q, r, c, bits[h], q[b, 0], k[b, 0], v[b, h], al[b, h], be[b, h])
            Q2, r2, c2 = pool.state(s, h)
            assert np.array_equal(Q2, o["Q"]) and np.array_equal(r2, o["r"]) and np.array_equal(c2, o["c"])
            assert np.array_equal(y[b, h], o["y"])
    assert not pool.block(0, 0).any() and not pool.block(2, 1).any()    # untouched slots stay zero
    with pytest.raises(IndexError):
        pool.decode_step(np.array([4, 0], np.int32), q, k, v, al, be)


# --------------------------------------------------------------------------- Proposition 1

def test_proposition1_error_recursion():
    """'The intuition: errors get carried forward' (Proposition 1): with
    E_t = S_hat_t - S_fp_t, A_t = (I - beta k k^T) D_t and eps_t the fresh
    quantization error, E_t = A_t E_{t-1} + eps_t.  A_t is built here from the
    inputs with numpy; the quantized and the exact trajectories come from the oracle."""
    rng = np.random.default_rng(12)
    for bits, gate in ((4, "gdn"), (6, "kda"), (8, "gdn")):
        S_fp = random_fp32_state(rng, steps=16).astype(np.float64)
        Q, r, c, _ = O.quantize(S_fp.astype(f32), bits)
        S_hat = O.dequantize(Q, r, c)
        E = S_hat - S_fp
        for t in range(12):
            q, k = unit(rng, 128), unit(rng, 128)
            v = rng.standard_normal(128).astype(f32)
            beta = f32(1 / (1 + np.exp(-rng.standard_normal())))
            alpha = (rng.uniform(0.6, 1.0, 128) if gate == "kda" else np.full(128, rng.uniform(0.6, 1.0))).astype(f32)
            o = O.step_state(Q, r, c, bits, q, k, v, alpha, beta)
            S_fp, _ = O.delta_step(S_fp, q, k, v, alpha, beta)
            kd = k.astype(np.float64)
            A = (np.eye(128) - float(beta) * np.outer(kd, kd)) @ np.diag(alpha.astype(np.float64))
            Q, r, c = o["Q"], o["r"], o["c"]
            S_hat = O.dequantize(Q, r, c)
            eps = S_hat - o["S_pre"]
            E_new = S_hat - S_fp
            scale = np.abs(E_new).max() + np.abs(S_fp).max()
            assert np.abs(E_new - (A @ E + eps)).max() <= 1e-12 * scale
            # the transition contracts: ||A||_2 <= max alpha for a unit key and beta in (0, 1)
            assert np.linalg.norm(A, 2) <= float(alpha.max()) * (1 + 1e-9)
            E = E_new


# --------------------------------------------------------------------------- fit invariants

@pytest.mark.parametrize("bits", [4, 6, 8])
def test_fit_invariants(bits):
    """No clipping, every live row reaches qmax, error at most half a step,
    and zero rows/columns encode as zero scale and zero codes."""
    rng = np.random.default_rng(20 + bits)
    qm = (1 << (bits - 1)) - 1
    for trial in range(6):
        S = random_fp32_state(rng, steps=4 + 6 * trial)
        S[3, :] = 0                                   # a zero row
        S[:, 9] = 0                                   # a zero column
        S[7, 11] = -S[7, 11] * 40 if trial % 2 else S[7, 11]   # an outlier
        Q, r, c, clipped = O.quantize(S, bits)
        assert clipped == 0
        x = S.astype(np.float64) / np.where(np.outer(r, c) > 0, np.outer(r, c), np.inf)
        assert np.abs(x).max() <= qm * (1 + 4 * F32_EPS)
        live = r > 0
        assert np.all(np.abs(Q[live]).max(axis=1) == qm)
        step = np.outer(r.astype(np.float64), c.astype(np.float64))
        err = np.abs(S.astype(np.float64) - Q * step)
        assert np.all(err <= 0.5 * step * (1 + 4 * F32_EPS) + 1e-300)
        assert r[3] == 0 and c[9] == 0 and not Q[3].any() and not Q[:, 9].any()


def test_fit_is_nearest_level_brute_force():
    """For tiny states, the code of every element is the level nearest to it among all
    2*qmax + 1 levels on its row/column grid (ties go to the even level)."""
    rng = np.random.default_rng(30)
    for d in (2, 4, 8):
        for bits in (4, 6, 8):
            qm = (1 << (bits - 1)) - 1
            levels = np.arange(-qm, qm + 1)
            for _ in range(200):
                S = (rng.standard_normal((d, d)) * rng.lognormal(0, 1.5, (d, 1))).astype(f32)
                Q, r, c, _ = O.quantize(S, bits)
                for i in range(d):
                    for j in range(d):
                        step = float(r[i]) * float(c[j])
                        if step == 0:
                            assert Q[i, j] == 0
                            continue
                        dist = np.abs(float(S[i, j]) - levels * step)
                        best = levels[dist == dist.min()]
                        assert Q[i, j] in best
                        if len(best) == 2:
                            assert Q[i, j] % 2 == 0


def test_power_of_two_fade_equivariance():
    """A step with alpha = 1/4, beta = 0 gives the same codes as alpha = 1, beta = 0
    from the same stored state, with r and c exactly halved."""
    rng = np.random.default_rng(31)
    for bits in (4, 6, 8):
        Q, r, c, _ = O.quantize(random_fp32_state(rng), bits)
        z = np.zeros(128, f32)
        one = O.step_state(Q, r, c, bits, z, z, z, 1.0, 0.0)
        quarter = O.step_state(Q, r, c, bits, z, z, z, 0.25, 0.0)
        assert np.array_equal(one["Q"], quarter["Q"])
        assert np.array_equal(one["r"] / 2, quarter["r"])
        assert np.array_equal(one["c"] / 2, quarter["c"])


def test_more_bits_less_error_brute_force():
    """On many tiny random states and short trajectories, 8-bit storage error stays below
    6-bit, which stays below 4-bit: in aggregate at every size, and per sample at d = 8."""
    rng = np.random.default_rng(32)
    for d in (2, 4, 8):
        tot = {4: 0.0, 6: 0.0, 8: 0.0}
        for s in range(400):
            S = (rng.standard_normal((d, d)) * rng.lognormal(0, 1, (1, d))).astype(f32)
            errs = {}
            for bits in (4, 6, 8):
                Q, r, c, _ = O.quantize(S, bits)
                errs[bits] = float(np.sum((S.astype(np.float64) - O.dequantize(Q, r, c)) ** 2))
                tot[bits] += errs[bits]
            if d == 8:
                assert errs[8] <= errs[6] <= errs[4]
        assert tot[8] < tot[6] < tot[4]
    # short quantized trajectories against the exact (double) trajectory
    d = 8
    tot = {4: 0.0, 6: 0.0, 8: 0.0}
    for s in range(60):
        seq = [(unit(rng, d), unit(rng, d), rng.standard_normal(d).astype(f32), f32(0.9), f32(0.5))
               for _ in range(10)]
        for bits in (4, 6, 8):
            Q, r, c = np.zeros((d, d), np.int32), np.zeros(d, f32), np.zeros(d, f32)
            S_fp = np.zeros((d, d))
            for (q, k, v, a, b) in seq:
                o = O.step_state(Q, r, c, bits, q, k, v, a, b)
                Q, r, c = o["Q"], o["r"], o["c"]
                S_fp, _ = O.delta_step(S_fp, q, k, v, a, b)
            tot[bits] += float(np.sum((O.dequantize(Q, r, c) - S_fp) ** 2))
    assert tot[8] < tot[6] < tot[4]


def test_dequantize_is_exact_product():
    """Q * r * c must be exact in double (an 8-bit integer times two fp32 values)."""
    rng = np.random.default_rng(33)
    Q, r, c, _ = O.quantize(random_fp32_state(rng), 8)
    S = O.dequantize(Q, r, c)
    from fractions import Fraction
    for (i, j) in [(0, 0), (5, 17), (127, 127), (64, 3)]:
        exact = Fraction(int(Q[i, j])) * Fraction(float(r[i])) * Fraction(float(c[j]))
        assert Fraction(S[i, j]) == exact


def test_single_flip_diverges_trajectory():
    """Property behind the trajectory-parity reading: one permitted +-1 code difference
    in a long-lived head grows, through the recurrence, into an output difference far
    above 1e-3 relative (errors along rarely-hit key directions persist when the gate
    sits near one)."""
    rng = np.random.default_rng(34)
    S = random_fp32_state(rng, steps=32, alpha=0.9998)
    Q, r, c, _ = O.quantize(S, 8)
    Q2 = Q.copy()
    Q2[5, 7] += 1 if Q2[5, 7] < 127 else -1
    A, B = (Q, r, c), (Q2, r.copy(), c.copy())
    num = den = 0.0
    for t in range(48):
        q, k = unit(rng, 128), unit(rng, 128)
        v = rng.standard_normal(128).astype(f32)
        a = O.step_state(*A, 8, q, k, v, 0.9998, 0.5)
        b = O.step_state(*B, 8, q, k, v, 0.9998, 0.5)
        A, B = (a["Q"], a["r"], a["c"]), (b["Q"], b["r"], b["c"])
        num += float(np.sum((a["y"] - b["y"]) ** 2))
        den += float(np.sum(a["y"] ** 2))
    assert np.sqrt(num / den) > 1e-3
