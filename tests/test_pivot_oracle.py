"""Pins of the oracle's FP16 pivot heads (STEPQuant summary, "Method" para 2: the
highest-risk units are kept in FP16 as sparse pivots).  A width-16 head stores its state as
binary16 values; its step fades, writes and reads out like every head and then stores the
state rounded to fp32 and to binary16 (nearest, ties to even)."""
import itertools

import numpy as np
import pytest

from oracle import oracle as O

f32 = np.float32


def test_fp16_rounding_matches_numpy():
    """binary16 rounding written from the format's definition against numpy's conversion
    (a library routine): ties to even, subnormals, the overflow threshold, signed zero."""
    special = [0.0, -0.0, 1.0, -1.0, 65504.0, 65519.99, 65520.0, -65520.0, 1e6, 2.0 ** -24, 2.0 ** -25,
               3 * 2.0 ** -25, 2.0 ** -14, 2.0 ** -14 * (1 - 2 ** -12), 1 + 2.0 ** -11, 1 + 3 * 2.0 ** -11,
               2048 + 1.0, 2048 + 3.0, 0.1, 1 / 3]
    rng = np.random.default_rng(0)
    x = np.concatenate([special, rng.standard_normal(200000) * 10.0 ** rng.uniform(-9, 5.2, 200000)])
    with np.errstate(over="ignore"):
        ref = x.astype(np.float16).view(np.uint16)
    assert np.array_equal(O.fp16_encode(x), ref)
    allbits = np.arange(65536, dtype=np.uint16)
    assert np.array_equal(O.fp16_decode(allbits), allbits.view(np.float16).astype(np.float64), equal_nan=True)


def _pivot_pool(rng, gate_mode=0):
    bits = [16, 6]
    pool = O.OraclePool(3, bits, 1 if gate_mode == 0 else 2, gate_mode)
    S = (rng.standard_normal((2, 2, 128, 128)) * 0.5).astype(f32)
    pool.load_fp32([2, 0], S)
    return pool, S


def test_pivot_load_and_dump_are_binary16_of_the_input():
    rng = np.random.default_rng(1)
    pool, S = _pivot_pool(rng)
    h16 = pool.state(2, 0)
    assert np.array_equal(h16, S[0, 0].astype(np.float16).view(np.uint16))
    assert O.block_bytes(16) == 32768
    back = pool.dump_fp32([2, 0])[:, 0]
    assert np.array_equal(back, S[:, 0].astype(np.float16).astype(f32))


def test_pivot_identity_step_keeps_state_and_reads_out():
    """alpha = 1, beta = 0: the stored state is unchanged bit for bit and y = S^T q."""
    rng = np.random.default_rng(2)
    pool, S = _pivot_pool(rng)
    before = pool.state(2, 0).copy()
    q = rng.standard_normal((1, 1, 128)).astype(f32)
    k = rng.standard_normal((1, 1, 128)).astype(f32)
    v = rng.standard_normal((1, 2, 128)).astype(f32)
    y = pool.decode_step([2], q, k, v, np.ones((1, 2), f32), np.zeros((1, 2), f32))
    assert np.array_equal(pool.state(2, 0), before)
    S16 = before.view(np.float16).astype(np.float64)
    np.testing.assert_allclose(y[0, 0], (S16.T @ q[0, 0].astype(np.float64)).astype(f32), rtol=2e-7, atol=1e-30)


def test_pivot_rank1_write_from_zero_state():
    """Zero state, k = e_5, any alpha: S = beta e_5 v^T, stored as binary16(fp32(beta v_j))
    in row 5, zero elsewhere; y_j = q_5 beta v_j."""
    pool = O.OraclePool(1, [16], 1)
    rng = np.random.default_rng(3)
    k = np.zeros((1, 1, 128), f32)
    k[0, 0, 5] = 1
    q = rng.standard_normal((1, 1, 128)).astype(f32)
    v = rng.standard_normal((1, 1, 128)).astype(f32)
    beta = f32(0.37)
    y = pool.decode_step([0], q, k, v, np.full((1, 1), 0.9, f32), np.full((1, 1), beta, f32))
    st = pool.state(0, 0)
    expect_row = (np.float64(beta) * v[0, 0].astype(np.float64)).astype(f32).astype(np.float16).view(np.uint16)
    assert np.array_equal(st[5], expect_row)
    assert not np.delete(st, 5, axis=0).any()
    np.testing.assert_allclose(y[0, 0], (np.float64(q[0, 0, 5]) * beta * v[0, 0].astype(np.float64)).astype(f32),
                               rtol=1e-7)


def test_pivot_step_equals_fp_step_rounded_to_binary16():
    """KDA pool with a pivot: one step of the pivot head equals the unquantized step from
    the binary16 state, rounded to fp32 and then to binary16 (numpy's conversion)."""
    rng = np.random.default_rng(4)
    pool, S = _pivot_pool(rng, gate_mode=1)
    S0 = pool.state(2, 0).view(np.float16).astype(np.float64)
    q = rng.standard_normal((1, 2, 128)).astype(f32)
    k = rng.standard_normal((1, 2, 128)).astype(f32)
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.standard_normal((1, 2, 128)).astype(f32)
    a = rng.uniform(0.5, 1, (1, 2, 128)).astype(f32)
    b = rng.uniform(0, 1, (1, 2)).astype(f32)
    y = pool.decode_step([2], q, k, v, a, b)
    Sx = np.ascontiguousarray(S0[None, None])
    y_fp = O.fp_decode_step(Sx, 1, 1, q[:, :1], k[:, :1], v[:, :1], a[:, :1], b[:, :1], round_fp32=True)
    assert np.array_equal(pool.state(2, 0), Sx[0, 0].astype(f32).astype(np.float16).view(np.uint16))
    assert np.array_equal(y[0, 0], y_fp[0, 0])


def test_pivot_selection_takes_highest_risk_units():
    hl = [2.0, 4096.0, 32.0, 900.0, 512.0]
    d = [[1.0, 0.5, 0.2], [0.1, 0.05, 0.01], [3.0, 2.0, 1.0], [0.2, 0.1, 0.03], [0.3, 0.2, 0.1]]
    cand = [4, 6, 8]
    risk = [O.lifetime_weight(h) * d[u][2] for u, h in enumerate(hl)]
    assert O.select_pivots(hl, d, cand, 2) == sorted(np.argsort(risk)[::-1][:2].tolist())
    assert O.select_pivots(hl, d, cand, 0) == []


def test_pivot_allocation_matches_bruteforce_on_the_rest():
    rng = np.random.default_rng(5)
    hl = list(2.0 ** rng.uniform(1, 12, 7))
    cand = [4, 6, 8]
    bits, obj = O.allocate_bits_pivots(hl, None, cand, 6.0, 2)
    piv = O.select_pivots(hl, None, cand, 2)
    assert [u for u, b in enumerate(bits) if b == 16] == piv
    rest = [u for u in range(7) if u not in piv]
    bb, bobj = O.allocate_bits_bruteforce([hl[u] for u in rest], None, cand, 6.0)
    assert [bits[u] for u in rest] == bb and obj == pytest.approx(bobj)
    assert sum(bits[u] for u in rest) <= 5 * 6
