"""Pins of the oracle's per-key-row widths (the ONTLE blog: the allocation unit of Kimi's
KDA is a single key row): the stored-row layout, the clip-free fit at each row's own
levels, the pool plumbing, and the per-row allocation."""
import json
import os

import numpy as np
import pytest

from oracle import oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
f32 = np.float32


def _golden_rb(g):
    rb = np.full(128, g["row_bits"]["default"], np.int32)
    for k, v in g["row_bits"].items():
        if k != "default":
            rb[int(k)] = v
    return rb


def test_rowbits_golden_bytes():
    g = json.load(open(os.path.join(GOLDEN, "rowbits_bytes.json")))
    rb = _golden_rb(g)
    Q = np.zeros((128, 128), np.int32)
    for i, j, code in g["codes"]:
        Q[i, j] = code
    buf = O.rows_pack(Q, rb)
    assert O.rows_block_bytes(rb) == g["block_bytes"]
    for off, expect in g["bytes_at"].items():
        off = int(off)
        assert list(buf[off:off + len(expect)]) == expect, off
    assert np.array_equal(O.rows_unpack(buf, rb), Q)
    assert list(O.rows_order(rb)[:4]) == [5, 0, 1, 3] and O.rows_order(rb)[-1] == 2


@pytest.mark.parametrize("bits", [4, 6, 8])
def test_uniform_rows_are_the_uniform_layout_and_fit(bits):
    rng = np.random.default_rng(bits)
    qm = (1 << (bits - 1)) - 1
    rb = np.full(128, bits, np.int32)
    Q = rng.integers(-qm, qm + 1, (128, 128)).astype(np.int32)
    assert np.array_equal(O.rows_pack(Q, rb), O.pack_codes(Q, bits))
    assert O.rows_block_bytes(rb) == O.block_bytes(bits)
    S = (rng.standard_normal((128, 128)) * np.exp(rng.normal(0, 1, 128))[:, None]).astype(f32)
    Qa, ra, ca, _ = O.rows_quantize(S, rb)
    Qb, rbb, cb = O.quantize(S, bits)[:3]
    assert np.array_equal(Qa, Qb) and np.array_equal(ra, rbb) and np.array_equal(ca, cb)


def test_mixed_rows_nearest_level_at_each_rows_width():
    """Brute force: every code is the nearest of its row's 2 qmax + 1 levels (ties even),
    the fit is clip-free, and each live row reaches its own qmax."""
    rng = np.random.default_rng(30)
    rb = rng.choice([4, 6, 8], 128).astype(np.int32)
    S = (rng.standard_normal((128, 128)) * np.exp(rng.normal(0, 1, 128))[:, None]).astype(f32)
    Q, r, c, clipped = O.rows_quantize(S, rb)
    assert clipped == 0
    for i in range(0, 128, 3):
        qm = (1 << (int(rb[i]) - 1)) - 1
        levels = np.arange(-qm, qm + 1, dtype=np.float64)
        x = S[i].astype(np.float64) / (np.float64(r[i]) * c.astype(np.float64))
        d = np.abs(x[:, None] - levels[None, :])
        best = levels[np.argmin(d, axis=1)]
        tie = np.isclose(np.sort(d, axis=1)[:, 1], np.sort(d, axis=1)[:, 0], rtol=0, atol=1e-12)
        assert np.all((Q[i] == best) | tie)
        assert np.abs(Q[i]).max() == qm


def test_rowbits_pool_plumbing():
    rng = np.random.default_rng(31)
    H = 2
    rbs = np.stack([rng.choice([4, 6, 8], 128), rng.choice([4, 8], 128)]).astype(np.int32)
    pool = O.OraclePool(3, [0, 0], H, 1, row_bits=rbs)
    S = (rng.standard_normal((2, H, 128, 128)) * 0.3).astype(f32)
    pool.load_fp32([2, 0], S)
    for h in range(H):
        Q, r, c = pool.state(2, h)
        Qe, re, ce, _ = O.rows_quantize(S[0, h], rbs[h])
        assert np.array_equal(Q, Qe) and np.array_equal(r, re) and np.array_equal(c, ce)
    off, stride = O.head_offsets([0, 0], row_bits=rbs)
    assert stride == O.rows_block_bytes(rbs[0]) + O.rows_block_bytes(rbs[1])
    # one KDA step through the pool equals the per-state step
    q = rng.standard_normal((1, H, 128)).astype(f32)
    k = rng.standard_normal((1, H, 128)).astype(f32)
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.standard_normal((1, H, 128)).astype(f32)
    a = rng.uniform(0.5, 1, (1, H, 128)).astype(f32)
    b = rng.uniform(0, 1, (1, H)).astype(f32)
    Q0, r0, c0 = pool.state(0, 1)
    y = pool.decode_step([0], q, k, v, a, b)
    Sh = O.dequantize(Q0, r0, c0)
    Sx = np.ascontiguousarray(Sh[None, None])
    y_fp = O.fp_decode_step(Sx, 1, 1, q[:, 1:], k[:, 1:], v[:, 1:], a[:, 1:], b[:, 1:], round_fp32=True)
    Qe, re, ce, _ = O.rows_quantize(Sx[0, 0].astype(f32), rbs[1])
    Q1, r1, c1 = pool.state(0, 1)
    assert np.array_equal(Q1, Qe) and np.array_equal(r1, re) and np.array_equal(c1, ce)
    assert np.array_equal(y[0, 1], y_fp[0, 0])


def test_mixed_pool_with_impact_scores_dispatches_each_fit():
    """One pool with a per-key-row head next to uniform heads and row-impact scores set: a KDA
    step through the pool equals, head by head, the unquantized step followed by the head's own
    fit -- the clip-free per-row fit for the per-row head, the impact-weighted fit for the
    uniform heads (the impact scores do not reach the per-row head)."""
    rng = np.random.default_rng(41)
    H = 3
    bits = [6, 0, 8]
    rbs = np.stack([np.full(128, 6), rng.choice([4, 6, 8], 128), np.full(128, 8)]).astype(np.int32)
    omega = np.exp(rng.normal(0, 1, (H, 128))).astype(f32)
    pool = O.OraclePool(2, bits, H, 1, row_bits=rbs, impact=omega)
    S = (rng.standard_normal((1, H, 128, 128)) * 0.3).astype(f32)
    pool.load_fp32([1], S)
    q = rng.standard_normal((1, H, 128)).astype(f32)
    k = rng.standard_normal((1, H, 128)).astype(f32)
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.standard_normal((1, H, 128)).astype(f32)
    a = rng.uniform(0.5, 1, (1, H, 128)).astype(f32)
    b = rng.uniform(0, 1, (1, H)).astype(f32)
    before = [pool.state(1, h) for h in range(H)]
    y = pool.decode_step([1], q, k, v, a, b)
    for h in range(H):
        Sx = np.ascontiguousarray(O.dequantize(*before[h])[None, None])
        sl = slice(h, h + 1)
        y_fp = O.fp_decode_step(Sx, 1, 1, q[:, sl], k[:, sl], v[:, sl], a[:, sl], b[:, sl], round_fp32=True)
        S32 = Sx[0, 0].astype(f32)
        if bits[h] == 0:
            Qe, re, ce, _ = O.rows_quantize(S32, rbs[h])
        else:
            Qe, re, ce, _ = O.quantize_impact(S32, bits[h], O.impact_normalize(omega[h]))
        Q1, r1, c1 = pool.state(1, h)
        assert np.array_equal(Q1, Qe) and np.array_equal(r1, re) and np.array_equal(c1, ce), h
        assert np.array_equal(y[0, h], y_fp[0, 0]), h
