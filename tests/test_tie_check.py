"""The element-wise code check that the GPU parity tests use where a flip-rate bar does not fit
(parity_helpers.flips_off_tie), pinned on the CPU on states whose rounding ties are placed by
hand.

A step from the zero state with a key k and beta = 1 writes S = k v^T.  For such a rank-one
state the clip-free fit gives every row of column j the same ratio
t_j = qmax * sqrt(|v_j| / max |v|) (the rank-one closed form of the fit), so choosing v places a
whole column at a rounding tie (t = 2.5) or far from one (t = 1.2)."""
import numpy as np

from oracle import oracle as O
from tests import parity_helpers as PH

BITS = 4
QMAX = 7


def _tie_step():
    rng = np.random.default_rng(5)
    bits, Hk, n = [BITS, BITS], 1, 1
    op = O.OraclePool(2, bits, Hk)
    ids = np.array([1], np.int32)
    before = op.slot_bytes(ids)                       # the zero state
    k = np.full((n, Hk, 128), 1.0 / np.sqrt(128.0), np.float32)
    q = rng.standard_normal((n, Hk, 128)).astype(np.float32)
    q /= np.linalg.norm(q)
    v = np.zeros((n, 2, 128), np.float32)
    v[0, :, 0] = 1.0                                  # the column maximum: t = qmax
    v[0, :, 1] = (2.5 / QMAX) ** 2                    # t = 2.5: a tie in every row
    v[0, :, 2] = (1.2 / QMAX) ** 2                    # t = 1.2: far from a tie
    v[0, :, 3] = -(4.5 / QMAX) ** 2                   # t = 4.5, negative codes
    x = dict(q=q, k=k, v=v, alpha=np.ones((n, 2), np.float32), beta=np.ones((n, 2), np.float32))
    op.decode_step(ids, x["q"], x["k"], x["v"], x["alpha"], x["beta"])
    return bits, Hk, before, op.slot_bytes(ids), x


def _edit(after, bits, h, fn):
    offs, _ = O.head_offsets(bits)
    out = after.copy()
    n = O.block_bytes(bits[h])
    Q, r, c = O.split_block(out[0, offs[h]:offs[h] + n], bits[h])
    Q = Q.copy()
    fn(Q)
    out[0, offs[h]:offs[h] + n] = O.make_block(Q, r, c, bits[h])
    return out


def test_closed_form_places_the_ties():
    bits, Hk, before, after, x = _tie_step()
    Q, r, c = O.split_block(after[0, :O.block_bytes(BITS)], BITS)
    assert np.all(Q[:, 0] == QMAX) and np.all(Q[:, 2] == 1) and np.all(np.abs(Q[:, 1] - 2.5) == 0.5)
    assert np.all(np.abs(Q[:, 3]) >= 4) and np.all(np.abs(Q[:, 3]) <= 5) and np.all(Q[:, 3] < 0)
    assert np.all(Q[:, 4:] == 0)


def test_oracle_against_itself_has_no_flip():
    bits, Hk, before, after, x = _tie_step()
    assert PH.flips_off_tie(after, before, bits, Hk, x) == (0, 0)


def test_a_whole_tie_column_rounded_the_other_way_passes():
    bits, Hk, before, after, x = _tie_step()

    def other_way(Q):
        Q[:, 1] = np.where(Q[:, 1] == 2, 3, 2)         # all 128 rows of the tie column
        Q[:, 3] = np.where(Q[:, 3] == -4, -5, -4)      # and the negative tie column
    assert PH.flips_off_tie(_edit(after, bits, 0, other_way), before, bits, Hk, x) == (0, 1)


def test_one_flip_away_from_a_tie_is_caught():
    bits, Hk, before, after, x = _tie_step()

    def one_off(Q):
        Q[17, 2] += 1                                  # t = 1.2: 1 is the only correct code
    assert PH.flips_off_tie(_edit(after, bits, 1, one_off), before, bits, Hk, x) == (1, 1)


def test_a_two_level_difference_is_reported():
    bits, Hk, before, after, x = _tie_step()

    def two_off(Q):
        Q[3, 1] = 4 if Q[3, 1] == 2 else 1             # two levels from the oracle's code
    off_tie, worst = PH.flips_off_tie(_edit(after, bits, 0, two_off), before, bits, Hk, x)
    assert worst == 2
