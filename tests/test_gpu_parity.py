"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle on the same seeded
inputs.  Every test here needs a B200 and the built libstepq.so."""
import json
import os

import numpy as np
import pytest

from oracle import oracle as O
from quantized_gated_delta_b200 import workloads as W
from tests import parity_helpers as PH

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
f32 = np.float32


@pytest.fixture(scope="module")
def S():
    from quantized_gated_delta_b200 import stepq
    stepq.load_library()
    return stepq


def dev(a, dtype=None):
    t = torch.from_numpy(np.ascontiguousarray(a))
    return t.cuda() if dtype is None else t.to(dtype).cuda()


def slots_t(ids):
    return dev(np.asarray(ids, dtype=np.int32))


def dump_bytes(pool, ids):
    out = torch.empty((len(ids), pool.slot_stride), dtype=torch.uint8, device="cuda")
    pool.dump_packed(slots_t(ids), out)
    torch.cuda.synchronize()
    return out.cpu().numpy()


def load_bytes(pool, ids, data):
    pool.load_packed(slots_t(ids), dev(data))


def unit(rng, n):
    x = rng.standard_normal(n)
    return (x / np.linalg.norm(x)).astype(f32)


def random_states(rng, n, H, steps=24, alpha=0.98):
    S_ = np.zeros((n, H, 128, 128))
    q = np.zeros((n, H, 128), f32)
    for _ in range(steps):
        x = dict(q=np.stack([[unit(rng, 128) for _ in range(H)] for _ in range(n)]),
                 k=np.stack([[unit(rng, 128) for _ in range(H)] for _ in range(n)]),
                 v=rng.standard_normal((n, H, 128)).astype(f32),
                 alpha=np.full((n, H), alpha, f32), beta=rng.uniform(0.1, 0.9, (n, H)).astype(f32))
        O.fp_decode_step(S_, H, 0, x["q"], x["k"], x["v"], x["alpha"], x["beta"], round_fp32=True)
    return S_.astype(f32)


# --------------------------------------------------------------------------- pool I/O

def test_load_fp32_matches_oracle_quantize(S):
    rng = np.random.default_rng(1)
    bits = [4, 6, 8, 8, 6, 4]
    n = 5
    st = random_states(rng, n, len(bits))
    st[0, 0, 3, :] = 0                      # zero row
    st[0, 1, :, 9] = 0                      # zero column
    st[1, 2, 7, 11] *= -50                  # outlier
    st[2, 3] = 0                            # all-zero state
    st[3, 4] *= 1e-30                       # tiny magnitudes
    st[4, 5] *= 1e20                        # huge magnitudes
    ids = np.array([7, 2, 0, 5, 3], np.int32)
    op = O.OraclePool(8, bits, len(bits))
    op.load_fp32(ids, st)
    gp = S.Pool(8, bits, len(bits), S.STEPQ_GATE_GDN, S.STEPQ_DTYPE_F32)
    gp.load_fp32(slots_t(ids), dev(st))
    res = PH.compare_slots(dump_bytes(gp, ids), op.slot_bytes(ids), bits)
    assert gp.get_error() == 0
    assert res["max_code_diff"] <= 1
    assert res["flips"] <= PH.CODE_FLIP_RATE * res["elements"] + 1e-12 or res["flips"] <= 1
    assert res["c_ulp"] == 0               # c = sqrt(max |S|): both sides correctly rounded
    assert res["r_ulp"] <= PH.R_ULP
    # untouched slots stay zero
    z = dump_bytes(gp, [1, 4, 6])
    assert not z.any()


def test_dump_fp32_is_exact(S):
    rng = np.random.default_rng(2)
    bits = [8, 4, 6]
    st = random_states(rng, 3, 3)
    ids = np.array([2, 0, 1], np.int32)
    op = O.OraclePool(3, bits, 3)
    op.load_fp32(ids, st)
    gp = S.Pool(3, bits, 3, S.STEPQ_GATE_GDN, S.STEPQ_DTYPE_F32)
    load_bytes(gp, ids, op.slot_bytes(ids))
    out = torch.empty((3, 3, 128, 128), dtype=torch.float32, device="cuda")
    gp.dump_fp32(slots_t(ids), out)
    assert np.array_equal(out.cpu().numpy(), op.dump_fp32(ids))


def test_packed_round_trip_bit_exact(S):
    rng = np.random.default_rng(3)
    bits = [6, 8, 4, 6]
    gp = S.Pool(16, bits, 2)
    stride = gp.slot_stride
    data = rng.integers(0, 256, (5, stride), dtype=np.uint8)
    ids = np.array([15, 3, 9, 0, 4], np.int32)
    load_bytes(gp, ids, data)
    assert np.array_equal(dump_bytes(gp, ids), data)
    assert np.array_equal(dump_bytes(gp, [15]), data[:1])


# --------------------------------------------------------------------------- hand-computed cases

@pytest.mark.parametrize("bits", [4, 6, 8])
def test_rank1_worked_case_on_gpu(S, bits):
    g = json.load(open(os.path.join(GOLDEN, "rank1_worked_case.json")))["step1"]
    gp = S.Pool(2, [bits], 1, S.STEPQ_GATE_GDN, S.STEPQ_DTYPE_F32)
    k = np.zeros((2, 1, 128), f32)
    k[:, 0, g["key_index"]] = 1
    v = np.zeros((2, 1, 128), f32)
    v[:, 0, :4] = g["v_head"]
    q = np.random.default_rng(4).standard_normal((2, 1, 128)).astype(f32)
    y = torch.empty((2, 1, 128), device="cuda")
    gp.decode_step(slots_t([1, 0]), dev(q), dev(k), dev(v), dev(np.full((2, 1), g["alpha"], f32)),
                   dev(np.full((2, 1), g["beta"], f32)), y)
    raw = dump_bytes(gp, [1, 0])
    for s in range(2):
        Q, r, c = O.split_block(raw[s], bits)
        assert list(Q[0, :4]) == g["codes_row0_head"][str(bits)]
        assert not Q[1:].any() and not Q[0, 4:].any()
        np.testing.assert_allclose(c[:4], g["c_head"], rtol=1e-6)
        assert r[0] == pytest.approx(g["r0"][str(bits)], rel=1e-6) and not r[1:].any()
    yh = y.cpu().numpy()
    np.testing.assert_allclose(yh[:, 0], q[:, 0, :1] * v[:, 0], rtol=1e-6, atol=1e-12)


def test_power_of_two_fade_equivariance_on_gpu(S):
    rng = np.random.default_rng(5)
    bits = [4, 6, 8]
    st = random_states(rng, 2, 3)
    op = O.OraclePool(2, bits, 3)
    op.load_fp32(np.arange(2, dtype=np.int32), st)
    outs = []
    for alpha in (1.0, 0.25):
        gp = S.Pool(2, bits, 3, S.STEPQ_GATE_GDN, S.STEPQ_DTYPE_F32)
        load_bytes(gp, [0, 1], op.slot_bytes([0, 1]))
        z = np.zeros((2, 3, 128), f32)
        y = torch.empty((2, 3, 128), device="cuda")
        gp.decode_step(slots_t([0, 1]), dev(z), dev(z), dev(z), dev(np.full((2, 3), alpha, f32)),
                       dev(np.zeros((2, 3), f32)), y)
        outs.append(dump_bytes(gp, [0, 1]))
    for s in range(2):
        for h, b in enumerate(bits):
            off, _ = O.head_offsets(bits)
            n = O.block_bytes(b)
            A = O.split_block(outs[0][s, off[h]:off[h] + n], b)
            B = O.split_block(outs[1][s, off[h]:off[h] + n], b)
            assert np.array_equal(A[0], B[0])
            assert np.array_equal(A[1] / 2, B[1]) and np.array_equal(A[2] / 2, B[2])


def test_decode_extreme_rows_vs_oracle(S):
    """One step from states with a row of subnormal magnitude whose key component is zero
    (the refit gives it a subnormal row factor), a state of huge magnitudes, and a zero
    state: single-step tolerances against the oracle."""
    rng = np.random.default_rng(11)
    bits = [4, 6, 8]
    n, H = 3, 3
    st = random_states(rng, n, H)
    st[0, :, 5, :] *= 1e-40                 # subnormal row in every head of request 0
    st[1] *= 1e30                           # huge magnitudes
    st[2, 1] = 0                            # zero state
    ids = np.array([2, 0, 1], np.int32)
    op = O.OraclePool(3, bits, H)
    op.load_fp32(ids, st)
    init = op.slot_bytes(ids)
    k = np.stack([[unit(rng, 128) for _ in range(H)] for _ in range(n)])
    k[0, :, 5] = 0
    k[0] /= np.linalg.norm(k[0], axis=-1, keepdims=True)
    x = dict(q=np.stack([[unit(rng, 128) for _ in range(H)] for _ in range(n)]), k=k.astype(f32),
             v=rng.standard_normal((n, H, 128)).astype(f32),
             alpha=rng.uniform(0.5, 1, (n, H)).astype(f32), beta=rng.uniform(0.1, 0.9, (n, H)).astype(f32))
    yg, sg, err = _run_gpu(S, bits, H, 0, S.STEPQ_DTYPE_F32, x, init, ids, 3)
    assert err == 0
    yo = op.decode_step(ids, x["q"], x["k"], x["v"], x["alpha"], x["beta"])
    ob = op.slot_bytes(ids)
    r0 = np.concatenate([O.split_block(ob[0, o:o + O.block_bytes(b)], b)[1]
                         for o, b in zip(O.head_offsets(bits)[0], bits)])
    assert np.any((r0 > 0) & (r0 < np.finfo(np.float32).tiny))      # the subnormal path is reached
    res = PH.compare_slots(sg, ob, bits)
    assert res["max_code_diff"] <= 1
    assert res["flips"] <= max(1, PH.CODE_FLIP_RATE * res["elements"])
    assert res["r_ulp"] <= PH.R_ULP and res["c_ulp"] <= PH.C_ULP
    assert PH.y_max_rel(yg, yo) <= PH.Y_MAX_REL


def test_pivot_heads_load_dump_and_step(S):
    """FP16 pivot heads next to quantized heads: load = binary16 of the input (bit-exact),
    dump exact, and one step (GDN fp32, KDA bf16) within the pivot bar and the usual bars."""
    rng = np.random.default_rng(12)
    bits = [16, 4, 16, 8]
    n, H = 3, 4
    st = random_states(rng, n, H)
    ids = np.array([1, 4, 2], np.int32)
    op = O.OraclePool(5, bits, H)
    op.load_fp32(ids, st)
    gp = S.Pool(5, bits, H, S.STEPQ_GATE_GDN, S.STEPQ_DTYPE_F32)
    gp.load_fp32(slots_t(ids), dev(st))
    gb, ob = dump_bytes(gp, ids), op.slot_bytes(ids)
    off, _ = O.head_offsets(bits)
    for s_ in range(n):
        for h in (0, 2):
            assert np.array_equal(O.pivot_state(gb[s_, off[h]:off[h] + 32768]),
                                  st[s_, h].astype(np.float16).view(np.uint16))
    out = torch.empty((n, H, 128, 128), dtype=torch.float32, device="cuda")
    load_bytes(gp, ids, ob)
    gp.dump_fp32(slots_t(ids), out)
    assert np.array_equal(out.cpu().numpy(), op.dump_fp32(ids))
    for gate, dtype, Hk in ((0, S.STEPQ_DTYPE_F32, H), (1, S.STEPQ_DTYPE_BF16, 2)):
        op2 = O.OraclePool(5, bits, Hk, gate)
        op2.load_fp32(ids, st)
        x = dict(q=W.round_bf16(np.stack([[unit(rng, 128) for _ in range(Hk)] for _ in range(n)])),
                 k=W.round_bf16(np.stack([[unit(rng, 128) for _ in range(Hk)] for _ in range(n)])),
                 v=W.round_bf16(rng.standard_normal((n, H, 128)).astype(f32)),
                 alpha=W.round_bf16(rng.uniform(0.6, 1, (n, H) if gate == 0 else (n, H, 128)).astype(f32)),
                 beta=W.round_bf16(rng.uniform(0.1, 0.9, (n, H)).astype(f32)))
        yg, sg, err = _run_gpu(S, bits, Hk, gate, dtype, x, op2.slot_bytes(ids), ids, 5)
        yo = op2.decode_step(ids, x["q"], x["k"], x["v"], x["alpha"], x["beta"])
        assert err == 0
        res = PH.compare_slots(sg, op2.slot_bytes(ids), bits)
        assert PH.pivots_ok(res), (res["pivot_flips"], res["pivot_elements"], res["pivot_ulp"])
        assert res["max_code_diff"] <= 1 and res["r_ulp"] <= PH.R_ULP and res["c_ulp"] <= PH.C_ULP
        assert PH.y_max_rel(yg, yo) <= PH.Y_MAX_REL


def _unit_rows(rng, shape):
    x = rng.standard_normal(shape + (128,))
    return (x / np.linalg.norm(x, axis=-1, keepdims=True)).astype(f32)


def test_max_heads_vs_oracle(S):
    """The largest pool shape a call accepts in heads: H = 256 value heads (every width, FP16
    pivot heads among them) on 128 key heads; one step from random states, every state
    against the oracle."""
    rng = np.random.default_rng(21)
    H, Hk, n = 256, 128, 3
    bits = [(4, 6, 8, 16, 6, 4, 8, 6)[h % 8] for h in range(H)]
    st = random_states(rng, n, H, steps=4)
    ids = np.array([4, 0, 2], np.int32)
    op = O.OraclePool(5, bits, Hk)
    op.load_fp32(ids, st)
    x = dict(q=_unit_rows(rng, (n, Hk)), k=_unit_rows(rng, (n, Hk)),
             v=rng.standard_normal((n, H, 128)).astype(f32),
             alpha=rng.uniform(0.7, 1, (n, H)).astype(f32), beta=rng.uniform(0.1, 0.9, (n, H)).astype(f32))
    yg, sg, err = _run_gpu(S, bits, Hk, 0, S.STEPQ_DTYPE_F32, x, op.slot_bytes(ids), ids, 5)
    assert err == 0
    yo = op.decode_step(ids, x["q"], x["k"], x["v"], x["alpha"], x["beta"])
    res = PH.compare_slots(sg, op.slot_bytes(ids), bits)
    assert PH.pivots_ok(res), (res["pivot_flips"], res["pivot_elements"], res["pivot_ulp"])
    assert res["max_code_diff"] <= 1 and res["flips"] <= max(1, PH.CODE_FLIP_RATE * res["elements"])
    assert res["r_ulp"] <= PH.R_ULP and res["c_ulp"] <= PH.C_ULP
    assert PH.y_max_rel(yg, yo) <= PH.Y_MAX_REL


def test_max_requests_sampled_vs_oracle(S):
    """The largest request count a call accepts: n = 65535 requests on a 65535-slot pool
    (every slot, in a random order), one launch; the oracle follows the first and the last
    request, four in between (loaded with random states) and two that start from the zeroed
    pool.  A state stepped from zero is rank one, so every row of a column carries the same
    code and a column at a rounding tie puts 128 elements at that tie at once: the codes are
    checked element by element instead of by a flip rate -- each code equals the oracle's,
    or differs by one where the oracle's S / (r c) is at a tie."""
    rng = np.random.default_rng(22)
    n, H, Hk, bits = 65535, 2, 1, [4, 8]
    slot_ids = rng.permutation(n).astype(np.int32)
    loaded = np.array([0, 1, 20000, 40000, 65533, 65534])
    fresh = np.array([7, 50001])
    sample = np.concatenate([loaded, fresh])
    st = random_states(rng, len(loaded), H, steps=8)
    op = O.OraclePool(len(sample), bits, Hk)
    op.load_fp32(np.arange(len(loaded), dtype=np.int32), st)
    gp = S.Pool(n, bits, Hk, S.STEPQ_GATE_GDN, S.STEPQ_DTYPE_BF16)
    load_bytes(gp, slot_ids[loaded], op.slot_bytes(np.arange(len(loaded))))
    x = dict(q=_unit_rows(rng, (n, Hk)), k=_unit_rows(rng, (n, Hk)),
             v=rng.standard_normal((n, H, 128)).astype(f32),
             alpha=rng.uniform(0.7, 1, (n, H)).astype(f32), beta=rng.uniform(0.1, 0.9, (n, H)).astype(f32))
    x = {key: W.round_bf16(val) for key, val in x.items()}
    tx = {key: dev(W.to_bf16_bits(val).view(np.int16)) for key, val in x.items()}
    y = torch.empty((n, H, 128), device="cuda")
    gp.decode_step(slots_t(slot_ids), tx["q"], tx["k"], tx["v"], tx["alpha"], tx["beta"], y)
    assert gp.get_error() == 0
    before = op.slot_bytes(np.arange(len(sample)))
    xs = {key: x[key][sample] for key in ("q", "k", "v", "alpha", "beta")}
    yo = op.decode_step(np.arange(len(sample), dtype=np.int32), xs["q"], xs["k"], xs["v"], xs["alpha"], xs["beta"])
    sg = dump_bytes(gp, slot_ids[sample])
    res = PH.compare_slots(sg, op.slot_bytes(np.arange(len(sample))), bits)
    assert res["r_ulp"] <= PH.R_ULP and res["c_ulp"] <= PH.C_ULP
    off_tie, worst = PH.flips_off_tie(sg, before, bits, Hk, xs)
    assert worst <= 1 and off_tie == 0
    assert PH.y_max_rel(y[torch.from_numpy(sample).cuda()].cpu().numpy(), yo) <= PH.Y_MAX_REL


def _run_gpu(S, bits, Hk, gate, dtype, x, init_bytes, ids, num_slots):
    gp = S.Pool(num_slots, bits, Hk, gate, dtype)
    load_bytes(gp, ids, init_bytes)
    tx = {}
    for key, val in x.items():
        if dtype == S.STEPQ_DTYPE_BF16:
            tx[key] = dev(W.to_bf16_bits(val).view(np.int16))
        else:
            tx[key] = dev(val)
    y = torch.empty(x["v"].shape, device="cuda")
    gp.decode_step(slots_t(ids), tx["q"], tx["k"], tx["v"], tx["alpha"], tx["beta"], y)
    return y.cpu().numpy(), dump_bytes(gp, ids), gp.get_error()


@pytest.mark.parametrize("H,Hk,gate,n", [(8, 2, 0, 37), (16, 1, 1, 5), (32, 4, 0, 19)],
                         ids=["group4-gdn-n37", "group16-kda-n5", "group8-gdn-n19"])
def test_key_head_groups_vs_oracle(S, H, Hk, gate, n):
    """Value heads sharing one key head in groups of 4, 8 and 16 (consecutive grouping,
    g(h) = h / (H / Hk)), every width and an FP16 pivot head, a batch size that fills no
    whole number of CTA passes, one step against the oracle with the single-step bars."""
    rng = np.random.default_rng(100 + H + Hk)
    bits = [(4, 6, 8, 16, 6, 4, 8, 6)[h % 8] for h in range(H)]
    num_slots = n + 3
    ids = rng.permutation(num_slots)[:n].astype(np.int32)
    st = random_states(rng, n, H, steps=6)
    op = O.OraclePool(num_slots, bits, Hk, gate)
    op.load_fp32(ids, st)
    x = dict(q=_unit_rows(rng, (n, Hk)), k=_unit_rows(rng, (n, Hk)),
             v=rng.standard_normal((n, H, 128)).astype(f32),
             alpha=rng.uniform(0.7, 1, (n, H) if gate == 0 else (n, H, 128)).astype(f32),
             beta=rng.uniform(0.1, 0.9, (n, H)).astype(f32))
    yg, sg, err = _run_gpu(S, bits, Hk, gate, S.STEPQ_DTYPE_F32, x, op.slot_bytes(ids), ids, num_slots)
    assert err == 0
    yo = op.decode_step(ids, x["q"], x["k"], x["v"], x["alpha"], x["beta"])
    res = PH.compare_slots(sg, op.slot_bytes(ids), bits)
    assert PH.pivots_ok(res), (res["pivot_flips"], res["pivot_elements"], res["pivot_ulp"])
    assert res["max_code_diff"] <= 1 and res["flips"] <= max(1, PH.CODE_FLIP_RATE * res["elements"])
    assert res["r_ulp"] <= PH.R_ULP and res["c_ulp"] <= PH.C_ULP
    assert PH.y_max_rel(yg, yo) <= PH.Y_MAX_REL


@pytest.mark.parametrize("bits,Hk,gate,n,num_slots,dtype", [
    ([6], 1, 0, 1, 1, 0),                 # one request, one head, a one-slot pool
    ([8, 4], 1, 1, 1, 3, 1),              # one request, a key head shared by two heads, KDA, bf16
    ([8] * 6, 3, 0, 3, 7, 1),             # every head 8-bit
    ([4] * 5 + [16], 1, 1, 2, 2, 0),      # every quantized head 4-bit plus a pivot, full pool
], ids=["n1-h1-slots1", "n1-h2-kda-bf16", "all8bit", "all4bit-pivot-fullpool"])
def test_smallest_shapes_vs_oracle(S, bits, Hk, gate, n, num_slots, dtype):
    """The degenerate end of the shape range: one request, one head, a pool with a single
    slot, a pool whose slots are all active, and pools of a single width.  Far fewer items
    than resident CTAs, so most CTAs of the persistent grid have nothing to do.  Two steps
    against the oracle.  Codes are checked element by element: each equals the oracle's or
    differs by one where the oracle's S / (r c) is at a rounding tie.  A flip-rate bar does
    not fit a pool of 8-bit heads only: the window of near-ties grows with qmax, and fp32
    arithmetic against the fp64 oracle flips about 1.4e-5 of such codes, all at ties."""
    rng = np.random.default_rng(7 * n + len(bits) + 3 * gate)
    H = len(bits)
    ids = rng.permutation(num_slots)[:n].astype(np.int32)
    op = O.OraclePool(num_slots, bits, Hk, gate)
    op.load_fp32(ids, random_states(rng, n, H, steps=5))
    gp = S.Pool(num_slots, bits, Hk, gate, dtype)
    load_bytes(gp, ids, op.slot_bytes(ids))
    for step in range(2):
        x = dict(q=_unit_rows(rng, (n, Hk)), k=_unit_rows(rng, (n, Hk)),
                 v=rng.standard_normal((n, H, 128)).astype(f32),
                 alpha=rng.uniform(0.7, 1, (n, H) if gate == 0 else (n, H, 128)).astype(f32),
                 beta=rng.uniform(0.1, 0.9, (n, H)).astype(f32))
        if dtype == S.STEPQ_DTYPE_BF16:         # both sides take the bf16-rounded inputs
            x = {k_: W.round_bf16(v_) for k_, v_ in x.items()}
            tx = {k_: dev(W.to_bf16_bits(v_).view(np.int16)) for k_, v_ in x.items()}
        else:
            tx = {k_: dev(v_) for k_, v_ in x.items()}
        y = torch.empty((n, H, 128), device="cuda")
        gp.decode_step(slots_t(ids), tx["q"], tx["k"], tx["v"], tx["alpha"], tx["beta"], y)
        before = op.slot_bytes(ids)
        yo = op.decode_step(ids, x["q"], x["k"], x["v"], x["alpha"], x["beta"])
        sg = dump_bytes(gp, ids)
        res = PH.compare_slots(sg, op.slot_bytes(ids), bits)
        assert PH.pivots_ok(res), (step, res["pivot_flips"], res["pivot_elements"], res["pivot_ulp"])
        off_tie, worst = PH.flips_off_tie(sg, before, bits, Hk, x)
        assert worst <= 1 and off_tie == 0, (step, worst, off_tie, res["flips"])
        assert res["r_ulp"] <= PH.R_ULP and res["c_ulp"] <= PH.C_ULP, step
        assert PH.y_max_rel(y.cpu().numpy(), yo) <= PH.Y_MAX_REL, step
        load_bytes(gp, ids, op.slot_bytes(ids))  # the next step starts from identical states
    assert gp.get_error() == 0
    gp.close()


def test_kda_equal_gates_gqa_and_bf16_identities(S):
    """Bit identities on the GPU: KDA with equal per-channel gates = GDN; Hk = 2 with
    H = 4 = repeated key heads; bf16 inputs = the same values given as fp32."""
    rng = np.random.default_rng(6)
    bits = [4, 6, 8, 6]
    n, H = 3, 4
    op = O.OraclePool(4, bits, H)
    ids = np.array([3, 1, 0], np.int32)
    op.load_fp32(ids, random_states(rng, n, H))
    init = op.slot_bytes(ids)
    q2 = W.round_bf16(np.stack([[unit(rng, 128) for _ in range(2)] for _ in range(n)]))
    k2 = W.round_bf16(np.stack([[unit(rng, 128) for _ in range(2)] for _ in range(n)]))
    v = W.round_bf16(rng.standard_normal((n, H, 128)).astype(f32))
    a = W.round_bf16(rng.uniform(0.5, 1, (n, H)).astype(f32))
    b = W.round_bf16(rng.uniform(0, 1, (n, H)).astype(f32))
    base = dict(q=q2, k=k2, v=v, alpha=a, beta=b)
    y0, s0, e0 = _run_gpu(S, bits, 2, 0, S.STEPQ_DTYPE_F32, base, init, ids, 4)
    rep = dict(base, q=np.repeat(q2, 2, 1), k=np.repeat(k2, 2, 1))
    y1, s1, e1 = _run_gpu(S, bits, 4, 0, S.STEPQ_DTYPE_F32, rep, init, ids, 4)
    kda = dict(base, alpha=np.repeat(a[:, :, None], 128, 2))
    y2, s2, e2 = _run_gpu(S, bits, 2, 1, S.STEPQ_DTYPE_F32, kda, init, ids, 4)
    y3, s3, e3 = _run_gpu(S, bits, 2, 0, S.STEPQ_DTYPE_BF16, base, init, ids, 4)
    assert e0 == e1 == e2 == e3 == 0
    for yy, ss in ((y1, s1), (y2, s2), (y3, s3)):
        assert np.array_equal(yy, y0)
        assert np.array_equal(ss, s0)


def test_slot_permutation_invariance_and_bad_slot(S):
    """The same requests placed in other slots give bit-identical results; an
    out-of-range slot id raises the device flag, is skipped, and leaves the others intact."""
    rng = np.random.default_rng(7)
    bits = [6, 8]
    n, H = 4, 2
    states = random_states(rng, n, H)
    op = O.OraclePool(n, bits, H)
    op.load_fp32(np.arange(n, dtype=np.int32), states)
    per_req = op.slot_bytes(np.arange(n))
    x = dict(q=np.stack([[unit(rng, 128) for _ in range(H)] for _ in range(n)]),
             k=np.stack([[unit(rng, 128) for _ in range(H)] for _ in range(n)]),
             v=rng.standard_normal((n, H, 128)).astype(f32),
             alpha=rng.uniform(0.8, 1, (n, H)).astype(f32), beta=rng.uniform(0, 1, (n, H)).astype(f32))
    ya, sa, ea = _run_gpu(S, bits, H, 0, S.STEPQ_DTYPE_F32, x, per_req, np.array([0, 1, 2, 3], np.int32), 8)
    yb, sb, eb = _run_gpu(S, bits, H, 0, S.STEPQ_DTYPE_F32, x, per_req, np.array([6, 2, 7, 0], np.int32), 8)
    assert ea == eb == 0
    assert np.array_equal(ya, yb) and np.array_equal(sa, sb)
    # bad slot: request 2 points outside the pool
    gp = S.Pool(8, bits, H, S.STEPQ_GATE_GDN, S.STEPQ_DTYPE_F32)
    load_bytes(gp, [0, 1, 3], per_req[[0, 1, 3]])
    y = torch.full((n, H, 128), 7.0, device="cuda")
    tx = {k_: dev(v_) for k_, v_ in x.items()}
    gp.decode_step(slots_t([0, 1, 99, 3]), tx["q"], tx["k"], tx["v"], tx["alpha"], tx["beta"], y)
    assert gp.get_error() == S.STEPQ_FLAG_BAD_SLOT
    assert gp.get_error() == 0                        # reading clears the flag
    yh = y.cpu().numpy()
    assert np.array_equal(yh[[0, 1, 3]], ya[[0, 1, 3]])
    assert np.all(yh[2] == 7.0)                       # skipped request: y untouched
    assert np.array_equal(dump_bytes(gp, [0, 1, 3]), sa[[0, 1, 3]])


def test_zero_requests_and_invalid_arguments(S):
    gp = S.Pool(4, [4, 8], 1)
    empty = torch.empty(0, dtype=torch.int32, device="cuda")
    t = torch.zeros(16, device="cuda")
    gp.decode_step(empty, t, t, t, t, t, t)           # n = 0: no-op
    lib = S.load_library()
    assert lib.stepq_decode_step(gp.handle, None, 1, None, None, None, None, None, None, None) == -1
    assert lib.stepq_pool_load_fp32(gp.handle, slots_t([0]).data_ptr(), 1, None, None) == -1
    with pytest.raises(S.StepqError):
        S.stepq_pool_create(4, [4, 5], 1)             # unsupported width
    with pytest.raises(S.StepqError):
        S.stepq_pool_create(4, [4, 8], 3)             # key heads must divide value heads
    assert gp.get_error() == 0


@pytest.mark.parametrize("gate,dtype", [(0, 1), (1, 0)], ids=["gdn-bf16", "kda-fp32"])
def test_host_buffer_steps_match_device_steps(S, gate, dtype):
    """stepq_decode_step_host (slot ids, inputs and y in host memory; copy-in, step and
    copy-out of consecutive calls overlapped through two staging buffers) gives outputs and
    states bit-identical to stepq_decode_step on device buffers, call after call: six calls
    enqueued back to back on pinned buffers (three with separate arrays, three with one
    contiguous input image copied in one transfer), then one on pageable buffers, then a
    larger batch that regrows the staging buffers.  GDN with bf16 inputs and KDA (per-channel gate
    vectors in the staging buffer) with fp32 inputs."""
    rng = np.random.default_rng(5)
    bits, H, Hk, num_slots = [4, 6, 8, 6], 4, 2, 12
    ids_all = np.array([6, 1, 3, 0, 5, 9, 11, 2], np.int32)
    S0 = torch.from_numpy(random_states(rng, len(ids_all), H)).cuda()
    pools = [S.Pool(num_slots, bits, Hk, gate, dtype) for _ in range(2)]
    for gp in pools:
        gp.load_fp32(slots_t(ids_all), S0)

    def inputs(n):
        ashape = (n, H, 128) if gate == S.STEPQ_GATE_KDA else (n, H)
        x = dict(q=np.stack([[unit(rng, 128) for _ in range(Hk)] for _ in range(n)]),
                 k=np.stack([[unit(rng, 128) for _ in range(Hk)] for _ in range(n)]),
                 v=rng.standard_normal((n, H, 128)).astype(f32),
                 alpha=rng.uniform(0.8, 1, ashape).astype(f32), beta=rng.uniform(0, 1, (n, H)).astype(f32))
        if dtype == S.STEPQ_DTYPE_F32:
            return {key: torch.from_numpy(val) for key, val in x.items()}
        return {key: torch.from_numpy(W.to_bf16_bits(val).view(np.int16)) for key, val in x.items()}

    # "pinned": six pinned arrays; "image": one pinned image at the offsets of
    # stepq_host_image_layout (one copy-in); "pageable": ordinary host memory
    plan = [(5, "pinned")] * 3 + [(5, "image")] * 3 + [(5, "pageable"), (8, "image")]
    steps = [(ids_all[:n], inputs(n), mode) for n, mode in plan]
    y_dev = []
    for ids, x, _ in steps:
        y = torch.empty((len(ids), H, 128), device="cuda")
        pools[0].decode_step(slots_t(ids), *[x[key].cuda() for key in ("q", "k", "v", "alpha", "beta")], y)
        y_dev.append(y.cpu().numpy())
    y_host = []
    for ids, x, mode in steps:
        hs = torch.from_numpy(ids.copy())
        yh = torch.full((len(ids), H, 128), float("nan"))
        if mode == "image":
            offs, total = pools[1].host_image_layout(len(ids))
            img = torch.zeros(total, dtype=torch.uint8).pin_memory()
            hx = {}
            for name, o, t in zip(("slots", "q", "k", "v", "alpha", "beta"), offs,
                                  [hs] + [x[key] for key in ("q", "k", "v", "alpha", "beta")]):
                nb = t.numel() * t.element_size()
                img[o:o + nb].copy_(t.reshape(-1).view(torch.uint8))
                hx[name] = img[o:o + nb].view(t.dtype)
            hs = hx.pop("slots")
            hx["image"] = img
            yh = yh.pin_memory()
        else:
            pinned = mode == "pinned"
            hx = {key: (val.pin_memory() if pinned else val.clone()) for key, val in x.items()}
            if pinned:
                hs, yh = hs.pin_memory(), yh.pin_memory()
        pools[1].decode_step_host(hs, hx["q"], hx["k"], hx["v"], hx["alpha"], hx["beta"], yh)
        y_host.append((yh, hx, hs))                 # keep the host buffers alive until the wait
    pools[1].host_wait()
    torch.cuda.synchronize()
    for t, (yd, (yh, _, _)) in enumerate(zip(y_dev, y_host)):
        assert np.array_equal(yd, yh.numpy()), "call %d" % t
    assert np.array_equal(dump_bytes(pools[0], ids_all), dump_bytes(pools[1], ids_all))
    assert pools[0].get_error() == 0 and pools[1].get_error() == 0


def test_bounded_wait_timeout_reports_and_context_survives(S):
    """The kernels' failure path: a bounded wait on a barrier that nothing completes gives up,
    raises the timeout flag for the host, and the context keeps working (a decode step right
    after it matches the same step on a fresh pool)."""
    rng = np.random.default_rng(11)
    bits, n, H = [4, 8], 3, 2
    states = random_states(rng, n, H)
    op = O.OraclePool(n, bits, H)
    op.load_fp32(np.arange(n, dtype=np.int32), states)
    per_req = op.slot_bytes(np.arange(n))
    x = dict(q=np.stack([[unit(rng, 128) for _ in range(H)] for _ in range(n)]),
             k=np.stack([[unit(rng, 128) for _ in range(H)] for _ in range(n)]),
             v=rng.standard_normal((n, H, 128)).astype(f32),
             alpha=rng.uniform(0.8, 1, (n, H)).astype(f32), beta=rng.uniform(0, 1, (n, H)).astype(f32))
    ids = np.arange(n, dtype=np.int32)
    y0, s0, e0 = _run_gpu(S, bits, H, 0, S.STEPQ_DTYPE_F32, x, per_req, ids, n)
    for _ in range(2):
        assert S.stepq_check_wait_timeout() == S.STEPQ_FLAG_TIMEOUT
    torch.cuda.synchronize()
    y1, s1, e1 = _run_gpu(S, bits, H, 0, S.STEPQ_DTYPE_F32, x, per_req, ids, n)
    assert e0 == e1 == 0
    assert np.array_equal(y0, y1) and np.array_equal(s0, s1)


# --------------------------------------------------------------------------- workload parity

CASES = [
    # (config, variant, batch, layer, sampled requests, steps compared)
    (1, "mixed6", None, 0, 4, 16),
    (2, "mixed6", None, 0, 8, 64),
    (3, "mixed6", None, 0, 6, 64),
    (4, "mixed6", None, 0, 6, 64),
    (4, "uniform4", None, 0, 6, 32),
    (4, "mixed6p", None, 0, 6, 32),
    (3, "mixed6p", None, 0, 4, 32),
    (2, "mixed6p", None, 0, 6, 32),
    (3, "rowbits", None, 0, 4, 32),
    (5, "mixed6", 64, 17, 3, 32),
    (5, "mixed6", 256, 17, 3, 32),
    (5, "mixed6", 1024, 0, 3, 32),
    (5, "mixed6", 1024, 35, 3, 32),
]


@pytest.mark.parametrize("config,variant,batch,layer,nsample,steps", CASES,
                         ids=["cfg%d-%s-b%s-l%d" % (c[0], c[1], c[2], c[3]) for c in CASES])
def test_trajectory_parity(S, config, variant, batch, layer, nsample, steps):
    """Full batch on the GPU (the launch configuration of the benchmark); the oracle
    follows a seeded sample of requests.  Every step: single-step tolerances (codes +-1
    at rate <= 1e-5, r/c ulps, y max-rel <= 1e-4).  Whole trajectory: y relative L2 <= 1e-3.
    A state whose codes came out +-1 from the oracle's is re-synchronised from the
    oracle's bytes before the next step (oracle -> GPU only): a single such flip is
    amplified by the recurrence itself, so free-running trajectories are not comparable."""
    w = W.make_workload(config, variant, batch)
    bits = PH.head_bits(w, layer)
    sub = W.sample_requests(w, nsample)
    sub_slots = w.slot_ids[sub]
    op = PH.oracle_pool_with_warmup(w, bits, sub, layer)
    rb = PH.row_bits(w, layer)
    gp = S.Pool(w.num_slots, bits, w.Hk, w.gate_mode, w.in_dtype, row_bits=rb)
    load_bytes(gp, sub_slots, op.slot_bytes(sub_slots))
    all_slots = slots_t(w.slot_ids)
    num = den = 0.0
    flips = elements = resyncs = 0
    pflips = pelements = 0
    worst = dict(max_code_diff=0, r_ulp=0, c_ulp=0, y=0.0, pivot_ulp=0)
    for t in range(steps):
        x = W.step_inputs(w, t, W.PHASE_RUN, layer)
        tx = PH.to_device(w, x, torch)
        y = torch.empty((w.B, w.H, w.dv), device="cuda")
        gp.decode_step(all_slots, tx["q"], tx["k"], tx["v"], tx["alpha"], tx["beta"], y)
        xs = PH.sub_inputs(x, sub)
        yo = op.decode_step(sub_slots, xs["q"], xs["k"], xs["v"], xs["alpha"], xs["beta"])
        yg = y[torch.from_numpy(sub).cuda()].cpu().numpy()
        num += float(np.sum((yg.astype(np.float64) - yo) ** 2))
        den += float(np.sum(yo.astype(np.float64) ** 2))
        worst["y"] = max(worst["y"], PH.y_max_rel(yg, yo))
        gb, ob = dump_bytes(gp, sub_slots), op.slot_bytes(sub_slots)
        res = PH.compare_slots(gb, ob, bits, row_bits=rb)
        flips += res["flips"]
        elements += res["elements"]
        pflips += res["pivot_flips"]
        pelements += res["pivot_elements"]
        for key in ("max_code_diff", "r_ulp", "c_ulp", "pivot_ulp"):
            worst[key] = max(worst[key], res[key])
        if not res["byte_equal"]:
            load_bytes(gp, sub_slots, ob)
            resyncs += 1
    assert gp.get_error() == 0
    rel = np.sqrt(num / den)
    print("\n%s: y rel L2 %.3e, worst %s, flips %d / %d (%.2e), pivot flips %d / %d, resyncs %d" %
          (w.name, rel, worst, flips, elements, flips / elements, pflips, pelements, resyncs))
    assert worst["pivot_ulp"] <= PH.PIVOT_ULP
    assert pflips <= max(1, PH.PIVOT_FLIP_RATE * pelements)
    assert worst["max_code_diff"] <= 1
    assert flips <= PH.CODE_FLIP_RATE * elements
    assert worst["r_ulp"] <= PH.R_ULP and worst["c_ulp"] <= PH.C_ULP
    assert worst["y"] <= PH.Y_MAX_REL
    assert rel <= PH.Y_TRAJ_REL_L2


# Free-running trajectories.  The per-step leg above re-synchronises a state whose codes came
# out one level apart, so it checks each step from identical stored states.  Here nothing is
# re-synchronised: the GPU runs the whole batch for the workload's full T, the oracle follows a
# sample of requests with its own quantized state, and both are compared with the oracle's
# unquantized (FP32-state) trajectory from the same starting state.  By the error recursion
# of "Paper Explained: STEPQuant", "The intuition: errors get carried forward"
# (E_t = A_t E_{t-1} + eps_t), the quantization error a trajectory accumulates is a property
# of the quantizer, not of where the roundings fall; a GPU path that quantizes like the
# oracle accumulates an error of the same size.  Bar: ||y_gpu - y_fp|| / ||y_oracle - y_fp||
# in [FREE_BAND_LO, FREE_BAND_HI] over the sampled requests and all T steps (two correct
# implementations of one quantizer land within a fraction of a percent of each other here).
FREE_BAND_LO, FREE_BAND_HI = 0.95, 1.05

FREE_CASES = [
    # (config, variant, batch, layer, sampled requests)
    (1, "mixed6", None, 0, 4),
    (2, "mixed6", None, 0, 8),
    (3, "mixed6", None, 0, 6),
    (4, "mixed6", None, 0, 6),
    (4, "uniform4", None, 0, 6),
    (4, "mixed6p", None, 0, 6),
    (3, "mixed6p", None, 0, 4),
    (2, "mixed6p", None, 0, 6),
    (3, "rowbits", None, 0, 4),
    (5, "mixed6", 64, 17, 3),
    (5, "mixed6", 1024, 35, 3),
]


@pytest.mark.parametrize("config,variant,batch,layer,nsample", FREE_CASES,
                         ids=["cfg%d-%s-b%s-l%d" % (c[0], c[1], c[2], c[3]) for c in FREE_CASES])
def test_free_running_trajectory(S, config, variant, batch, layer, nsample):
    w = W.make_workload(config, variant, batch)
    bits = PH.head_bits(w, layer)
    sub = W.sample_requests(w, nsample)
    sub_slots = w.slot_ids[sub]
    op = PH.oracle_pool_with_warmup(w, bits, sub, layer)
    rb = PH.row_bits(w, layer)
    gp = S.Pool(w.num_slots, bits, w.Hk, w.gate_mode, w.in_dtype, row_bits=rb)
    load_bytes(gp, sub_slots, op.slot_bytes(sub_slots))
    # the unquantized run starts from the same (dequantized) state
    S_fp = op.dump_fp32(sub_slots).astype(np.float64)
    all_slots = slots_t(w.slot_ids)
    sub_t = torch.from_numpy(sub).cuda()
    d_gpu = d_ora = d_go = n_ora = n_fp = 0.0
    for t in range(w.T):
        x = W.step_inputs(w, t, W.PHASE_RUN, layer)
        tx = PH.to_device(w, x, torch)
        y = torch.empty((w.B, w.H, w.dv), device="cuda")
        gp.decode_step(all_slots, tx["q"], tx["k"], tx["v"], tx["alpha"], tx["beta"], y)
        xs = PH.sub_inputs(x, sub)
        yo = op.decode_step(sub_slots, xs["q"], xs["k"], xs["v"], xs["alpha"], xs["beta"]).astype(np.float64)
        yf = O.fp_decode_step(S_fp, w.Hk, w.gate_mode, xs["q"], xs["k"], xs["v"], xs["alpha"], xs["beta"],
                              round_fp32=True).astype(np.float64)
        yg = y[sub_t].cpu().numpy().astype(np.float64)
        d_gpu += float(np.sum((yg - yf) ** 2))
        d_ora += float(np.sum((yo - yf) ** 2))
        d_go += float(np.sum((yg - yo) ** 2))
        n_ora += float(np.sum(yo ** 2))
        n_fp += float(np.sum(yf ** 2))
    assert gp.get_error() == 0
    ratio = np.sqrt(d_gpu / d_ora)
    print("\n%s free-running T=%d: quantization error vs FP32 state: gpu %.3e, oracle %.3e (ratio %.4f); "
          "gpu vs oracle y rel L2 %.3e" % (w.name, w.T, np.sqrt(d_gpu / n_fp), np.sqrt(d_ora / n_fp), ratio,
                                          np.sqrt(d_go / n_ora)))
    assert FREE_BAND_LO <= ratio <= FREE_BAND_HI


# --------------------------------------------------------------------------- checkpoint and debug mode

def test_checkpoint_restore_continues_bit_identically(S):
    """Dump a pool's packed slots after a few steps, restore them into a fresh pool with
    load_packed, and continue both pools with the same inputs: y and the packed states stay
    bit-identical (the pool layout is the whole state of a request)."""
    w = W.make_workload(4, "mixed6p")
    bits = PH.head_bits(w)
    n = 64
    ids = w.slot_ids[:n]
    rng = np.random.default_rng(404)
    S0 = random_states(rng, n, w.H, steps=16)
    a = S.Pool(w.num_slots, bits, w.Hk, w.gate_mode, w.in_dtype)
    a.load_fp32(slots_t(ids), dev(S0))
    xs = []
    for t in range(12):
        x = PH.sub_inputs(W.step_inputs(w, t), np.arange(n))
        xs.append(PH.to_device(w, x, torch))
    y = torch.empty((n, w.H, w.dv), device="cuda")
    for t in range(4):
        a.decode_step(slots_t(ids), xs[t]["q"], xs[t]["k"], xs[t]["v"], xs[t]["alpha"], xs[t]["beta"], y)
    ckpt = dump_bytes(a, ids)
    b = S.Pool(w.num_slots, bits, w.Hk, w.gate_mode, w.in_dtype)
    load_bytes(b, ids, ckpt)
    ya = torch.empty_like(y)
    yb = torch.empty_like(y)
    for t in range(4, 12):
        a.decode_step(slots_t(ids), xs[t]["q"], xs[t]["k"], xs[t]["v"], xs[t]["alpha"], xs[t]["beta"], ya)
        b.decode_step(slots_t(ids), xs[t]["q"], xs[t]["k"], xs[t]["v"], xs[t]["alpha"], xs[t]["beta"], yb)
        torch.cuda.synchronize()
        assert torch.equal(ya, yb)
    assert np.array_equal(dump_bytes(a, ids), dump_bytes(b, ids))
    assert a.get_error() == 0 and b.get_error() == 0
    a.close()
    b.close()


@pytest.mark.parametrize("variant,fit", [("mixed6", "clipfree"), ("mixed6p", "clipfree"), ("mixed6", "impact")])
def test_graph_replay_matches_eager_steps(S, variant, fit):
    """The launch configuration the benchmark times: config-4 decode steps (512 requests on a
    1024-slot pool) captured as one CUDA graph on a side stream, programmatic dependent
    launches between the steps, the FP16 pivot heads' kernel on the pool's forked stream
    (mixed6p), and the impact-weighted fit.  Replays of the graph must give the eager launches'
    y and packed states bit for bit (the kernels are deterministic), so the oracle parity of
    the eager path carries over to the timed path."""
    w = W.make_workload(4, variant)
    bits = PH.head_bits(w)
    ids = slots_t(w.slot_ids)
    a = S.Pool(w.num_slots, bits, w.Hk, w.gate_mode, w.in_dtype)
    b = S.Pool(w.num_slots, bits, w.Hk, w.gate_mode, w.in_dtype)
    if fit == "impact":
        scores = _impact_scores(np.random.default_rng(91), w.H)
        a.set_impact(scores)
        b.set_impact(scores)
    xs = [PH.to_device(w, W.step_inputs(w, t), torch) for t in range(12)]
    nstep = 4
    ya = torch.empty((nstep, w.B, w.H, w.dv), device="cuda")
    yb = torch.empty_like(ya)

    def steps(pool, y, first):
        for t in range(nstep):
            x = xs[first + t]
            pool.decode_step(ids, x["q"], x["k"], x["v"], x["alpha"], x["beta"], y[t])

    # both pools leave the zero state through the same eager steps (deterministic: identical)
    steps(a, ya, 0)
    steps(b, yb, 0)
    torch.cuda.synchronize()
    assert torch.equal(ya, yb)
    graph = torch.cuda.CUDAGraph()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        with torch.cuda.graph(graph, stream=side):
            steps(a, ya, 4)
    torch.cuda.current_stream().wait_stream(side)
    for rep in range(2):
        graph.replay()
        steps(b, yb, 4)
        torch.cuda.synchronize()
        assert torch.equal(ya, yb), rep
        assert np.array_equal(dump_bytes(a, w.slot_ids), dump_bytes(b, w.slot_ids)), rep
    assert a.get_error() == 0 and b.get_error() == 0
    del graph
    a.close()
    b.close()


def test_debug_mode_rejects_duplicate_slot_ids(S):
    """With STEPQ_DEBUG_SLOTS a step with a repeated or out-of-range slot id is refused before
    any device work (the states stay as they were); distinct ids give the same step as
    without the debug mode."""
    bits = np.array([4, 6, 8, 16], np.int32)
    rng = np.random.default_rng(5)
    n, H, Hk = 4, 4, 2
    S0 = random_states(rng, n, H)
    ids = np.array([5, 1, 6, 2], np.int32)
    pools = [S.Pool(8, bits, Hk, 0, 0) for _ in range(2)]
    for p in pools:
        p.load_fp32(slots_t(ids), dev(S0))
    pools[1].set_debug(S.STEPQ_DEBUG_SLOTS)
    x = dict(q=np.stack([[unit(rng, 128) for _ in range(Hk)] for _ in range(n)]),
             k=np.stack([[unit(rng, 128) for _ in range(Hk)] for _ in range(n)]),
             v=rng.standard_normal((n, H, 128)).astype(f32), alpha=np.full((n, H), 0.9, f32),
             beta=np.full((n, H), 0.5, f32))
    tx = {k_: dev(v_) for k_, v_ in x.items()}
    y = torch.zeros((n, H, 128), device="cuda")
    before = dump_bytes(pools[1], ids)
    for bad in ([5, 1, 5, 2], [5, 1, 8, 2], [5, -1, 6, 2]):
        with pytest.raises(S.StepqError) as err:
            pools[1].decode_step(slots_t(bad), tx["q"], tx["k"], tx["v"], tx["alpha"], tx["beta"], y)
        assert err.value.status == -1
    assert np.array_equal(dump_bytes(pools[1], ids), before)
    assert float(y.abs().max()) == 0.0
    ys = []
    for p in pools:
        yp = torch.empty((n, H, 128), device="cuda")
        p.decode_step(slots_t(ids), tx["q"], tx["k"], tx["v"], tx["alpha"], tx["beta"], yp)
        torch.cuda.synchronize()
        ys.append(yp.cpu().numpy())
    assert np.array_equal(ys[0], ys[1])
    assert np.array_equal(dump_bytes(pools[0], ids), dump_bytes(pools[1], ids))
    for p in pools:
        assert p.get_error() == 0
        p.close()


# --------------------------------------------------------------------------- impact-weighted fit

def _impact_scores(rng, H):
    """Synthetic row-impact scores (positive, spread over two decades, as calibration gives)."""
    return np.exp(rng.normal(0, 1.2, (H, 128))).astype(f32)


def test_impact_fit_load_and_step_vs_oracle(S):
    """Pool with row-impact scores: quantize-in and one decode step (GDN fp32, KDA bf16)
    against the oracle's impact-weighted fit: r within 8 ulp, c within 2e-5, codes +-1 at a
    rate <= 1e-3, y as always."""
    rng = np.random.default_rng(13)
    bits = [4, 6, 8, 6]
    n, H = 3, 4
    omega = _impact_scores(rng, H)
    st = random_states(rng, n, H)
    ids = np.array([2, 0, 1], np.int32)
    op = O.OraclePool(3, bits, H, impact=omega)
    op.load_fp32(ids, st)
    gp = S.Pool(3, bits, H, S.STEPQ_GATE_GDN, S.STEPQ_DTYPE_F32)
    gp.set_impact(omega)
    gp.load_fp32(slots_t(ids), dev(st))
    res = PH.compare_slots(dump_bytes(gp, ids), op.slot_bytes(ids), bits)
    assert res["max_code_diff"] <= 1 and res["r_ulp"] <= PH.R_ULP
    assert PH.impact_scales_ok(res), res
    assert res["flips_near"] <= max(1, PH.CODE_FLIP_RATE_IMPACT * res["elements"]), res
    for gate, dtype, Hk in ((0, S.STEPQ_DTYPE_F32, H), (1, S.STEPQ_DTYPE_BF16, 2)):
        op2 = O.OraclePool(3, bits, Hk, gate, impact=omega)
        op2.load_fp32(ids, st)
        x = dict(q=W.round_bf16(np.stack([[unit(rng, 128) for _ in range(Hk)] for _ in range(n)])),
                 k=W.round_bf16(np.stack([[unit(rng, 128) for _ in range(Hk)] for _ in range(n)])),
                 v=W.round_bf16(rng.standard_normal((n, H, 128)).astype(f32)),
                 alpha=W.round_bf16(rng.uniform(0.6, 1, (n, H) if gate == 0 else (n, H, 128)).astype(f32)),
                 beta=W.round_bf16(rng.uniform(0.1, 0.9, (n, H)).astype(f32)))
        gp2 = S.Pool(3, bits, Hk, gate, dtype)
        gp2.set_impact(omega)
        load_bytes(gp2, ids, op2.slot_bytes(ids))
        tx = {}
        for key, val in x.items():
            tx[key] = dev(W.to_bf16_bits(val).view(np.int16)) if dtype == S.STEPQ_DTYPE_BF16 else dev(val)
        y = torch.empty((n, H, 128), device="cuda")
        gp2.decode_step(slots_t(ids), tx["q"], tx["k"], tx["v"], tx["alpha"], tx["beta"], y)
        yo = op2.decode_step(ids, x["q"], x["k"], x["v"], x["alpha"], x["beta"])
        assert gp2.get_error() == 0
        res = PH.compare_slots(dump_bytes(gp2, ids), op2.slot_bytes(ids), bits)
        assert res["max_code_diff"] <= 1 and res["r_ulp"] <= PH.R_ULP, res
        assert PH.impact_scales_ok(res), res
        assert res["flips_near"] <= max(1, PH.CODE_FLIP_RATE_IMPACT * res["elements"]), res
        assert PH.y_max_rel(y.cpu().numpy(), yo) <= PH.Y_MAX_REL


def test_impact_fit_trajectory_config4(S):
    """Config-4 pool with synthetic row-impact scores, full batch on the GPU, a sampled
    trajectory on the oracle (re-synchronised after a code difference, as for the clip-free
    fit); unit scores select the impact fit too, and clearing them returns to the clip-free fit."""
    w = W.make_workload(4, "mixed6")
    bits = PH.head_bits(w)
    rng = np.random.default_rng(14)
    omega = _impact_scores(rng, w.H)
    sub = W.sample_requests(w, 4)
    sub_slots = w.slot_ids[sub]
    op = PH.oracle_pool_with_warmup(w, bits, sub)
    op_imp = O.OraclePool(w.num_slots, bits, w.Hk, w.gate_mode, impact=omega)
    op_imp.data[:] = op.data
    gp = S.Pool(w.num_slots, bits, w.Hk, w.gate_mode, w.in_dtype)
    gp.set_impact(omega)
    load_bytes(gp, sub_slots, op_imp.slot_bytes(sub_slots))
    all_slots = slots_t(w.slot_ids)
    flips = elements = c_far = c_cols = 0
    worst = dict(r_ulp=0, c_rel=0.0, y=0.0)
    for t in range(24):
        x = W.step_inputs(w, t)
        tx = PH.to_device(w, x, torch)
        y = torch.empty((w.B, w.H, w.dv), device="cuda")
        gp.decode_step(all_slots, tx["q"], tx["k"], tx["v"], tx["alpha"], tx["beta"], y)
        xs = PH.sub_inputs(x, sub)
        yo = op_imp.decode_step(sub_slots, xs["q"], xs["k"], xs["v"], xs["alpha"], xs["beta"])
        yg = y[torch.from_numpy(sub).cuda()].cpu().numpy()
        worst["y"] = max(worst["y"], PH.y_max_rel(yg, yo))
        gb, ob = dump_bytes(gp, sub_slots), op_imp.slot_bytes(sub_slots)
        res = PH.compare_slots(gb, ob, bits)
        assert res["max_code_diff"] <= 1 and res.get("zero_c_mismatch", 0) == 0
        flips += res["flips"]
        elements += res["elements"]
        c_far += res.get("c_far", 0)
        c_cols += res.get("c_cols", 0)
        worst["r_ulp"] = max(worst["r_ulp"], res["r_ulp"])
        worst["c_rel"] = max(worst["c_rel"], res.get("c_rel", 0.0))
        if not res["byte_equal"]:
            load_bytes(gp, sub_slots, ob)
    print("\nimpact fit: worst %s, flips %d / %d (%.2e), columns with c off > 2e-5: %d / %d" %
          (worst, flips, elements, flips / elements, c_far, c_cols))
    assert gp.get_error() == 0
    assert worst["r_ulp"] <= PH.R_ULP and worst["y"] <= PH.Y_MAX_REL
    assert c_far <= max(1, PH.C_FAR_RATE_IMPACT * c_cols)
    assert flips <= PH.CODE_FLIP_RATE_IMPACT * elements
    # clearing the scores returns to the clip-free fit
    gp.set_impact(None)
    load_bytes(gp, sub_slots, op.slot_bytes(sub_slots))
    x = W.step_inputs(w, 0)
    tx = PH.to_device(w, x, torch)
    y = torch.empty((w.B, w.H, w.dv), device="cuda")
    gp.decode_step(all_slots, tx["q"], tx["k"], tx["v"], tx["alpha"], tx["beta"], y)
    xs = PH.sub_inputs(x, sub)
    op.decode_step(sub_slots, xs["q"], xs["k"], xs["v"], xs["alpha"], xs["beta"])
    res = PH.compare_slots(dump_bytes(gp, sub_slots), op.slot_bytes(sub_slots), bits)
    assert res["max_code_diff"] <= 1 and res["c_ulp"] <= PH.C_ULP


# --------------------------------------------------------------------------- per-key-row widths

def test_rowbits_heads_load_dump_and_step(S):
    """Heads with per-key-row widths next to uniform heads: quantize-in, exact dump, and one
    KDA bf16 step against the oracle (the usual single-step bars)."""
    rng = np.random.default_rng(15)
    H = 4
    bits = [0, 8, 0, 4]
    rb = np.stack([rng.choice([4, 6, 8], 128, p=[0.45, 0.35, 0.2]) for _ in range(H)]).astype(np.int32)
    rb[2, :] = 4
    rb[2, 3] = 6                                    # one 6-bit row among 4-bit rows
    n = 3
    st = random_states(rng, n, H)
    ids = np.array([1, 3, 0], np.int32)
    op = O.OraclePool(4, bits, 2, 1, row_bits=rb)
    op.load_fp32(ids, st)
    gp = S.Pool(4, bits, 2, S.STEPQ_GATE_KDA, S.STEPQ_DTYPE_BF16, row_bits=rb)
    assert gp.slot_stride == op.slot_stride
    gp.load_fp32(slots_t(ids), dev(st))
    res = PH.compare_slots(dump_bytes(gp, ids), op.slot_bytes(ids), bits, row_bits=rb)
    assert res["max_code_diff"] <= 1 and res["c_ulp"] == 0 and res["r_ulp"] <= PH.R_ULP, res
    load_bytes(gp, ids, op.slot_bytes(ids))
    out = torch.empty((n, H, 128, 128), dtype=torch.float32, device="cuda")
    gp.dump_fp32(slots_t(ids), out)
    assert np.array_equal(out.cpu().numpy(), op.dump_fp32(ids))
    x = dict(q=W.round_bf16(np.stack([[unit(rng, 128) for _ in range(2)] for _ in range(n)])),
             k=W.round_bf16(np.stack([[unit(rng, 128) for _ in range(2)] for _ in range(n)])),
             v=W.round_bf16(rng.standard_normal((n, H, 128)).astype(f32)),
             alpha=W.round_bf16(rng.uniform(0.6, 1, (n, H, 128)).astype(f32)),
             beta=W.round_bf16(rng.uniform(0.1, 0.9, (n, H)).astype(f32)))
    tx = {k_: dev(W.to_bf16_bits(v_).view(np.int16)) for k_, v_ in x.items()}
    y = torch.empty((n, H, 128), device="cuda")
    gp.decode_step(slots_t(ids), tx["q"], tx["k"], tx["v"], tx["alpha"], tx["beta"], y)
    yo = op.decode_step(ids, x["q"], x["k"], x["v"], x["alpha"], x["beta"])
    assert gp.get_error() == 0
    res = PH.compare_slots(dump_bytes(gp, ids), op.slot_bytes(ids), bits, row_bits=rb)
    assert res["max_code_diff"] <= 1 and res["r_ulp"] <= PH.R_ULP and res["c_ulp"] <= PH.C_ULP, res
    assert res["flips"] <= max(1, PH.CODE_FLIP_RATE * res["elements"])
    assert PH.y_max_rel(y.cpu().numpy(), yo) <= PH.Y_MAX_REL


def test_rowbits_and_impact_fit_in_one_pool(S):
    """A pool with per-key-row heads next to uniform heads and row-impact scores set: the
    uniform heads take the impact-weighted fit, the per-row heads keep the clip-free fit at
    each row's levels (both fit options in one kernel).  One KDA bf16 step against the oracle:
    the impact bars on the uniform heads, the single-step bars on the per-row heads."""
    rng = np.random.default_rng(16)
    H, n = 4, 3
    bits = [0, 8, 0, 6]
    rb = np.stack([rng.choice([4, 6, 8], 128, p=[0.4, 0.4, 0.2]) for _ in range(H)]).astype(np.int32)
    omega = _impact_scores(rng, H)
    st = random_states(rng, n, H)
    ids = np.array([2, 0, 3], np.int32)
    op = O.OraclePool(4, bits, 2, 1, row_bits=rb, impact=omega)
    op.load_fp32(ids, st)
    gp = S.Pool(4, bits, 2, S.STEPQ_GATE_KDA, S.STEPQ_DTYPE_BF16, row_bits=rb)
    gp.set_impact(omega)
    load_bytes(gp, ids, op.slot_bytes(ids))
    x = dict(q=W.round_bf16(np.stack([[unit(rng, 128) for _ in range(2)] for _ in range(n)])),
             k=W.round_bf16(np.stack([[unit(rng, 128) for _ in range(2)] for _ in range(n)])),
             v=W.round_bf16(rng.standard_normal((n, H, 128)).astype(f32)),
             alpha=W.round_bf16(rng.uniform(0.6, 1, (n, H, 128)).astype(f32)),
             beta=W.round_bf16(rng.uniform(0.1, 0.9, (n, H)).astype(f32)))
    tx = {k_: dev(W.to_bf16_bits(v_).view(np.int16)) for k_, v_ in x.items()}
    y = torch.empty((n, H, 128), device="cuda")
    gp.decode_step(slots_t(ids), tx["q"], tx["k"], tx["v"], tx["alpha"], tx["beta"], y)
    yo = op.decode_step(ids, x["q"], x["k"], x["v"], x["alpha"], x["beta"])
    assert gp.get_error() == 0
    gb, ob = dump_bytes(gp, ids), op.slot_bytes(ids)
    offs, _ = O.head_offsets(bits, row_bits=rb)
    for h, b in enumerate(bits):                       # one head block at a time
        sl = slice(int(offs[h]), int(offs[h]) + (O.block_bytes(b) if b else O.rows_block_bytes(rb[h])))
        res = PH.compare_slots(gb[:, sl], ob[:, sl], [b], row_bits=rb[h:h + 1])
        assert res["max_code_diff"] <= 1 and res["r_ulp"] <= PH.R_ULP, (h, res)
        if b:
            assert PH.impact_scales_ok(res), (h, res)
            assert res["flips_near"] <= max(1, PH.CODE_FLIP_RATE_IMPACT * res["elements"]), (h, res)
        else:
            assert res["c_ulp"] <= PH.C_ULP, (h, res)
            assert res["flips"] <= max(1, PH.CODE_FLIP_RATE * res["elements"]), (h, res)
    assert PH.y_max_rel(y.cpu().numpy(), yo) <= PH.Y_MAX_REL
    gp.close()
