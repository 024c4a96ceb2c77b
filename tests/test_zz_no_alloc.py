"""The allocation-free decode entry point (stepq_decode_step_noalloc).

Some callers cannot allocate device memory: a serving engine or framework that hands out
all device memory from its own arena or caching allocator, or code embedded where new
allocations are not allowed.  They hold the packed state buffer themselves and call this
entry point, whose scratch is a fixed device array inside the library.  Here it must give
the same results as the pool-based stepq_decode_step on two calls in a row.

This file is collected last on purpose (its scratch is shared library state); it must pass
on its own in a fresh process and after every other test.
"""
import numpy as np
import pytest

from oracle import oracle as O
from quantized_gated_delta_b200 import workloads as W
from tests import parity_helpers as PH

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


def dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def unit(rng, shape):
    x = rng.standard_normal(shape)
    return (x / np.linalg.norm(x, axis=-1, keepdims=True)).astype(np.float32)


@pytest.mark.parametrize("gate_mode,in_dtype", [(0, 1), (1, 0)])
def test_noalloc_matches_pool_entry_point(gate_mode, in_dtype):
    from quantized_gated_delta_b200 import stepq as S
    rng = np.random.default_rng(77 + gate_mode)
    bits = np.array([6, 4, 8, 6], np.int32)
    num_slots, H, Hk, n = 8, 4, 2, 5
    ids = np.array([7, 2, 0, 5, 3], np.int32)
    # a non-trivial starting state for the requests (oracle-quantized fp32 states)
    st = np.zeros((n, H, 128, 128))
    for _ in range(12):
        O.fp_decode_step(st, H, 0, unit(rng, (n, H, 128)), unit(rng, (n, H, 128)),
                         rng.standard_normal((n, H, 128)).astype(np.float32),
                         np.full((n, H), 0.97, np.float32), rng.uniform(0.2, 0.8, (n, H)).astype(np.float32),
                         round_fp32=True)
    op = O.OraclePool(num_slots, bits, Hk)
    op.load_fp32(ids, st.astype(np.float32))

    pool = S.Pool(num_slots, bits, Hk, gate_mode, in_dtype)
    pool.load_packed(dev(ids), dev(op.slot_bytes(ids)))
    state = torch.zeros(num_slots * pool.slot_stride, dtype=torch.uint8, device="cuda")
    image = torch.empty((n, pool.slot_stride), dtype=torch.uint8, device="cuda")
    pool.dump_packed(dev(ids), image)
    for r, s in enumerate(ids):
        state[int(s) * pool.slot_stride:(int(s) + 1) * pool.slot_stride] = image[r]
    flag = torch.full((1,), -1, dtype=torch.int32, device="cuda")

    for call in range(2):
        x = dict(q=unit(rng, (n, Hk, 128)), k=unit(rng, (n, Hk, 128)),
                 v=rng.standard_normal((n, H, 128)).astype(np.float32),
                 alpha=(rng.uniform(0.5, 1.0, (n, H, 128)) if gate_mode == 1 else rng.uniform(0.5, 1.0, (n, H))),
                 beta=rng.uniform(0.0, 1.0, (n, H)))
        tx = {}
        for key, val in x.items():
            val = np.asarray(val, np.float32)
            tx[key] = dev(W.to_bf16_bits(val).view(np.int16)) if in_dtype == 1 else dev(val)
        y_pool = torch.empty((n, H, 128), device="cuda")
        y_free = torch.empty((n, H, 128), device="cuda")
        pool.decode_step(dev(ids), tx["q"], tx["k"], tx["v"], tx["alpha"], tx["beta"], y_pool)
        S.stepq_decode_step_noalloc(num_slots, bits, Hk, gate_mode, in_dtype, state, dev(ids), tx["q"], tx["k"],
                                    tx["v"], tx["alpha"], tx["beta"], y_free, flag_out=flag)
        torch.cuda.synchronize()
        assert int(flag.item()) == 0
        assert pool.get_error() == 0
        yp, yf = y_pool.cpu().numpy(), y_free.cpu().numpy()
        assert PH.y_max_rel(yf, yp) <= PH.Y_MAX_REL
        np.testing.assert_array_equal(yf, yp)            # same kernel, same inputs: identical
        pool.dump_packed(dev(ids), image)
        got = state.view(num_slots, pool.slot_stride)[torch.from_numpy(ids.astype(np.int64)).cuda()]
        assert torch.equal(got, image)
    pool.close()


def test_noalloc_rejects_too_many_heads():
    from quantized_gated_delta_b200 import stepq as S
    t = torch.zeros(256, dtype=torch.float32, device="cuda")
    ids = torch.zeros(1, dtype=torch.int32, device="cuda")
    state = torch.zeros(1024, dtype=torch.uint8, device="cuda")
    with pytest.raises(S.StepqError) as err:
        S.stepq_decode_step_noalloc(1, [4] * 257, 1, 0, 0, state, ids, t, t, t, t, t, t)
    assert err.value.status == -4


def test_noalloc_calls_replay_from_a_cuda_graph():
    """After its first call on a device, the entry point may be captured: the tables reach the
    scratch as a kernel argument, so a replayed graph refreshes them without touching host
    memory.  Two captured calls, replayed three times with new inputs written in place, must
    give the pool entry point's y and state bytes bit for bit."""
    from quantized_gated_delta_b200 import stepq as S
    rng = np.random.default_rng(4242)
    bits = np.array([8, 6, 4, 6, 4, 8], np.int32)
    num_slots, H, Hk, n = 12, 6, 3, 7
    ids = rng.permutation(num_slots)[:n].astype(np.int32)
    st = np.zeros((n, H, 128, 128))
    for _ in range(10):
        O.fp_decode_step(st, H, 0, unit(rng, (n, H, 128)), unit(rng, (n, H, 128)),
                         rng.standard_normal((n, H, 128)).astype(np.float32),
                         np.full((n, H), 0.95, np.float32), rng.uniform(0.2, 0.8, (n, H)).astype(np.float32),
                         round_fp32=True)
    op = O.OraclePool(num_slots, bits, Hk)
    op.load_fp32(ids, st.astype(np.float32))
    pool = S.Pool(num_slots, bits, Hk, 0, 1)
    pool.load_packed(dev(ids), dev(op.slot_bytes(ids)))
    state = torch.zeros(num_slots * pool.slot_stride, dtype=torch.uint8, device="cuda")
    image = torch.empty((n, pool.slot_stride), dtype=torch.uint8, device="cuda")
    pool.dump_packed(dev(ids), image)
    for r, s in enumerate(ids):
        state[int(s) * pool.slot_stride:(int(s) + 1) * pool.slot_stride] = image[r]
    d_ids = dev(ids)
    flag = torch.full((1,), -1, dtype=torch.int32, device="cuda")

    def draw():
        x = dict(q=unit(rng, (2, n, Hk, 128)), k=unit(rng, (2, n, Hk, 128)),
                 v=rng.standard_normal((2, n, H, 128)).astype(np.float32),
                 alpha=rng.uniform(0.5, 1.0, (2, n, H)), beta=rng.uniform(0.0, 1.0, (2, n, H)))
        return {key: dev(W.to_bf16_bits(np.asarray(val, np.float32)).view(np.int16)) for key, val in x.items()}

    bufs = draw()
    y_free = torch.empty((2, n, H, 128), device="cuda")

    def two_calls():
        for t in range(2):
            S.stepq_decode_step_noalloc(num_slots, bits, Hk, 0, 1, state, d_ids, bufs["q"][t], bufs["k"][t],
                                        bufs["v"][t], bufs["alpha"][t], bufs["beta"][t], y_free[t], flag_out=flag)

    # the first call on the device resolves the scratch address and configures the kernels
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        two_calls()
    torch.cuda.current_stream().wait_stream(side)
    y_pool = torch.empty((n, H, 128), device="cuda")
    for t in range(2):                               # the pool follows the same two steps
        pool.decode_step(d_ids, bufs["q"][t], bufs["k"][t], bufs["v"][t], bufs["alpha"][t], bufs["beta"][t], y_pool)
        assert torch.equal(y_pool, y_free[t])
    torch.cuda.synchronize()

    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        two_calls()
    for rep in range(3):
        new = draw()
        for key in bufs:
            bufs[key].copy_(new[key])
        graph.replay()
        for t in range(2):
            pool.decode_step(d_ids, bufs["q"][t], bufs["k"][t], bufs["v"][t], bufs["alpha"][t], bufs["beta"][t],
                             y_pool)
            torch.cuda.synchronize()
            assert torch.equal(y_pool, y_free[t]), (rep, t)
        assert int(flag.item()) == 0
        pool.dump_packed(d_ids, image)
        got = state.view(num_slots, pool.slot_stride)[torch.from_numpy(ids.astype(np.int64)).cuda()]
        assert torch.equal(got, image), rep
    assert pool.get_error() == 0
    del graph
    pool.close()
