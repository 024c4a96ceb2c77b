"""Multi-process paths on CPU (gloo, world size 2): request sharding, max-over-ranks
timing and the optional output gather.  The per-rank decode step is run by the CPU oracle
here, standing in for each rank's GPU; what is under test is the plumbing around it."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    from oracle import oracle as O
    from quantized_gated_delta_b200 import dist as D
    from quantized_gated_delta_b200 import workloads as W
    r, wsz, _ = D.init_from_env("gloo", timeout_s=60)
    assert (r, wsz) == (rank, world)
    # one batch of requests split across the ranks; every rank owns a pool of its own
    w = W.make_workload(1)
    mine = list(D.shard_requests(w.B, wsz, r))
    bits = np.asarray(w.head_bits[0], np.int32)
    pool = O.OraclePool(w.num_slots, bits, w.Hk, w.gate_mode)
    slots = w.slot_ids[mine]
    ys = []
    for t in range(3):
        x = W.step_inputs(w, t)
        xs = {k: np.ascontiguousarray(v[mine]) for k, v in x.items()}
        ys.append(pool.decode_step(slots, nthreads=1, **xs))
    y = torch.from_numpy(np.stack(ys, axis=1))                        # [mine, T, H, dv]
    counts = [len(D.shard_requests(w.B, wsz, k)) for k in range(wsz)]
    y_all = D.gather_outputs(y, counts)
    t_max = D.max_over_ranks(10.0 + rank)
    n_all = D.sum_over_ranks(len(mine))
    D.barrier()
    if rank == 0:
        np.save(os.path.join(out_dir, "y_all.npy"), y_all.numpy())
        np.save(os.path.join(out_dir, "scalars.npy"), np.array([t_max, n_all]))
    D.finalize()


def test_shard_requests_cover_each_request_once():
    from quantized_gated_delta_b200 import dist as D
    for n in (1, 5, 64, 513):
        for world in (1, 2, 3, 8):
            parts = [list(D.shard_requests(n, world, r)) for r in range(world)]
            assert sum(parts, []) == list(range(n))
            assert max(map(len, parts)) - min(map(len, parts)) <= 1


def test_two_ranks_gloo_match_single_process(tmp_path):
    from oracle import oracle as O
    from quantized_gated_delta_b200 import workloads as W
    world = 2
    ctx = mp.get_context("spawn")
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, str(tmp_path))) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=180)
        assert p.exitcode == 0
    y_all = np.load(tmp_path / "y_all.npy")
    t_max, n_all = np.load(tmp_path / "scalars.npy")
    assert t_max == 11.0 and n_all == 4
    # single process, whole batch, one pool
    w = W.make_workload(1)
    pool = O.OraclePool(w.num_slots, np.asarray(w.head_bits[0], np.int32), w.Hk, w.gate_mode)
    ys = [pool.decode_step(w.slot_ids, nthreads=1, **W.step_inputs(w, t)) for t in range(3)]
    assert np.array_equal(y_all, np.stack(ys, axis=1))
