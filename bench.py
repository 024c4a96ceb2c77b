"""Benchmark of the fused quantized gated Delta-rule decode step on B200.

A step is one decode step of the whole hot path (dequantize, fade, Delta write, readout,
dual-axis refit, requantize, repack) for every (request, value head) of one batch.
Workload: the high-concurrency GDN pool -- 512 requests scattered over a 1024-slot pool,
32 value heads sharing 16 key heads, d_k = d_v = 128, 6-bit-nominal mixed widths from the
lifetime-aware allocator, bf16 inputs, fp32 outputs.

  python bench.py [--gpus N --steps K --warmup W] [--impl reference]
Multi-GPU (torchrun): every rank owns its own pool and requests (the units are
independent; no collective on the data path): weak scaling, time = max over ranks.
"""
from __future__ import annotations

import argparse
import hashlib
import re
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "quantized-state updates/s (req·head·step) and achieved HBM GB/s vs peak"
UNIT = "updates/s"
N_INPUT_SETS = 64          # distinct per-step input batches cycled through (1.1 GB on device)
E2E_HOST_SETS = 8          # distinct pinned host batches for the end-to-end leg
GRAPH_CHUNK = 16           # decode steps per captured CUDA graph in the device-timed leg
EVENT_STEPS = 256          # plain launches timed one by one (informational)


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=4096)
    ap.add_argument("--warmup", type=int, default=32)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--variant", default="mixed6", choices=["mixed6", "uniform4", "mixed6p", "rowbits"],
                    help="mixed6: 6-bit nominal allocation; uniform4; mixed6p: mixed6 plus one FP16 pivot head; "
                         "rowbits (--workload kda): per-key-row widths")
    ap.add_argument("--e2e-steps", type=int, default=256)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--input-sets", type=int, default=N_INPUT_SETS,
                    help="distinct per-step input batches kept on the device and cycled")
    ap.add_argument("--fit", default="clipfree", choices=["clipfree", "impact"],
                    help="dual-axis fit: clip-free (the headline) or impact-weighted with synthetic row-impact scores")
    ap.add_argument("--workload", default="pool", choices=["pool", "stack", "kda"],
                    help="pool: the high-concurrency pool (the headline); stack: the 36-layer stack sweep; "
                         "kda: the KDA layer (per-channel gates)")
    ap.add_argument("--batch", type=int, default=1024, choices=[64, 256, 1024],
                    help="requests of the stack sweep")
    ap.add_argument("--no-sweep", action="store_true",
                    help="skip the device-timed sweep of the other workloads after the headline line's legs")
    return ap.parse_args()


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as fh:
            p = json.load(fh)
        return float(p["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


def _code_only(src: str) -> str:
    """C/C++ source without comments and with whitespace runs collapsed (string literals in
    these files hold no comment markers)."""
    src = re.sub(r"/\*.*?\*/", " ", src, flags=re.S)
    src = re.sub(r"//[^\n]*", " ", src)
    return " ".join(src.split())


def kernel_source_hash(csrc: str | None = None) -> str:
    """Hash of the library's code (comments and layout excluded): a recorded ncu traffic
    figure is reported only for the code it was measured on."""
    h = hashlib.sha256()
    csrc = csrc or os.path.join(ROOT, "quantized_gated_delta_b200", "csrc")
    for f in sorted(os.listdir(csrc)):
        with open(os.path.join(csrc, f), encoding="utf-8") as fh:
            h.update(f.encode() + b"\0" + _code_only(fh.read()).encode())
    return h.hexdigest()[:16]


def recorded_traffic(workload_name: str):
    """DRAM bytes per launch from the committed ncu summary, if it was taken on this source."""
    try:
        with open(os.path.join(ROOT, "profiles", "decode_traffic.json")) as fh:
            rec = json.load(fh)
        if rec.get("source_hash") == kernel_source_hash() and rec.get("workload") == workload_name:
            return float(rec["dram_bytes_per_launch"])
    except Exception:
        pass
    return None


def copy_link_rates(hin, hout, reps: int = 20) -> dict:
    """Copy rates between the device and the given pinned host buffers (the host-buffer leg's
    own input image and y, since the rate depends on where the host pages sit): each direction
    alone, then both at once on two streams, as in the leg."""
    import torch
    hin, hout = hin.view(torch.uint8).reshape(-1), hout.view(torch.uint8).reshape(-1)
    h2d_bytes, d2h_bytes = hin.numel(), hout.numel()
    din = torch.empty(h2d_bytes, dtype=torch.uint8, device="cuda")
    dout = torch.empty(d2h_bytes, dtype=torch.uint8, device="cuda")
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()

    def timed(do_in, do_out):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        e0.record()
        s_in.wait_event(e0)
        s_out.wait_event(e0)
        for _ in range(reps):
            if do_in:
                with torch.cuda.stream(s_in):
                    din.copy_(hin, non_blocking=True)
            if do_out:
                with torch.cuda.stream(s_out):
                    hout.copy_(dout, non_blocking=True)
        torch.cuda.current_stream().wait_stream(s_in)
        torch.cuda.current_stream().wait_stream(s_out)
        e1.record()
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / 1e3 / reps

    timed(True, True)                                # warm-up
    t_in, t_out, t_both = timed(True, False), timed(False, True), timed(True, True)
    return {"h2d_gbs": h2d_bytes / t_in / 1e9, "d2h_gbs": d2h_bytes / t_out / 1e9,
            "both_h2d_gbs": h2d_bytes / t_both / 1e9, "both_d2h_gbs": d2h_bytes / t_both / 1e9}


class ClockSampler:
    """nvidia-smi clock / throttle sampling during the timed region."""

    def __init__(self, device_index: int):
        self.dev = device_index
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            import torch
            ident = str(torch.cuda.get_device_properties(self.dev).uuid)
            ident = ident if ident.startswith("GPU-") else "GPU-" + ident
        except Exception:
            ident = str(self.dev)
        q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", ident, "--query-gpu=" + q,
                                          "--format=csv,noheader,nounits", "-lms", "50"],
                                         stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
        time.sleep(0.3)

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.1)
        self.proc.terminate()
        self.proc.wait()
        rows = []
        for line in open(self.path):
            f = [x.strip() for x in line.split(",")]
            if len(f) >= 9:
                rows.append(f)
        os.unlink(self.path)
        if not rows:
            return None
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        reasons = set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            for n, v in zip(names, r[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": float(rows[0][2]) if rows[0][2].replace(".", "").isdigit() else None,
                "reasons": sorted(reasons), "samples": len(rows)}


def block_bytes(bits: int, dk: int = 128, dv: int = 128) -> int:
    """Packed head block: codes (dk*dv*bits/8 bytes) + fp32 row and column factors; an FP16
    pivot head (width 16) is the binary16 state alone."""
    if bits == 16:
        return 2 * dk * dv
    return dk * dv * bits // 8 + 4 * dk + 4 * dv


def algorithmic_bytes_per_step(w, bits, slot_stride=None) -> float:
    """State read once + written once per (request, head), plus the step's inputs and outputs
    (slot_stride: the pool's bytes per request, for heads with per-key-row widths)."""
    per_slot = slot_stride if slot_stride is not None else sum(block_bytes(int(b), w.dk, w.dv) for b in bits)
    state = 2.0 * w.B * per_slot
    esz = 2 if w.in_dtype == 1 else 4
    io = w.B * w.Hk * 2 * w.dk * esz            # q, k (shared by H / Hk value heads)
    io += w.B * w.H * w.dv * esz                # v
    io += w.B * w.H * (w.dk if w.gate_mode == 1 else 1) * esz   # alpha
    io += w.B * w.H * esz                       # beta
    io += w.B * w.H * w.dv * 4                  # y (fp32)
    io += w.B * 4                               # slot ids
    return state + io


def _oracle_sample(w, bits, nreq: int):
    from oracle import oracle as O
    from quantized_gated_delta_b200 import workloads as W
    sub = W.sample_requests(w, nreq)
    pool = O.OraclePool(w.num_slots, bits, w.Hk, w.gate_mode)
    xs = [{k: np.ascontiguousarray(v[sub]) for k, v in W.step_inputs(w, t).items()} for t in range(4)]
    return pool, w.slot_ids[sub], xs


def cpu_baseline(w, bits, seconds: float):
    """The CPU oracle, as it stands, on this host's cores on a bounded sample of the workload."""
    from oracle import oracle as O
    pool, sl, xs = _oracle_sample(w, bits, 16)
    pool.decode_step(sl, **xs[0])                        # first touch, thread start
    steps = 0
    t0 = time.perf_counter()
    while True:
        pool.decode_step(sl, **xs[steps % len(xs)])
        steps += 1
        el = time.perf_counter() - t0
        if el >= seconds:
            break
    value = steps * len(sl) * w.H / el
    # the same oracle on one core, over a shorter bounded sample
    one = 0
    t1 = time.perf_counter()
    while True:
        pool.decode_step(sl[:2], **{k: v[:2] for k, v in xs[one % len(xs)].items()}, nthreads=1)
        one += 1
        el1 = time.perf_counter() - t1
        if el1 >= seconds / 3:
            break
    return {"value": value, "unit": UNIT, "cores": O.default_threads(), "kind": "oracle",
            "sample": "%d requests x %d heads x %d decode steps of %s (%.1f s)" % (len(sl), w.H, steps, w.name, el),
            "one_core_value": one * 2 * w.H / el1, "host_cpus": os.cpu_count(), "cpu_model": _cpu_model()}


def _cpu_model() -> str:
    try:
        for line in open("/proc/cpuinfo"):
            if line.startswith("model name"):
                return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def slot_stride_of(bits) -> int:
    """Bytes of one slot: per head, codes + r + c (an FP16 pivot head: 2 bytes per value)."""
    return sum(2 * 128 * 128 if int(b) == 16 else 128 * 128 * int(b) // 8 + 8 * 128 for b in bits)


def pool_config(w, bits, row_bits, fit, world, slot_stride):
    """The `config` of a bench line on the single-pool workloads (both arms: the workload only;
    each arm reports the number of input batches it cycles in its own `input_sets` key)."""
    return {"workload": "%s: B=%d of %d slots, H=%d, Hk=%d, d_k=d_v=%d, %s inputs, bits %s%s"
                        % (w.name, w.B, w.num_slots, w.H, w.Hk, w.dk, w.dtype_name,
                           "".join(str(int(b)) for b in bits) if row_bits is None else "per key row (4/6/8: %s)"
                           % "/".join(str(int(np.sum(row_bits == x))) for x in (4, 6, 8)),
                           ", impact-weighted fit" if fit == "impact" else ""),
            "avg_bits": float(np.mean(bits if row_bits is None else row_bits)),
            "parallelism": "dp%d (independent pools)" % world,
            "l2": "no flush: %.0f MB of packed state read and written per step (> 126 MB L2)"
                  % (w.B * slot_stride / 1e6)}


def run_reference(args):
    """Reference arm: the oracle, as it stands, timed on the host cores.  Each step is a
    bounded sample of the workload's requests, sized so the whole run takes a few minutes."""
    if int(os.environ.get("RANK", "0")) != 0:
        return
    from oracle import oracle as O
    from quantized_gated_delta_b200 import workloads as W
    w = W.make_workload(4, args.variant)
    if w.head_bits is None:
        if w.n_pivots:
            bits, _ = O.allocate_bits_pivots(list(w.half_life[0]), None, [4, 6, 8], w.avg_bits, w.n_pivots)
        else:
            bits, _ = O.allocate_bits_dp(list(w.half_life[0]), None, [4, 6, 8], w.avg_bits)
    else:
        bits = list(w.head_bits[0])
    pool, sl, xs = _oracle_sample(w, bits, 16)
    t0 = time.perf_counter()
    pool.decode_step(sl, **xs[0])
    per_req = (time.perf_counter() - t0) / len(sl)
    budget = 120.0 / max(1, args.steps + args.warmup)
    nreq = int(max(1, min(16, budget // max(per_req, 1e-6))))
    pool, sl, xs = _oracle_sample(w, bits, nreq)
    for i in range(args.warmup):
        pool.decode_step(sl, **xs[i % len(xs)])
    t0 = time.perf_counter()
    for i in range(args.steps):
        pool.decode_step(sl, **xs[i % len(xs)])
    el = time.perf_counter() - t0
    value = args.steps * len(sl) * w.H / el
    cores = O.default_threads()
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": el * 1e3 / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic",
            "config": pool_config(w, bits, None, "clipfree", args.gpus, slot_stride_of(bits)),
            "input_sets": len(xs),
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                             "sample": "%d requests x %d heads per step, %d steps of %s"
                                       % (len(sl), w.H, args.steps, w.name)},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line))


def _time_stack(batch: int, steps: int, warmup: int, clocks_too: bool = False) -> dict:
    """36-layer stack sweep: a step runs layers 0..35 in order, each a decode step of its own
    pool (per-layer allocation).  Timed twice on the device: 36 plain launches per step, and
    the step captured once as a CUDA graph and replayed."""
    import torch

    from quantized_gated_delta_b200 import stepq
    from quantized_gated_delta_b200 import workloads as W

    w = W.make_workload(5, batch=batch)
    L = w.layers
    pools, bits_all = [], []
    for layer in range(L):
        bits = np.asarray(stepq.stepq_allocate_bits(w.half_life[layer], None, (4, 6, 8), w.avg_bits), np.uint8)
        bits_all.append(bits)
        pools.append(stepq.Pool(w.num_slots, bits, w.Hk, w.gate_mode, w.in_dtype))
    slots = torch.from_numpy(w.slot_ids).cuda()

    def dev_inputs(x):
        return {k: torch.from_numpy(W.as_device_dtype(w, v).view(np.int16)).cuda() for k, v in x.items()}
    nsets = 2
    sets = [[dev_inputs(W.step_inputs(w, t, W.PHASE_RUN, layer)) for layer in range(L)] for t in range(nsets)]
    y = torch.empty((w.B, w.H, w.dv), device="cuda")

    def step(i):
        xs = sets[i % nsets]
        for layer in range(L):
            x = xs[layer]
            pools[layer].decode_step(slots, x["q"], x["k"], x["v"], x["alpha"], x["beta"], y)

    for i in range(max(3, warmup)):
        step(i)
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream()
    sampler = ClockSampler(0) if clocks_too else None
    if sampler:
        sampler.start()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for i in range(steps):
        step(i)
    e1.record(stream)
    torch.cuda.synchronize()
    ms_plain = e0.elapsed_time(e1)
    # the same step as one CUDA graph (inputs of set 0), replayed
    g = torch.cuda.CUDAGraph()
    side = torch.cuda.Stream()
    side.wait_stream(stream)
    with torch.cuda.stream(side):
        with torch.cuda.graph(g, stream=side):
            step(0)
    stream.wait_stream(side)
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize()
    e0.record(stream)
    for _ in range(steps):
        g.replay()
    e1.record(stream)
    torch.cuda.synchronize()
    ms_graph = e0.elapsed_time(e1)
    clocks = sampler.stop() if sampler else None
    for p_ in pools:
        if p_.get_error() != 0:
            raise RuntimeError("device flag set in the stack sweep")
    units = w.B * w.H * L * steps
    # the same pool with FP32 states (d_k x d_v float32 per head, no scales): the pages'
    # reference point for the state-pool memory
    fp32_bytes = int(L * w.num_slots * w.H * w.dk * w.dv * 4)
    pool_bytes = int(sum(p_.total_bytes for p_ in pools))
    alg = sum(algorithmic_bytes_per_step(w, b) for b in bits_all)          # one step, all layers
    peak, peak_kind = peaks()
    achieved = alg * steps / (ms_graph / 1e3) / 1e9
    del g
    for p_ in pools:
        p_.close()
    return {"workload": w.name, "w": w, "B": w.B, "L": L, "steps": steps, "ms_graph": ms_graph,
            "ms_plain": ms_plain, "us_per_layer_step": ms_graph * 1e3 / (steps * L),
            "us_per_layer_step_plain": ms_plain * 1e3 / (steps * L), "updates_per_s": units / (ms_graph / 1e3),
            "achieved_gbs": achieved, "frac": achieved / peak, "peak": peak, "peak_kind": peak_kind,
            "alg": alg, "pool_bytes": pool_bytes, "fp32_pool_bytes": fp32_bytes, "clocks": clocks}


def run_stack(args):
    """The 36-layer stack sweep as its own bench line (--workload stack)."""
    import torch
    torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", "0")))
    r = _time_stack(args.batch, args.steps, args.warmup, clocks_too=True)
    w = r["w"]
    line = {"metric": "quantized-state updates/s (req·head·layer-step), 36-layer stack", "value": r["updates_per_s"],
            "unit": UNIT, "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": r["ms_graph"] / args.steps, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": {"workload": "%s: %d layers x H=%d, Hk=%d, B=%d, per-layer allocation (6.0 avg), bf16 inputs"
                                   % (w.name, r["L"], w.H, w.Hk, w.B),
                       "pool_bytes": r["pool_bytes"],
                       "fp32_pool_bytes": r["fp32_pool_bytes"],
                       "fp32_over_packed": r["fp32_pool_bytes"] / float(r["pool_bytes"]),
                       "l2": "no flush: each layer's pool is re-read after the other 35 (stack > 126 MB L2)"},
            "us_per_layer_step_graph": r["us_per_layer_step"],
            "us_per_layer_step_plain": r["us_per_layer_step_plain"],
            "roofline": {"bound": "hbm", "achieved": r["achieved_gbs"], "peak": r["peak"], "unit": "GB/s",
                         "frac": r["frac"], "peak_source": r["peak_kind"], "traffic": None,
                         "algorithmic_bytes_per_step": r["alg"], "kernel": "decode_kernel (36 launches per step)"},
            "gpu_launches": args.steps * r["L"], "clocks": r["clocks"]}
    print(json.dumps(line))


def _time_pool_workload(config: int, variant: str, fit: str, steps: int) -> dict:
    """Device time of one single-pool workload: a 16-step CUDA graph of decode steps replayed
    (inputs resident in HBM, cycling through 4 sets), after 4 warm-up steps."""
    import torch

    from quantized_gated_delta_b200 import stepq
    from quantized_gated_delta_b200 import workloads as W

    w = W.make_workload(config, variant)
    row_bits = None
    if w.row_half_life is not None:
        rb = stepq.stepq_allocate_bits(np.ravel(w.row_half_life[0]), None, (4, 6, 8), w.avg_bits)
        row_bits = np.asarray(rb, np.uint8).reshape(w.H, w.dk)
        bits = np.zeros(w.H, dtype=np.uint8)
    elif w.head_bits is not None:
        bits = np.asarray(w.head_bits[0], np.uint8)
    elif w.n_pivots:
        bits = np.asarray(stepq.stepq_allocate_bits_pivots(w.half_life[0], None, (4, 6, 8), w.avg_bits,
                                                           w.n_pivots), np.uint8)
    else:
        bits = np.asarray(stepq.stepq_allocate_bits(w.half_life[0], None, (4, 6, 8), w.avg_bits), np.uint8)
    pool = stepq.Pool(w.num_slots, bits, w.Hk, w.gate_mode, w.in_dtype, row_bits=row_bits)
    if fit == "impact":
        pool.set_impact(W.impact_scores(w))
    slots = torch.from_numpy(w.slot_ids).cuda()
    sets = [{k: torch.from_numpy(W.as_device_dtype(w, v).view(np.int16)).cuda()
             for k, v in W.step_inputs(w, t).items()} for t in range(4)]
    y = torch.empty((w.B, w.H, w.dv), device="cuda")
    stream = torch.cuda.current_stream()
    for t in range(4):
        x = sets[t]
        pool.decode_step(slots, x["q"], x["k"], x["v"], x["alpha"], x["beta"], y, stream)
    g = torch.cuda.CUDAGraph()
    side = torch.cuda.Stream()
    side.wait_stream(stream)
    with torch.cuda.stream(side):
        with torch.cuda.graph(g, stream=side):
            for t in range(GRAPH_CHUNK):
                x = sets[t % 4]
                pool.decode_step(slots, x["q"], x["k"], x["v"], x["alpha"], x["beta"], y, side)
    stream.wait_stream(side)
    g.replay()
    torch.cuda.synchronize()
    reps = max(1, steps // GRAPH_CHUNK)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(reps):
        g.replay()
    e1.record(stream)
    torch.cuda.synchronize()
    if pool.get_error() != 0:
        raise RuntimeError("device flag set in the %s sweep" % w.name)
    us = e0.elapsed_time(e1) * 1e3 / (reps * GRAPH_CHUNK)
    alg = algorithmic_bytes_per_step(w, bits, pool.slot_stride)
    peak, _ = peaks()
    del g
    pool.close()
    return {"workload": w.name + (" (impact-weighted fit)" if fit == "impact" else ""), "B": w.B, "H": w.H,
            "Hk": w.Hk, "steps": reps * GRAPH_CHUNK, "us_per_step": us, "updates_per_s": w.B * w.H / (us / 1e6),
            "achieved_gbs": alg / (us / 1e6) / 1e9, "frac": alg / (us / 1e6) / 1e9 / peak,
            "algorithmic_bytes_per_step": alg}


def workload_sweep() -> list:
    """The other workloads, device-timed after the headline measurement: the
    hybrid GDN layer, the KDA layer (per-head and per-key-row widths), the high-concurrency
    pool's uniform 4-bit, FP16-pivot and impact-fit variants, and the 36-layer stack at three
    batch sizes (per layer-step, as one CUDA graph per step)."""
    out = []
    for config, variant, fit, steps in ((2, "mixed6", "clipfree", 1024), (3, "mixed6", "clipfree", 1024),
                                        (3, "rowbits", "clipfree", 512), (4, "uniform4", "clipfree", 512),
                                        (4, "mixed6p", "clipfree", 512), (4, "mixed6", "impact", 512)):
        out.append(_time_pool_workload(config, variant, fit, steps))
    for batch in (64, 256, 1024):
        r = _time_stack(batch, 16, 3)
        out.append({k: r[k] for k in ("workload", "B", "steps", "us_per_layer_step", "updates_per_s",
                                      "achieved_gbs", "frac", "pool_bytes", "fp32_pool_bytes")})
    return out


def main():
    args = parse()
    if args.impl == "reference":
        run_reference(args)
        return
    if args.workload == "stack":
        run_stack(args)
        return
    import torch

    from quantized_gated_delta_b200 import dist as D
    from quantized_gated_delta_b200 import stepq
    from quantized_gated_delta_b200 import workloads as W

    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    rank, world, local = D.init_from_env("nccl", timeout_s=120)

    w = W.make_workload(3 if args.workload == "kda" else 4, args.variant)
    w.seed = D.shard_seed(w.seed, rank)              # each rank serves its own requests
    row_bits = None
    if w.row_half_life is not None:
        # the allocation unit is the key row: widths over the layer's H * d_k rows
        rb = stepq.stepq_allocate_bits(np.ravel(w.row_half_life[0]), None, (4, 6, 8), w.avg_bits)
        row_bits = np.asarray(rb, np.uint8).reshape(w.H, w.dk)
        bits = np.zeros(w.H, dtype=np.uint8)
    elif w.head_bits is not None:
        bits = w.head_bits[0]
    elif w.n_pivots:
        bits = stepq.stepq_allocate_bits_pivots(w.half_life[0], None, (4, 6, 8), w.avg_bits, w.n_pivots)
    else:
        bits = stepq.stepq_allocate_bits(w.half_life[0], None, (4, 6, 8), w.avg_bits)
    bits = np.asarray(bits, dtype=np.uint8)
    pool = stepq.Pool(w.num_slots, bits, w.Hk, w.gate_mode, w.in_dtype, row_bits=row_bits)
    if args.fit == "impact":
        pool.set_impact(W.impact_scores(w))
    slots = torch.from_numpy(w.slot_ids).cuda()

    # per-step inputs, resident in HBM (bf16 bit patterns)
    def dev_inputs(x):
        return {k: torch.from_numpy(W.as_device_dtype(w, v).view(np.int16)).cuda() for k, v in x.items()}
    nsets = max(1, min(args.input_sets, args.steps + args.warmup))
    host_sets = [W.step_inputs(w, t) for t in range(nsets)]
    sets = [dev_inputs(x) for x in host_sets]
    y = torch.empty((w.B, w.H, w.dv), device="cuda")
    stream = torch.cuda.current_stream()

    def step(i):
        x = sets[i % nsets]
        pool.decode_step(slots, x["q"], x["k"], x["v"], x["alpha"], x["beta"], y, stream)

    # the decode loop as a serving engine launches it: a chunk of GRAPH_CHUNK steps (one kernel
    # each, inputs cycling through the resident sets) captured once as a CUDA graph
    chunk = torch.cuda.CUDAGraph()
    side = torch.cuda.Stream()
    side.wait_stream(stream)
    try:
        with torch.cuda.stream(side):
            with torch.cuda.graph(chunk, stream=side):
                for t in range(GRAPH_CHUNK):
                    x = sets[t % nsets]
                    pool.decode_step(slots, x["q"], x["k"], x["v"], x["alpha"], x["beta"], y, side)
        graphed = GRAPH_CHUNK
    except Exception as exc:                       # no capture: the timed steps are plain launches
        graphed = 0
        capture_error = type(exc).__name__
        torch.cuda.synchronize()
    stream.wait_stream(side)

    for i in range(args.warmup):
        step(i)
    if graphed:
        chunk.replay()                             # uploads the graph (untimed)
    torch.cuda.synchronize()
    if pool.get_error() != 0:
        raise RuntimeError("device flag set during warm-up")

    # ---- device-timed leg: exactly K steps, inputs resident in HBM: K // GRAPH_CHUNK replays
    # of the chunk, then K % GRAPH_CHUNK plain launches
    sampler = ClockSampler(local) if rank == 0 else None
    if sampler:
        sampler.start()
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    D.barrier()
    torch.cuda.synchronize()
    t_start.record(stream)
    replays = args.steps // graphed if graphed else 0
    for _ in range(replays):
        chunk.replay()
    for i in range(args.steps - replays * graphed):
        step(args.warmup + i)
    t_end.record(stream)
    torch.cuda.synchronize()
    D.barrier()
    clocks = sampler.stop() if sampler else None
    ms_total = D.max_over_ranks(t_start.elapsed_time(t_end), "cuda")
    err = pool.get_error()
    if err != 0:
        raise RuntimeError("device flag %d set during the timed region" % err)
    units_per_step = w.B * w.H
    value = units_per_step * args.steps * world / (ms_total / 1e3)
    avg_kernel_s = ms_total / args.steps / 1e3    # per launch, gaps between the kernels included
    alg_bytes = algorithmic_bytes_per_step(w, bits, pool.slot_stride)
    peak, peak_kind = peaks()
    achieved = alg_bytes / avg_kernel_s / 1e9

    # ---- informational: plain launches, each bracketed by its own pair of events
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(EVENT_STEPS)]
    torch.cuda.synchronize()
    for i in range(EVENT_STEPS):
        ev[i][0].record(stream)
        step(i)
        ev[i][1].record(stream)
    torch.cuda.synchronize()
    event_us = statistics.median(a.elapsed_time(b) * 1e3 for a, b in ev)
    del chunk
    if pool.get_error() != 0:
        raise RuntimeError("device flag set in the plain-launch leg")

    # ---- end-to-end leg: the host-buffer entry point.  Slot ids, inputs and y live in pinned
    # host memory; every step the library copies that step's inputs in and its y out, through
    # two staging buffers, so the copies of one step overlap the neighbouring steps' kernels.
    # each step's slot ids and inputs sit in one pinned image at the offsets the library gives
    # (stepq_host_image_layout), so the call copies them in one transfer
    offs, img_bytes = pool.host_image_layout(w.B)
    names = ("slots", "q", "k", "v", "alpha", "beta")
    host, images = [], []
    for x in host_sets[:E2E_HOST_SETS]:
        img = torch.zeros(img_bytes, dtype=torch.uint8).pin_memory()
        images.append(img)
        arrays = [np.ascontiguousarray(w.slot_ids, dtype=np.int32)] + \
                 [W.as_device_dtype(w, x[k]).view(np.int16) for k in names[1:]]
        views = {}
        for name, o, a in zip(names, offs, arrays):
            t = torch.from_numpy(a.reshape(-1))
            img[o:o + t.numel() * t.element_size()].copy_(t.view(torch.uint8))
            views[name] = img[o:o + t.numel() * t.element_size()].view(t.dtype)
        host.append(views)
    y_host = torch.empty((w.B, w.H, w.dv), dtype=torch.float32).pin_memory()
    h2d = img_bytes
    d2h = y_host.numel() * 4

    def e2e_step(i):
        hx = host[i % len(host)]
        pool.decode_step_host(hx["slots"], hx["q"], hx["k"], hx["v"], hx["alpha"], hx["beta"], y_host, stream)

    for i in range(3):
        e2e_step(i)
    pool.host_wait(stream)
    torch.cuda.synchronize()
    D.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for i in range(args.e2e_steps):
        e2e_step(i)
    pool.host_wait(stream)
    e1.record(stream)
    torch.cuda.synchronize()
    ms_e2e = D.max_over_ranks(e0.elapsed_time(e1), "cuda")
    e2e_value = units_per_step * args.e2e_steps * world / (ms_e2e / 1e3)
    link = copy_link_rates(images[0], y_host)
    # what the leg can reach: the slowest of the kernel, the input copy and the y copy, the two
    # copies running at once in opposite directions
    bound_us = max(avg_kernel_s * 1e6, h2d / (link["both_h2d_gbs"] * 1e3), d2h / (link["both_d2h_gbs"] * 1e3))

    base = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline and row_bits is None:
        base = cpu_baseline(w, bits, args.cpu_seconds)
    sweep = None
    if world == 1 and not args.no_sweep and args.workload == "pool" and args.variant == "mixed6" \
            and args.fit == "clipfree":
        sweep = workload_sweep()

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_total / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": pool_config(w, bits, row_bits, args.fit, world, pool.slot_stride),
            "input_sets": nsets,
            "achieved_gbs": achieved,
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                         "frac": achieved / peak, "peak_source": peak_kind,
                         "traffic": recorded_traffic(w.name),
                         "algorithmic_bytes_per_launch": alg_bytes,
                         "kernel": "decode_kernel", "avg_kernel_us": avg_kernel_s * 1e6},
            "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                    "steps": args.e2e_steps,
                    "us_per_step": ms_e2e * 1e3 / args.e2e_steps,
                    "copy_link": link, "bound_us_per_step": bound_us,
                    "frac_of_bound": bound_us / (ms_e2e * 1e3 / args.e2e_steps),
                    "api": "stepq_decode_step_host: one pinned input image per step (stepq_host_image_layout), "
                           "one host-to-device and one device-to-host copy per step, copies of consecutive steps "
                           "overlapped"},
            "timing": ("device leg: %d-step CUDA-graph chunks replayed" % graphed if graphed else
                       "device leg: plain launches (graph capture failed: %s)" % capture_error)
                      + " (kernel time = region / steps); plain launches with one event pair each: %.1f us median"
                      % event_us,
            "gpu_launches": args.steps * (2 if int(np.sum(bits == 16)) else 1),   # + pivot kernel
            "clocks": clocks,
            "cpu_baseline": base,
            "workloads": sweep,
        }
        print(json.dumps(line))
    pool.close()
    D.finalize()


if __name__ == "__main__":
    main()
