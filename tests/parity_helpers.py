"""Shared helpers of the GPU parity tests: workload set-up on the oracle side, moving
inputs to the device, and comparison of packed states (codes +-1 rule, scale ulps)."""
from __future__ import annotations

import numpy as np

from oracle import oracle as O
from quantized_gated_delta_b200 import workloads as W

# Tolerances (the reading of the single-step bar; see the design notes):
CODE_FLIP_RATE = 1e-5       # codes may differ by exactly 1 at this rate
R_ULP = 6                   # row factors r within 6 ulp of the oracle's
C_ULP = 4                   # column factors c within 4 ulp
Y_MAX_REL = 1e-4            # per (request, head): max_j |dy_j| / max_j |y_j|
Y_TRAJ_REL_L2 = 1e-3        # whole trajectory: ||dy||_2 / ||y||_2
# Impact-weighted fit: the column scale c_j is the least-squares scale of the intermediate
# codes Q0, a quotient of two sums of up to 128 non-negative terms; fp32 sums differ from the
# oracle's double sums by at most ~(n-1) u, so c within 2e-5 relative.  An intermediate code
# at a near tie may round one level apart (as any code may), which moves c_j by
# w r^2 |P| / sum w r^2 Q0^2 -- a few percent in a column that a few rows carry; such columns
# are counted like code flips and may be at most 3e-4 of the columns (about 1e-4 seen over a
# 256-step trajectory of the 512-request pool).  The codes of such a column follow its c and
# are not held to a flip rate; in every other column codes are +-1 at <= 1e-5, the
# single-step bar of the clip-free fit (1.3e-6 seen).
C_REL_IMPACT = 2e-5
C_FAR_RATE_IMPACT = 3e-4
CODE_FLIP_RATE_IMPACT = 1e-5
PIVOT_ULP = 1               # FP16 pivot states: binary16 values within 1 ulp ...
PIVOT_FLIP_RATE = 1e-3      # ... and off by one ulp at most at this rate (see pivots_ok)


def head_bits(w: W.Workload, layer: int = 0) -> np.ndarray:
    """Fixed widths of the workload, else the oracle's lifetime-aware allocation."""
    if w.head_bits is not None:
        return np.asarray(w.head_bits[layer], dtype=np.int32)
    if w.row_half_life is not None:
        return np.zeros(w.H, dtype=np.int32)          # every head: per-key-row widths
    if w.n_pivots:
        bits, _ = O.allocate_bits_pivots(list(w.half_life[layer]), None, [4, 6, 8], w.avg_bits, w.n_pivots)
        return np.asarray(bits, dtype=np.int32)
    bits, _ = O.allocate_bits_dp(list(w.half_life[layer]), None, [4, 6, 8], w.avg_bits)
    return np.asarray(bits, dtype=np.int32)


_ROW_BITS_CACHE = {}


def row_bits(w: W.Workload, layer: int = 0):
    """Per-key-row widths [H, dk] of a workload whose allocation unit is the key row, from
    the oracle's exact allocation over the layer's H * dk rows (None otherwise)."""
    if w.row_half_life is None:
        return None
    key = (w.name, w.seed, layer)
    if key not in _ROW_BITS_CACHE:
        hl = list(np.asarray(w.row_half_life[layer], dtype=np.float64).ravel())
        bits, _ = O.allocate_bits_dp_vec(hl, None, [4, 6, 8], w.avg_bits)
        _ROW_BITS_CACHE[key] = np.asarray(bits, dtype=np.int32).reshape(w.H, w.dk)
    return _ROW_BITS_CACHE[key]


def sub_inputs(x: dict, idx) -> dict:
    return {k: np.ascontiguousarray(v[idx]) for k, v in x.items()}


def oracle_pool_with_warmup(w: W.Workload, bits, req_idx, layer: int = 0) -> O.OraclePool:
    """Oracle pool whose slots slot_ids[req_idx] hold the quantized state reached after the
    workload's FP32 warm-up steps (unquantized steps from zero, fp32-stored)."""
    pool = O.OraclePool(w.num_slots, bits, w.Hk, w.gate_mode, row_bits=row_bits(w, layer))
    req_idx = np.asarray(req_idx)
    S = np.zeros((len(req_idx), w.H, w.dk, w.dv))
    for t in range(w.warmup_steps):
        x = sub_inputs(W.step_inputs(w, t, W.PHASE_WARMUP, layer), req_idx)
        O.fp_decode_step(S, w.Hk, w.gate_mode, x["q"], x["k"], x["v"], x["alpha"], x["beta"],
                         round_fp32=True)
    pool.load_fp32(w.slot_ids[req_idx], S.astype(np.float32))
    return pool


def to_device(w: W.Workload, x: dict, torch):
    """Inputs of one step as CUDA tensors in the device dtype (bf16 as its bit patterns)."""
    out = {}
    for key, val in x.items():
        a = W.as_device_dtype(w, val)
        t = torch.from_numpy(a.view(np.int16) if a.dtype == np.uint16 else a)
        out[key] = t.cuda()
    return out


def ulp_diff(a: np.ndarray, b: np.ndarray) -> np.ndarray:
    """Distance in units in the last place between same-signed float32 arrays."""
    ia = a.astype(np.float32).view(np.int32).astype(np.int64)
    ib = b.astype(np.float32).view(np.int32).astype(np.int64)
    return np.abs(ia - ib)


def fp16_ulp_diff(a: np.ndarray, b: np.ndarray) -> np.ndarray:
    """Distance in binary16 ulps between two arrays of binary16 bit patterns (ordered
    through zero: +0 and -0 coincide)."""
    def key(h):
        h = h.astype(np.int64)
        return np.where(h & 0x8000, -(h & 0x7FFF), h)
    return np.abs(key(a) - key(b))


TIE_DIST = 2e-4        # code units: a few fp32 ulps of S / (r c) at qmax, plus the r / c ulps allowed


def flips_off_tie(gpu_bytes, ora_before, bits, Hk, x, dk=128, dv=128):
    """Codes of a GPU step that differ from the oracle's and are not at a rounding tie.

    For each state and head the oracle's own step (from the slot bytes before the step,
    ora_before [n, slot_stride], and the inputs x of those n requests, GDN) gives the
    updated state before rounding and the fitted r, c; a code may differ by one only where
    |S / (r c)| lies within TIE_DIST of a half-integer (both roundings are then correct).
    x["alpha"][s, h] is a head's gate (GDN) or its 128 per-channel gates (KDA).  FP16 pivot
    heads (width 16) hold no codes and are skipped; compare_slots checks them.
    Returns (count of differing codes off a tie, largest code difference)."""
    offs, _ = O.head_offsets(bits, dk, dv)
    H = len(bits)
    off_tie, worst = 0, 0
    for s in range(gpu_bytes.shape[0]):
        for h, b in enumerate(bits):
            b = int(b)
            if b == 16:
                continue
            n = O.block_bytes(b, dk, dv)
            Q0, r0, c0 = O.split_block(ora_before[s, offs[h]:offs[h] + n], b, dk, dv)
            g = h // (H // Hk)
            out = O.step_state(Q0, r0, c0, b, x["q"][s, g], x["k"][s, g], x["v"][s, h], x["alpha"][s, h],
                               float(x["beta"][s, h]))
            Qg = O.split_block(gpu_bytes[s, offs[h]:offs[h] + n], b, dk, dv)[0]
            d = np.abs(Qg.astype(np.int64) - out["Q"])
            worst = max(worst, int(d.max()))
            den = np.outer(out["r"].astype(np.float64), out["c"].astype(np.float64))
            S32 = out["S_pre"].astype(np.float32).astype(np.float64)
            t = np.abs(np.divide(S32, den, out=np.zeros_like(S32), where=den > 0))
            at_tie = np.abs(t - np.floor(t) - 0.5) < TIE_DIST
            off_tie += int(np.sum((d > 0) & ~at_tie))
    return off_tie, worst


def compare_slots(gpu_bytes: np.ndarray, ora_bytes: np.ndarray, bits, dk=128, dv=128, row_bits=None) -> dict:
    """Compare slot images [n, slot_stride] head by head (FP16 pivot heads by binary16 ulps;
    heads of width 0 by their per-key-row widths row_bits [H, dk])."""
    offs, stride = O.head_offsets(bits, dk, dv, row_bits)
    res = dict(max_code_diff=0, flips=0, elements=0, r_ulp=0, c_ulp=0, byte_equal=True,
               pivot_ulp=0, pivot_flips=0, pivot_elements=0)
    for s in range(gpu_bytes.shape[0]):
        for h, b in enumerate(bits):
            o = int(offs[h])
            n = O.block_bytes(int(b), dk, dv) if int(b) else O.rows_block_bytes(row_bits[h], dv)
            g, r = gpu_bytes[s, o:o + n], ora_bytes[s, o:o + n]
            if int(b) == 16:
                d16 = fp16_ulp_diff(O.pivot_state(g, dk, dv), O.pivot_state(r, dk, dv))
                res["pivot_ulp"] = max(res["pivot_ulp"], int(d16.max()))
                res["pivot_flips"] += int((d16 > 0).sum())
                res["pivot_elements"] += d16.size
                res["byte_equal"] &= bool(np.array_equal(g, r))
                continue
            if np.array_equal(g, r):
                res["elements"] += dk * dv
                continue
            res["byte_equal"] = False
            if int(b):
                Qg, rg, cg = O.split_block(g, int(b), dk, dv)
                Qo, ro, co = O.split_block(r, int(b), dk, dv)
            else:
                Qg, rg, cg = O.rows_split_block(g, row_bits[h], dv)
                Qo, ro, co = O.rows_split_block(r, row_bits[h], dv)
            d = np.abs(Qg - Qo)
            res["max_code_diff"] = max(res["max_code_diff"], int(d.max()))
            res["flips"] += int((d > 0).sum())
            res["elements"] += d.size
            res["r_ulp"] = max(res["r_ulp"], int(ulp_diff(rg, ro).max()))
            res["c_ulp"] = max(res["c_ulp"], int(ulp_diff(cg, co).max()))
            nz = co != 0
            rel_all = np.zeros(co.shape)
            rel_all[nz] = np.abs(cg[nz].astype(np.float64) - co[nz]) / np.abs(co[nz])
            rel = rel_all[nz] if nz.any() else np.zeros(1)
            res["c_rel"] = max(res.get("c_rel", 0.0), float(rel.max()))
            res["c_far"] = res.get("c_far", 0) + int(np.sum(rel > C_REL_IMPACT))
            res["c_cols"] = res.get("c_cols", 0) + int(cg.size)
            # code flips outside the columns whose scale moved (impact fit, see C_FAR_RATE_IMPACT)
            near = rel_all <= C_REL_IMPACT
            res["flips_near"] = res.get("flips_near", 0) + int(((d > 0) & near[None, :]).sum())
            res["zero_c_mismatch"] = res.get("zero_c_mismatch", 0) + int(np.sum((co == 0) != (cg == 0)))
    return res


def y_max_rel(yg: np.ndarray, yo: np.ndarray) -> float:
    """Largest per-(request, head) max_j |dy_j| / max_j |y_j| (y shaped [..., dv])."""
    num = np.abs(yg - yo).max(axis=-1)
    den = np.abs(yo).max(axis=-1)
    den = np.where(den > 0, den, 1.0)
    return float((num / den).max())


def pivots_ok(res: dict) -> bool:
    """The FP16 pivot bar: every binary16 value within PIVOT_ULP, off-by-one at a rate of at
    most PIVOT_FLIP_RATE.  The kernel rounds an fp32-computed value to binary16, the oracle its
    fp64 value (to fp32, then binary16): they part only where the value lies within the fp32
    error of a binary16 rounding boundary, a share of about 2^-12 k of the values for an error
    of k fp32 ulps (k up to ~4 where the fade and the write nearly cancel).  Trajectories show
    3-4e-5; single steps from fresh random states more."""
    if res["pivot_elements"] == 0:
        return True
    return res["pivot_ulp"] <= PIVOT_ULP and res["pivot_flips"] <= max(1, PIVOT_FLIP_RATE * res["pivot_elements"])


def impact_scales_ok(res: dict) -> bool:
    """The impact-fit column-scale bar (see C_REL_IMPACT): c within 2e-5 relative except in at
    most a 1e-3 share of the compared columns, and zero exactly where the oracle's is zero."""
    cols = res.get("c_cols", 0)
    return res.get("zero_c_mismatch", 0) == 0 and res.get("c_far", 0) <= max(1, C_FAR_RATE_IMPACT * cols)
