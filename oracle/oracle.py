"""Python face of the CPU oracle for the quantized gated Delta-rule decode step.

TEST INFRASTRUCTURE ONLY: the tests, the smoke check and the CPU-baseline leg of
the benchmark may import this module; the product path never does.  It shares
no code with the CUDA path.  The arithmetic lives in ``stepq_oracle.c`` (plain C,
double precision); this module compiles it with gcc on first use, marshals numpy
arrays into it, and holds the plain-Python bit-allocation oracle.

Citations name the web pages on STEPQuant (arXiv 2609.38169) by title and section:
  [SUM]  hyper.ai paper summary, "Method"
  [EXP]  "Paper Explained: STEPQuant -- When and Where Quantization Errors Matter in
         Delta-Rule Recurrent States", "The mechanism: rewriting state with the delta rule"
         and "The intuition: errors get carried forward"
  [BLOG] ONTLE blog post on STEPQuant, paragraphs on lifetime-aware bit allocation
"""
from __future__ import annotations

import ctypes
import itertools
import math
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "stepq_oracle.c")
_LIB = os.path.join(_HERE, "liboracle_stepq.so")
GCC_FLAGS = ["-O2", "-std=c11", "-fopenmp", "-fno-fast-math", "-ffp-contract=off",
             "-shared", "-fPIC", "-Wall", "-Wextra"]

_lib = None


def build(force: bool = False) -> str:
    """Compile the C oracle into ``liboracle_stepq.so`` next to its source."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + ".tmp.%d" % os.getpid()
        subprocess.check_call(["gcc", *GCC_FLAGS, "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is not None:
        return _lib
    lib = ctypes.CDLL(build())
    P = ctypes.c_void_p
    I = ctypes.c_int
    L = ctypes.c_long
    F = ctypes.c_float
    sig = {
        "oracle_qmax": (I, [I]),
        "oracle_codes_bytes": (L, [I, I, I]),
        "oracle_block_bytes": (L, [I, I, I]),
        "oracle_pack_codes": (None, [I, I, I, P, P]),
        "oracle_unpack_codes": (None, [I, I, I, P, P]),
        "oracle_quantize": (I, [I, I, I, P, P, P, P]),
        "oracle_dequantize": (None, [I, I, P, P, P, P]),
        "oracle_delta_step": (None, [I, I, P, P, P, P, P, F, P]),
        "oracle_step_state": (I, [I, I, I, P, P, P, P, P, P, P, F, P, P, P, P, P]),
        "oracle_head_offsets": (L, [I, P, I, I, P, P]),
        "oracle_decode_step": (L, [I, I, I, I, I, P, I, P, P, I, P, P, P, P, P, P, I, P, P]),
        "oracle_pool_load": (L, [I, I, I, P, I, P, P, I, P, I, P, P]),
        "oracle_impact_normalize": (None, [I, P, P]),
        "oracle_quantize_impact": (I, [I, I, I, P, P, P, P, P]),
        "oracle_pool_dump": (I, [I, I, I, P, I, P, P, I, P, I, P]),
        "oracle_rows_order": (None, [I, P, P]),
        "oracle_rows_panel_bytes": (L, [I, P]),
        "oracle_rows_block_bytes": (L, [I, I, P]),
        "oracle_rows_pack": (None, [I, I, P, P, P]),
        "oracle_rows_unpack": (None, [I, I, P, P, P]),
        "oracle_rows_quantize": (I, [I, I, P, P, P, P, P]),
        "oracle_fp_decode_step": (None, [I, I, I, I, I, I, P, P, P, P, P, P, P, I, I]),
        "oracle_fp16_encode": (None, [L, P, P]),
        "oracle_fp16_decode": (None, [L, P, P]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib


def _p(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def default_threads() -> int:
    return max(1, len(os.sched_getaffinity(0)))


# --------------------------------------------------------------------------- layout

def qmax(bits: int) -> int:
    return _load().oracle_qmax(bits)


def codes_bytes(bits: int, dk: int = 128, dv: int = 128) -> int:
    return _load().oracle_codes_bytes(bits, dk, dv)


def block_bytes(bits: int, dk: int = 128, dv: int = 128) -> int:
    return _load().oracle_block_bytes(bits, dk, dv)


def head_offsets(head_bits, dk: int = 128, dv: int = 128, row_bits=None):
    """(offsets[H], slot_stride) of the head blocks inside one slot (a head of width 0 takes
    its per-key-row widths from row_bits [H, dk])."""
    hb = _c(head_bits, np.int32)
    off = np.zeros(len(hb), dtype=np.int64)
    rb = None if row_bits is None else _c(row_bits, np.int32)
    stride = _load().oracle_head_offsets(len(hb), _p(hb), dk, dv, _p(off), None if rb is None else _p(rb))
    return off, int(stride)


# --------------------------------------------------------------------------- per-key-row widths

def rows_order(rb) -> np.ndarray:
    """Stored position -> key row of a head with per-row widths rb [dk]."""
    rb = _c(rb, np.int32)
    out = np.zeros(len(rb), dtype=np.int32)
    _load().oracle_rows_order(len(rb), _p(rb), _p(out))
    return out


def rows_block_bytes(rb, dv: int = 128) -> int:
    rb = _c(rb, np.int32)
    return int(_load().oracle_rows_block_bytes(len(rb), dv, _p(rb)))


def rows_pack(Q: np.ndarray, rb) -> np.ndarray:
    Q = _c(Q, np.int32)
    rb = _c(rb, np.int32)
    dk, dv = Q.shape
    out = np.zeros(rows_block_bytes(rb, dv) - 4 * dk - 4 * dv, dtype=np.uint8)
    _load().oracle_rows_pack(dk, dv, _p(rb), _p(Q), _p(out))
    return out


def rows_unpack(buf: np.ndarray, rb, dv: int = 128) -> np.ndarray:
    buf = _c(buf, np.uint8)
    rb = _c(rb, np.int32)
    Q = np.zeros((len(rb), dv), dtype=np.int32)
    _load().oracle_rows_unpack(len(rb), dv, _p(rb), _p(buf), _p(Q))
    return Q


def rows_split_block(blk: np.ndarray, rb, dv: int = 128):
    """Per-row head block -> (Q [dk, dv], r [dk] by key row, c [dv])."""
    rb = _c(rb, np.int32)
    dk = len(rb)
    blk = _c(blk, np.uint8)
    cb = rows_block_bytes(rb, dv) - 4 * dk - 4 * dv
    Q = rows_unpack(blk[:cb], rb, dv)
    r = np.zeros(dk, dtype=np.float32)
    r[rows_order(rb)] = blk[cb:cb + 4 * dk].view(np.float32)
    c = blk[cb + 4 * dk:cb + 4 * dk + 4 * dv].view(np.float32).copy()
    return Q, r, c


def rows_quantize(S32: np.ndarray, rb):
    """Clip-free fit at each row's own levels -> (Q, r, c, clipped)."""
    S32 = _c(S32, np.float32)
    rb = _c(rb, np.int32)
    dk, dv = S32.shape
    Q = np.zeros((dk, dv), dtype=np.int32)
    r = np.zeros(dk, dtype=np.float32)
    c = np.zeros(dv, dtype=np.float32)
    n = _load().oracle_rows_quantize(dk, dv, _p(rb), _p(S32), _p(Q), _p(r), _p(c))
    return Q, r, c, int(n)


def pack_codes(Q: np.ndarray, bits: int) -> np.ndarray:
    Q = _c(Q, np.int32)
    dk, dv = Q.shape
    out = np.zeros(codes_bytes(bits, dk, dv), dtype=np.uint8)
    _load().oracle_pack_codes(bits, dk, dv, _p(Q), _p(out))
    return out


def unpack_codes(buf: np.ndarray, bits: int, dk: int = 128, dv: int = 128) -> np.ndarray:
    buf = _c(buf, np.uint8)
    Q = np.zeros((dk, dv), dtype=np.int32)
    _load().oracle_unpack_codes(bits, dk, dv, _p(buf), _p(Q))
    return Q


def split_block(blk: np.ndarray, bits: int, dk: int = 128, dv: int = 128):
    """Head block bytes -> (codes Q [dk,dv] int32, r [dk] fp32, c [dv] fp32)."""
    blk = _c(blk, np.uint8)
    cb = codes_bytes(bits, dk, dv)
    Q = unpack_codes(blk[:cb], bits, dk, dv)
    r = blk[cb:cb + 4 * dk].view(np.float32).copy()
    c = blk[cb + 4 * dk:cb + 4 * dk + 4 * dv].view(np.float32).copy()
    return Q, r, c


def fp16_encode(x) -> np.ndarray:
    """Nearest binary16 values of x (float64 array, ties to even), as uint16 bit patterns."""
    x = _c(x, np.float64)
    out = np.zeros(x.shape, dtype=np.uint16)
    _load().oracle_fp16_encode(x.size, _p(x), _p(out))
    return out


def fp16_decode(h) -> np.ndarray:
    h = _c(h, np.uint16)
    out = np.zeros(h.shape, dtype=np.float64)
    _load().oracle_fp16_decode(h.size, _p(h), _p(out))
    return out


def pivot_state(blk: np.ndarray, dk: int = 128, dv: int = 128) -> np.ndarray:
    """FP16 pivot head block bytes -> the state's binary16 bit patterns [dk, dv]."""
    return _c(blk, np.uint8)[:2 * dk * dv].view(np.uint16).reshape(dk, dv).copy()


def impact_normalize(omega) -> np.ndarray:
    """Row-impact scores normalized to mean 1 (fp32 of the double quotient)."""
    omega = _c(omega, np.float32)
    w = np.zeros(omega.shape, dtype=np.float32)
    _load().oracle_impact_normalize(len(omega), _p(omega), _p(w))
    return w


def quantize_impact(S32: np.ndarray, bits: int, w):
    """Impact-weighted fit of an fp32 state with normalized weights w -> (Q, r, c, clipped)."""
    S32 = _c(S32, np.float32)
    dk, dv = S32.shape
    Q = np.zeros((dk, dv), dtype=np.int32)
    r = np.zeros(dk, dtype=np.float32)
    c = np.zeros(dv, dtype=np.float32)
    n = _load().oracle_quantize_impact(bits, dk, dv, _p(S32), _p(_c(w, np.float32)), _p(Q), _p(r), _p(c))
    return Q, r, c, int(n)


def make_block(Q, r, c, bits: int) -> np.ndarray:
    Q = _c(Q, np.int32)
    dk, dv = Q.shape
    return np.concatenate([pack_codes(Q, bits), _c(r, np.float32).view(np.uint8),
                           _c(c, np.float32).view(np.uint8)])


# --------------------------------------------------------------------------- one state

def quantize(S32: np.ndarray, bits: int):
    """Dual-axis clip-free fit + nearest-level codes of an fp32 state ([SUM] Method).

    Returns (Q int32 [dk,dv], r fp32 [dk], c fp32 [dv], clip_count)."""
    S32 = _c(S32, np.float32)
    dk, dv = S32.shape
    Q = np.zeros((dk, dv), dtype=np.int32)
    r = np.zeros(dk, dtype=np.float32)
    c = np.zeros(dv, dtype=np.float32)
    clipped = _load().oracle_quantize(bits, dk, dv, _p(S32), _p(Q), _p(r), _p(c))
    return Q, r, c, clipped


def dequantize(Q, r, c) -> np.ndarray:
    """S_hat = Q * r_i * c_j in double."""
    Q = _c(Q, np.int32)
    r = _c(r, np.float32)
    c = _c(c, np.float32)
    dk, dv = Q.shape
    S = np.zeros((dk, dv), dtype=np.float64)
    _load().oracle_dequantize(dk, dv, _p(Q), _p(r), _p(c), _p(S))
    return S


def delta_step(S: np.ndarray, q, k, v, alpha, beta: float):
    """Unquantized gated Delta-rule step ([EXP] mechanism) on a copy of a double state.

    alpha is a scalar (GDN) or a [dk] vector (KDA).  Returns (S_new, y) in double."""
    S = np.array(S, dtype=np.float64, order="C")
    dk, dv = S.shape
    al = _c(np.broadcast_to(np.asarray(alpha, dtype=np.float32), (dk,)), np.float32)
    y = np.zeros(dv, dtype=np.float64)
    _load().oracle_delta_step(dk, dv, _p(S), _p(_c(q, np.float32)), _p(_c(k, np.float32)),
                              _p(_c(v, np.float32)), _p(al), float(beta), _p(y))
    return S, y


def step_state(Q, r, c, bits: int, q, k, v, alpha, beta: float):
    """One quantized decode step of one state.

    Returns dict(Q, r, c, y (fp32), S_pre (double, the updated state before
    quantization), clipped)."""
    Q = _c(Q, np.int32)
    dk, dv = Q.shape
    al = _c(np.broadcast_to(np.asarray(alpha, dtype=np.float32), (dk,)), np.float32)
    Qo = np.zeros_like(Q)
    ro = np.zeros(dk, dtype=np.float32)
    co = np.zeros(dv, dtype=np.float32)
    y = np.zeros(dv, dtype=np.float32)
    S_pre = np.zeros((dk, dv), dtype=np.float64)
    clipped = _load().oracle_step_state(
        dk, dv, bits, _p(Q), _p(_c(r, np.float32)), _p(_c(c, np.float32)),
        _p(_c(q, np.float32)), _p(_c(k, np.float32)), _p(_c(v, np.float32)), _p(al), float(beta),
        _p(Qo), _p(ro), _p(co), _p(y), _p(S_pre))
    return dict(Q=Qo, r=ro, c=co, y=y, S_pre=S_pre, clipped=clipped)


# --------------------------------------------------------------------------- pools

class OraclePool:
    """Host pool with the packed layout: slot-major, heads in order, each head block
    = [codes | r fp32[dk] | c fp32[dv]] (an FP16 pivot head, width 16: the state as
    binary16 values).  A zeroed pool is the zero state."""

    def __init__(self, num_slots: int, head_bits, num_key_heads: int, gate_mode: int = 0,
                 dk: int = 128, dv: int = 128, impact=None, row_bits=None):
        self.head_bits = _c(head_bits, np.int32)
        self.H = len(self.head_bits)
        self.Hk = int(num_key_heads)
        if self.H % self.Hk:
            raise ValueError("key heads must divide value heads")
        self.dk, self.dv = dk, dv
        self.gate_mode = int(gate_mode)
        self.num_slots = int(num_slots)
        self.row_bits = None if row_bits is None else _c(row_bits, np.int32)
        if (self.head_bits == 0).any():
            assert self.row_bits is not None and self.row_bits.shape == (self.H, dk)
        self.offsets, self.slot_stride = head_offsets(self.head_bits, dk, dv, self.row_bits)
        self.data = np.zeros(self.num_slots * self.slot_stride, dtype=np.uint8)
        # row-impact scores [H, dk] -> the impact-weighted fit for every quantized head
        self.impact_w = None
        if impact is not None:
            impact = _c(impact, np.float32)
            assert impact.shape == (self.H, dk) and (impact > 0).all()
            self.impact_w = np.stack([impact_normalize(row) for row in impact])

    def block_size(self, h: int) -> int:
        b = int(self.head_bits[h])
        return block_bytes(b, self.dk, self.dv) if b else rows_block_bytes(self.row_bits[h], self.dv)

    def block(self, slot: int, h: int) -> np.ndarray:
        o = slot * self.slot_stride + int(self.offsets[h])
        return self.data[o:o + self.block_size(h)]

    def state(self, slot: int, h: int):
        """(Q, r, c) of a quantized head; the binary16 bit patterns of an FP16 pivot head."""
        if int(self.head_bits[h]) == 16:
            return pivot_state(self.block(slot, h), self.dk, self.dv)
        if int(self.head_bits[h]) == 0:
            return rows_split_block(self.block(slot, h), self.row_bits[h], self.dv)
        return split_block(self.block(slot, h), int(self.head_bits[h]), self.dk, self.dv)

    def set_state(self, slot: int, h: int, Q, r, c):
        self.block(slot, h)[:] = make_block(Q, r, c, int(self.head_bits[h]))

    def _rb(self):
        return None if self.row_bits is None else _p(self.row_bits)

    def slot_bytes(self, slot_ids) -> np.ndarray:
        s = self.slot_stride
        return np.stack([self.data[int(i) * s:(int(i) + 1) * s] for i in slot_ids])

    def load_fp32(self, slot_ids, S, nthreads: int | None = None) -> int:
        """Quantize fp32 states S [n, H, dk, dv] into the given slots."""
        sl = _c(slot_ids, np.int32)
        S = _c(S, np.float32)
        assert S.shape == (len(sl), self.H, self.dk, self.dv)
        rc = _load().oracle_pool_load(self.H, self.dk, self.dv, _p(self.head_bits), self.num_slots,
                                      _p(self.data), _p(sl), len(sl), _p(S), nthreads or default_threads(),
                                      None if self.impact_w is None else _p(self.impact_w), self._rb())
        if rc < 0:
            raise IndexError("slot id out of range")
        return int(rc)

    def dump_fp32(self, slot_ids, nthreads: int | None = None) -> np.ndarray:
        sl = _c(slot_ids, np.int32)
        S = np.zeros((len(sl), self.H, self.dk, self.dv), dtype=np.float32)
        rc = _load().oracle_pool_dump(self.H, self.dk, self.dv, _p(self.head_bits), self.num_slots,
                                      _p(self.data), _p(sl), len(sl), _p(S), nthreads or default_threads(),
                                      self._rb())
        if rc < 0:
            raise IndexError("slot id out of range")
        return S

    def decode_step(self, slot_ids, q, k, v, alpha, beta, nthreads: int | None = None) -> np.ndarray:
        """One quantized decode step for the requests in slot_ids; returns y [n, H, dv] fp32."""
        sl = _c(slot_ids, np.int32)
        n = len(sl)
        q = _c(q, np.float32)
        k = _c(k, np.float32)
        v = _c(v, np.float32)
        alpha = _c(alpha, np.float32)
        beta = _c(beta, np.float32)
        assert q.shape == (n, self.Hk, self.dk) and k.shape == q.shape
        assert v.shape == (n, self.H, self.dv) and beta.shape == (n, self.H)
        assert alpha.shape == ((n, self.H) if self.gate_mode == 0 else (n, self.H, self.dk))
        y = np.zeros((n, self.H, self.dv), dtype=np.float32)
        rc = _load().oracle_decode_step(self.H, self.Hk, self.dk, self.dv, self.gate_mode,
                                        _p(self.head_bits), self.num_slots, _p(self.data), _p(sl), n,
                                        _p(q), _p(k), _p(v), _p(alpha), _p(beta), _p(y),
                                        nthreads or default_threads(),
                                        None if self.impact_w is None else _p(self.impact_w), self._rb())
        if rc < 0:
            raise IndexError("slot id out of range")
        if rc > 0:
            raise AssertionError("oracle fit clipped %d codes" % rc)
        return y


def fp_decode_step(S: np.ndarray, Hk: int, gate_mode: int, q, k, v, alpha, beta,
                   round_fp32: bool, nthreads: int | None = None) -> np.ndarray:
    """Unquantized step on double states S [n, H, dk, dv] in place; returns y [n, H, dv]."""
    assert S.dtype == np.float64 and S.flags.c_contiguous
    n, H, dk, dv = S.shape
    y = np.zeros((n, H, dv), dtype=np.float32)
    _load().oracle_fp_decode_step(H, Hk, dk, dv, gate_mode, n, _p(S), _p(_c(q, np.float32)),
                                  _p(_c(k, np.float32)), _p(_c(v, np.float32)),
                                  _p(_c(alpha, np.float32)), _p(_c(beta, np.float32)), _p(y),
                                  1 if round_fp32 else 0, nthreads or default_threads())
    return y


# --------------------------------------------------------------------------- bit allocation
# [SUM] Method para 2; [BLOG] lifetime-aware bit allocation.  Reading: lifetime of a
# unit from its mean log retention, rho = exp(mean log alpha) = 2^(-1/half_life);
# error retention after j updates ~ rho^j, so the lifetime weight is
# sum_j rho^j = 1 / (1 - rho); choose widths from the candidate set minimising
# sum_u w_u * D_u(b_u) subject to sum_u b_u <= N * avg_bits.  Without a measured
# distortion table, D_u(b) = 2^(-2b) (a uniform quantizer's error power scaling).

def lifetime_weight(half_life: float) -> float:
    rho = 2.0 ** (-1.0 / half_life)
    return 1.0 / (1.0 - rho)


def _distortion(distortion, u: int, ci: int, cand) -> float:
    if distortion is None:
        return 2.0 ** (-2 * cand[ci])
    return float(distortion[u][ci])


def allocation_objective(bits, half_life, distortion, cand) -> float:
    cand = list(cand)
    return sum(lifetime_weight(h) * _distortion(distortion, u, cand.index(b), cand)
               for u, (b, h) in enumerate(zip(bits, half_life)))


def allocate_bits_bruteforce(half_life, distortion, cand, avg_bits):
    """Exhaustive search over every assignment (tiny N only)."""
    N = len(half_life)
    budget = math.floor(N * avg_bits + 1e-9)
    best, best_bits = None, None
    for combo in itertools.product(range(len(cand)), repeat=N):
        if sum(cand[c] for c in combo) > budget:
            continue
        obj = sum(lifetime_weight(half_life[u]) * _distortion(distortion, u, combo[u], cand)
                  for u in range(N))
        if best is None or obj < best:
            best, best_bits = obj, [cand[c] for c in combo]
    return best_bits, best


def select_pivots(half_life, distortion, cand, n_pivots: int):
    """Indices of the FP16 pivot units ([SUM] Method para 2: the highest-risk units are kept
    in FP16).  Reading: risk = lifetime weight x the distortion left at the widest candidate
    width; the n_pivots units of highest risk, ties to the lower index."""
    cand = list(cand)
    top = cand.index(max(cand))
    risk = [(-lifetime_weight(h) * _distortion(distortion, u, top, cand), u) for u, h in enumerate(half_life)]
    return sorted(u for _, u in sorted(risk)[:n_pivots])


def allocate_bits_pivots(half_life, distortion, cand, avg_bits, n_pivots: int):
    """Pivots first (width 16, outside the budget), then the exact DP over the other units
    with the budget floor((N - n_pivots) * avg_bits)."""
    piv = set(select_pivots(half_life, distortion, cand, n_pivots))
    rest = [u for u in range(len(half_life)) if u not in piv]
    sub_d = None if distortion is None else [distortion[u] for u in rest]
    bits_rest, obj = allocate_bits_dp([half_life[u] for u in rest], sub_d, cand, avg_bits)
    bits = [16] * len(half_life)
    for u, b in zip(rest, bits_rest):
        bits[u] = b
    return bits, obj


def allocate_bits_dp_vec(half_life, distortion, cand, avg_bits):
    """The same exact programme vectorised over the bits spent (numpy), for thousands of
    units (one unit per key row).  Ties resolve as in the library's allocator: for each total
    the widest candidate that reaches the best value first, then the smallest total."""
    N = len(half_life)
    budget = math.floor(N * avg_bits + 1e-9)
    cand = list(cand)
    order = sorted(range(len(cand)), key=lambda ci: -cand[ci])          # widest first
    best = np.full(budget + 1, np.inf)
    best[0] = 0.0
    choice = np.full((N, budget + 1), -1, dtype=np.int8)
    for u in range(N):
        w = -1.0 / math.expm1(-math.log(2.0) / half_life[u])
        nxt = np.full(budget + 1, np.inf)
        pick = np.full(budget + 1, -1, dtype=np.int8)
        for ci in order:
            b = cand[ci]
            v = np.full(budget + 1, np.inf)
            if b <= budget:                      # a width above the whole budget never fits
                v[b:] = best[:budget + 1 - b] + w * _distortion(distortion, u, ci, cand)
            better = v < nxt
            nxt = np.where(better, v, nxt)
            pick = np.where(better, ci, pick)
        best, choice[u] = nxt, pick
    if not np.isfinite(best).any():
        raise ValueError("budget too small for the candidate widths")
    s = int(np.argmin(best))
    bits = [0] * N
    for u in range(N - 1, -1, -1):
        ci = int(choice[u, s])
        bits[u] = cand[ci]
        s -= cand[ci]
    return bits, float(np.min(best))


def allocate_bits_dp(half_life, distortion, cand, avg_bits):
    """Exact dynamic programme over the bits spent so far (any N)."""
    N = len(half_life)
    budget = math.floor(N * avg_bits + 1e-9)
    INF = float("inf")
    # best[s] = (objective, choices) over the units seen so far, spending exactly s bits
    best = {0: (0.0, [])}
    for u in range(N):
        w = lifetime_weight(half_life[u])
        nxt = {}
        for s, (obj, ch) in best.items():
            for ci, b in enumerate(cand):
                s2 = s + b
                if s2 > budget:
                    continue
                o2 = obj + w * _distortion(distortion, u, ci, cand)
                if o2 < nxt.get(s2, (INF, None))[0]:
                    nxt[s2] = (o2, ch + [b])
        best = nxt
    if not best:
        raise ValueError("budget too small for the candidate widths")
    obj, ch = min(best.values(), key=lambda t: t[0])
    return ch, obj
