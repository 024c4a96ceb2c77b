"""Seeded synthetic workloads for the quantized gated Delta-rule decode step.

This module only draws inputs: shapes, seeds and value distributions of the
serving workloads (many concurrent requests, hybrid-model head shapes).  It holds
none of the decode step's arithmetic; both the CUDA path and the CPU oracle
consume exactly the arrays produced here.

Recipes (the STEPQuant pages describe GDN/KDA hybrids served with many concurrent
requests; they print no input data, so every input is synthetic):
  q, k   ~ N(0, 1), then L2-normalised per (request, key head) vector
  v      ~ N(0, 1)
  beta   = sigmoid(N(0, 1))
  GDN    alpha = 2^(-1/h) per value head, h its half-life (constant over steps)
  KDA    alpha_i = exp(-softplus(x)), x ~ N(mu_h, 1), fresh per (request, head, step,
         key channel); mu_h set so that the head's mean-log-retention half-life
         ln 2 / E[softplus(x)] equals h_h, with h_h log-spaced over [2, 4096]
  bf16   inputs are rounded to bfloat16 (round to nearest even); every consumer
         uses the rounded values
Random streams: numpy PCG64 seeded by (seed, layer, phase, step); phase 0 is the
warm-up, phase 1 the timed trajectory, so any step can be redrawn on its own.
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np

GATE_GDN = 0
GATE_KDA = 1
DTYPE_FP32 = 0
DTYPE_BF16 = 1

PHASE_WARMUP = 0
PHASE_RUN = 1


# --------------------------------------------------------------------------- bf16

def to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """float32 -> bfloat16 bit patterns, round to nearest even (finite inputs)."""
    b = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    # no uint32 overflow for finite inputs: the largest pattern 0xFF7FFFFF + 0x8000 < 2^32
    b = (b + np.uint32(0x7FFF) + ((b >> np.uint32(16)) & np.uint32(1))) >> np.uint32(16)
    return b.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def round_bf16(x: np.ndarray) -> np.ndarray:
    return bf16_bits_to_f32(to_bf16_bits(x))


# --------------------------------------------------------------------------- workloads

@dataclasses.dataclass
class Workload:
    name: str
    B: int                    # concurrent requests
    H: int                    # value heads
    Hk: int                   # key heads (divides H; value head h reads key head h // (H // Hk))
    T: int                    # decode steps
    gate_mode: int            # GATE_GDN or GATE_KDA
    in_dtype: int             # DTYPE_FP32 or DTYPE_BF16 (q, k, v, alpha, beta)
    num_slots: int            # pool slots
    seed: int
    half_life: np.ndarray     # [layers, H] nominal half-life per head (GDN: exact; KDA: mean)
    slot_ids: np.ndarray      # [B] int32, distinct, in [0, num_slots)
    head_bits: np.ndarray | None = None   # [layers, H] fixed widths, or None (set by an allocator)
    avg_bits: float = 6.0     # nominal average width for the allocator
    n_pivots: int = 0         # FP16 pivot heads per layer chosen by the allocator
    layers: int = 1
    warmup_steps: int = 32
    kda_mu: np.ndarray | None = None      # [layers, H], or [layers, H, dk] (per-channel gates)
    row_half_life: np.ndarray | None = None   # [layers, H, dk]: per-key-row widths (KDA, unit = key row)
    dk: int = 128
    dv: int = 128

    @property
    def dtype_name(self) -> str:
        return "bf16" if self.in_dtype == DTYPE_BF16 else "f32"


def _rng(seed: int, *key: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, *key])))


def _softplus(x):
    return np.logaddexp(0.0, x)


def kda_mu_for_half_lives(h: np.ndarray) -> np.ndarray:
    """kda_mu_for_half_life over an array (vectorised bisection on the same quadrature)."""
    nodes, weights = np.polynomial.hermite_e.hermegauss(64)
    weights = weights / weights.sum()
    target = math.log(2.0) / np.asarray(h, dtype=np.float64)
    lo = np.full(target.shape, -40.0)
    hi = np.full(target.shape, 10.0)
    for _ in range(200):
        mid = 0.5 * (lo + hi)
        ms = (_softplus(mid[..., None] + nodes) * weights).sum(-1)
        big = ms > target
        hi = np.where(big, mid, hi)
        lo = np.where(big, lo, mid)
    return 0.5 * (lo + hi)


def kda_mu_for_half_life(h: float) -> float:
    """mu such that ln2 / E[softplus(x)] = h for x ~ N(mu, 1) (64-node Gauss-Hermite, bisection)."""
    nodes, weights = np.polynomial.hermite_e.hermegauss(64)
    weights = weights / weights.sum()
    target = math.log(2.0) / h

    def mean_softplus(mu):
        return float(np.dot(weights, _softplus(mu + nodes)))

    lo, hi = -40.0, 10.0
    for _ in range(200):
        mid = 0.5 * (lo + hi)
        if mean_softplus(mid) > target:
            hi = mid
        else:
            lo = mid
    return 0.5 * (lo + hi)


def _loguniform_half_life(seed: int, layers: int, H: int) -> np.ndarray:
    r = _rng(seed, 1000)
    return np.exp(r.uniform(0.0, math.log(4096.0), size=(layers, H)))


def make_workload(config: int, variant: str = "mixed6", batch: int | None = None) -> Workload:
    """The five serving workloads, shaped like the pages' many-request hybrid-model serving.

    1  GDN toy: B=4, H=Hk=4, T=16, fp32, half-lives [2,32,512,4096], bits [4,6,8,8], seed 0
    2  GDN hybrid layer: B=64, H=32, Hk=16, T=64, bf16, log-uniform half-lives, 6-bit nominal
    3  KDA layer: B=256, H=Hk=32, T=64, bf16, per-channel gates, 6-bit nominal
    4  high-concurrency GDN pool: B=512 of 1024 slots (random slot ids), H=32, Hk=16, T=256,
       bf16; variant "mixed6" (6-bit nominal) or "uniform4"
    Variant "mixed6p" (configs 2-4): 6-bit nominal plus one FP16 pivot head per layer, the
    smallest nonzero share at 32 heads (the pages keep 1.39% of the heads in FP16)
    5  36-layer GDN stack: H=32, Hk=16, T=32 per layer, B in {64, 256, 1024} (``batch``), bf16
    """
    if variant not in ("mixed6", "mixed6p", "uniform4", "rowbits") or (variant == "uniform4" and config != 4) \
            or (variant == "mixed6p" and config not in (2, 3, 4)) or (variant == "rowbits" and config != 3):
        raise ValueError("variant %r of workload %r" % (variant, config))
    w = _make_workload(config, variant, batch)
    if variant == "rowbits":
        # every key channel its own mean gate: half-lives log-uniform over [2, 4096] per
        # (head, channel); the allocation unit is the key row
        rhl = np.exp(_rng(w.seed, 0, 6000).uniform(math.log(2.0), math.log(4096.0), (1, w.H, w.dk)))
        w.row_half_life = rhl
        w.kda_mu = kda_mu_for_half_lives(rhl)
        w.name += "_rowbits"
    if variant == "mixed6p":
        w.n_pivots = 1
        w.name += "_p"
    return w


def _make_workload(config: int, variant: str, batch: int | None) -> Workload:
    if config == 1:
        return Workload("gdn_toy", B=4, H=4, Hk=4, T=16, gate_mode=GATE_GDN, in_dtype=DTYPE_FP32,
                        num_slots=4, seed=0,
                        half_life=np.array([[2.0, 32.0, 512.0, 4096.0]]),
                        slot_ids=np.arange(4, dtype=np.int32),
                        head_bits=np.array([[4, 6, 8, 8]], dtype=np.int32))
    if config == 2:
        return Workload("gdn_hybrid", B=64, H=32, Hk=16, T=64, gate_mode=GATE_GDN,
                        in_dtype=DTYPE_BF16, num_slots=64, seed=2,
                        half_life=_loguniform_half_life(2, 1, 32),
                        slot_ids=np.arange(64, dtype=np.int32))
    if config == 3:
        hl = np.exp(np.linspace(math.log(2.0), math.log(4096.0), 32))[None, :]
        mu = np.array([[kda_mu_for_half_life(h) for h in hl[0]]])
        return Workload("kda", B=256, H=32, Hk=32, T=64, gate_mode=GATE_KDA, in_dtype=DTYPE_BF16,
                        num_slots=256, seed=3, half_life=hl, kda_mu=mu,
                        slot_ids=np.arange(256, dtype=np.int32))
    if config == 4:
        perm = _rng(4, 2000).permutation(1024).astype(np.int32)
        w = Workload("gdn_pool_" + variant.rstrip("p"), B=512, H=32, Hk=16, T=256, gate_mode=GATE_GDN,
                     in_dtype=DTYPE_BF16, num_slots=1024, seed=4,
                     half_life=_loguniform_half_life(4, 1, 32), slot_ids=perm[:512])
        if variant == "uniform4":
            w.head_bits = np.full((1, 32), 4, dtype=np.int32)
        return w
    if config == 5:
        B = 1024 if batch is None else int(batch)
        if B not in (64, 256, 1024):
            raise ValueError("stack sweep batch must be 64, 256 or 1024")
        return Workload("gdn_stack_b%d" % B, B=B, H=32, Hk=16, T=32, gate_mode=GATE_GDN,
                        in_dtype=DTYPE_BF16, num_slots=B, seed=5, layers=36,
                        half_life=_loguniform_half_life(5, 36, 32),
                        slot_ids=np.arange(B, dtype=np.int32))
    raise ValueError("unknown workload %r" % config)


def impact_scores(w: Workload, layer: int = 0) -> np.ndarray:
    """Synthetic row-impact scores [H, d_k] for the impact-weighted fit: positive, spread over
    about two decades (log-normal, sigma 1.2), seeded by (seed, layer).  The pages calibrate
    them as expected squared readout weights over WikiText-2 tokens; no model or data here."""
    return np.exp(_rng(w.seed, layer, 7000).normal(0.0, 1.2, (w.H, w.dk))).astype(np.float32)


# --------------------------------------------------------------------------- per-step inputs

def step_inputs(w: Workload, t: int, phase: int = PHASE_RUN, layer: int = 0) -> dict:
    """Inputs of decode step t: float32 arrays holding exactly the values every consumer uses.

    Keys: q, k [B, Hk, dk]; v [B, H, dv]; beta [B, H]; alpha [B, H] (GDN) or
    [B, H, dk] (KDA)."""
    r = _rng(w.seed, layer, phase, t)
    B, H, Hk, dk, dv = w.B, w.H, w.Hk, w.dk, w.dv
    f32 = np.float32
    q = r.standard_normal((B, Hk, dk), dtype=f32)
    k = r.standard_normal((B, Hk, dk), dtype=f32)
    q /= np.sqrt(np.einsum("bhd,bhd->bh", q, q))[..., None]
    k /= np.sqrt(np.einsum("bhd,bhd->bh", k, k))[..., None]
    v = r.standard_normal((B, H, dv), dtype=f32)
    beta = 1.0 / (1.0 + np.exp(-r.standard_normal((B, H), dtype=f32)))
    if w.gate_mode == GATE_GDN:
        alpha = np.broadcast_to((2.0 ** (-1.0 / w.half_life[layer])).astype(f32), (B, H))
    else:
        mu = np.asarray(w.kda_mu[layer])
        x = r.standard_normal((B, H, dk)) + (mu[None, :, None] if mu.ndim == 1 else mu[None, :, :])
        alpha = np.exp(-_softplus(x))
    out = dict(q=q, k=k, v=v, beta=beta, alpha=alpha)
    for key in out:
        a = np.ascontiguousarray(out[key], dtype=np.float32)
        out[key] = round_bf16(a) if w.in_dtype == DTYPE_BF16 else a
    return out


def as_device_dtype(w: Workload, x: np.ndarray) -> np.ndarray:
    """Host array in the dtype the device path reads: float32, or bf16 bit patterns (uint16)."""
    return to_bf16_bits(x) if w.in_dtype == DTYPE_BF16 else np.ascontiguousarray(x, dtype=np.float32)


def sample_requests(w: Workload, count: int, seed_key: int = 3000) -> np.ndarray:
    """A seeded sample of request indices (sorted), always including the first and last."""
    if count >= w.B:
        return np.arange(w.B)
    r = _rng(w.seed, seed_key)
    pick = set(r.choice(w.B, size=max(count - 2, 0), replace=False).tolist()) | {0, w.B - 1}
    return np.array(sorted(pick))
