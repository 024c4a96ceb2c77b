"""ctypes binding of libstepq, with the names of the C ABI in include/stepq.h.

Argument marshalling only: tensors are passed by device pointer, every step of the
decode path runs in the library's CUDA kernels.  The library must be built
(``python quantized_gated_delta_b200/build.py``); importing a missing or stale
library raises instead of falling back to anything else.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libstepq.so")

STEPQ_OK = 0
STEPQ_GATE_GDN = 0
STEPQ_GATE_KDA = 1
STEPQ_DTYPE_F32 = 0
STEPQ_DTYPE_BF16 = 1
STEPQ_FLAG_BAD_SLOT = 1
STEPQ_FLAG_TIMEOUT = 2
STEPQ_DEBUG_SLOTS = 1

EXPORTED = [
    "stepq_pool_create", "stepq_pool_destroy", "stepq_pool_bytes", "stepq_pool_head_offset",
    "stepq_pool_load_fp32", "stepq_pool_load_packed", "stepq_pool_dump_fp32",
    "stepq_pool_dump_packed", "stepq_decode_step", "stepq_pool_get_error",
    "stepq_allocate_bits", "stepq_status_string", "stepq_decode_step_noalloc",
    "stepq_allocate_bits_pivots", "stepq_pool_set_impact", "stepq_pool_create_rows",
    "stepq_check_wait_timeout", "stepq_decode_step_host", "stepq_pool_host_wait",
    "stepq_pool_set_debug", "stepq_check_slot_ids", "stepq_host_image_layout",
]


class StepqError(RuntimeError):
    def __init__(self, status: int, what: str):
        super().__init__("%s failed: %s (%d)" % (what, stepq_status_string(status), status))
        self.status = status


class stepq_pool_desc(ctypes.Structure):
    _fields_ = [("num_slots", ctypes.c_int32), ("num_heads", ctypes.c_int32),
                ("num_key_heads", ctypes.c_int32), ("d_k", ctypes.c_int32), ("d_v", ctypes.c_int32),
                ("gate_mode", ctypes.c_int32), ("in_dtype", ctypes.c_int32),
                ("head_bits", ctypes.POINTER(ctypes.c_uint8))]


_lib = None


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError("libstepq.so is not built (run: python quantized_gated_delta_b200/build.py)")
    lib = ctypes.CDLL(path)
    P, I, Z = ctypes.c_void_p, ctypes.c_int32, ctypes.c_size_t
    sig = {
        "stepq_pool_create": [ctypes.POINTER(stepq_pool_desc), ctypes.POINTER(P)],
        "stepq_pool_destroy": [P],
        "stepq_pool_bytes": [P, ctypes.POINTER(Z), ctypes.POINTER(Z)],
        "stepq_pool_head_offset": [P, I, ctypes.POINTER(Z)],
        "stepq_pool_load_fp32": [P, P, I, P, P],
        "stepq_pool_load_packed": [P, P, I, P, P],
        "stepq_pool_dump_fp32": [P, P, I, P, P],
        "stepq_pool_dump_packed": [P, P, I, P, P],
        "stepq_decode_step": [P, P, I, P, P, P, P, P, P, P],
        "stepq_pool_get_error": [P, ctypes.POINTER(I)],
        "stepq_allocate_bits": [P, P, I, P, I, ctypes.c_double, P],
        "stepq_allocate_bits_pivots": [P, P, I, P, I, ctypes.c_double, I, P],
        "stepq_pool_set_impact": [P, P],
        "stepq_check_wait_timeout": [ctypes.POINTER(I), P],
        "stepq_decode_step_host": [P, P, I, P, P, P, P, P, P, P],
        "stepq_pool_host_wait": [P, P],
        "stepq_pool_create_rows": [ctypes.POINTER(stepq_pool_desc), P, ctypes.POINTER(P)],
        "stepq_decode_step_noalloc": [ctypes.POINTER(stepq_pool_desc), P, P, I, P, P, P, P, P, P, P, P],
        "stepq_pool_set_debug": [P, I],
        "stepq_check_slot_ids": [P, I, I],
        "stepq_host_image_layout": [P, I, P, ctypes.POINTER(Z)],
    }
    for name, args in sig.items():
        fn = getattr(lib, name)
        fn.argtypes = args
        fn.restype = ctypes.c_int
    lib.stepq_status_string.argtypes = [ctypes.c_int]
    lib.stepq_status_string.restype = ctypes.c_char_p
    _lib = lib
    return lib


def _check(status: int, what: str):
    if status != STEPQ_OK:
        raise StepqError(status, what)


def _ptr(t) -> int | None:
    return None if t is None else t.data_ptr()


def _stream(stream) -> int | None:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    return stream if isinstance(stream, int) else stream.cuda_stream


def _dev(t, name):
    if not t.is_cuda or not t.is_contiguous():
        raise ValueError("%s must be a contiguous CUDA tensor" % name)
    return t.data_ptr()


# ------------------------------------------------------------------------------ C ABI names

def stepq_status_string(status: int) -> str:
    return load_library().stepq_status_string(status).decode()


def stepq_pool_create(num_slots: int, head_bits, num_key_heads: int, gate_mode: int = STEPQ_GATE_GDN,
                      in_dtype: int = STEPQ_DTYPE_BF16, d_k: int = 128, d_v: int = 128) -> int:
    hb = np.ascontiguousarray(head_bits, dtype=np.uint8)
    desc = stepq_pool_desc(int(num_slots), len(hb), int(num_key_heads), d_k, d_v, gate_mode, in_dtype,
                           hb.ctypes.data_as(ctypes.POINTER(ctypes.c_uint8)))
    handle = ctypes.c_void_p()
    _check(load_library().stepq_pool_create(ctypes.byref(desc), ctypes.byref(handle)), "stepq_pool_create")
    return handle.value


def stepq_pool_create_rows(num_slots: int, head_bits, num_key_heads: int, row_bits, gate_mode: int = STEPQ_GATE_KDA,
                           in_dtype: int = STEPQ_DTYPE_BF16, d_k: int = 128, d_v: int = 128) -> int:
    """Pool whose heads of width 0 take per-key-row widths from row_bits [H, d_k]."""
    hb = np.ascontiguousarray(head_bits, dtype=np.uint8)
    rb = np.ascontiguousarray(row_bits, dtype=np.uint8)
    if rb.shape != (len(hb), d_k):
        raise ValueError("row_bits must be [H, d_k]")
    desc = stepq_pool_desc(int(num_slots), len(hb), int(num_key_heads), d_k, d_v, gate_mode, in_dtype,
                           hb.ctypes.data_as(ctypes.POINTER(ctypes.c_uint8)))
    handle = ctypes.c_void_p()
    _check(load_library().stepq_pool_create_rows(ctypes.byref(desc), rb.ctypes.data, ctypes.byref(handle)),
           "stepq_pool_create_rows")
    return handle.value


def stepq_pool_destroy(pool: int):
    _check(load_library().stepq_pool_destroy(pool), "stepq_pool_destroy")


def stepq_pool_bytes(pool: int):
    a, b = ctypes.c_size_t(), ctypes.c_size_t()
    _check(load_library().stepq_pool_bytes(pool, ctypes.byref(a), ctypes.byref(b)), "stepq_pool_bytes")
    return a.value, b.value


def stepq_pool_head_offset(pool: int, h: int) -> int:
    o = ctypes.c_size_t()
    _check(load_library().stepq_pool_head_offset(pool, h, ctypes.byref(o)), "stepq_pool_head_offset")
    return o.value


def stepq_pool_load_fp32(pool: int, slot_ids, S, stream=None):
    _check(load_library().stepq_pool_load_fp32(pool, _dev(slot_ids, "slot_ids"), slot_ids.numel(),
                                               _dev(S, "S"), _stream(stream)), "stepq_pool_load_fp32")


def stepq_pool_load_packed(pool: int, slot_ids, data, stream=None):
    _check(load_library().stepq_pool_load_packed(pool, _dev(slot_ids, "slot_ids"), slot_ids.numel(),
                                                 _dev(data, "bytes"), _stream(stream)), "stepq_pool_load_packed")


def stepq_pool_dump_fp32(pool: int, slot_ids, S_out, stream=None):
    _check(load_library().stepq_pool_dump_fp32(pool, _dev(slot_ids, "slot_ids"), slot_ids.numel(),
                                               _dev(S_out, "S_out"), _stream(stream)), "stepq_pool_dump_fp32")


def stepq_pool_dump_packed(pool: int, slot_ids, out, stream=None):
    _check(load_library().stepq_pool_dump_packed(pool, _dev(slot_ids, "slot_ids"), slot_ids.numel(),
                                                 _dev(out, "bytes_out"), _stream(stream)), "stepq_pool_dump_packed")


def stepq_decode_step(pool: int, slot_ids, q, k, v, alpha, beta, y, stream=None):
    _check(load_library().stepq_decode_step(
        pool, _dev(slot_ids, "slot_ids"), slot_ids.numel(), _dev(q, "q"), _dev(k, "k"), _dev(v, "v"),
        _dev(alpha, "alpha"), _dev(beta, "beta"), _dev(y, "y"), _stream(stream)), "stepq_decode_step")


def _host(t, name):
    if t.is_cuda or not t.is_contiguous():
        raise ValueError("%s must be a contiguous host tensor" % name)
    return t.data_ptr()


def stepq_decode_step_host(pool: int, slot_ids, q, k, v, alpha, beta, y, stream=None):
    """Decode step with every per-step buffer in host memory (pinned for overlapped copies):
    copy-in, step and copy-out are asynchronous; ``stepq_pool_host_wait`` orders a stream
    after the copies."""
    _check(load_library().stepq_decode_step_host(
        pool, _host(slot_ids, "slot_ids"), slot_ids.numel(), _host(q, "q"), _host(k, "k"), _host(v, "v"),
        _host(alpha, "alpha"), _host(beta, "beta"), _host(y, "y"), _stream(stream)), "stepq_decode_step_host")


def stepq_pool_host_wait(pool: int, stream=None):
    _check(load_library().stepq_pool_host_wait(pool, _stream(stream)), "stepq_pool_host_wait")


def stepq_decode_step_noalloc(num_slots: int, head_bits, num_key_heads: int, gate_mode: int, in_dtype: int,
                              state, slot_ids, q, k, v, alpha, beta, y, flag_out=None, stream=None):
    """Decode step on a caller-owned packed state buffer; the library allocates nothing.

    For callers whose device memory all comes from their own allocator or arena (``state``
    is such a buffer, in the pool layout).  ``flag_out``: optional int32 CUDA tensor that
    receives the call's device flag bits."""
    hb = np.ascontiguousarray(head_bits, dtype=np.uint8)
    desc = stepq_pool_desc(int(num_slots), len(hb), int(num_key_heads), 128, 128, gate_mode, in_dtype,
                           hb.ctypes.data_as(ctypes.POINTER(ctypes.c_uint8)))
    _check(load_library().stepq_decode_step_noalloc(
        ctypes.byref(desc), _dev(state, "state"), _dev(slot_ids, "slot_ids"), slot_ids.numel(),
        _dev(q, "q"), _dev(k, "k"), _dev(v, "v"), _dev(alpha, "alpha"), _dev(beta, "beta"), _dev(y, "y"),
        None if flag_out is None else _dev(flag_out, "flag_out"), _stream(stream)), "stepq_decode_step_noalloc")


def stepq_pool_set_impact(pool: int, impact=None):
    """Row-impact scores [H, d_k] (host array) for the impact-weighted fit, or None."""
    if impact is None:
        _check(load_library().stepq_pool_set_impact(pool, None), "stepq_pool_set_impact")
        return
    w = np.ascontiguousarray(impact, dtype=np.float32)
    _check(load_library().stepq_pool_set_impact(pool, w.ctypes.data), "stepq_pool_set_impact")


def stepq_pool_set_debug(handle: int, flags: int) -> None:
    _check(load_library().stepq_pool_set_debug(handle, int(flags)), "stepq_pool_set_debug")


def stepq_check_slot_ids(slot_ids, num_slots: int) -> int:
    """Status of the host-side slot-id check (0 when distinct and in range)."""
    ids = np.ascontiguousarray(slot_ids, dtype=np.int32)
    return load_library().stepq_check_slot_ids(ids.ctypes.data if ids.size else None, int(ids.size), int(num_slots))


def stepq_host_image_layout(handle: int, n: int):
    """(offsets of slot_ids, q, k, v, alpha, beta; total bytes) of the contiguous host input
    image of n requests."""
    offs = (ctypes.c_size_t * 6)()
    total = ctypes.c_size_t()
    _check(load_library().stepq_host_image_layout(handle, int(n), offs, ctypes.byref(total)),
           "stepq_host_image_layout")
    return [int(o) for o in offs], int(total.value)


def stepq_check_wait_timeout(stream=None) -> int:
    """Run the kernels' bounded-wait failure path on a barrier nothing completes; returns the
    flag bits it raised (STEPQ_FLAG_TIMEOUT when the path works)."""
    f = ctypes.c_int32()
    _check(load_library().stepq_check_wait_timeout(ctypes.byref(f), _stream(stream)), "stepq_check_wait_timeout")
    return f.value


def stepq_pool_get_error(pool: int) -> int:
    f = ctypes.c_int32()
    _check(load_library().stepq_pool_get_error(pool, ctypes.byref(f)), "stepq_pool_get_error")
    return f.value


def stepq_allocate_bits(half_life, distortion=None, cand=(4, 6, 8), avg_bits: float = 6.0) -> np.ndarray:
    hl = np.ascontiguousarray(half_life, dtype=np.float64)
    cd = np.ascontiguousarray(cand, dtype=np.uint8)
    dist = None if distortion is None else np.ascontiguousarray(distortion, dtype=np.float64)
    if dist is not None and dist.shape != (len(hl), len(cd)):
        raise ValueError("distortion must be [N, C]")
    out = np.zeros(len(hl), dtype=np.uint8)
    _check(load_library().stepq_allocate_bits(hl.ctypes.data, None if dist is None else dist.ctypes.data,
                                              len(hl), cd.ctypes.data, len(cd), float(avg_bits),
                                              out.ctypes.data), "stepq_allocate_bits")
    return out


def stepq_allocate_bits_pivots(half_life, distortion=None, cand=(4, 6, 8), avg_bits: float = 6.0,
                               n_pivots: int = 0) -> np.ndarray:
    hl = np.ascontiguousarray(half_life, dtype=np.float64)
    cd = np.ascontiguousarray(cand, dtype=np.uint8)
    dist = None if distortion is None else np.ascontiguousarray(distortion, dtype=np.float64)
    if dist is not None and dist.shape != (len(hl), len(cd)):
        raise ValueError("distortion must be [N, C]")
    out = np.zeros(len(hl), dtype=np.uint8)
    _check(load_library().stepq_allocate_bits_pivots(hl.ctypes.data, None if dist is None else dist.ctypes.data,
                                                     len(hl), cd.ctypes.data, len(cd), float(avg_bits),
                                                     int(n_pivots), out.ctypes.data), "stepq_allocate_bits_pivots")
    return out


# ------------------------------------------------------------------------------ convenience

class Pool:
    """Owning wrapper around a stepq_pool handle (device memory freed on close)."""

    def __init__(self, num_slots: int, head_bits, num_key_heads: int, gate_mode: int = STEPQ_GATE_GDN,
                 in_dtype: int = STEPQ_DTYPE_BF16, row_bits=None):
        self.head_bits = np.ascontiguousarray(head_bits, dtype=np.uint8)
        self.num_slots, self.H, self.Hk = int(num_slots), len(self.head_bits), int(num_key_heads)
        self.gate_mode, self.in_dtype = gate_mode, in_dtype
        self.handle = None
        if row_bits is None:
            self.handle = stepq_pool_create(num_slots, self.head_bits, num_key_heads, gate_mode, in_dtype)
        else:
            self.handle = stepq_pool_create_rows(num_slots, self.head_bits, num_key_heads, row_bits, gate_mode,
                                                 in_dtype)
        self.slot_stride, self.total_bytes = stepq_pool_bytes(self.handle)

    def close(self):
        if self.handle:
            stepq_pool_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def decode_step(self, slot_ids, q, k, v, alpha, beta, y, stream=None):
        stepq_decode_step(self.handle, slot_ids, q, k, v, alpha, beta, y, stream)

    def decode_step_host(self, slot_ids, q, k, v, alpha, beta, y, stream=None):
        stepq_decode_step_host(self.handle, slot_ids, q, k, v, alpha, beta, y, stream)

    def host_wait(self, stream=None):
        stepq_pool_host_wait(self.handle, stream)

    def load_fp32(self, slot_ids, S, stream=None):
        stepq_pool_load_fp32(self.handle, slot_ids, S, stream)

    def load_packed(self, slot_ids, data, stream=None):
        stepq_pool_load_packed(self.handle, slot_ids, data, stream)

    def dump_fp32(self, slot_ids, S_out, stream=None):
        stepq_pool_dump_fp32(self.handle, slot_ids, S_out, stream)

    def dump_packed(self, slot_ids, out, stream=None):
        stepq_pool_dump_packed(self.handle, slot_ids, out, stream)

    def host_image_layout(self, n: int):
        return stepq_host_image_layout(self.handle, n)

    def set_debug(self, flags: int) -> None:
        stepq_pool_set_debug(self.handle, flags)

    def get_error(self) -> int:
        return stepq_pool_get_error(self.handle)

    def set_impact(self, impact=None):
        if impact is not None and np.shape(impact) != (self.H, 128):
            raise ValueError("impact must be [H, 128]")
        stepq_pool_set_impact(self.handle, impact)
