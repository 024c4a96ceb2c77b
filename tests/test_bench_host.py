"""Host-side arithmetic of bench.py (no GPU): the algorithmic bytes behind the roofline, the
slot stride of the reference arm, and the code hash that keys the recorded DRAM traffic."""
import os
import shutil
import types

import pytest

import bench
from oracle import oracle as O


def _w(B, H, Hk, gate, bf16=True):
    return types.SimpleNamespace(B=B, H=H, Hk=Hk, dk=128, dv=128, gate_mode=gate, in_dtype=1 if bf16 else 0)


@pytest.mark.parametrize("bits,Hk_ratio,gate,expect", [
    # bytes moved per (request, head) update: the state read and written once
    # (2 x (d_k d_v b / 8 + 4 d_k + 4 d_v)), q and k shared by H / H_k heads, v, y in fp32,
    # the gates, and the request's slot id spread over its heads
    (6, 2, 0, 2 * (128 * 128 * 6 // 8 + 1024) + (2 * 256) // 2 + 256 + 512 + 2 + 2),
    (4, 2, 0, 2 * (128 * 128 * 4 // 8 + 1024) + (2 * 256) // 2 + 256 + 512 + 2 + 2),
    (6, 1, 1, 2 * (128 * 128 * 6 // 8 + 1024) + 2 * 256 + 256 + 512 + 256 + 2),
])
def test_algorithmic_bytes_per_update(bits, Hk_ratio, gate, expect):
    H = 32
    w = _w(B=16, H=H, Hk=H // Hk_ratio, gate=gate)
    per_update = bench.algorithmic_bytes_per_step(w, [bits] * H) / (w.B * w.H)
    assert per_update == pytest.approx(expect + 4 / H, abs=1e-9)


def test_algorithmic_bytes_match_the_published_per_update_figures():
    """The per-update totals of the measurement plan: 6-bit GQA about 27,652 B, KDA 6-bit
    about 28,164 B, uniform 4-bit about 19,460 B (slot ids aside)."""
    H = 32
    for bits, Hk, gate, figure in ((6, 16, 0, 27652), (6, 32, 1, 28164), (4, 16, 0, 19460)):
        w = _w(B=8, H=H, Hk=Hk, gate=gate)
        per_update = bench.algorithmic_bytes_per_step(w, [bits] * H) / (w.B * H) - 4 / H
        assert abs(per_update - figure) <= 4, (bits, gate, per_update)


@pytest.mark.parametrize("bits", [[4, 6, 8], [8] * 5, [16, 4, 16, 8], [6] * 32])
def test_slot_stride_of_matches_the_oracle_layout(bits):
    assert bench.slot_stride_of(bits) == O.head_offsets(bits)[1]


def test_code_hash_ignores_comments_but_not_code(tmp_path):
    src = os.path.join(bench.ROOT, "quantized_gated_delta_b200", "csrc")
    dst = tmp_path / "csrc"
    shutil.copytree(src, dst)
    h0 = bench.kernel_source_hash(str(dst))
    assert h0 == bench.kernel_source_hash(src)
    f = dst / "stepq_tile.cuh"
    text = f.read_text()
    f.write_text("// a new comment line\n" + text.replace("namespace stepq {", "namespace stepq {   /* note */", 1))
    assert bench.kernel_source_hash(str(dst)) == h0
    f.write_text(text.replace("constexpr int PANEL = 16;", "constexpr int PANEL = 32;", 1))
    assert bench.kernel_source_hash(str(dst)) != h0
