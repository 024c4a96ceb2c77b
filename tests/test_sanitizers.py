"""Host code under AddressSanitizer, LeakSanitizer and UndefinedBehaviorSanitizer (no GPU).

Two drivers are built here with the sanitizers on:
- tests/sanitize/oracle_driver.c runs every function of the CPU oracle on random inputs and
  edge cases (zero rows and columns, subnormal values, every head kind, bad slot ids);
- tests/sanitize/capi_fakes.cpp links the library's host code (the C ABI and the bit
  allocator) against fake CUDA runtime calls that work on host memory, then runs pool
  creation and destruction, an allocation failure injected at each device allocation of
  pool creation (STEPQ_OUT_OF_MEMORY, no leak), the slot-id debug mode, the host-buffer
  staging path, the impact-score normalization and the allocator.
A sanitizer report or a failed check makes the driver program exit non-zero.
"""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HERE = os.path.join(ROOT, "tests", "sanitize")
CSRC = os.path.join(ROOT, "quantized_gated_delta_b200", "csrc")
SAN = ["-fsanitize=address,undefined", "-fno-sanitize-recover=all", "-fno-omit-frame-pointer", "-g", "-O1"]
ENV = dict(os.environ, ASAN_OPTIONS="detect_leaks=1:abort_on_error=0:halt_on_error=1",
           UBSAN_OPTIONS="print_stacktrace=1:halt_on_error=1")


def _host_flags():
    """SAN for nvcc's host compiler: one -Xcompiler per flag (nvcc splits its value on commas)."""
    out = []
    for f in SAN:
        parts = ["-fsanitize=" + x for x in f.split("=", 1)[1].split(",")] if f.startswith("-fsanitize=") else [f]
        out += ["-Xcompiler=" + x for x in parts]
    return out


def _run(cmd, cwd=None, env=None, timeout=600):
    p = subprocess.run(cmd, cwd=cwd, env=env, capture_output=True, text=True, timeout=timeout)
    return p.returncode, p.stdout + p.stderr


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
def test_oracle_under_sanitizers(tmp_path):
    exe = str(tmp_path / "oracle_driver")
    rc, out = _run(["gcc", "-std=c11", *SAN, "-o", exe, os.path.join(HERE, "oracle_driver.c"),
                    os.path.join(ROOT, "oracle", "stepq_oracle.c"), "-lm"])
    assert rc == 0, out
    rc, out = _run([exe], env=ENV)
    assert rc == 0, out
    assert "AddressSanitizer" not in out and "runtime error" not in out, out


@pytest.mark.skipif(shutil.which("g++") is None or not os.path.exists("/usr/local/cuda/bin/nvcc"),
                    reason="needs g++ and nvcc")
def test_c_abi_host_code_under_sanitizers(tmp_path):
    nvcc = "/usr/local/cuda/bin/nvcc"
    inc = ["-I" + os.path.join(ROOT, "include"), "-I" + CSRC]
    capi = str(tmp_path / "capi.o")
    rc, out = _run([nvcc, "-std=c++17", "-O1", "-g", "-gencode", "arch=compute_100a,code=sm_100a",
                    *_host_flags(), *inc, "-c", os.path.join(CSRC, "stepq_capi.cu"), "-o", capi])
    assert rc == 0, out
    exe = str(tmp_path / "capi_fakes")
    rc, out = _run(["g++", "-std=c++17", *SAN, *inc, "-I/usr/local/cuda/include", "-o", exe,
                    os.path.join(HERE, "capi_fakes.cpp"), os.path.join(CSRC, "stepq_alloc.cpp"), capi])
    assert rc == 0, out
    rc, out = _run([exe], env=ENV)
    assert rc == 0, out
    assert "0 failures" in out and "AddressSanitizer" not in out and "runtime error" not in out, out
