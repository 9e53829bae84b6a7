"""Host code under AddressSanitizer and UndefinedBehaviorSanitizer (no GPU needed).

Two native drivers in tests/native are built with -fsanitize=address,undefined and run in a
subprocess (a sanitized build cannot be loaded into this Python process):
  - the oracle's C source with every entry point, mode bit, ragged and empty sequences,
    snapshots, decode through a slot map and the argument checks;
  - the host side of libkda's C ABI (csrc/kda_api.cu: validation, the work plan, the
    sequence split, snapshot rows, workspace sizing) with its kernel launchers and CUDA runtime
    calls replaced by recording stubs, whose recorded plans are checked against invariants.
Any memory error, leak or undefined behaviour aborts the driver, and the test fails.
"""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
NATIVE = os.path.join(ROOT, "tests", "native")
CSRC = os.path.join(ROOT, "linear_attention_serving_rule_b200", "csrc")
SAN = ["-g", "-O1", "-fsanitize=address,undefined", "-fno-sanitize-recover=all", "-fno-omit-frame-pointer"]
ENV = dict(os.environ, ASAN_OPTIONS="detect_leaks=1:abort_on_error=0", UBSAN_OPTIONS="print_stacktrace=1")


def _cuda_include():
    for d in (os.environ.get("CUDA_HOME"), "/usr/local/cuda"):
        if d and os.path.exists(os.path.join(d, "include", "cuda_runtime.h")):
            return os.path.join(d, "include")
    return None


def _run(cmd_build, exe, tmp_path):
    b = subprocess.run(cmd_build, capture_output=True, text=True)
    if b.returncode != 0 and "sanitize" in (b.stderr or "") and "not supported" in (b.stderr or ""):
        pytest.skip("the host compiler has no sanitizer runtime")
    assert b.returncode == 0, b.stderr[-4000:]
    r = subprocess.run([exe], capture_output=True, text=True, env=ENV, timeout=300)
    assert r.returncode == 0, (r.stdout + r.stderr)[-4000:]
    assert "runtime error" not in r.stderr and "ERROR: AddressSanitizer" not in r.stderr
    return r.stdout


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
def test_oracle_under_asan_ubsan(tmp_path):
    exe = str(tmp_path / "oracle_driver")
    cmd = ["gcc", "-std=c11", *SAN, "-Wall", "-Wextra", "-Wno-unknown-pragmas",
           "-I", os.path.join(ROOT, "oracle"), os.path.join(NATIVE, "oracle_sanitize_driver.c"),
           os.path.join(ROOT, "oracle", "kda_ref.c"), "-lm", "-o", exe]
    assert "oracle sanitizer driver ok" in _run(cmd, exe, tmp_path)


@pytest.mark.skipif(shutil.which("g++") is None or _cuda_include() is None,
                    reason="needs g++ and the CUDA headers")
def test_api_host_code_under_asan_ubsan(tmp_path):
    exe = str(tmp_path / "api_driver")
    cmd = ["g++", "-std=c++17", *SAN, "-Wall", "-I", os.path.join(ROOT, "include"), "-I", CSRC,
           "-I", _cuda_include(), "-x", "c++", os.path.join(CSRC, "kda_api.cu"), "-x", "none",
           os.path.join(NATIVE, "api_host_driver.cpp"), "-o", exe]
    assert "api host driver ok" in _run(cmd, exe, tmp_path)
