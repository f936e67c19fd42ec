"""The library memoizes its one-time set-up (kernel shared-memory limits,
occupancy answers, the device address of the allocation-free entry point's
scratch array) per CUDA context, keyed on the context's process-unique id,
so that a context made again after a device reset is set up afresh rather
than handed a stale address.  The memo is plain C++; this compiles it with
a host-only driver (tests/cpp/ctx_memo_check.cpp) and runs the checks."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "bit_nf4_quantized_13_b200", "csrc")
SRC = os.path.join(ROOT, "tests", "cpp", "ctx_memo_check.cpp")


@pytest.mark.skipif(shutil.which("g++") is None, reason="needs g++")
def test_context_memo_keys_on_context_id(tmp_path):
    exe = tmp_path / "ctx_memo_check"
    subprocess.run(["g++", "-std=c++17", "-O1", "-pthread", "-I", CSRC, SRC, "-o", str(exe)], check=True)
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0, r.stdout + r.stderr
