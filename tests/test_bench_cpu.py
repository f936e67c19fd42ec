"""The benchmark's host side on CPU: the algorithmic byte and FLOP counts it
divides by, checked against the oracle's own output sizes and against the
products the linear consists of, and the reference arm's JSON line (the
oracle timed on the host cores) on one process and under a two-rank
launch, where rank 0 alone prints."""
import json
import os
import socket
import subprocess
import sys

import numpy as np
import pytest

import bench
import oracle

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.parametrize("numel", [1, 2, 63, 64, 65, 1000, 64 * 256, 64 * 256 + 1, 64 * 256 * 3 + 17])
def test_quant_and_dequant_bytes_match_the_stored_format(numel):
    """The quantized weight's bytes are what the oracle stores: codes, one
    FP8 constant per 64-block, one fp32 per 256 constants, the mean."""
    d = oracle.quantize_nf4_dq(np.linspace(-1, 1, numel, dtype=np.float32))
    stored = d["codes"].nbytes + d["c2_fp8"].nbytes + d["c1"].nbytes + np.float32(d["mean"]).nbytes
    assert bench.quant_bytes(numel) == 4 * numel + stored
    for out_bytes in (2, 4):
        assert bench.dequant_bytes(numel, out_bytes) == stored + out_bytes * numel


def test_decode_bytes_count_the_weight_and_the_activations():
    M, N, K, r = 4, 512, 256, 16
    d = oracle.quantize_nf4_dq(np.ones(N * K, np.float32))
    weight = d["codes"].nbytes + d["c2_fp8"].nbytes + d["c1"].nbytes
    act = 2 * (M * K + r * K + N * r + M * N + M * r)  # X, A, B read; Y, T written (bf16)
    assert bench.decode_bytes(M, N, K, r) == weight + act


def test_flop_counts_are_the_sum_of_the_linears_products():
    M, N, K, r = 7, 24, 64, 4

    def mm(m, n, k):
        return 2 * m * n * k

    fwd = mm(M, N, K) + mm(M, r, K) + mm(M, N, r)  # X W'^T, T = X A^T, T B^T
    bwd = mm(M, K, N) + mm(M, r, N) + mm(M, K, r) + mm(r, K, M) + mm(N, r, M)  # dY W', U, U A, dA, dB
    assert bench.fwd_flops(M, N, K, r) == fwd
    assert bench.linear_flops(M, N, K, r) == fwd + bwd


def _json_lines(text):
    out = []
    for ln in text.splitlines():
        ln = ln.strip()
        if ln.startswith("{"):
            out.append(json.loads(ln))
    return out


def _check_reference_line(line, n):
    for k in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
              "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert k in line, k
    assert line["impl"] == "reference" and line["n_gpus"] == n
    assert line["metric"] == bench.METRIC and line["unit"] == "TFLOP/s"
    assert line["value"] > 0 and line["higher_is_better"] is True
    assert line["steps"] == 1 and line["warmup"] == 3
    assert line["config"]["workload"] == bench.WORKLOAD
    cb = line["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] == line["value"] and cb["cores"] >= 1 and cb["sample"]
    e2e = line["e2e"]
    assert e2e["value"] == line["value"] and e2e["unit"] == line["unit"]
    assert e2e["h2d_bytes_per_step"] == 0 and e2e["d2h_bytes_per_step"] == 0


def test_reference_arm_prints_one_contract_line():
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--steps", "1", "--warmup", "3"],
                       cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = _json_lines(r.stdout)
    assert len(lines) == 1, r.stdout
    _check_reference_line(lines[0], 1)


def test_reference_arm_two_ranks_rank0_prints():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), "bench.py", "--gpus", "2",
           "--impl", "reference", "--steps", "1", "--warmup", "3"]
    r = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = _json_lines(r.stdout)
    assert len(lines) == 1, r.stdout
    _check_reference_line(lines[0], 2)
