"""The FP4 (E2M1) and Int4 comparison types (study notes 5.1.2, Table 2)
through the typed C-ABI entry points, against the oracle: the library's
tables equal the oracle's bit for bit; codes, FP8 constants, c1 and the mean
bit-exact; dequantized fp32 and bf16 bit-exact; the linear forward and
backward within the parity tolerance (including the small-batch path)."""
import numpy as np
import pytest
import torch

import oracle
import synth
from helpers import bits_of, check_close, dev_bf16, dev_f32, host_f64

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a CUDA GPU", allow_module_level=True)

import bit_nf4_quantized_13_b200 as q  # noqa: E402

TYPES = [("fp4", q.TYPE_FP4), ("int4", q.TYPE_INT4), ("nf4", q.TYPE_NF4)]


@pytest.mark.parametrize("name,qt", TYPES)
def test_tables_match_oracle(name, qt):
    np.testing.assert_array_equal(q.qlora_codebook(qt).view(np.uint32), oracle.codebook(name).view(np.uint32))


@pytest.mark.parametrize("name,qt", TYPES)
@pytest.mark.parametrize("n", [1, 63, 64 * 256 + 7, 4096 * 1024])
def test_quantize_dequantize_bit_exact(name, qt, n):
    w = synth.weight_student_t(2, 700 + n % 31, (n,))
    wq = q.qlora_quantize_nf4_dq(dev_f32(w), qtype=qt)
    d = oracle.quantize_nf4_dq(w, qtype=name)
    np.testing.assert_array_equal(wq.codes.cpu().numpy(), d["codes"])
    np.testing.assert_array_equal(wq.c2_fp8.cpu().numpy(), d["c2_fp8"])
    np.testing.assert_array_equal(wq.c1.cpu().numpy()[:d["c1"].size].view(np.uint32), d["c1"].view(np.uint32))
    assert wq.mean.cpu().numpy().view(np.uint32)[0] == np.float32(d["mean"]).view(np.uint32)
    ref = oracle.dequantize(d["codes"], d["c2_fp8"], d["c1"], d["mean"], n, qtype=name)
    got = q.qlora_dequantize(wq, torch.float32).cpu().numpy().reshape(-1)
    np.testing.assert_array_equal(got.view(np.uint32), ref.view(np.uint32))
    gotb = bits_of(q.qlora_dequantize(wq, torch.bfloat16)).reshape(-1)
    np.testing.assert_array_equal(gotb, oracle.bf16_rne(ref))


@pytest.mark.parametrize("name,qt", TYPES[:2])
@pytest.mark.parametrize("M,N,K,r", [(16, 512, 512, 8), (300, 1024, 768, 64), (4, 2048, 1024, 16)])
def test_linear_other_types(name, qt, M, N, K, r):
    case = synth.linear_case(f"{name}m{M}n{N}k{K}", M, N, K, r, 16.0, seed=13, outlier_frac=0.001)
    d = oracle.quantize_nf4_dq(case.W, qtype=name)
    Wb = oracle.bf16_rne(oracle.dequantize(d["codes"], d["c2_fp8"], d["c1"], d["mean"], case.W.size,
                                           qtype=name)).reshape(N, K)
    wq = q.qlora_quantize_nf4_dq(dev_f32(case.W), qtype=qt)
    X, A, B, dY = dev_bf16(case.X), dev_bf16(case.A), dev_bf16(case.B), dev_bf16(case.dY)
    Y, T = q.qlora_linear_fwd(X, wq, A, B, case.s)
    dX, dA, dB = q.qlora_linear_bwd(dY, X, wq, A, B, case.s, T=T)
    torch.cuda.synchronize()
    assert q.qlora_device_error(reset=True) == 0
    Yr, _ = oracle.linear_fwd(case.X, Wb, case.A, case.B, case.s)
    dXr, dAr, dBr = oracle.linear_bwd(case.dY, case.X, Wb, case.A, case.B, case.s)
    check_close(host_f64(Y), Yr, f"Y {name}")
    check_close(host_f64(dX), dXr, f"dX {name}")
    check_close(host_f64(dA), dAr, f"dA {name}")
    check_close(host_f64(dB), dBr, f"dB {name}")


def test_unknown_type_is_refused():
    P = 1 << 20
    assert q.lib.qlora_quantize_4bit_dq(7, P, 64, 64, 256, P, P, P, P, P, 1 << 16, None, None) == 1
    out = np.zeros(16, np.float32)
    import ctypes
    assert q.lib.qlora_codebook(3, out.ctypes.data_as(ctypes.c_void_p)) == 1
