"""Failure detection on the GPU without a fault: every pipeline wait in the
tensor-core kernels is bounded by GPU time and, when the bound passes,
records QLORA_ERR_TIMEOUT in a sticky device word and lets the kernel
return.  The self-test kernel waits (1 ms limit) on a barrier nothing ever
signals, with no copy or MMA in flight; the host then reads the status, and
a normal quantize + forward + backward afterwards still matches the oracle
(the context stayed usable)."""
import numpy as np
import pytest
import torch

import oracle
import synth
from helpers import check_close, dev_bf16, dev_f32, host_f64

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a CUDA GPU", allow_module_level=True)

import bit_nf4_quantized_13_b200 as q  # noqa: E402


def test_bounded_wait_gives_up_and_reports_timeout():
    assert q.qlora_device_error(reset=True) in (0, 6)
    assert q.qlora_device_error() == 0
    n0 = q.qlora_kernel_launch_count()
    q.qlora_debug_wait_timeout(1_000_000)  # 1 ms
    torch.cuda.synchronize()
    assert q.qlora_kernel_launch_count() - n0 == 1
    assert q.qlora_device_error() == 6          # read, not cleared
    assert q.qlora_device_error(reset=True) == 6
    assert q.qlora_device_error() == 0          # cleared


def test_library_still_works_after_a_timeout():
    q.qlora_debug_wait_timeout(1_000_000)
    torch.cuda.synchronize()
    assert q.qlora_device_error(reset=True) == 6
    case = synth.linear_case("after_timeout", 96, 384, 512, 16, 16.0, seed=31)
    d = oracle.quantize_nf4_dq(case.W)
    Wb = oracle.bf16_rne(oracle.dequantize(d["codes"], d["c2_fp8"], d["c1"], d["mean"],
                                           case.W.size)).reshape(case.N, case.K)
    wq = q.qlora_quantize_nf4_dq(dev_f32(case.W))
    X, A, B, dY = dev_bf16(case.X), dev_bf16(case.A), dev_bf16(case.B), dev_bf16(case.dY)
    Y, T = q.qlora_linear_fwd(X, wq, A, B, case.s)
    dX, dA, dB = q.qlora_linear_bwd(dY, X, wq, A, B, case.s, T=T)
    torch.cuda.synchronize()
    assert q.qlora_device_error() == 0
    np.testing.assert_array_equal(wq.codes.cpu().numpy(), d["codes"])
    Yr, _ = oracle.linear_fwd(case.X, Wb, case.A, case.B, case.s)
    dXr, dAr, dBr = oracle.linear_bwd(case.dY, case.X, Wb, case.A, case.B, case.s)
    check_close(host_f64(Y), Yr, "Y")
    check_close(host_f64(dX), dXr, "dX")
    check_close(host_f64(dA), dAr, "dA")
    check_close(host_f64(dB), dBr, "dB")
