"""GPU parity of the small-batch forward (1 <= M <= 16 tokens, the weight
streamed once) against the fp64 CPU oracle, through the C ABI: Y and T
within relative Frobenius error 5e-3 and max-abs error 2e-2 * max|ref|.
The frozen weight is the library's own quantization, pinned bit-exactly to
the oracle's by the quantization tests (and re-checked here)."""
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


def _fwd_case(case, expect_launches=1):
    d_ref = oracle.quantize_nf4_dq(case.W)
    w32 = oracle.dequantize(d_ref["codes"], d_ref["c2_fp8"], d_ref["c1"], d_ref["mean"], case.W.size)
    Wb = oracle.bf16_rne(w32).reshape(case.N, case.K)
    wq = q.qlora_quantize_nf4_dq(dev_f32(case.W))
    X, A, B = dev_bf16(case.X), dev_bf16(case.A), dev_bf16(case.B)
    torch.cuda.synchronize()
    n0 = q.qlora_kernel_launch_count()
    Y, T = q.qlora_linear_fwd(X, wq, A, B, case.s)
    n1 = q.qlora_kernel_launch_count()
    torch.cuda.synchronize()
    np.testing.assert_array_equal(wq.codes.cpu().numpy(), d_ref["codes"])
    np.testing.assert_array_equal(wq.c2_fp8.cpu().numpy(), d_ref["c2_fp8"])
    assert q.qlora_device_error(reset=True) == 0
    if expect_launches is not None:
        assert n1 - n0 == expect_launches
    Yr, T0 = oracle.linear_fwd(case.X, Wb, case.A, case.B, case.s)
    check_close(host_f64(T), case.s * T0, "T")
    check_close(host_f64(Y), Yr, "Y")
    return wq, X, A, B, Y, T


@pytest.mark.parametrize("which", [0, 1])
@pytest.mark.parametrize("M", [1, 4, 16])
def test_decode13b_shapes(which, M):
    """W 5120x5120 / 13824x5120, X M x 5120, r=16, alpha=16 (s=1), seed 0."""
    _fwd_case(synth.decode13b_linear(which, M, seed=0))


@pytest.mark.parametrize("M,N,K,r", [(1, 16, 64, 8), (2, 48, 1984, 24), (5, 512, 512, 8), (8, 256, 4096, 64),
                                     (9, 4096, 4096, 64), (3, 11008, 4096, 64), (16, 1024, 16384, 64),
                                     (7, 4096, 11008, 64), (12, 160, 640, 40), (16, 64, 128, 16)])
def test_small_batch_shapes(M, N, K, r):
    """Token counts 1..16 on both token tiles, one to many units per
    cluster, K from one block to 256 blocks, ranks not a multiple of 16."""
    case = synth.linear_case(f"m{M}n{N}k{K}r{r}", M, N, K, r, 16.0, seed=7, outlier_frac=0.001)
    _fwd_case(case)


@pytest.mark.parametrize("M,N,K,r", [(4, 100, 192, 8), (4, 128, 22016, 64), (16, 96, 256, 4)])
def test_small_batch_other_path(M, N, K, r):
    """Shapes the weight-streaming path does not take (N % 16, K > 16384,
    r % 8) still match through the general path."""
    case = synth.linear_case(f"o{M}n{N}k{K}r{r}", M, N, K, r, 16.0, seed=8)
    _fwd_case(case, expect_launches=None)


def test_small_batch_deterministic_and_saves_T():
    case = synth.linear_case("det", 16, 2048, 2048, 16, 16.0, seed=9)
    wq, X, A, B, Y, T = _fwd_case(case)
    Y2, T2 = q.qlora_linear_fwd(X, wq, A, B, case.s)
    torch.cuda.synchronize()
    assert torch.equal(Y, Y2) and torch.equal(T, T2)
    # the saved T feeds the backward exactly as a recomputed one would
    dY = dev_bf16(synth.bf16_normal(9, 77, (16, 2048)))
    a = q.qlora_linear_bwd(dY, X, wq, A, B, case.s, T=T)
    assert q.qlora_device_error(reset=True) == 0
    assert all(torch.isfinite(t.float()).all() for t in a)
