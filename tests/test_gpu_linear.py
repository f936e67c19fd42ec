"""GPU parity of the QLoRA linear forward and backward against the fp64 CPU
oracle, through the C ABI: Y, dX, dA, dB within relative Frobenius error
5e-3 and max-abs error 2e-2 * max|ref|; T (= bf16(s X A^T)) likewise.  The
frozen weight seen by both sides is the library's own quantization, which
the quantization tests pin bit-exactly to the oracle's."""
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


def _run_case(case, rows=None, want_dx=True, pass_T=True):
    """Quantize on both sides, run fwd + bwd on the GPU, compare with the
    oracle on the selected rows (all when rows is None)."""
    d_ref = oracle.quantize_nf4_dq(case.W)
    w32 = oracle.dequantize(d_ref["codes"], d_ref["c2_fp8"], d_ref["c1"], d_ref["mean"], case.W.size)
    Wb = oracle.bf16_rne(w32).reshape(case.N, case.K)

    wq = q.qlora_quantize_nf4_dq(dev_f32(case.W))
    X, A, B, dY = dev_bf16(case.X), dev_bf16(case.A), dev_bf16(case.B), dev_bf16(case.dY)
    Y, T = q.qlora_linear_fwd(X, wq, A, B, case.s)
    dX, dA, dB = q.qlora_linear_bwd(dY, X, wq, A, B, case.s, T=T if pass_T else None,
                                    want_dx=want_dx)
    torch.cuda.synchronize()
    # the quantized weight is the oracle's, bit for bit
    np.testing.assert_array_equal(wq.codes.cpu().numpy(), d_ref["codes"])
    np.testing.assert_array_equal(wq.c2_fp8.cpu().numpy(), d_ref["c2_fp8"])
    assert wq.mean.cpu().numpy().view(np.uint32)[0] == np.float32(d_ref["mean"]).view(np.uint32)
    np.testing.assert_array_equal(bits_of(q.qlora_dequantize(wq, torch.bfloat16)).reshape(-1),
                                  Wb.reshape(-1))

    Yr, T0 = oracle.linear_fwd(case.X, Wb, case.A, case.B, case.s, rows=rows)
    dXr, dAr, dBr = oracle.linear_bwd(case.dY, case.X, Wb, case.A, case.B, case.s, rows=rows,
                                      want_dx=want_dx)
    assert q.qlora_device_error(reset=True) == 0
    sel = slice(None) if rows is None else rows
    check_close(host_f64(T)[sel], case.s * T0, "T")
    check_close(host_f64(Y)[sel], Yr, "Y")
    if want_dx:
        check_close(host_f64(dX)[sel], dXr, "dX")
    check_close(host_f64(dA), dAr, "dA")
    check_close(host_f64(dB), dBr, "dB")
    return Y, T, dX, dA, dB


def test_tiny_config():
    """W 512x512, X 16x512, r=8, alpha=16 (s=2), seed 0."""
    _run_case(synth.tiny(0))


@pytest.mark.parametrize("M,N,K,r", [(1, 64, 64, 1), (3, 100, 192, 8), (17, 513, 128, 16),
                                     (130, 257, 320, 64), (64, 128, 256, 256), (200, 96, 512, 3),
                                     (129, 200, 64, 33), (300, 520, 192, 16), (257, 1000, 256, 72),
                                     (77, 136, 448, 24)])
def test_ragged_shapes(M, N, K, r):
    case = synth.linear_case(f"m{M}n{N}k{K}r{r}", M, N, K, r, 16.0, seed=1, outlier_frac=0.001)
    _run_case(case)


def test_tile_spanning_shape():
    """Several tiles in every dimension plus ragged tails."""
    case = synth.linear_case("m333n777k1024r64", 333, 777, 1024, 64, 16.0, seed=2, outlier_frac=0.001)
    _run_case(case)


@pytest.mark.parametrize("M,N,K", [(830, 4864, 128), (1001, 4864, 128), (1090, 4864, 128), (1200, 4864, 128),
                                   (830, 128, 4864), (1001, 128, 4864), (1090, 128, 4864), (1200, 128, 4864)])
def test_partial_rounds_and_split_tiles(M, N, K):
    """Tile counts that leave the GEMMs' last round of tiles partly empty:
    the forward with 19 weight-row tiles (N = 4864) x 2-3 token tiles of
    512, and the dX product with 19 row tiles (K = 4864) over a contraction
    of only two 64-blocks plus the LoRA slab, each with a ragged token tail,
    so the last round's stages are split between SM pairs and finished
    through the workspace; 64 sampled rows."""
    case = synth.linear_case(f"w{M}n{N}k{K}", M, N, K, 16, 16.0, seed=21, outlier_frac=0.001)
    rows = np.sort(synth.rng(0, 121).choice(M, 64, replace=False)).astype(np.int64)
    _run_case(case, rows=rows)


def test_T_recompute_matches_saved_T():
    case = synth.linear_case("m96n256k256r16", 96, 256, 256, 16, 16.0, seed=3)
    wq = q.qlora_quantize_nf4_dq(dev_f32(case.W))
    X, A, B, dY = dev_bf16(case.X), dev_bf16(case.A), dev_bf16(case.B), dev_bf16(case.dY)
    _, T = q.qlora_linear_fwd(X, wq, A, B, case.s)
    a = q.qlora_linear_bwd(dY, X, wq, A, B, case.s, T=T)
    b = q.qlora_linear_bwd(dY, X, wq, A, B, case.s, T=None)
    for x, y in zip(a, b):
        assert torch.equal(x, y)
    # no dX requested: dA, dB unchanged
    _, dA, dB = q.qlora_linear_bwd(dY, X, wq, A, B, case.s, T=T, want_dx=False)
    assert torch.equal(dA, a[1]) and torch.equal(dB, a[2])


def test_empty_batch_gives_zero_adapter_gradients():
    case = synth.linear_case("m0", 1, 64, 128, 8, 16.0, seed=4)
    wq = q.qlora_quantize_nf4_dq(dev_f32(case.W))
    A, B = dev_bf16(case.A), dev_bf16(case.B)
    X = torch.empty((0, 128), dtype=torch.bfloat16, device="cuda")
    dY = torch.empty((0, 64), dtype=torch.bfloat16, device="cuda")
    Y, T = q.qlora_linear_fwd(X, wq, A, B, case.s)
    assert Y.shape == (0, 64)
    dA = torch.full((8, 128), 1.0, dtype=torch.bfloat16, device="cuda")
    dB = torch.full((64, 8), 1.0, dtype=torch.bfloat16, device="cuda")
    q.qlora_linear_bwd(dY, X, wq, A, B, case.s, dA=dA, dB=dB)
    torch.cuda.synchronize()
    assert torch.count_nonzero(dA) == 0 and torch.count_nonzero(dB) == 0


def test_unsupported_shapes_raise():
    case = synth.linear_case("bad", 4, 64, 128, 8, 16.0, seed=5)
    wq = q.qlora_quantize_nf4_dq(dev_f32(case.W))
    X, A, B = dev_bf16(case.X), dev_bf16(case.A), dev_bf16(case.B)
    with pytest.raises(q.QloraError) as e:  # K % 64 != 0, operands consistent: refused by the library
        Xbad = torch.zeros((4, 100), dtype=torch.bfloat16, device="cuda")
        Abad = torch.zeros((8, 100), dtype=torch.bfloat16, device="cuda")
        q.qlora_linear_fwd(Xbad, q.Nf4Weight(wq.codes, wq.c2_fp8, wq.c1, wq.mean, (64, 100)), Abad, B, 1.0)
    assert e.value.status == 2
    with pytest.raises(ValueError):  # operands that disagree: refused by the binding
        q.qlora_linear_fwd(X, wq, torch.zeros((8, 64), dtype=torch.bfloat16, device="cuda"), B, 1.0)
    Abig = torch.zeros((257, 128), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(q.QloraError):
        q.qlora_linear_fwd(X, wq, Abig, torch.zeros((64, 257), dtype=torch.bfloat16, device="cuda"), 1.0)


@pytest.mark.parametrize("which", [0, 1])
def test_llama7b_shapes_sampled_rows(which):
    """W 4096x4096 / 11008x4096, X 4096 tokens, r=64, alpha=16: Y and dX on
    64 seeded rows, T on those rows, dA and dB in full."""
    case = synth.llama7b_linear(which, seed=0)
    rows = np.sort(synth.rng(0, 99 + which).choice(case.M, 64, replace=False)).astype(np.int64)
    _run_case(case, rows=rows)


# q/o (8192 x 8192), gate/up (22016 x 8192) and down (8192 x 22016: the
# 344-block contraction) of a LLaMA-65B-shaped layer
LLAMA65B_DISTINCT = [0, 4, 6]


@pytest.mark.parametrize("M", [512, 8192])
@pytest.mark.parametrize("which", LLAMA65B_DISTINCT)
def test_llama65b_shapes(which, M):
    """LLaMA-65B-shaped linears, r=64, alpha=16: Y, T and dX on 512 seeded
    token rows (all rows at M = 512), dA and dB in full."""
    case = synth.llama65b_linear(which, M, seed=0)
    rows = None
    if M > 512:
        rows = np.sort(synth.rng(0, 650 + which).choice(M, 512, replace=False)).astype(np.int64)
    _run_case(case, rows=rows)


def test_unfused_library_path_agrees():
    """Second opinion: dequantize to bf16 with the library, then torch.matmul
    (cuBLAS) for X W'^T + (s X A^T) B^T and dY W' + (s dY B) A; the fused
    kernels agree within the same tolerance."""
    case = synth.linear_case("k9", 512, 1536, 2048, 64, 16.0, seed=11, outlier_frac=0.001)
    wq = q.qlora_quantize_nf4_dq(dev_f32(case.W))
    X, A, B, dY = dev_bf16(case.X), dev_bf16(case.A), dev_bf16(case.B), dev_bf16(case.dY)
    Y, T = q.qlora_linear_fwd(X, wq, A, B, case.s)
    dX, _, _ = q.qlora_linear_bwd(dY, X, wq, A, B, case.s, T=T)
    Wd = q.qlora_dequantize(wq, torch.bfloat16).view(case.N, case.K)
    Tk = (X.float() @ A.float().t() * case.s).bfloat16()
    Yk = X.float() @ Wd.float().t() + Tk.float() @ B.float().t()
    Uk = (dY.float() @ B.float() * case.s).bfloat16()
    dXk = dY.float() @ Wd.float() + Uk.float() @ A.float()
    torch.cuda.synchronize()
    check_close(host_f64(Y), Yk.double().cpu().numpy(), "Y vs unfused")
    check_close(host_f64(dX), dXk.double().cpu().numpy(), "dX vs unfused")
