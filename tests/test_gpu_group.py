"""GPU parity of the grouped QLoRA linears (q/k/v or gate/up: G linears on
one input, each with its own frozen 4-bit weight and rank-r adapter, run as
one stacked forward GEMM and one dX GEMM) against the fp64 CPU oracle run
linear by linear: Y_g, T_g, dA_g and dB_g against the oracle's single-linear
results, dX against the sum of the oracle's per-linear dX.  Same tolerance
as the single linears (relative Frobenius error 5e-3, max-abs 2e-2 *
max|ref|)."""
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


def _run_group(cases, rows=None, pass_T=True, want_dx=True):
    """cases: LinearCase per linear, all with the same M, K, r, alpha; the
    first case's X is the group's input."""
    X = cases[0].X
    s = cases[0].s
    r = cases[0].r
    Ns = [c.N for c in cases]
    starts = np.concatenate([[0], np.cumsum(Ns)])
    Wbs = []
    for c in cases:
        d = oracle.quantize_nf4_dq(c.W)
        w32 = oracle.dequantize(d["codes"], d["c2_fp8"], d["c1"], d["mean"], c.W.size)
        Wbs.append(oracle.bf16_rne(w32).reshape(c.N, c.K))

    wqs = [q.qlora_quantize_nf4_dq(dev_f32(c.W)) for c in cases]
    Xd = dev_bf16(X)
    A_cat = dev_bf16(np.concatenate([c.A for c in cases], axis=0))
    B_cat = dev_bf16(np.concatenate([c.B for c in cases], axis=0))
    dY = dev_bf16(np.concatenate([c.dY for c in cases], axis=1))
    Y, T = q.qlora_linear_group_fwd(Xd, wqs, A_cat, B_cat, s)
    dX, dA, dB = q.qlora_linear_group_bwd(dY, Xd, wqs, A_cat, B_cat, s, T=T if pass_T else None,
                                          want_dx=want_dx)
    torch.cuda.synchronize()
    assert q.qlora_device_error(reset=True) == 0

    sel = slice(None) if rows is None else rows
    Yh, Th = host_f64(Y)[sel], host_f64(T)[sel]
    dAh, dBh = host_f64(dA), host_f64(dB)
    dX_ref = 0.0
    for g, c in enumerate(cases):
        Yr, T0 = oracle.linear_fwd(X, Wbs[g], c.A, c.B, s, rows=rows)
        dXr, dAr, dBr = oracle.linear_bwd(c.dY, X, Wbs[g], c.A, c.B, s, rows=rows, want_dx=want_dx)
        check_close(Th[:, g * r:(g + 1) * r], s * T0, f"T_{g}")
        check_close(Yh[:, starts[g]:starts[g + 1]], Yr, f"Y_{g}")
        check_close(dAh[g * r:(g + 1) * r], dAr, f"dA_{g}")
        check_close(dBh[starts[g]:starts[g + 1]], dBr, f"dB_{g}")
        if want_dx:
            dX_ref = dX_ref + dXr
    if want_dx:
        check_close(host_f64(dX)[sel], dX_ref, "dX")
    return Y, T, dX, dA, dB


def _cases(M, Ns, K, r, seed):
    return [synth.linear_case(f"g{g}_m{M}n{N}k{K}r{r}", M, N, K, r, 16.0, seed=seed, wid=g,
                              outlier_frac=0.001) for g, N in enumerate(Ns)]


@pytest.mark.parametrize("M,Ns,K,r", [
    (600, (512, 256, 256), 320, 16),   # q/k/v with narrower k/v, ragged token tail
    (130, (768, 768), 256, 64),        # gate/up
    (1, (256,), 128, 8),               # one linear, one token
    (77, (256, 256, 256, 256), 192, 64),  # four linears, total rank 256
    (1100, (1024, 256, 256), 512, 32),  # several token tiles
])
def test_group_shapes(M, Ns, K, r):
    _run_group(_cases(M, Ns, K, r, seed=31))


def test_group_recomputed_T_and_no_dx():
    cases = _cases(300, (256, 512), 256, 16, seed=32)
    a = _run_group(cases, pass_T=True)
    b = _run_group(cases, pass_T=False, want_dx=False)
    assert torch.equal(a[3], b[3]) and torch.equal(a[4], b[4])


def test_group_fp4_weights():
    """The grouped GEMMs read the type's table like the single ones."""
    cases = _cases(200, (256, 256), 256, 16, seed=33)
    X = cases[0].X
    s, r = cases[0].s, cases[0].r
    wqs = [q.qlora_quantize_nf4_dq(dev_f32(c.W), qtype=q.TYPE_FP4) for c in cases]
    Xd = dev_bf16(X)
    A_cat = dev_bf16(np.concatenate([c.A for c in cases], axis=0))
    B_cat = dev_bf16(np.concatenate([c.B for c in cases], axis=0))
    Y, T = q.qlora_linear_group_fwd(Xd, wqs, A_cat, B_cat, s)
    torch.cuda.synchronize()
    n0 = 0
    for g, c in enumerate(cases):
        d = oracle.quantize_nf4_dq(c.W, qtype="fp4")
        w32 = oracle.dequantize(d["codes"], d["c2_fp8"], d["c1"], d["mean"], c.W.size, qtype="fp4")
        Wb = oracle.bf16_rne(w32).reshape(c.N, c.K)
        Yr, T0 = oracle.linear_fwd(X, Wb, c.A, c.B, s)
        check_close(host_f64(Y)[:, n0:n0 + c.N], Yr, f"Y_{g} (fp4)")
        check_close(host_f64(T)[:, g * r:(g + 1) * r], s * T0, f"T_{g} (fp4)")
        n0 += c.N


def test_group_empty_batch():
    cases = _cases(1, (256, 256), 128, 8, seed=34)
    wqs = [q.qlora_quantize_nf4_dq(dev_f32(c.W)) for c in cases]
    A_cat = dev_bf16(np.concatenate([c.A for c in cases], axis=0))
    B_cat = dev_bf16(np.concatenate([c.B for c in cases], axis=0))
    X = torch.empty((0, 128), dtype=torch.bfloat16, device="cuda")
    dY = torch.empty((0, 512), dtype=torch.bfloat16, device="cuda")
    Y, _ = q.qlora_linear_group_fwd(X, wqs, A_cat, B_cat, 2.0)
    assert Y.shape == (0, 512)
    dA = torch.full((16, 128), 1.0, dtype=torch.bfloat16, device="cuda")
    dB = torch.full((512, 8), 1.0, dtype=torch.bfloat16, device="cuda")
    q.qlora_linear_group_bwd(dY, X, wqs, A_cat, B_cat, 2.0, dA_cat=dA, dB_cat=dB)
    torch.cuda.synchronize()
    assert torch.count_nonzero(dA) == 0 and torch.count_nonzero(dB) == 0


def test_group_unsupported_shapes_raise():
    cases = _cases(16, (256, 200), 128, 8, seed=35)  # N_2 not a multiple of 256
    wqs = [q.qlora_quantize_nf4_dq(dev_f32(c.W)) for c in cases]
    A_cat = dev_bf16(np.concatenate([c.A for c in cases], axis=0))
    B_cat = dev_bf16(np.concatenate([c.B for c in cases], axis=0))
    with pytest.raises(q.QloraError) as e:
        q.qlora_linear_group_fwd(dev_bf16(cases[0].X), wqs, A_cat, B_cat, 2.0)
    assert e.value.status == 2


@pytest.mark.parametrize("group,M", [((0, 1, 2), 2048), ((4, 5), 512)])
def test_llama65b_groups(group, M):
    """A LLaMA-65B-shaped layer's q/k/v group (3 x 8192 x 8192) at 2048
    tokens and gate/up group (2 x 22016 x 8192) at 512 tokens, r=64,
    alpha=16: Y, T, dX on 32 seeded rows, dA and dB in full."""
    cases = [synth.llama65b_linear(w, M, seed=0) for w in group]
    rows = np.sort(synth.rng(0, 700 + group[0]).choice(M, 32, replace=False)).astype(np.int64)
    _run_group(cases, rows=rows)
