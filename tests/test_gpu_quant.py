"""GPU parity of the quantization path against the CPU oracle, through the
C ABI (the Python binding only marshals pointers): NF4 codes, FP8 constant
bytes, c1 and the mean bit-exact; dequantized weights exact in fp32 (the
contract allows 1 ulp) and in bf16."""
import numpy as np
import pytest
import torch

import oracle
import synth
from helpers import dev_f32

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():  # the CPU suite never selects these
    pytest.skip("needs a CUDA GPU", allow_module_level=True)

import bit_nf4_quantized_13_b200 as q  # noqa: E402


def _quant_both(w):
    d_ref = oracle.quantize_nf4_dq(w)
    W = dev_f32(w.reshape(-1))
    status = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    wq = q.qlora_quantize_nf4_dq(W, status=status)
    torch.cuda.synchronize()
    return d_ref, wq, int(status.item())


def _assert_quant_equal(d_ref, wq):
    np.testing.assert_array_equal(wq.codes.cpu().numpy(), d_ref["codes"])
    np.testing.assert_array_equal(wq.c2_fp8.cpu().numpy(), d_ref["c2_fp8"])
    np.testing.assert_array_equal(wq.c1.cpu().numpy().view(np.uint32), d_ref["c1"].view(np.uint32))
    assert wq.mean.cpu().numpy().view(np.uint32)[0] == np.float32(d_ref["mean"]).view(np.uint32)


NUMELS = [1, 2, 3, 63, 64, 65, 100, 511, 512, 513, 1000, 64 * 256, 64 * 256 + 7, 64 * 256 * 3 + 130,
          (1 << 20) + 37, 512 * 512]


@pytest.mark.parametrize("numel", NUMELS)
def test_quantize_bit_exact(numel):
    w = synth.weight_normal(0, 1000 + numel % 977, (numel,), 0.02, 0.001)
    if numel >= 256:
        w[64:128] = 0.0   # an all-zero block
        w[200] = 0.0
    d_ref, wq, st = _quant_both(w)
    assert st == 0
    _assert_quant_equal(d_ref, wq)


@pytest.mark.parametrize("shape,tid", [((4096, 4096), 1), ((11008, 4096), 11)])
def test_quantize_bit_exact_llama7b_shapes(shape, tid):
    w = synth.weight_normal(0, tid, shape, 0.02, 0.001)
    d_ref, wq, st = _quant_both(w)
    assert st == 0
    _assert_quant_equal(d_ref, wq)


def test_quantize_student_t_and_wide_range():
    w = synth.weight_student_t(0, 5, (64 * 1000,))
    # blocks whose constants span many binades exercise the exact mean
    scale = np.repeat(np.exp2(synth.rng(0, 6).integers(-60, 60, 1000)).astype(np.float32), 64)
    d_ref, wq, st = _quant_both(w * scale)
    assert st == 0
    _assert_quant_equal(d_ref, wq)


def test_quantize_all_zero_and_constant():
    for w in (np.zeros(64 * 300, np.float32), np.full(64 * 300 + 5, 0.5, np.float32)):
        d_ref, wq, st = _quant_both(w)
        assert st == 0
        _assert_quant_equal(d_ref, wq)


def test_quantize_reports_nonfinite():
    w = synth.normal_f32(0, 8, (64 * 40,), 0.02)
    w[777] = np.nan
    _, _, st = _quant_both(w)
    assert st == 5
    w[777] = np.inf
    _, _, st = _quant_both(w)
    assert st == 5


def test_encode_near_every_decision_boundary():
    """Weights placed within a few ulps of every midpoint between adjacent
    codes, for block maxima spanning the fp32 range."""
    qv = oracle.nf4_codebook().astype(np.float64)
    mids = (qv[1:] + qv[:-1]) / 2
    rows = []
    scales = [1.0, 0.0731, 3.3e-5, 1.7e3, 2.0 ** -100, 1.0e30, 2.0 ** 126 * 1.5, 2.0 ** -125, 2.0 ** -119.5,
              2.0 ** 119.5, 2.0 ** 121]
    scales += list(np.exp2(synth.rng(0, 4242).uniform(-118, 118, 24)))
    for a in scales:
        for m in mids:
            c = np.float32(m * a)
            near = (c.view(np.uint32).astype(np.int64) + np.arange(-3, 4)).astype(np.uint32).view(np.float32)
            rows.append(near)
        blk_rows = np.concatenate(rows)
        rows = []
        # pack into 64-blocks whose first element sets the absmax a
        per = 63
        nblk = -(-blk_rows.size // per)
        w = np.zeros((nblk, 64), np.float32)
        w[:, 0] = np.float32(a)
        flat = np.zeros(nblk * per, np.float32)
        flat[: blk_rows.size] = blk_rows
        w[:, 1:] = flat.reshape(nblk, per)
        d_ref, wq, st = _quant_both(w.reshape(-1))
        assert st == 0
        np.testing.assert_array_equal(wq.codes.cpu().numpy(), d_ref["codes"], err_msg=f"a={a}")


@pytest.mark.slow
def test_encode_exhaustive_unit_block():
    """Every fp32 n in [-1, 1] (in chunks), in blocks whose absmax is 1 so
    that n = w exactly."""
    top = np.uint32(0x3F800000)
    chunk = 1 << 26
    for s in (0, 1):
        for lo in range(0, int(top) + 1, chunk):
            hi = min(lo + chunk, int(top) + 1)
            vals = np.arange(lo, hi, dtype=np.uint64).astype(np.uint32)
            if s:
                vals |= np.uint32(0x80000000)
            vals = vals.view(np.float32)
            per = 63
            nblk = -(-vals.size // per)
            w = np.zeros((nblk, 64), np.float32)
            w[:, 0] = 1.0
            flat = np.zeros(nblk * per, np.float32)
            flat[: vals.size] = vals
            w[:, 1:] = flat.reshape(nblk, per)
            codes_ref, _, _ = oracle.quantize_nf4(w.reshape(-1))
            W = dev_f32(w.reshape(-1))
            wq = q.qlora_quantize_nf4_dq(W)
            np.testing.assert_array_equal(wq.codes.cpu().numpy(), codes_ref)


@pytest.mark.parametrize("numel", [1, 3, 64, 1000, 64 * 256 * 2 + 77, 4096 * 4096])
def test_dequantize_matches_oracle(numel):
    w = synth.weight_normal(1, 2000 + numel % 991, (numel,), 0.02, 0.001)
    w[::7] = 0.0
    d_ref = oracle.quantize_nf4_dq(w)
    ref = oracle.dequantize(d_ref["codes"], d_ref["c2_fp8"], d_ref["c1"], d_ref["mean"], numel)
    wq = q.qlora_quantize_nf4_dq(dev_f32(w))
    got32 = q.qlora_dequantize(wq, torch.float32).cpu().numpy()
    # fp32: within 1 ulp (the kernels round every step like the oracle, so exact)
    diff = np.abs(got32.view(np.int32).astype(np.int64) - ref.view(np.int32).astype(np.int64))
    assert diff.max() <= 1
    assert np.array_equal(got32, ref)
    got16 = q.qlora_dequantize(wq, torch.bfloat16).view(torch.int16).cpu().numpy().view(np.uint16)
    np.testing.assert_array_equal(got16, oracle.bf16_rne(ref))
    assert np.all(got32[::7] == 0.0)


def test_fp8_encoder_matches_oracle_sweep():
    # every 7th fp32 bit pattern in one call chunk, plus all rounding boundaries
    pats = np.arange(0, 2 ** 32, 7, dtype=np.uint64).astype(np.uint32).view(np.float32)
    x = pats[np.isfinite(pats)]
    got = q.qlora_fp8_e4m3_encode(dev_f32(x)).cpu().numpy()
    ref = oracle.e4m3_encode(x)
    bad = np.nonzero(got != ref)[0]
    assert bad.size == 0, (x[bad[:5]], got[bad[:5]], ref[bad[:5]])
    special = np.float32([np.inf, -np.inf, 448.0, 464.0, 465.0, -1e-30, 2.0 ** -10, 3 * 2.0 ** -11])
    np.testing.assert_array_equal(q.qlora_fp8_e4m3_encode(dev_f32(special)).cpu().numpy(),
                                  oracle.e4m3_encode(special))


def test_quantize_is_deterministic_and_stream_ordered():
    w = synth.weight_normal(3, 3, (2048, 4096), 0.02, 0.001)
    W = dev_f32(w)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        a = q.qlora_quantize_nf4_dq(W)
        b = q.qlora_quantize_nf4_dq(W)
    s.synchronize()
    for x, y in ((a.codes, b.codes), (a.c2_fp8, b.c2_fp8), (a.c1, b.c1), (a.mean, b.mean)):
        assert torch.equal(x, y)
