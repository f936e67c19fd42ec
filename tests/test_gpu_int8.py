"""GPU parity of the block-wise Int8 absmax quantization (study notes 3.1,
eq. 1) and dequantization (eq. 2) against the CPU oracle, through the C ABI:
codes and per-block constants bit-exact, dequantized fp32 bit-exact (both
sides compute RN32(127/absmax), RN32(c x), round half away from zero and
RN32(code / c)).  Ragged tails, zero blocks, every supported block size, and
the non-finite status."""
import numpy as np
import pytest
import torch

import oracle
import synth
from helpers import dev_f32

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a CUDA GPU", allow_module_level=True)

import bit_nf4_quantized_13_b200 as q  # noqa: E402


def _check(x, block):
    codes, c = q.qlora_int8_quantize(dev_f32(x), block)
    deq = q.qlora_int8_dequantize(codes, c, block)
    torch.cuda.synchronize()
    rc, rcc = oracle.int8_quant_blocks(x, block)
    np.testing.assert_array_equal(codes.cpu().numpy().reshape(-1), rc)
    np.testing.assert_array_equal(c.cpu().numpy()[:rcc.size].view(np.uint32), rcc.view(np.uint32))
    rd = oracle.int8_dequant_blocks(rc, rcc, block)
    np.testing.assert_array_equal(deq.cpu().numpy().reshape(-1).view(np.uint32), rd.view(np.uint32))


@pytest.mark.parametrize("block", [32, 64, 128, 256])
@pytest.mark.parametrize("n", [1, 31, 64, 1000, 64 * 4097 + 5, 1 << 20])
def test_int8_matches_oracle(block, n):
    x = synth.weight_normal(3, 900 + n % 97, (n,), 0.02, 0.001)
    _check(x, block)


def test_int8_zero_blocks_and_extremes():
    x = synth.weight_student_t(4, 901, (64 * 300 + 7,))
    x[64 * 10:64 * 12] = 0.0                 # two zero blocks: c = 0, codes 0, dequant 0
    x[64 * 20:64 * 21] = 3.0e38              # a block at the top of the fp32 range
    x[64 * 30:64 * 31] = 1.0e-30             # tiny values (c stays finite)
    x[64 * 40 + 5] = -7.5                    # an outlier
    _check(x, 64)


def test_int8_llama7b_shaped_weight():
    x = synth.weight_normal(0, 902, (4096, 4096), 0.02, 0.001).reshape(-1)
    _check(x, 64)


def test_int8_nonfinite_status():
    x = synth.weight_normal(5, 903, (64 * 50,), 0.02).copy()
    st = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    q.qlora_int8_quantize(dev_f32(x), 64, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    x[64 * 7 + 3] = np.nan
    q.qlora_int8_quantize(dev_f32(x), 64, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 5
