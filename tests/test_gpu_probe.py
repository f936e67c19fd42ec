"""The DRAM-ceiling probes the bench measures with: the fill writes every
word, the read pass folds what it reads (observable through its `never`
word)."""
import pytest
import torch

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a CUDA GPU", allow_module_level=True)

import bit_nf4_quantized_13_b200 as q  # noqa: E402


@pytest.mark.parametrize("n_words", [4, 4096, (1 << 20) + 12, 3 * (1 << 22)])
def test_fill_writes_every_word(n_words):
    buf = torch.zeros(n_words, dtype=torch.int32, device="cuda")
    q.qlora_debug_fill(buf, 0xDEADBEEF)
    torch.cuda.synchronize()
    assert torch.all(buf == torch.tensor(0xDEADBEEF, dtype=torch.int64).to(torch.int32).item())


def test_read_folds_what_it_reads():
    src = torch.arange(1, 9, dtype=torch.int32, device="cuda")  # two 16-byte runs
    sink = torch.zeros(1, dtype=torch.int32, device="cuda")
    q.qlora_debug_read(src, sink, never=1 ^ 2 ^ 3 ^ 4)  # the first run's fold
    torch.cuda.synchronize()
    assert sink.item() == 1 ^ 2 ^ 3 ^ 4
    sink.zero_()
    q.qlora_debug_read(src, sink, never=0x7FFFFFFF)  # no thread folds to this
    torch.cuda.synchronize()
    assert sink.item() == 0
