"""The allocation-free quantize entry point, for callers that cannot
allocate device memory (for example a plugin whose host application owns
the whole device-memory budget, or a loop that cannot pay cudaMalloc's
implicit synchronisation).  Through the C ABI it must give the same bytes
as qlora_quantize_nf4_dq with a caller workspace, on two calls in a row
(the second on a different input, so stale scratch contents would show),
and refuse inputs beyond its built-in scratch.  Collected last on purpose."""
import ctypes

import numpy as np
import pytest
import torch

import synth

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a CUDA GPU", allow_module_level=True)

import bit_nf4_quantized_13_b200 as q  # noqa: E402


def _p(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else None


def _via_abi_noalloc(W):
    """Call qlora_quantize_nf4_dq_noalloc through the C ABI with raw pointers."""
    out = q.alloc_nf4_weight(tuple(W.shape), W.device)
    status = torch.full((1,), -1, dtype=torch.int32, device=W.device)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    st = q.lib.qlora_quantize_nf4_dq_noalloc(_p(W), W.numel(), 64, 256, _p(out.codes), _p(out.c2_fp8),
                                             _p(out.c1), _p(out.mean), _p(status), stream)
    assert st == 0
    return out, status


def _via_abi_workspace(W):
    out = q.alloc_nf4_weight(tuple(W.shape), W.device)
    n = W.numel()
    ws = torch.empty(q.qlora_quantize_workspace_size(n), dtype=torch.uint8, device=W.device)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    st = q.lib.qlora_quantize_nf4_dq(_p(W), n, 64, 256, _p(out.codes), _p(out.c2_fp8), _p(out.c1),
                                     _p(out.mean), _p(ws), ws.numel(), None, stream)
    assert st == 0
    return out


def _same(a, b):
    for x, y in ((a.codes, b.codes), (a.c2_fp8, b.c2_fp8), (a.c1, b.c1), (a.mean, b.mean)):
        assert torch.equal(x, y)


def test_noalloc_matches_workspace_entry_on_two_calls_in_a_row():
    W1 = torch.from_numpy(synth.weight_normal(0, 501, (11008, 4096), 0.02, 0.001)).cuda()
    W2 = torch.from_numpy(synth.weight_student_t(0, 502, (3000 * 64 + 17,))).cuda()
    first, s1 = _via_abi_noalloc(W1)
    second, s2 = _via_abi_noalloc(W2)
    torch.cuda.synchronize()
    assert int(s1.item()) == 0 and int(s2.item()) == 0
    _same(first, _via_abi_workspace(W1))
    _same(second, _via_abi_workspace(W2))
    # and once more on the first input after the second call used the scratch
    again, _ = _via_abi_noalloc(W1)
    _same(again, first)


@pytest.mark.parametrize("numel", [1, 17, 63, 64, 65, 64 * 257 + 3])
def test_noalloc_small_and_ragged_sizes(numel):
    W = torch.from_numpy(synth.weight_normal(0, 503, (numel,), 0.02, 0.01)).cuda()
    got, st = _via_abi_noalloc(W)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    _same(got, _via_abi_workspace(W))


def test_noalloc_empty_input_launches_nothing():
    n0 = q.qlora_kernel_launch_count()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    assert q.lib.qlora_quantize_nf4_dq_noalloc(None, 0, 64, 256, None, None, None, None, None, stream) == 0
    assert q.qlora_kernel_launch_count() == n0


def test_noalloc_call_takes_no_device_memory():
    """With torch's caching allocator holding everything the call needs, a
    warmed-up call leaves the device's free memory exactly where it was."""
    W = torch.from_numpy(synth.weight_normal(0, 504, (4096, 1024), 0.02, 0.001)).cuda()
    out = q.alloc_nf4_weight(tuple(W.shape), W.device)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)

    def call():
        st = q.lib.qlora_quantize_nf4_dq_noalloc(_p(W), W.numel(), 64, 256, _p(out.codes), _p(out.c2_fp8),
                                                 _p(out.c1), _p(out.mean), None, stream)
        assert st == 0

    call()  # first call in this context: the scratch address is looked up here
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    for _ in range(3):
        call()
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    assert free1 == free0


def test_noalloc_rejects_sizes_beyond_its_scratch():
    P = 1 << 20  # never dereferenced: the size check comes first
    st = q.lib.qlora_quantize_nf4_dq_noalloc(P, q.NOALLOC_MAX_NUMEL + 1, 64, 256, P, P, P, P, None, None)
    assert st == 3
