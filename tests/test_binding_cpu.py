"""The Python binding's argument checks and marshalling, on the CPU: the
library is replaced by a recorder so that no kernel runs.  Shapes that
disagree, wrong dtypes and buffers too small for the weight are refused
before anything reaches the library (its kernels would read out of bounds);
consistent operands reach it with the right sizes."""
import numpy as np
import pytest
import torch

import bit_nf4_quantized_13_b200 as q


class FakeLib:
    def __init__(self, status=0):
        self.calls = []
        self.status = status

    def __getattr__(self, name):
        def fn(*args):
            self.calls.append((name, args))
            if name.endswith("_workspace_size"):
                return 64
            return self.status
        return fn


@pytest.fixture
def fake(monkeypatch):
    lib = FakeLib()
    monkeypatch.setattr(q, "_get_lib", lambda: lib)
    monkeypatch.setattr(q, "_need_cuda", lambda *ts: None)
    monkeypatch.setattr(q, "_stream", lambda stream=None: None)
    return lib


def bf16(*shape):
    return torch.zeros(shape, dtype=torch.bfloat16)


def weight(N, K):
    return q.alloc_nf4_weight((N, K), "cpu")


@pytest.mark.parametrize("M,N,K,r", [(1, 64, 64, 8), (0, 64, 128, 8), (333, 777, 1024, 64),
                                     (4096, 11008, 4096, 64), (16, 5120, 5120, 16)])
def test_consistent_operands_reach_the_library(fake, M, N, K, r):
    w = weight(N, K)
    Y, T = q.qlora_linear_fwd(bf16(M, K), w, bf16(r, K), bf16(N, r), 0.25)
    assert Y.shape == (M, N) and T.shape == (M, r)
    name, args = fake.calls[-1]  # the typed entry point: the data type first
    assert name == "qlora_linear_fwd_4bit" and args[0] == q.TYPE_NF4
    assert args[2:5] == (M, N, K) and args[11] == r
    dX, dA, dB = q.qlora_linear_bwd(bf16(M, N), bf16(M, K), w, bf16(r, K), bf16(N, r), 0.25, T=T)
    assert dX.shape == (M, K) and dA.shape == (r, K) and dB.shape == (N, r)
    name, args = fake.calls[-1]
    assert name == "qlora_linear_bwd_4bit" and args[0] == q.TYPE_NF4
    assert args[3:6] == (M, N, K) and args[12] == r


def test_disagreeing_operands_are_refused(fake):
    M, N, K, r = 8, 128, 256, 16
    w = weight(N, K)
    X, A, B, dY = bf16(M, K), bf16(r, K), bf16(N, r), bf16(M, N)
    bad_fwd = [
        (bf16(M, K + 64), w, A, B),                 # X and the weight disagree on K
        (X, w, bf16(r, K - 64), B),                 # A's K
        (X, w, A, bf16(N + 1, r)),                  # B's N
        (X, w, A, bf16(N, r + 8)),                  # B's r
        (X.float(), w, A, B),                       # dtype
        (X, q.Nf4Weight(w.codes[:10], w.c2_fp8, w.c1, w.mean, (N, K)), A, B),  # codes too small
        (X, q.Nf4Weight(w.codes, w.c2_fp8, w.c1.double(), w.mean, (N, K)), A, B),  # c1 dtype
        (bf16(M, K, 1), w, A, B),                   # not 2-D
    ]
    for args in bad_fwd:
        with pytest.raises(ValueError):
            q.qlora_linear_fwd(*args, 1.0)
    with pytest.raises(ValueError):
        q.qlora_linear_fwd(X, w, A, B, 1.0, Y=bf16(M, N + 1))
    with pytest.raises(ValueError):
        q.qlora_linear_fwd(X, w, A, B, 1.0, T_save=bf16(M, r + 1))
    for kw in ({"T": bf16(M + 1, r)}, {"dX": bf16(M, K + 1)}, {"dA": bf16(r, K + 1)}, {"dB": bf16(N, r + 1)}):
        with pytest.raises(ValueError):
            q.qlora_linear_bwd(dY, X, w, A, B, 1.0, **kw)
    with pytest.raises(ValueError):
        q.qlora_linear_bwd(bf16(M, N + 1), X, w, A, B, 1.0)
    assert fake.calls == [], "nothing may reach the library"


def test_library_status_becomes_an_exception(fake):
    fake.status = 2
    with pytest.raises(q.QloraError) as e:
        q.qlora_linear_fwd(bf16(4, 100), weight(64, 100), bf16(8, 100), bf16(64, 8), 1.0)
    assert e.value.status == 2


def test_quantize_and_dequantize_buffers_are_checked(fake):
    W = torch.zeros((64, 128), dtype=torch.float32)
    w = q.qlora_quantize_nf4_dq(W)
    assert fake.calls[-1][0] == "qlora_quantize_4bit_dq" and fake.calls[-1][1][0] == q.TYPE_NF4
    assert fake.calls[-1][1][2] == W.numel()
    wf = q.qlora_quantize_nf4_dq(W, qtype=q.TYPE_FP4)  # the data type reaches the library and stays with the weight
    assert fake.calls[-1][1][0] == q.TYPE_FP4 and wf.qtype == q.TYPE_FP4
    q.qlora_dequantize(wf, torch.float32)
    assert fake.calls[-1][0] == "qlora_dequantize_4bit" and fake.calls[-1][1][0] == q.TYPE_FP4
    small = q.Nf4Weight(w.codes[:100], w.c2_fp8, w.c1, w.mean, (64, 128))
    with pytest.raises(ValueError):
        q.qlora_quantize_nf4_dq(W, out=small)
    with pytest.raises(ValueError):
        q.qlora_dequantize(small, torch.bfloat16)
    with pytest.raises(ValueError):
        q.qlora_dequantize(w, torch.bfloat16, out=torch.zeros(10, dtype=torch.bfloat16))
    with pytest.raises(ValueError):
        q.qlora_dequantize(w, torch.bfloat16, out=torch.zeros(64 * 128, dtype=torch.float32))
    out = q.qlora_dequantize(w, torch.bfloat16)
    assert out.shape == (64, 128) and out.dtype == torch.bfloat16
    with pytest.raises(ValueError):
        q.qlora_fp8_e4m3_encode(torch.zeros(8, dtype=torch.float64))
    with pytest.raises(ValueError):
        q.qlora_quantize_nf4_dq(W, status=torch.zeros(1, dtype=torch.int64))
    q.qlora_quantize_nf4_dq(W, status=torch.zeros(1, dtype=torch.int32))


def test_cpu_tensors_are_refused_without_the_fake():
    with pytest.raises(ValueError):
        q._need_cuda(torch.zeros(4))


def test_group_operands_reach_the_library(fake):
    M, K, r = 48, 256, 16
    ws_ = [weight(512, K), weight(256, K), weight(256, K)]
    A_cat, B_cat = bf16(3 * r, K), bf16(1024, r)
    Y, T = q.qlora_linear_group_fwd(bf16(M, K), ws_, A_cat, B_cat, 0.5)
    assert Y.shape == (M, 1024) and T.shape == (M, 3 * r)
    name, args = fake.calls[-1]
    assert name == "qlora_linear_group_fwd" and args[0] == q.TYPE_NF4
    assert args[2:4] == (M, K) and args[5] == 3 and args[8] == r
    desc = args[4]  # the host array of weight descriptors
    assert [desc[i].N for i in range(3)] == [512, 256, 256]
    assert desc[1].codes == ws_[1].codes.data_ptr()
    dX, dA, dB = q.qlora_linear_group_bwd(bf16(M, 1024), bf16(M, K), ws_, A_cat, B_cat, 0.5, T=T)
    assert dX.shape == (M, K) and dA.shape == (3 * r, K) and dB.shape == (1024, r)
    name, args = fake.calls[-1]
    assert name == "qlora_linear_group_bwd" and args[3:5] == (M, K) and args[6] == 3 and args[9] == r


def test_group_disagreeing_operands_are_refused(fake):
    M, K, r = 8, 128, 8
    w1, w2 = weight(256, K), weight(256, K)
    X, A_cat, B_cat = bf16(M, K), bf16(2 * r, K), bf16(512, r)
    bad = [
        (X, [w1, weight(256, K + 64)], A_cat, B_cat),        # the weights disagree on K
        (X, [w1, w2], bf16(2 * r + 1, K), B_cat),            # A_cat rows not G r
        (X, [w1, w2], A_cat, bf16(511, r)),                  # B_cat rows not sum N_g
        (X, [w1, w2, w1, w2, w1], bf16(5 * r, K), bf16(1280, r)),  # more than four linears
        (X, [], A_cat, B_cat),                               # no linear
        (X.float(), [w1, w2], A_cat, B_cat),                 # dtype
    ]
    for args in bad:
        with pytest.raises(ValueError):
            q.qlora_linear_group_fwd(*args, 1.0)
    w_fp4 = q.alloc_nf4_weight((256, K), "cpu", q.TYPE_FP4)
    with pytest.raises(ValueError):  # one 4-bit type per group
        q.qlora_linear_group_fwd(X, [w1, w_fp4], A_cat, B_cat, 1.0)
    with pytest.raises(ValueError):
        q.qlora_linear_group_bwd(bf16(M, 511), X, [w1, w2], A_cat, B_cat, 1.0)
    assert fake.calls == [], "nothing may reach the library"
