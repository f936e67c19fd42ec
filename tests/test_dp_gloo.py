"""The data-parallel path on CPU: two gloo ranks split the tokens, compute
their adapter gradients with the oracle, and all-reduce them; the sum must
equal the single-process gradients of the whole batch (dA and dB are sums
over tokens)."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from bit_nf4_quantized_13_b200.dp import allreduce_adapter_grads, shard_rows


def test_shard_rows_partition():
    for M in (0, 1, 7, 4096, 4097):
        for world in (1, 2, 3, 8):
            spans = [shard_rows(M, r, world) for r in range(world)]
            assert spans[0][0] == 0 and spans[-1][1] == M
            assert all(spans[i][1] == spans[i + 1][0] for i in range(world - 1))
            sizes = [b - a for a, b in spans]
            assert max(sizes) - min(sizes) <= 1
    with pytest.raises(ValueError):
        shard_rows(10, 2, 2)


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=__import__("datetime").timedelta(seconds=60))
    try:
        import oracle
        import synth
        case = synth.linear_case("dp", 10, 24, 64, 4, 16.0, seed=7)
        Wb = synth.bf16_normal(7, 99, (case.N, case.K), 0.02)
        a, b = shard_rows(case.M, rank, world)
        _, dA, dB = oracle.linear_bwd(case.dY[a:b], case.X[a:b], Wb, case.A, case.B, case.s,
                                      want_dx=False)
        tA, tB = torch.from_numpy(dA.copy()), torch.from_numpy(dB.copy())
        allreduce_adapter_grads(tA, tB)
        if rank == 0:
            _, rA, rB = oracle.linear_bwd(case.dY, case.X, Wb, case.A, case.B, case.s, want_dx=False)
            out.put((float(np.max(np.abs(tA.numpy() - rA))), float(np.max(np.abs(tB.numpy() - rB))),
                     float(np.max(np.abs(rA))), float(np.max(np.abs(rB)))))
    finally:
        dist.destroy_process_group()


def test_two_rank_allreduce_matches_full_batch():
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
    assert all(p.exitcode == 0 for p in procs)
    eA, eB, mA, mB = out.get(timeout=5)
    # fp32 transport of fp64 partial sums
    assert eA <= 1e-6 * max(mA, 1e-30) and eB <= 1e-6 * max(mB, 1e-30)
