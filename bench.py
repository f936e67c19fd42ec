#!/usr/bin/env python
"""Benchmark of the QLoRA NF4 linear hot path on B200.

Workload (one step): for each of the two LLaMA-7B-shaped linears -- W
4096x4096 and 11008x4096 fp32 ~N(0, 0.02) with 0.1% of entries x8, X 4096
tokens x 4096 bf16, rank r = 64, alpha = 16 -- quantize W to NF4 with double
quantization, run the forward Y = X W'^T + s (X A^T) B^T, and the backward
(dX, dA, dB).  Synthetic, seeded inputs (synth.py).  The metric is the
algorithmic fwd+bwd FLOP rate, 4MNK + 6Mr(N+K) per linear, over the whole
step (quantization included).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl native|reference]

Under torchrun each rank runs its own token batch against replicated frozen
weights (weak scaling) and the adapter gradients are all-reduced every step.
Rank 0 prints one JSON line.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

import synth  # noqa: E402

METRIC = "QLoRA linear fwd+bwd TFLOP/s & NF4 quant/dequant GB/s, % of roofline"
WORKLOAD = "llama7b_linears_w4096x4096_w11008x4096_m4096_r64_alpha16_quantize_fwd_bwd"
M_TOKENS, RANK, ALPHA = 4096, 64, 16.0
L2_FLUSH_BYTES = 256 << 20
PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# DRAM bytes (read + write) per call of the dX GEMM, mean over the two linears, from one ncu
# capture of the kernel as it is now (profiles/k_nf4_gemm_pair_llama7b_m4096.md: 43.73 MB for
# the 4096x4096 linear, whose 33.5 MB dX is still in L2 when the launch ends, and 174.99 MB for
# the 11008x4096 one); None when the kernel has changed since then.
DX_TRAFFIC_BYTES = 109.36e6


def linear_flops(M, N, K, r):
    return 4 * M * N * K + 6 * M * r * (N + K)


def fwd_flops(M, N, K, r):
    return 2 * M * N * K + 2 * M * r * (N + K)


def quant_bytes(numel):
    nb = -(-numel // 64)
    return 4 * numel + (numel + 1) // 2 + nb + 4 * (-(-nb // 256)) + 4


def dequant_bytes(numel, out_bytes):
    nb = -(-numel // 64)
    return (numel + 1) // 2 + nb + 4 * (-(-nb // 256)) + 4 + out_bytes * numel


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(PEAKS_FALLBACK), "fallback"


class NvmlClockSampler:
    """SM clock and clock-event reasons read through NVML (read-only
    queries) every millisecond from a thread, so that even a timed region of
    a few milliseconds holds many samples.  Raises if NVML is unavailable."""
    REASONS = (("hw_slowdown", "nvmlClocksEventReasonHwSlowdown"),
               ("hw_thermal_slowdown", "nvmlClocksEventReasonHwThermalSlowdown"),
               ("sw_thermal_slowdown", "nvmlClocksEventReasonSwThermalSlowdown"),
               ("sw_power_cap", "nvmlClocksEventReasonSwPowerCap"))

    def __init__(self, torch_device_index: int, interval_s: float = 0.001):
        import pynvml
        import torch
        self.nv = pynvml
        pynvml.nvmlInit()
        handle = None
        try:  # the CUDA device's own GPU, whatever the visible-device mapping
            pr = torch.cuda.get_device_properties(torch_device_index)
            bus = f"{pr.pci_domain_id:08x}:{pr.pci_bus_id:02x}:{pr.pci_device_id:02x}.0"
            handle = pynvml.nvmlDeviceGetHandleByPciBusId(bus)
        except Exception:
            handle = pynvml.nvmlDeviceGetHandleByIndex(torch_device_index)
        self.h = handle
        self.max_mhz = float(pynvml.nvmlDeviceGetMaxClockInfo(handle, pynvml.NVML_CLOCK_SM))
        self.masks = [(nm, getattr(pynvml, attr)) for nm, attr in self.REASONS]
        self.lines = []
        self.stop_flag = False
        self.interval = interval_s
        self.t = threading.Thread(target=self._poll, daemon=True)
        self.t.start()

    def _poll(self):
        nv = self.nv
        while not self.stop_flag:
            try:
                sm = float(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
                rs = int(nv.nvmlDeviceGetCurrentClocksEventReasons(self.h))
                self.lines.append((time.time(), sm, rs))
            except Exception:
                pass
            time.sleep(self.interval)

    def stop(self):
        self.stop_flag = True
        self.t.join(timeout=5)

    def summary(self, t0, t1):
        rows = [x for x in self.lines if t0 <= x[0] <= t1] or list(self.lines)
        if not rows:
            return None
        reasons = sorted({nm for (_, _, rs) in rows for nm, m in self.masks if rs & m})
        return {"sm_mhz": statistics.median(r[1] for r in rows), "sm_max_mhz": self.max_mhz,
                "reasons": reasons, "samples": len(rows), "source": "nvml, 1 ms polling"}


def clock_sampler(device_index: int):
    try:
        return NvmlClockSampler(device_index)
    except Exception:
        return ClockSampler(device_index)


class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons during a window."""
    FIELDS = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int, interval_ms: int = 10):
        self.lines = []
        self.proc = None
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-i", str(device_index), "-lms", str(interval_ms)],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except (OSError, FileNotFoundError):
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append((time.time(), line.strip()))

    def stop(self):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self, t0, t1):
        if self.proc is None:
            return None
        rows = [l for (t, l) in self.lines if t0 <= t <= t1] or [l for (_, l) in self.lines]
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for l in rows:
            parts = [p.strip() for p in l.split(",")]
            if len(parts) < 10:
                continue
            try:
                sm.append(float(parts[2]))
                mx.append(float(parts[3]))
            except ValueError:
                continue
            for nm, v in zip(names, parts[6:10]):
                if v.lower().startswith("active"):
                    reasons.add(nm)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm)}


class L2Flush:
    """Leaves the L2 cache holding only clean lines of a buffer no kernel
    uses: a write of one buffer larger than L2, then a read of another one.
    The read evicts the write's dirty lines (their write-back happens here,
    outside any timed region), so the next timed kernel neither finds its
    inputs in L2 nor pays for writing back someone else's dirty lines."""

    def __init__(self, torch, dev, nbytes: int = L2_FLUSH_BYTES):
        self.w = torch.empty(nbytes, dtype=torch.uint8, device=dev)
        self.r = torch.ones(nbytes // 4, dtype=torch.int32, device=dev)
        self.sink = torch.empty((), dtype=torch.int32, device=dev)

    def __call__(self):
        self.w.zero_()
        self.sink.copy_(self.r.max())


def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


# ---------------------------------------------------------------- oracle arm

def oracle_weight_bf16(case):
    """The bf16 weight the linear consumes, from the oracle's own NF4 round
    trip (computed once per linear, outside any timing)."""
    import oracle
    W = case.W.reshape(-1)
    d = oracle.quantize_nf4_dq(W)
    return oracle.bf16_rne(oracle.dequantize(d["codes"], d["c2_fp8"], d["c1"], d["mean"],
                                             W.size)).reshape(case.N, case.K)


def oracle_sample(case, Wb, rows_m: int, quant_elems: int):
    """Time the CPU oracle on a bounded sample of one linear: quantization of
    the first `quant_elems` weights, and fwd+bwd on the first `rows_m`
    tokens against the full weight.  Returns (t_quant, t_linear, flops, bytes)."""
    import oracle
    W = case.W.reshape(-1)
    t0 = time.perf_counter()
    oracle.quantize_nf4_dq(W[:quant_elems])
    tq = time.perf_counter() - t0
    X, dY = case.X[:rows_m], case.dY[:rows_m]
    t1 = time.perf_counter()
    oracle.linear_fwd(X, Wb, case.A, case.B, case.s)
    oracle.linear_bwd(dY, X, Wb, case.A, case.B, case.s)
    tl = time.perf_counter() - t1
    return tq, tl, linear_flops(rows_m, case.N, case.K, case.r), quant_bytes(quant_elems)


def oracle_baseline(cases, wbs, rows_m=4, quant_elems=1 << 22):
    import oracle
    tq_tot = tl_tot = fl_tot = qb_tot = 0.0
    for c, wb in zip(cases, wbs):
        tq, tl, fl, qb = oracle_sample(c, wb, rows_m, quant_elems)
        tq_tot += tq
        tl_tot += tl
        fl_tot += fl
        qb_tot += qb
    return {"value": fl_tot / tl_tot / 1e12, "unit": "TFLOP/s", "cores": oracle.threads(),
            "kind": "oracle",
            "sample": (f"fwd+bwd of {rows_m} tokens per linear (full N, K, r=64) and quantization of "
                       f"the first {quant_elems} weights per linear, both linears"),
            "quant_gbs": qb_tot / tq_tot / 1e9, "seconds": tl_tot + tq_tot}


def oracle_decode_baseline():
    """The oracle's small-batch forward at the LLaMA-13B decode shapes, in
    full: W 5120x5120 and 13824x5120, one token, r = 16 (the forward over
    the oracle's own bf16 dequantized weight; its NF4 round trip is done
    beforehand, untimed).  GB/s counts the same algorithmic bytes as the
    GPU's decode entries."""
    import oracle
    out = {}
    for which in range(2):
        c = synth.decode13b_linear(which, 1, seed=0)
        wb = oracle_weight_bf16(c)
        t0 = time.perf_counter()
        oracle.linear_fwd(c.X, wb, c.A, c.B, c.s)
        dt = time.perf_counter() - t0
        nbytes = decode_bytes(1, c.N, c.K, c.r)
        out[f"{c.N}x{c.K}_m1"] = {"ms": dt * 1e3, "gbs": nbytes / dt / 1e9}
    return out


def run_reference(args, world, rank):
    if rank != 0:
        return 0
    cases = [synth.llama7b_linear(i, seed=0, M=M_TOKENS) for i in range(2)]
    wbs = [oracle_weight_bf16(c) for c in cases]
    for _ in range(args.warmup):
        oracle_baseline(cases, wbs, rows_m=1, quant_elems=1 << 16)
    vals = []
    t_all = 0.0
    for _ in range(args.steps):
        b = oracle_baseline(cases, wbs, rows_m=2, quant_elems=1 << 20)
        vals.append(b["value"])
        t_all += b["seconds"]
    value = statistics.mean(vals)
    line = {"metric": METRIC, "value": value, "unit": "TFLOP/s", "impl": "reference", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * t_all / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": {"workload": WORKLOAD, "sample": "2 tokens per linear"},
            "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": b["cores"], "kind": "oracle",
                             "sample": "fwd+bwd of 2 tokens per linear and quantization of 2^20 weights "
                                       "per linear, per step"},
            "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------- native arm

def run_native(args, world, rank, local):
    import torch
    import torch.distributed as dist

    import bit_nf4_quantized_13_b200 as q
    from bit_nf4_quantized_13_b200.dp import allreduce_adapter_grads

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)

    def to_bf16(bits):
        return torch.from_numpy(bits.view(np.int16)).to(dev).view(torch.bfloat16)

    cases = []
    for i in range(2):
        c = synth.llama7b_linear(i, seed=0, M=M_TOKENS)
        if world > 1:  # every rank its own tokens, the same frozen weight and adapters
            xc = synth.linear_case("x", M_TOKENS, c.N, c.K, RANK, ALPHA, seed=1000 + rank,
                                   wid=i)
            c.X, c.dY = xc.X, xc.dY
        cases.append(c)

    bufs = []
    for c in cases:
        b = {"case": c}
        b["W"] = torch.from_numpy(c.W).to(dev)
        b["X"], b["A"], b["B"], b["dY"] = to_bf16(c.X), to_bf16(c.A), to_bf16(c.B), to_bf16(c.dY)
        b["wq"] = q.alloc_nf4_weight((c.N, c.K), dev)
        b["qws"] = torch.empty(q.qlora_quantize_workspace_size(c.W.size), dtype=torch.uint8, device=dev)
        b["Y"] = torch.empty((c.M, c.N), dtype=torch.bfloat16, device=dev)
        b["T"] = torch.empty((c.M, c.r), dtype=torch.bfloat16, device=dev)
        b["dX"] = torch.empty((c.M, c.K), dtype=torch.bfloat16, device=dev)
        b["dA"] = torch.empty((c.r, c.K), dtype=torch.bfloat16, device=dev)
        b["dB"] = torch.empty((c.N, c.r), dtype=torch.bfloat16, device=dev)
        b["bws"] = torch.empty(q.qlora_linear_bwd_workspace_size(c.M, c.N, c.K, c.r), dtype=torch.uint8,
                               device=dev)
        b["Wdq"] = torch.empty((c.N, c.K), dtype=torch.bfloat16, device=dev)
        bufs.append(b)
    flush = L2Flush(torch, dev)
    stream = torch.cuda.current_stream()

    def step(ev=None):
        for i, b in enumerate(bufs):
            c = b["case"]
            if ev is not None:
                ev[i][0].record(stream)
            q.qlora_quantize_nf4_dq(b["W"], out=b["wq"], ws=b["qws"])
            if ev is not None:
                ev[i][1].record(stream)
            q.qlora_linear_fwd(b["X"], b["wq"], b["A"], b["B"], c.s, Y=b["Y"], T_save=b["T"], ws=b["bws"])
            if ev is not None:
                ev[i][2].record(stream)
            q.qlora_linear_bwd(b["dY"], b["X"], b["wq"], b["A"], b["B"], c.s, T=b["T"], dX=b["dX"],
                               dA=b["dA"], dB=b["dB"], ws=b["bws"])
            if world > 1:
                allreduce_adapter_grads(b["dA"], b["dB"])
            if ev is not None:
                ev[i][3].record(stream)

    def new_events():
        return [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in bufs]

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()

    clocks = clock_sampler(local)
    time.sleep(0.3)
    launches0 = q.qlora_kernel_launch_count()
    steps_ev, phase_ev = [], []
    t_wall0 = time.time()
    for _ in range(args.steps):
        flush()  # L2 flush between timed steps (outside the step's events)
        s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        pe = new_events()
        s0.record(stream)
        step(pe)
        s1.record(stream)
        steps_ev.append((s0, s1))
        phase_ev.append(pe)
    torch.cuda.synchronize()
    t_wall1 = time.time()
    launches = q.qlora_kernel_launch_count() - launches0
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    clocks.stop()

    step_ms = [a.elapsed_time(b) for a, b in steps_ev]
    total_ms = sum(step_ms)
    if world > 1:
        t = torch.tensor([total_ms], dtype=torch.float64, device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        total_ms = float(t.item())
    ms_per_step = total_ms / args.steps
    flops_step = sum(linear_flops(c.M, c.N, c.K, c.r) for c in cases)
    value = flops_step * world / (ms_per_step * 1e-3) / 1e12

    # per-phase breakdown (rank-local)
    qt = sum(pe[i][0].elapsed_time(pe[i][1]) for pe in phase_ev for i in range(2))
    ft = sum(pe[i][1].elapsed_time(pe[i][2]) for pe in phase_ev for i in range(2))
    bt = sum(pe[i][2].elapsed_time(pe[i][3]) for pe in phase_ev for i in range(2))
    qbytes = sum(quant_bytes(c.W.size) for c in cases) * args.steps
    fflops = sum(fwd_flops(c.M, c.N, c.K, c.r) for c in cases) * args.steps
    bflops = sum(linear_flops(c.M, c.N, c.K, c.r) - fwd_flops(c.M, c.N, c.K, c.r) for c in cases) * args.steps

    # standalone dequantization (row a7), timed separately after the steps
    dq_ms, dq_bytes = 0.0, 0
    for _ in range(3):
        for b in bufs:
            q.qlora_dequantize(b["wq"], torch.bfloat16, out=b["Wdq"])
    for _ in range(max(3, args.steps // 4)):
        for b in bufs:
            flush()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            q.qlora_dequantize(b["wq"], torch.bfloat16, out=b["Wdq"])
            e1.record(stream)
            torch.cuda.synchronize()
            dq_ms += e0.elapsed_time(e1)
            dq_bytes += dequant_bytes(b["case"].W.size, 2)
    # the same to fp32 (the other output type of row a7), into one buffer sized
    # for the larger weight
    dq32_ms, dq32_bytes = 0.0, 0
    w32buf = torch.empty(max(b["case"].W.size for b in bufs), dtype=torch.float32, device=dev)
    for rep in range(max(3, args.steps // 4) + 2):
        for b in bufs:
            n = b["case"].W.size
            flush()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            q.qlora_dequantize(b["wq"], torch.float32, out=w32buf[:n])
            e1.record(stream)
            torch.cuda.synchronize()
            if rep >= 2:
                dq32_ms += e0.elapsed_time(e1)
                dq32_bytes += dequant_bytes(n, 4)
    del w32buf
    other_types = run_other_types(q, torch, dev, stream, flush, bufs, peaks_hbm=load_peaks()[0]["hbm_gbs"])
    # the DRAM ceilings these kernels meet, from the library's own probe
    # kernels (16-byte streaming stores / loads) over a 2 GiB buffer, 16x the
    # L2, so that the cache absorbs a negligible part; torch's fill beside
    ceil_buf = torch.empty(1 << 29, dtype=torch.float32, device=dev)
    ceil_sink = torch.zeros(1, dtype=torch.int32, device=dev)

    def ceiling_gbs(fn):
        ms = 0.0
        for rep in range(5):
            flush()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            fn()
            e1.record(stream)
            torch.cuda.synchronize()
            if rep >= 2:
                ms += e0.elapsed_time(e1)
        return 3 * 4 * ceil_buf.numel() / (ms * 1e-3) / 1e9

    fill_gbs = ceiling_gbs(lambda: q.qlora_debug_fill(ceil_buf, 0x3F800000))
    read_gbs = ceiling_gbs(lambda: q.qlora_debug_read(ceil_buf, ceil_sink))
    torch_fill_gbs = ceiling_gbs(lambda: ceil_buf.fill_(1.0))
    del ceil_buf, ceil_sink
    # time the output bytes alone take at that rate, over the dequant's time
    dq32_write_frac = (sum(4 * b["case"].W.size for b in bufs) / (fill_gbs * 1e9)) / \
        (dq32_ms * 1e-3 / (max(3, args.steps // 4))) if dq32_ms else None
    dq16_write_frac = (sum(2 * b["case"].W.size for b in bufs) / (fill_gbs * 1e9)) / \
        (dq_ms * 1e-3 / (max(3, args.steps // 4))) if dq_ms else None

    # the dominant kernel: the backward's dX GEMM (dX = dY W' + U A), timed
    # live as the backward with dX minus the backward without it, per call,
    # L2 flushed before each
    dx_ms, dx_flops, dx_reps = 0.0, 0.0, max(5, args.steps // 4)
    for rep in range(dx_reps + 2):
        for b in bufs:
            c = b["case"]
            tt = []
            for want in (True, False):
                flush()
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record(stream)
                q.qlora_linear_bwd(b["dY"], b["X"], b["wq"], b["A"], b["B"], c.s, T=b["T"],
                                   dX=b["dX"] if want else None, dA=b["dA"], dB=b["dB"], ws=b["bws"],
                                   want_dx=want)
                e1.record(stream)
                tt.append((e0, e1))
            torch.cuda.synchronize()
            if rep >= 2:
                dx_ms += tt[0][0].elapsed_time(tt[0][1]) - tt[1][0].elapsed_time(tt[1][1])
                dx_flops += 2.0 * c.M * c.N * c.K + 2.0 * c.M * c.r * c.K

    # unfused comparator: dequantize to a bf16 W in HBM, then library GEMMs
    # (torch.matmul / cuBLAS) for the base product and the LoRA path
    k9_ms = 0.0
    k9_reps = max(3, args.steps // 4)
    for rep in range(k9_reps + 2):
        for b in bufs:
            c = b["case"]
            flush()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            q.qlora_dequantize(b["wq"], torch.bfloat16, out=b["Wdq"])
            yk = torch.matmul(b["X"], b["Wdq"].t())
            tk = torch.matmul(b["X"], b["A"].t()).mul_(c.s)
            yk.addmm_(tk, b["B"].t())
            e1.record(stream)
            torch.cuda.synchronize()
            if rep >= 2:
                k9_ms += e0.elapsed_time(e1)
    k9_tflops = sum(fwd_flops(c.M, c.N, c.K, c.r) for c in cases) * k9_reps / (k9_ms * 1e-3) / 1e12

    decode = run_decode(q, torch, dev, stream, flush, args) if rank == 0 and not args.no_decode else None
    peaks, peak_src = load_peaks()
    full7b = run_full_7b_set(q, torch, dev, stream, peaks) if rank == 0 and not args.no_c3 else None
    l65b = run_llama65b_layer(q, torch, dev, stream, flush, peaks, args) if rank == 0 and not args.no_c4 else None

    # the GEMM is timed in short bursts between L2 flushes: the burst peak
    tc_peak = peaks["bf16_tflops"]
    fwd_tflops = fflops / (ft * 1e-3) / 1e12
    if decode:
        for v in decode.values():
            v["frac_hbm"] = v["gbs"] / peaks["hbm_gbs"]
            v["graph_frac_hbm"] = v["graph_gbs"] / peaks["hbm_gbs"]
    dx_tflops = dx_flops / (dx_ms * 1e-3) / 1e12
    roofline = {"kernel": "k_nf4_gemm_pair<1>: dX = dY W' + U A of qlora_linear_bwd "
                          "(largest share of the step in the ncu launch list)",
                "bound": "tensor", "achieved": dx_tflops, "peak": tc_peak, "unit": "TFLOP/s",
                "frac": dx_tflops / tc_peak, "traffic": DX_TRAFFIC_BYTES, "peak_source": peak_src,
                "algorithmic": "2MNK + 2MrK per call (both linears, M=4096, r=64)",
                "timing": "per call: backward with dX minus backward without dX, CUDA events, L2 flushed",
                "peak_kind": "burst (clocks stay at max in the timed region)"}

    # end to end through the C ABI with host buffers: H2D of the step's
    # inputs from pinned memory, the step, D2H of its outputs
    e2e = None
    if not args.no_e2e:
        hin, hout = [], []
        for b in bufs:
            hin.append({k: b[k].cpu().pin_memory() for k in ("W", "X", "A", "B", "dY")})
            hout.append({k: torch.empty_like(b[k], device="cpu").pin_memory() for k in ("Y", "dX", "dA", "dB")})
        h2d = sum(t.numel() * t.element_size() for h in hin for t in h.values())
        d2h = sum(t.numel() * t.element_size() for h in hout for t in h.values())

        def e2e_step():
            for b, hi, ho in zip(bufs, hin, hout):
                for k, t in hi.items():
                    b[k].copy_(t, non_blocking=True)
            step()
            for b, ho in zip(bufs, hout):
                for k, t in ho.items():
                    t.copy_(b[k], non_blocking=True)

        for _ in range(2):
            e2e_step()
        torch.cuda.synchronize()
        ee = []
        for _ in range(max(3, args.steps // 2)):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            e2e_step()
            e1.record(stream)
            ee.append((e0, e1))
        torch.cuda.synchronize()
        e_ms = statistics.mean(a.elapsed_time(b) for a, b in ee)
        if world > 1:
            t = torch.tensor([e_ms], dtype=torch.float64, device=dev)
            dist.all_reduce(t, op=dist.ReduceOp.MAX)
            e_ms = float(t.item())
        e2e = {"value": flops_step * world / (e_ms * 1e-3) / 1e12, "unit": "TFLOP/s",
               "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h), "ms_per_step": e_ms}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = oracle_baseline(cases, [oracle_weight_bf16(c) for c in cases], rows_m=256, quant_elems=1 << 24)
        cpu["decode_13b"] = oracle_decode_baseline()
        cpu["sample"] += "; plus the 13B decode forward (M = 1, both shapes) in full"

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": WORKLOAD, "linears": ["4096x4096", "11008x4096"], "tokens_per_gpu": M_TOKENS,
                       "rank": RANK, "alpha": ALPHA, "block": 64, "block2": 256,
                       "l2": ("flushed between timed steps (256 MiB write, then a 256 MiB read of another buffer, "
                              "so L2 holds only clean lines); inputs also exceed L2"),
                       "parallelism": f"dp{world}"},
            "gpu_launches": int(launches),
            "roofline": roofline,
            "components": {
                "quantize_gbs": qbytes / (qt * 1e-3) / 1e9,
                "quantize_frac_hbm": qbytes / (qt * 1e-3) / 1e9 / peaks["hbm_gbs"],
                "dequant_bf16_gbs": dq_bytes / (dq_ms * 1e-3) / 1e9 if dq_ms else None,
                "dequant_bf16_frac_hbm": (dq_bytes / (dq_ms * 1e-3) / 1e9 / peaks["hbm_gbs"]) if dq_ms else None,
                "dequant_fp32_gbs": dq32_bytes / (dq32_ms * 1e-3) / 1e9 if dq32_ms else None,
                "dequant_fp32_frac_hbm": (dq32_bytes / (dq32_ms * 1e-3) / 1e9 / peaks["hbm_gbs"]) if dq32_ms else None,
                "write_ceiling_gbs": fill_gbs,
                "read_ceiling_gbs": read_gbs,
                "torch_fill_gbs": torch_fill_gbs,
                "quantize_frac_read_ceiling": (sum(4.0 * c.W.size for c in cases) * args.steps / (read_gbs * 1e9))
                / (qt * 1e-3),
                "dequant_fp32_frac_write_ceiling": dq32_write_frac,
                "dequant_bf16_frac_write_ceiling": dq16_write_frac,
                "full_set_dequant_fp32_frac_write_ceiling": (
                    (4.0 * full7b["params"] / (fill_gbs * 1e9)) / (full7b["dequant_fp32_ms"] * 1e-3)
                    if full7b else None),
                "full_set_dequant_bf16_frac_write_ceiling": (
                    (2.0 * full7b["params"] / (fill_gbs * 1e9)) / (full7b["dequant_bf16_ms"] * 1e-3)
                    if full7b else None),
                "ceiling_note": ("ceilings: qlora_debug_fill / qlora_debug_read over a 2 GiB buffer, L2 "
                                 "flushed; frac_write_ceiling = output bytes at the write ceiling over the "
                                 "dequant's time (it also reads 0.52 B per weight), frac_read_ceiling = the "
                                 "4 B per weight read at the read ceiling over the quantize time"),
                "fwd_tflops": fwd_tflops, "fwd_frac_tensor": fwd_tflops / tc_peak,
                "bwd_tflops": bflops / (bt * 1e-3) / 1e12, "dx_path_tflops": dx_tflops,
                "unfused_fwd_tflops": k9_tflops,
                "other_types": other_types,
                "decode": decode,
                "full_llama7b_weight_set": full7b,
                "llama65b_layer": l65b,
                "ms": {"quantize": qt / args.steps, "fwd": ft / args.steps, "bwd": bt / args.steps},
                "peaks": {"hbm_gbs": peaks["hbm_gbs"], "bf16_tflops": tc_peak, "source": peak_src}},
            "clocks": clocks.summary(t_wall0, t_wall1),
            "e2e": e2e,
            "cpu_baseline": cpu,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def run_full_7b_set(q, torch, dev, stream, peaks):
    """The full LLaMA-7B-shaped weight set (224 tensors: 32 layers x q, k, v,
    o 4096^2, gate, up 11008x4096, down 4096x11008; 6 476 005 376 weights,
    Student-t df=5 rescaled to std 0.02), all resident in HBM: quantized
    tensor by tensor, back to back, then dequantized to fp32 and to bf16 the
    same way.  Every pass reads data written long before (26 GB of inputs
    against a 126 MB L2), so no flush is needed.  bits/param counts the four
    stored buffers of every tensor."""
    shapes = synth.llama7b_weight_shapes()
    Ws, wqs = [], []
    for i, (_, n, k) in enumerate(shapes):
        Ws.append(synth.student_t_device(0, 1000 + i, n * k, dev).view(n, k))
        wqs.append(q.alloc_nf4_weight((n, k), dev))
    params = sum(n * k for _, n, k in shapes)
    qws = torch.empty(q.qlora_quantize_workspace_size(max(n * k for _, n, k in shapes)), dtype=torch.uint8,
                      device=dev)
    stored = sum(w.nbytes() for w in wqs)

    def timed(fn, reps=2):
        best = None
        for _ in range(reps):
            torch.cuda.synchronize()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            fn()
            e1.record(stream)
            torch.cuda.synchronize()
            ms = e0.elapsed_time(e1)
            best = ms if best is None else min(best, ms)
        return best

    def quant_all():
        for W, wq in zip(Ws, wqs):
            q.qlora_quantize_nf4_dq(W, out=wq, ws=qws)

    quant_all()  # warm-up (first launches)
    tq = timed(quant_all)
    qbytes = sum(quant_bytes(n * k) for _, n, k in shapes)
    del Ws
    out32 = torch.empty(params, dtype=torch.float32, device=dev)
    offs = np.cumsum([0] + [n * k for _, n, k in shapes])

    def dq_all(dtype, out):
        for j, wq in enumerate(wqs):
            q.qlora_dequantize(wq, dtype, out=out[offs[j]:offs[j + 1]])

    dq_all(torch.float32, out32)
    t32 = timed(lambda: dq_all(torch.float32, out32))
    out16 = out32.view(torch.bfloat16)[:params]
    dq_all(torch.bfloat16, out16)
    t16 = timed(lambda: dq_all(torch.bfloat16, out16))
    b32 = sum(dequant_bytes(n * k, 4) for _, n, k in shapes)
    b16 = sum(dequant_bytes(n * k, 2) for _, n, k in shapes)
    del out32, out16, wqs
    hbm = peaks["hbm_gbs"]
    one = run_one_large_tensor(q, torch, dev, stream, hbm, timed)
    return {"tensors": len(shapes), "params": params, "bits_per_param": 8.0 * stored / params,
            "stored_bytes": stored,
            "quantize_ms": tq, "quantize_gbs": qbytes / (tq * 1e-3) / 1e9,
            "quantize_frac_hbm": qbytes / (tq * 1e-3) / 1e9 / hbm,
            "dequant_fp32_ms": t32, "dequant_fp32_gbs": b32 / (t32 * 1e-3) / 1e9,
            "dequant_fp32_frac_hbm": b32 / (t32 * 1e-3) / 1e9 / hbm,
            "dequant_bf16_ms": t16, "dequant_bf16_gbs": b16 / (t16 * 1e-3) / 1e9,
            "dequant_bf16_frac_hbm": b16 / (t16 * 1e-3) / 1e9 / hbm,
            "inputs": "Student-t df=5 x 0.02/sqrt(5/3), generated on the GPU (synth.student_t_device, seed 0)",
            "one_tensor_32768x32768": one}


def run_one_large_tensor(q, torch, dev, stream, hbm, timed):
    """One 32768 x 32768 weight (2^30 weights, Student-t as the 7B set, 4 GiB
    of fp32 against a 126 MB L2): quantize, dequantize to fp32 and to bf16,
    each timed alone, so that the per-call fixed cost (launches, the bins'
    clearing, the double quantization) is small against the streaming."""
    n = 1 << 30
    W = synth.student_t_device(0, 5000, n, dev).view(32768, 32768)
    wq = q.alloc_nf4_weight((32768, 32768), dev)
    qws = torch.empty(q.qlora_quantize_workspace_size(n), dtype=torch.uint8, device=dev)
    q.qlora_quantize_nf4_dq(W, out=wq, ws=qws)
    tq = timed(lambda: q.qlora_quantize_nf4_dq(W, out=wq, ws=qws), reps=3)
    del W
    out = {"quantize_ms": tq, "quantize_gbs": quant_bytes(n) / (tq * 1e-3) / 1e9}
    for name, dtype, nbytes in (("fp32", torch.float32, 4), ("bf16", torch.bfloat16, 2)):
        o = torch.empty((32768, 32768), dtype=dtype, device=dev)
        q.qlora_dequantize(wq, dtype, out=o)
        t = timed(lambda: q.qlora_dequantize(wq, dtype, out=o), reps=3)
        out[f"dequant_{name}_ms"] = t
        out[f"dequant_{name}_gbs"] = dequant_bytes(n, nbytes) / (t * 1e-3) / 1e9
        del o
    for k in [k for k in out if k.endswith("_gbs")]:
        out[k.replace("_gbs", "_frac_hbm")] = out[k] / hbm
    return out


def run_llama65b_layer(q, torch, dev, stream, flush, peaks, args):
    """A LLaMA-65B-shaped decoder layer's seven linears (q, k, v, o 8192^2,
    gate, up 22016x8192, down 8192x22016; r=64, alpha=16, LoRA on every
    linear): per token count M in 512/2048/8192, the forward and backward
    (dX, dA, dB) of all seven, timed per linear with CUDA events; one layer
    pass per timed iteration, L2 flushed between iterations."""
    layer = synth.LLAMA65B_LAYER
    wqs = []
    for i, (_, n, k) in enumerate(layer):
        W = synth.normal_device(0, 2000 + i, (n, k), dev, std=0.02)
        wqs.append(q.qlora_quantize_nf4_dq(W))
        del W
    reps = max(3, min(10, args.steps // 5))
    out = {}
    tc_b, tc_s = peaks["bf16_tflops"], peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"])
    sampler = clock_sampler(dev.index if dev.index is not None else 0)  # clocks of these long dense runs
    for M in synth.LLAMA65B_TOKENS:
        lin = []
        for i, (nm, n, k) in enumerate(layer):
            d = {"name": nm, "N": n, "K": k}
            d["X"] = synth.normal_device(1, 3000 + 10 * i, (M, k), dev, dtype=torch.bfloat16)
            d["dY"] = synth.normal_device(1, 3001 + 10 * i, (M, n), dev, dtype=torch.bfloat16)
            d["A"] = synth.normal_device(1, 3002 + 10 * i, (RANK, k), dev, std=0.01, dtype=torch.bfloat16)
            d["B"] = synth.normal_device(1, 3003 + 10 * i, (n, RANK), dev, std=0.01, dtype=torch.bfloat16)
            d["Y"] = torch.empty((M, n), dtype=torch.bfloat16, device=dev)
            d["T"] = torch.empty((M, RANK), dtype=torch.bfloat16, device=dev)
            d["dX"] = torch.empty((M, k), dtype=torch.bfloat16, device=dev)
            d["dA"] = torch.empty((RANK, k), dtype=torch.bfloat16, device=dev)
            d["dB"] = torch.empty((n, RANK), dtype=torch.bfloat16, device=dev)
            d["ws"] = torch.empty(q.qlora_linear_bwd_workspace_size(M, n, k, RANK), dtype=torch.uint8, device=dev)
            lin.append(d)
        s_lora = ALPHA / RANK

        def layer_pass(ev=None):
            for i, (d, wq) in enumerate(zip(lin, wqs)):
                if ev is not None:
                    ev[i][0].record(stream)
                q.qlora_linear_fwd(d["X"], wq, d["A"], d["B"], s_lora, Y=d["Y"], T_save=d["T"], ws=d["ws"])
                if ev is not None:
                    ev[i][1].record(stream)
                q.qlora_linear_bwd(d["dY"], d["X"], wq, d["A"], d["B"], s_lora, T=d["T"], dX=d["dX"],
                                   dA=d["dA"], dB=d["dB"], ws=d["ws"])
                if ev is not None:
                    ev[i][2].record(stream)

        block_pass, parts = grouped_block(q, torch, dev, lin, wqs, M)
        layer_pass()
        block_pass()
        torch.cuda.synchronize()
        tw0 = time.time()
        fwd_ms = [0.0] * len(layer)
        bwd_ms = [0.0] * len(layer)
        tot_ms, blk_ms = 0.0, 0.0
        # the layer linear by linear and as a grouped block, in turn, so that
        # both meet the same clock and power state
        for _ in range(reps):
            flush()
            ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in layer]
            layer_pass(ev)
            torch.cuda.synchronize()
            for i in range(len(layer)):
                fwd_ms[i] += ev[i][0].elapsed_time(ev[i][1]) / reps
                bwd_ms[i] += ev[i][1].elapsed_time(ev[i][2]) / reps
            tot_ms += ev[0][0].elapsed_time(ev[-1][2]) / reps
            flush()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            block_pass()
            b.record(stream)
            torch.cuda.synchronize()
            blk_ms += a.elapsed_time(b) / reps
        del parts
        per = []
        fl_tot = 0.0
        for i, (nm, n, k) in enumerate(layer):
            ff, fb = fwd_flops(M, n, k, RANK), linear_flops(M, n, k, RANK) - fwd_flops(M, n, k, RANK)
            fl_tot += ff + fb
            per.append({"linear": f"{nm} {n}x{k}", "fwd_ms": fwd_ms[i], "bwd_ms": bwd_ms[i],
                        "fwd_tflops": ff / (fwd_ms[i] * 1e-3) / 1e12, "bwd_tflops": fb / (bwd_ms[i] * 1e-3) / 1e12,
                        "fwd_bwd_tflops": (ff + fb) / ((fwd_ms[i] + bwd_ms[i]) * 1e-3) / 1e12})
        tf = fl_tot / (tot_ms * 1e-3) / 1e12
        tw1 = time.time()
        grouped = {"layer_ms": blk_ms, "layer_tflops": fl_tot / (blk_ms * 1e-3) / 1e12,
                   "vs_per_linear": tot_ms / blk_ms, "groups": "qkv, o, gate+up, down"}
        out[f"m{M}"] = {"layer_ms": tot_ms, "layer_flops": fl_tot, "layer_tflops": tf,
                        "frac_burst": tf / tc_b, "frac_sustained": tf / tc_s, "linears": per,
                        "clocks": sampler.summary(tw0, tw1), "grouped": grouped}
        del lin
    sampler.stop()
    return out


def run_other_types(q, torch, dev, stream, flush, bufs, peaks_hbm):
    """The comparison types on the same two 7B-shaped weights: quantization
    to FP4 (E2M1) and Int4 with the NF4 path's kernels (the type's table),
    and block-wise Int8 (block 64) quantize and dequantize; per call, L2
    flushed, mean over 3 timed rounds after 2."""
    def timed(fn):
        ms = 0.0
        for rep in range(5):
            for b in bufs:
                flush()
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record(stream)
                fn(b)
                e1.record(stream)
                torch.cuda.synchronize()
                if rep >= 2:
                    ms += e0.elapsed_time(e1)
        return ms / 3
    out = {}
    nbytes_q = sum(quant_bytes(b["case"].W.size) for b in bufs)
    for name, qt in (("fp4", q.TYPE_FP4), ("int4", q.TYPE_INT4)):
        ws_ = [q.alloc_nf4_weight(b["case"].W.shape, dev, qt) for b in bufs]
        idx = {id(b): i for i, b in enumerate(bufs)}
        ms = timed(lambda b: q.qlora_quantize_nf4_dq(b["W"], out=ws_[idx[id(b)]], ws=b["qws"], qtype=qt))
        out[f"{name}_quantize_gbs"] = nbytes_q / (ms * 1e-3) / 1e9
        out[f"{name}_quantize_frac_hbm"] = out[f"{name}_quantize_gbs"] / peaks_hbm
        del ws_
    n_all = sum(b["case"].W.size for b in bufs)
    i8 = [(torch.empty(b["case"].W.size, dtype=torch.int8, device=dev),
           torch.empty(-(-b["case"].W.size // 64), dtype=torch.float32, device=dev),
           torch.empty(b["case"].W.size, dtype=torch.float32, device=dev)) for b in bufs]
    idx = {id(b): i for i, b in enumerate(bufs)}
    int8_bytes = n_all * (4 + 1) + 4 * sum(-(-b["case"].W.size // 64) for b in bufs)
    ms = timed(lambda b: q.qlora_int8_quantize(b["W"].view(-1), 64, codes=i8[idx[id(b)]][0], c=i8[idx[id(b)]][1]))
    out["int8_quantize_gbs"] = int8_bytes / (ms * 1e-3) / 1e9
    ms = timed(lambda b: q.qlora_int8_dequantize(i8[idx[id(b)]][0], i8[idx[id(b)]][1], 64, out=i8[idx[id(b)]][2]))
    out["int8_dequant_gbs"] = int8_bytes / (ms * 1e-3) / 1e9
    out["int8_quantize_frac_hbm"] = out["int8_quantize_gbs"] / peaks_hbm
    out["int8_dequant_frac_hbm"] = out["int8_dequant_gbs"] / peaks_hbm
    out["note"] = "both 7B-shaped weights per round; Int8 bytes: 4 B fp32 + 1 B code per element + 4 B per 64-block"
    del i8
    return out


def grouped_block(q, torch, dev, lin, wqs, M):
    """The same layer as a decoder block runs it: q, k, v read one input and
    run as one grouped linear, gate and up likewise; o and down alone.  Same
    FLOPs as the seven separate linears.  Returns the pass and its buffers."""
    s_lora = ALPHA / RANK
    parts = []
    for idx in ((0, 1, 2), (3,), (4, 5), (6,)):
        ds = [lin[i] for i in idx]
        n_all, k = sum(d["N"] for d in ds), ds[0]["K"]
        G = len(idx)
        g = {"w": [wqs[i] for i in idx], "X": ds[0]["X"],
             "A": torch.cat([d["A"] for d in ds]).contiguous(), "B": torch.cat([d["B"] for d in ds]).contiguous(),
             "dY": torch.cat([d["dY"] for d in ds], dim=1).contiguous(),
             "Y": torch.empty((M, n_all), dtype=torch.bfloat16, device=dev),
             "T": torch.empty((M, G * RANK), dtype=torch.bfloat16, device=dev),
             "dX": torch.empty((M, k), dtype=torch.bfloat16, device=dev),
             "dA": torch.empty((G * RANK, k), dtype=torch.bfloat16, device=dev),
             "dB": torch.empty((n_all, RANK), dtype=torch.bfloat16, device=dev)}
        g["ws"] = torch.empty(q.qlora_linear_group_bwd_workspace_size(M, G, RANK), dtype=torch.uint8, device=dev)
        parts.append(g)

    def block_pass():
        for g in parts:
            q.qlora_linear_group_fwd(g["X"], g["w"], g["A"], g["B"], s_lora, Y=g["Y"], T_save=g["T"], ws=g["ws"])
        for g in reversed(parts):
            q.qlora_linear_group_bwd(g["dY"], g["X"], g["w"], g["A"], g["B"], s_lora, T=g["T"], dX=g["dX"],
                                     dA_cat=g["dA"], dB_cat=g["dB"], ws=g["ws"])

    return block_pass, parts


def decode_bytes(M, N, K, r):
    """Algorithmic bytes of one small-batch forward: the quantized weight
    (0.5 + 1/64 + 1/4096 B/param) plus X, A, B read and Y, T written."""
    return N * K // 2 + N * K // 64 + -(-(N * K // 64) // 256) * 4 + 2 * (M * K + r * K + N * r + M * N + M * r)


def run_decode(q, torch, dev, stream, flush, args):
    """LLaMA-13B-shaped decode forward (W 5120x5120 and 13824x5120, M = 1,
    4, 16 tokens, r = 16): per call device time with L2 flushed before
    each call, launched directly and replayed from a CUDA graph."""
    out = {}
    reps = max(10, args.steps)
    for which in range(2):
        if args.decode_case and not args.decode_case.startswith(f"{synth.DECODE13B[which][1]}x"):
            continue
        base = synth.decode13b_linear(which, 16, seed=0)
        W = torch.from_numpy(base.W).to(dev)
        wq = q.qlora_quantize_nf4_dq(W)
        del W
        for M in (1, 4, 16):
            if args.decode_case and not args.decode_case.endswith(f"_m{M}"):
                continue
            c = synth.decode13b_linear(which, M, seed=0) if M != 16 else base
            X = torch.from_numpy(c.X.view(np.int16)).to(dev).view(torch.bfloat16)
            A = torch.from_numpy(c.A.view(np.int16)).to(dev).view(torch.bfloat16)
            B = torch.from_numpy(c.B.view(np.int16)).to(dev).view(torch.bfloat16)
            Y = torch.empty((M, c.N), dtype=torch.bfloat16, device=dev)
            T = torch.empty((M, c.r), dtype=torch.bfloat16, device=dev)
            ws = torch.empty(q.qlora_linear_fwd_workspace_size(M, c.N, c.K, c.r), dtype=torch.uint8, device=dev)

            def call():
                q.qlora_linear_fwd(X, wq, A, B, c.s, Y=Y, T_save=T, ws=ws)

            for _ in range(3):
                call()
            torch.cuda.synchronize()
            direct = []
            for _ in range(reps):
                flush()
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record(stream)
                call()
                e1.record(stream)
                direct.append((e0, e1))
            torch.cuda.synchronize()
            ms = statistics.median(a.elapsed_time(b) for a, b in direct)
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                call()
            g.replay()
            torch.cuda.synchronize()
            graphed = []
            for _ in range(reps):
                flush()
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record(stream)
                g.replay()
                e1.record(stream)
                graphed.append((e0, e1))
            torch.cuda.synchronize()
            gms = statistics.median(a.elapsed_time(b) for a, b in graphed)
            del g
            # unfused comparator: the library's dequantize to a bf16 W in HBM,
            # then torch.matmul (cuBLAS) for the base and LoRA products
            Wdq = torch.empty((c.N, c.K), dtype=torch.bfloat16, device=dev)

            def unfused():
                q.qlora_dequantize(wq, torch.bfloat16, out=Wdq)
                yk = torch.matmul(X, Wdq.t())
                tk = torch.matmul(X, A.t()).mul_(c.s)
                yk.addmm_(tk, B.t())

            for _ in range(3):
                unfused()
            torch.cuda.synchronize()
            uf = []
            for _ in range(reps):
                flush()
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record(stream)
                unfused()
                e1.record(stream)
                uf.append((e0, e1))
            torch.cuda.synchronize()
            ums = statistics.median(a.elapsed_time(b) for a, b in uf)
            del Wdq
            nbytes = decode_bytes(M, c.N, c.K, c.r)
            out[f"{c.N}x{c.K}_m{M}"] = {"bytes": nbytes, "ms": ms, "gbs": nbytes / (ms * 1e-3) / 1e9,
                                        "graph_ms": gms, "graph_gbs": nbytes / (gms * 1e-3) / 1e9,
                                        "unfused_ms": ums}
    return out


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["native", "reference"], default="native")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--no-c3", action="store_true", help="skip the full LLaMA-7B-shaped weight set")
    ap.add_argument("--no-c4", action="store_true", help="skip the LLaMA-65B-shaped layer")
    ap.add_argument("--decode-only", action="store_true",
                    help="time only the small-batch forward (LLaMA-13B decode shapes) and print it")
    ap.add_argument("--decode-case", default="", help="e.g. 13824x5120_m16: one decode configuration")
    args = ap.parse_args(argv)
    world, rank, local = dist_setup()
    if args.decode_only:
        import torch

        import bit_nf4_quantized_13_b200 as q
        dev = torch.device("cuda", local)
        torch.cuda.set_device(dev)
        flush = L2Flush(torch, dev)
        res = run_decode(q, torch, dev, torch.cuda.current_stream(), flush, args)
        peaks, src = load_peaks()
        for v in res.values():
            v["frac_hbm"] = v["gbs"] / peaks["hbm_gbs"]
            v["graph_frac_hbm"] = v["graph_gbs"] / peaks["hbm_gbs"]
        print(json.dumps({"decode": res, "hbm_peak_gbs": peaks["hbm_gbs"], "peak_source": src}), flush=True)
        return 0
    if args.impl == "reference":
        return run_reference(args, world, rank)
    return run_native(args, world, rank, local)


if __name__ == "__main__":
    sys.exit(main())
