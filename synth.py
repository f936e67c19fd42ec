"""Seeded synthetic inputs for the QLoRA NF4 linear layer.

This module holds none of the method's arithmetic: it only draws numbers.
Both the tests (for the CPU oracle and for the CUDA library) and ``bench.py``
take their inputs from here, so the two sides see identical bytes.

Generator: numpy's Philox counter-based bit generator (Philox4x64-10,
Salmon et al., SC'11), keyed by (seed, tensor id), so every tensor has its
own independent stream.  Normals come from numpy's standard_normal; the
compute-type tensors (X, A, B, dY) are drawn in fp32 and rounded to bf16
(nearest even), and are thereafter *defined* as those bf16 values.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np

# tensor ids: one independent stream per role
TID_W, TID_X, TID_A, TID_B, TID_DY, TID_OUTLIER = 1, 2, 3, 4, 5, 6


def rng(seed: int, tid: int) -> np.random.Generator:
    key = np.array([int(tid) & 0xFFFFFFFFFFFFFFFF, int(seed) & 0xFFFFFFFFFFFFFFFF], np.uint64)
    return np.random.Generator(np.random.Philox(key=key))


def normal_f32(seed: int, tid: int, shape, std: float = 1.0) -> np.ndarray:
    x = rng(seed, tid).standard_normal(size=shape, dtype=np.float32)
    if std != 1.0:
        x *= np.float32(std)
    return x


def to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """fp32 -> bf16 bit patterns, nearest even (inputs are finite)."""
    u = np.ascontiguousarray(x, np.float32).view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return u.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.ascontiguousarray(b, np.uint16).astype(np.uint32) << 16).view(np.float32)


def bf16_normal(seed: int, tid: int, shape, std: float = 1.0) -> np.ndarray:
    return to_bf16_bits(normal_f32(seed, tid, shape, std))


def weight_normal(seed: int, tid: int, shape, std: float = 0.02,
                  outlier_frac: float = 0.0, outlier_scale: float = 8.0) -> np.ndarray:
    """fp32 W ~ N(0, std^2); a Bernoulli(outlier_frac) subset (own stream) is
    multiplied by outlier_scale -- the heavy tail of LLM weight matrices."""
    w = normal_f32(seed, tid, shape, std)
    if outlier_frac > 0.0:
        mask = rng(seed, tid * 1000 + TID_OUTLIER).random(size=shape) < outlier_frac
        w[mask] *= np.float32(outlier_scale)
    return w


def weight_student_t(seed: int, tid: int, shape, df: float = 5.0, std: float = 0.02) -> np.ndarray:
    """fp32 W ~ Student-t(df) rescaled to the given standard deviation."""
    t = rng(seed, tid).standard_t(df, size=shape)
    return (t * (std / math.sqrt(df / (df - 2.0)))).astype(np.float32)


def student_t_device(seed: int, tid: int, numel: int, device, df: int = 5, std: float = 0.02):
    """fp32 torch tensor of `numel` Student-t(df) draws, rescaled to the given
    standard deviation, generated on `device` by torch's counter-based
    generator seeded with (seed, tid).  For integer df the variate is built
    from its definition: Z / sqrt(V / df) with Z ~ N(0,1) and V the sum of
    df squared N(0,1) draws.  Used where a workload is too large to draw on
    the host (the full LLaMA-7B-shaped weight set)."""
    import torch
    g = torch.Generator(device=device)
    g.manual_seed((int(seed) << 24) ^ int(tid))
    z = torch.randn(numel, generator=g, device=device, dtype=torch.float32)
    v = torch.zeros(numel, device=device, dtype=torch.float32)
    for _ in range(int(df)):
        v.add_(torch.randn(numel, generator=g, device=device, dtype=torch.float32).square_())
    z.div_(v.div_(float(df)).sqrt_())
    return z.mul_(std / math.sqrt(df / (df - 2.0)))


def normal_device(seed: int, tid: int, shape, device, std: float = 1.0, dtype=None):
    """N(0, std^2) draws generated on `device` by torch's counter-based
    generator seeded with (seed, tid), optionally cast (round to nearest
    even) to `dtype`.  Used for the activations of the largest workloads."""
    import torch
    g = torch.Generator(device=device)
    g.manual_seed((int(seed) << 24) ^ int(tid))
    x = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
    if std != 1.0:
        x.mul_(std)
    return x if dtype is None else x.to(dtype)


@dataclass
class LinearCase:
    """One QLoRA linear: W (N x K) fp32, X (M x K), A (r x K), B (N x r) and dY
    (M x N) as bf16 bits, and the LoRA scalar s = alpha / r."""
    name: str
    M: int
    N: int
    K: int
    r: int
    alpha: float
    W: np.ndarray
    X: np.ndarray
    A: np.ndarray
    B: np.ndarray
    dY: np.ndarray
    meta: dict = field(default_factory=dict)

    @property
    def s(self) -> float:
        return self.alpha / self.r


def linear_case(name: str, M: int, N: int, K: int, r: int, alpha: float, seed: int = 0,
                w_std: float = 0.02, outlier_frac: float = 0.0, wid: int = 0,
                ab_std: float = 0.01, with_dy: bool = True) -> LinearCase:
    base = 10 * wid
    W = weight_normal(seed, base + TID_W, (N, K), w_std, outlier_frac)
    X = bf16_normal(seed, base + TID_X, (M, K))
    A = bf16_normal(seed, base + TID_A, (r, K), ab_std)
    B = bf16_normal(seed, base + TID_B, (N, r), ab_std)
    dY = bf16_normal(seed, base + TID_DY, (M, N)) if with_dy else None
    return LinearCase(name, M, N, K, r, alpha, W, X, A, B, dY)


# --- the workloads -----------------------------------------------------------

def tiny(seed: int = 0) -> LinearCase:
    """W 512x512 ~N(0,0.02); X 16x512 ~N(0,1); r=8, alpha=16; A,B ~N(0,0.01)."""
    return linear_case("tiny_512x512_m16_r8", 16, 512, 512, 8, 16.0, seed)


LLAMA7B_LINEARS = [("w4096x4096", 4096, 4096), ("w11008x4096", 11008, 4096)]


def llama7b_linear(which: int, seed: int = 0, M: int = 4096) -> LinearCase:
    """LLaMA-7B-shaped linear: W ~N(0,0.02) with 0.1% entries x8; X 4096 tokens
    (16 x 256); r=64, alpha=16."""
    name, N, K = LLAMA7B_LINEARS[which]
    return linear_case(f"llama7b_{name}_m{M}_r64", M, N, K, 64, 16.0, seed,
                       outlier_frac=0.001, wid=which)


def llama7b_weight_shapes():
    """The 224 linear weights of a LLaMA-7B-shaped model (32 layers x q,k,v,o
    4096^2, gate/up 11008x4096, down 4096x11008)."""
    shapes = []
    for layer in range(32):
        for nm in ("q", "k", "v", "o"):
            shapes.append((f"l{layer}.{nm}", 4096, 4096))
        shapes.append((f"l{layer}.gate", 11008, 4096))
        shapes.append((f"l{layer}.up", 11008, 4096))
        shapes.append((f"l{layer}.down", 4096, 11008))
    return shapes


LLAMA65B_LAYER = [("q", 8192, 8192), ("k", 8192, 8192), ("v", 8192, 8192), ("o", 8192, 8192),
                  ("gate", 22016, 8192), ("up", 22016, 8192), ("down", 8192, 22016)]

LLAMA65B_TOKENS = (512, 2048, 8192)


def llama65b_linear(which: int, M: int, seed: int = 0, r: int = 64, with_dy: bool = True) -> LinearCase:
    """One linear of a LLaMA-65B-shaped decoder layer (LLAMA65B_LAYER[which]):
    W ~N(0,0.02) with 0.1% entries x8 (the 7B-shaped recipe; the 65B case
    states no distribution), X M x K ~N(0,1) bf16 with M in 512/2048/8192,
    r=64, alpha=16."""
    name, N, K = LLAMA65B_LAYER[which]
    return linear_case(f"llama65b_{name}_{N}x{K}_m{M}_r{r}", M, N, K, r, 16.0, seed,
                       outlier_frac=0.001, wid=20 + which, with_dy=with_dy)


DECODE13B = [("w5120x5120", 5120, 5120), ("w13824x5120", 13824, 5120)]


def decode13b_linear(which: int, M: int, seed: int = 0) -> LinearCase:
    """LLaMA-13B-shaped decode linear: W 5120x5120 or 13824x5120 ~N(0,0.02)
    without outliers; X M x 5120 (M in 1, 4, 16) ~N(0,1) bf16; r=16,
    alpha=16 (s=1); forward only."""
    name, N, K = DECODE13B[which]
    return linear_case(f"decode13b_{name}_m{M}_r16", M, N, K, 16, 16.0, seed, wid=2 + which,
                       with_dy=False)
