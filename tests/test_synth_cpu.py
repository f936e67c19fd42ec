"""The seeded input recipe: deterministic per (seed, tensor id), independent
streams, the stated distributions, and bf16 rounding that matches torch's."""
import numpy as np
import torch

import synth


def test_same_key_same_bytes_and_streams_differ():
    a = synth.normal_f32(3, synth.TID_X, (64, 64))
    b = synth.normal_f32(3, synth.TID_X, (64, 64))
    assert np.array_equal(a.view(np.uint32), b.view(np.uint32))
    c = synth.normal_f32(3, synth.TID_A, (64, 64))
    d = synth.normal_f32(4, synth.TID_X, (64, 64))
    assert not np.array_equal(a, c) and not np.array_equal(a, d)
    # independent streams: no correlation to speak of
    assert abs(np.corrcoef(a.ravel(), c.ravel())[0, 1]) < 0.05


def test_bf16_rounding_matches_torch():
    x = synth.normal_f32(0, 9, (1 << 16,), std=3.0)
    x[:8] = np.float32([1.0, -1.0, 1.00390625, 1.01171875, 0.0, -0.0, 3.0e-39, 65504.0])
    ours = synth.to_bf16_bits(x)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, ref)
    back = synth.bf16_bits_to_f32(ours)
    assert np.array_equal(back, torch.from_numpy(x).to(torch.bfloat16).float().numpy())


def test_weight_distribution_and_outliers():
    n = 1 << 20
    w = synth.weight_normal(0, synth.TID_W, (n,), std=0.02)
    assert abs(float(w.mean())) < 0.02 * 5 / np.sqrt(n)
    assert abs(float(w.std()) / 0.02 - 1.0) < 0.01
    wo = synth.weight_normal(0, synth.TID_W, (n,), std=0.02, outlier_frac=0.001, outlier_scale=8.0)
    scaled = np.count_nonzero(wo != w)
    # Bernoulli(0.001) over 2^20 entries: mean 1049, sd 32
    assert abs(scaled - 0.001 * n) < 6 * np.sqrt(0.001 * n)
    changed = wo != w
    assert np.allclose(wo[changed], 8.0 * w[changed])


def test_student_t_weights_have_the_stated_std():
    w = synth.weight_student_t(0, synth.TID_W, (1 << 20,), df=5.0, std=0.02)
    assert abs(float(w.std()) / 0.02 - 1.0) < 0.05
    # heavier tails than a normal of the same spread
    assert np.mean(np.abs(w) > 4 * 0.02) > 2 * 6.3e-5


def test_workload_shapes():
    c = synth.tiny(0)
    assert (c.W.shape, c.X.shape, c.A.shape, c.B.shape, c.dY.shape) == \
        ((512, 512), (16, 512), (8, 512), (512, 8), (16, 512))
    assert c.s == 2.0 and c.W.dtype == np.float32 and c.X.dtype == np.uint16
    d = synth.decode13b_linear(1, 4)
    assert (d.N, d.K, d.M, d.r, d.s) == (13824, 5120, 4, 16, 1.0) and d.dY is None
    shapes = synth.llama7b_weight_shapes()
    assert len(shapes) == 224 and sum(n * k for _, n, k in shapes) == 32 * (4 * 4096 * 4096 + 3 * 11008 * 4096)
