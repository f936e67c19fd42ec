"""Pins for the CPU oracle: each test checks the oracle against something other
than itself -- a value the pages print, a closed form, a library routine for a
special case, an invariant, or brute force on tiny inputs.  Page citations
name "QLoRA: Efficient Finetuning of Quantized LLMs" study notes
(gitcode.csdn.net) by section and equation."""
import math
import os

import numpy as np
import pytest
import torch
from scipy.special import ndtr, ndtri

import oracle
import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden(name):
    out = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            k, v = line.split(":", 1)
            out[k.strip()] = [float(t) for t in v.split()]
    return out


# ---------------------------------------------------------------- a1 codebook

def test_norm_ppf_matches_library_quantile():
    """AS 241 against scipy's ndtri (an independent implementation)."""
    ps = np.concatenate([np.linspace(1e-6, 1 - 1e-6, 2001), [1e-300, 1e-30, 1e-12, 0.02425,
                                                              0.075, 0.425, 0.5, 0.575, 0.925,
                                                              0.96770833333, 1 - 1e-12]])
    for p in ps:
        ref = float(ndtri(p))
        got = oracle.norm_ppf(float(p))
        assert abs(got - ref) <= 2e-15 * max(1.0, abs(ref)), (p, got, ref)


def test_norm_ppf_inverts_the_cdf():
    """Closed form: Q(Phi(x)) = x with Phi(x) = erfc(-x/sqrt 2)/2."""
    assert oracle.norm_ppf(0.5) == 0.0
    for x in np.linspace(-6, 6, 241):
        p = 0.5 * math.erfc(-x / math.sqrt(2.0))
        # p carries one rounding (<= 2^-53 relative); dQ/dp = 1/phi(x)
        phi = math.exp(-x * x / 2) / math.sqrt(2 * math.pi)
        tol = 4e-15 * max(1.0, abs(x)) + 2.0 ** -52 * p / phi
        assert abs(oracle.norm_ppf(p) - x) <= tol, (x, p)


def test_codebook_structure():
    """Section 3.2: 2^k = 16 values in [-1, 1]; an exact zero; the negative
    half from 2^(k-1) quantiles and the positive half from 2^(k-1)+1, the
    shared zero kept once -> 7 negative, 1 zero, 8 positive."""
    q = oracle.nf4_codebook()
    assert q.dtype == np.float32 and q.size == 16
    assert np.all(np.diff(q) > 0)
    assert q[0] == -1.0 and q[15] == 1.0
    assert np.count_nonzero(q == 0.0) == 1 and q[7] == 0.0
    assert np.count_nonzero(q < 0) == 7 and np.count_nonzero(q > 0) == 8
    # asymmetric: the type is not symmetric about zero
    assert not np.allclose(q[:7], -q[15:8:-1])


def test_codebook_equal_probability_bins():
    """Section 3.2 (quantile quantization): each half's values sit at evenly
    spaced probabilities of N(0,1) between 1/2 and the common tail
    probability delta.  Checked with scipy's CDF, independent of the oracle's
    quantile routine; the fp32 rounding of q bounds the error (< 1e-7)."""
    q = oracle.nf4_codebook().astype(np.float64)
    delta = oracle.nf4_delta()
    scale = ndtri(delta)  # the normaliser: the outermost quantile
    pos = ndtr(q[8:] * scale) - 0.5
    neg = 0.5 - ndtr(q[:7][::-1] * scale)
    np.testing.assert_allclose(pos, (delta - 0.5) * np.arange(1, 9) / 8, atol=1e-7, rtol=0)
    np.testing.assert_allclose(neg, (delta - 0.5) * np.arange(1, 8) / 7, atol=1e-7, rtol=0)
    # delta lies between the outermost-bin centres of the 15- and 16-bin grids
    assert 1 - 1 / 30 < delta < 1 - 1 / 32


# ------------------------------------------------------------ a2/a3 encoding

def _py_bruteforce(w, block=64):
    """Pure-Python brute force, fp32 arithmetic through numpy scalars."""
    q = [np.float32(v) for v in oracle.nf4_codebook()]
    n = len(w)
    codes, c2 = [], []
    for lo in range(0, n, block):
        blk = [np.float32(v) for v in w[lo:lo + block]]
        a = max(abs(v) for v in blk)
        c2.append(a)
        for v in blk:
            if a == 0:
                codes.append(7)
                continue
            x = np.float32(v / a)
            best, bd = 0, abs(np.float32(x - q[0]))
            for i in range(1, 16):
                d = abs(np.float32(x - q[i]))
                if d < bd:
                    best, bd = i, d
            codes.append(best)
    if n % 2:
        codes.append(0)
    packed = [(codes[2 * t] << 4) | codes[2 * t + 1] for t in range(len(codes) // 2)]
    return np.array(packed, np.uint8), np.array(c2, np.float32)


@pytest.mark.parametrize("n", [1, 2, 63, 64, 65, 127, 128, 300, 641])
def test_encode_matches_python_brute_force(n):
    w = synth.normal_f32(7, 100 + n, (n,), 0.02)
    w[::11] = 0.0
    codes, c2, st = oracle.quantize_nf4(w)
    pc, pa = _py_bruteforce(w)
    assert st == oracle.OK
    np.testing.assert_array_equal(codes, pc)
    np.testing.assert_array_equal(c2, pa)


def test_absmax_worked_example():
    """Section 3.1: the block [-5, 3, -2] has absmax 5."""
    g = _golden("int8_absmax_worked_example.txt")
    blk = np.zeros(64, np.float32)
    blk[:3] = g["block"]
    _, c2, _ = oracle.quantize_nf4(blk)
    assert c2.tolist() == g["absmax"]


def test_encode_special_values():
    q = oracle.nf4_codebook()
    # the block maximum maps to an end of the type; codebook points map to themselves
    w = np.zeros(64, np.float32)
    w[0] = 1.0
    w[1:17] = q
    codes, c2, _ = oracle.quantize_nf4(w)
    nib = np.stack([codes >> 4, codes & 15], 1).reshape(-1)
    assert c2[0] == 1.0 and nib[0] == 15
    np.testing.assert_array_equal(nib[1:17], np.arange(16))
    assert np.all(nib[17:] == 7)
    # nibble order: element 2t in the high nibble
    w2 = np.zeros(64, np.float32)
    w2[0], w2[1] = 1.0, -1.0
    c, _, _ = oracle.quantize_nf4(w2)
    assert c[0] == 0xF0
    # a negative maximum maps to code 0
    w3 = np.zeros(64, np.float32)
    w3[5] = -3.0
    c, a, _ = oracle.quantize_nf4(w3)
    assert a[0] == 3.0 and (c[2] >> 4) == 7 and (c[2] & 15) == 0
    # all-zero W: zero constants and the zero code everywhere
    c, a, _ = oracle.quantize_nf4(np.zeros(200, np.float32))
    assert np.all(c == 0x77) and np.all(a == 0)
    # odd length: the pad nibble is zero
    c, _, _ = oracle.quantize_nf4(np.zeros(3, np.float32))
    assert c.tolist() == [0x77, 0x70]


def test_encode_ties_go_to_lower_index():
    """Where fp32 |n - q_j| equals |n - q_(j+1)|, the lower index wins."""
    q = oracle.nf4_codebook()
    found = 0
    for j in range(15):
        mid = np.float32((np.float64(q[j]) + np.float64(q[j + 1])) / 2)
        for cand in (np.nextafter(mid, np.float32(-2)), mid, np.nextafter(mid, np.float32(2))):
            dl = abs(np.float32(cand - q[j]))
            du = abs(np.float32(q[j + 1] - cand))
            if dl == du:
                w = np.zeros(64, np.float32)
                w[0], w[1] = 1.0, cand
                c, _, _ = oracle.quantize_nf4(w)
                assert (c[0] & 15) == j, (j, cand)
                found += 1
    assert found >= 1


def test_encode_is_monotone_and_within_half_gap():
    q = oracle.nf4_codebook().astype(np.float64)
    w = np.sort(synth.normal_f32(3, 1, (64,), 1.0))
    w[np.argmax(np.abs(w))] = np.float32(2.5) * np.sign(w[np.argmax(np.abs(w))])
    codes, c2, _ = oracle.quantize_nf4(w)
    nib = np.stack([codes >> 4, codes & 15], 1).reshape(-1)
    assert np.all(np.diff(nib.astype(int)) >= 0)
    n = w.astype(np.float64) / c2[0]
    gap = np.max(np.diff(q)) / 2
    assert np.max(np.abs(n - q[nib])) <= gap + 1e-7


def test_nonfinite_is_reported():
    w = np.zeros(128, np.float32)
    w[70] = np.inf
    assert oracle.quantize_nf4(w)[2] == oracle.ERR_NONFINITE
    w[70] = np.nan
    assert oracle.quantize_nf4(w)[2] == oracle.ERR_NONFINITE


# --------------------------------------------------------------------- a4 mean

def test_mean_is_exact_sum_correctly_rounded():
    """mu = RN32(RN64(S)/nb) for the exact sum S: math.fsum returns the
    correctly rounded sum of floats (Shewchuk), an independent route."""
    r = synth.rng(0, 77)
    cases = [
        np.abs(r.standard_normal(4097)).astype(np.float32) * np.float32(0.05),
        np.exp(r.uniform(-80, 80, 1000)).astype(np.float32),  # huge dynamic range
        np.array([2.0 ** 100] + [2.0 ** -100] * 1000 + [1.0], np.float32),
        np.array([3.4e38, 3.4e38], np.float32) / np.float32(4),
        np.array([1e-45, 1e-45, 3e-45], np.float32),  # subnormals
        np.array([0.0], np.float32),
    ]
    for c2 in cases:
        mu, s, st = oracle.mean_exact(c2)
        assert st == oracle.OK
        ref_s = math.fsum(float(v) for v in c2)
        assert s == ref_s
        assert mu == np.float32(ref_s / c2.size)
        # order independence
        mu2, _, _ = oracle.mean_exact(c2[::-1].copy())
        assert mu2 == mu


def test_mean_rejects_nonfinite():
    assert oracle.mean_exact(np.array([1.0, np.inf], np.float32))[2] == oracle.ERR_NONFINITE


# ---------------------------------------------------------------------- FP8

def _e4m3_by_definition(b):
    s = -1.0 if b & 0x80 else 1.0
    e, m = (b >> 3) & 15, b & 7
    if e == 15 and m == 7:
        return math.nan
    if e == 0:
        return s * m * 2.0 ** -9
    return s * (1 + m / 8) * 2.0 ** (e - 7)


def test_e4m3_decode_table():
    """All 256 bytes: the OCP E4M3 definition, and torch's float8_e4m3fn."""
    b = np.arange(256, dtype=np.uint8)
    got = oracle.e4m3_decode(b)
    ref = np.array([_e4m3_by_definition(int(v)) for v in b], np.float64)
    tor = torch.from_numpy(b.copy()).view(torch.float8_e4m3fn).float().numpy()
    for i in range(256):
        if math.isnan(ref[i]):
            assert np.isnan(got[i]) and np.isnan(tor[i])
        else:
            assert got[i] == ref[i] == tor[i], i
    assert np.nanmax(got) == 448.0


def _e4m3_sweep_values():
    # every 61st fp32 bit pattern, plus every pattern within +-4 ulps of each
    # midpoint between adjacent E4M3 values (the rounding boundaries)
    pats = np.arange(0, 2 ** 32, 61, dtype=np.uint64).astype(np.uint32)
    vals = [pats.view(np.float32)]
    pos = np.array([_e4m3_by_definition(b) for b in range(0x7f)], np.float64)
    mids = ((pos[1:] + pos[:-1]) / 2).astype(np.float32)
    mids = np.concatenate([mids, np.float32([448.0, 464.0, 480.0, 2.0 ** -10])])
    near = (mids.view(np.uint32)[:, None].astype(np.int64) + np.arange(-4, 5)[None, :])
    near = near.astype(np.uint32).view(np.float32).reshape(-1)
    vals += [near, -near]
    v = np.concatenate(vals)
    return v[np.isfinite(v)]


def test_e4m3_encode_matches_library_conversion():
    """RNE with saturation to +-448: torch's float8_e4m3fn conversion of the
    value clamped to [-448, 448] (clamping first gives the satfinite
    result)."""
    x = _e4m3_sweep_values()
    got = oracle.e4m3_encode(x)
    ref = torch.from_numpy(np.clip(x, -448, 448)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    bad = np.nonzero(got != ref)[0]
    assert bad.size == 0, (x[bad[:5]], got[bad[:5]], ref[bad[:5]])
    assert oracle.e4m3_encode(np.float32([np.inf, -np.inf, 1e30])).tolist() == [0x7e, 0xfe, 0x7e]


def test_bf16_rne_matches_library_conversion():
    pats = np.arange(0, 2 ** 32, 97, dtype=np.uint64).astype(np.uint32)
    x = pats.view(np.float32)
    x = x[np.isfinite(x)]
    got = oracle.bf16_rne(x)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(got, ref)


# ------------------------------------------------------------- a5 double quant

def test_double_quant_bits_per_param():
    """Section 3.3: 32/64 = 0.5 bits of constants per parameter without DQ;
    8/64 + 32/(64*256) = 0.127 with it; saving 0.373 bits, ~3 GB at 65B."""
    g = _golden("double_quant_bits.txt")
    numel = 64 * 256 * 3 + 64 * 10 + 5  # ragged at both levels
    w = synth.normal_f32(0, 1, (numel,), 0.02)
    d = oracle.quantize_nf4_dq(w)
    assert d["codes"].size == (numel + 1) // 2
    assert d["c2_fp8"].size == -(-numel // 64) and d["c1"].size == -(-numel // (64 * 256))
    # at a full multiple of the blocks, the constant overhead is exact
    numel = 64 * 256 * 4
    d = oracle.quantize_nf4_dq(synth.normal_f32(0, 2, (numel,), 0.02))
    const_bits = (d["c2_fp8"].size * 8 + d["c1"].size * 32) / numel
    assert const_bits == 8 / 64 + 32 / (64 * 256) == 0.126953125
    assert abs(const_bits - g["dq_constants_bits"][0]) < 5e-4
    assert 32 / 64 == g["fp32_constants_bits"][0]
    saving = 0.5 - const_bits
    assert abs(saving - g["saving_bits"][0]) < 5e-4
    assert abs(65e9 * saving / 8 / 1e9 - g["saving_65b_gb_approx"][0]) < 0.1
    total_bits = (d["codes"].size * 8 + d["c2_fp8"].size * 8 + d["c1"].size * 32 + 32) / numel
    assert total_bits == 4 + 0.126953125 + 32 / numel


def test_double_quant_error_bound():
    """E4M3 keeps 3 mantissa bits: |c2' - c2| <= 2^-4 |y| (normal range) plus
    2^-10 c1 (subnormal spacing) plus a few fp32 roundings."""
    w = synth.weight_normal(0, 9, (64 * 256 * 5 + 64 * 3,), 0.02, 0.001)
    d = oracle.quantize_nf4_dq(w)
    c2, mu = d["c2"].astype(np.float64), float(d["mean"])
    c2p = oracle.dequant_constants(d["c2_fp8"], d["c1"], d["mean"]).astype(np.float64)
    c1 = np.repeat(d["c1"].astype(np.float64), 256)[: c2.size]
    y = np.abs(c2 - mu)
    ulp = np.spacing(np.maximum(np.abs(c2p), abs(mu)).astype(np.float32)).astype(np.float64)
    bound = 2.0 ** -4 * y * (1 + 1e-6) + 2.0 ** -10 * c1 + 4 * ulp
    assert np.all(np.abs(c2p - c2) <= bound)
    # c1 is the group absmax of y over the E4M3 maximum
    g0 = c2[:256] - mu
    assert d["c1"][0] == np.float32(np.float32(np.max(np.abs(np.float32(g0)))) / np.float32(448))


def test_double_quant_zero_group():
    c2 = np.full(300, 0.25, np.float32)
    mu, _, _ = oracle.mean_exact(c2)
    b, c1 = oracle.double_quant(c2, mu)
    assert mu == np.float32(0.25) and np.all(c1 == 0) and np.all(b == 0)


# -------------------------------------------------------------- a6/a7 dequant

def test_dequant_round_trip_bound_and_exact_zero():
    """Section 3.2: zeros quantize without error.  Away from zero the error
    is at most half the widest code gap times the block constant, plus the
    double-quant error of the constant."""
    q = oracle.nf4_codebook().astype(np.float64)
    n = 64 * 256 * 2 + 100
    w = synth.weight_normal(1, 1, (n,), 0.02, 0.001)
    w[::5] = 0.0
    d = oracle.quantize_nf4_dq(w)
    wd = oracle.dequantize(d["codes"], d["c2_fp8"], d["c1"], d["mean"], n)
    assert np.all(wd[::5] == 0.0)
    c2 = np.repeat(d["c2"].astype(np.float64), 64)[:n]
    c2p = np.repeat(oracle.dequant_constants(d["c2_fp8"], d["c1"], d["mean"]).astype(np.float64), 64)[:n]
    halfgap = np.max(np.diff(q)) / 2
    err = np.abs(wd.astype(np.float64) - w)
    assert np.all(err <= halfgap * c2 + np.abs(c2p - c2) + 1e-6 * c2)
    # all-zero W round-trips exactly
    z = np.zeros(1000, np.float32)
    dz = oracle.quantize_nf4_dq(z)
    assert np.all(oracle.dequantize(dz["codes"], dz["c2_fp8"], dz["c1"], dz["mean"], 1000) == 0)


def test_dequant_definition_small():
    """a6/a7 spelled out for one block: w' = q[code] * (e4m3 * c1 + mu)."""
    q = oracle.nf4_codebook()
    codes = np.array([0x0F, 0x7A], np.uint8)
    b = np.array([0x38], np.uint8)  # 1.0 in E4M3
    c1 = np.array([0.5], np.float32)
    mu = np.float32(0.25)
    out = oracle.dequantize(codes, b, c1, mu, 4)
    cp = np.float32(np.float32(1.0 * 0.5) + mu)
    np.testing.assert_array_equal(out, np.float32([q[0] * cp, q[15] * cp, q[7] * cp, q[10] * cp]))


# ---------------------------------------------------------- a8-a10 the linear

def _grid_bf16(seed, tid, shape, step=0.125, span=6):
    """Values k*step, |k| <= span: exact in bf16 with room for +-step."""
    k = synth.rng(seed, tid).integers(-span, span + 1, size=shape)
    return synth.to_bf16_bits((k * step).astype(np.float32))


def _bits(x):
    return synth.to_bf16_bits(np.asarray(x, np.float32))


def _f(bits):
    return synth.bf16_bits_to_f32(bits).astype(np.float64)


def test_linear_reduces_to_plain_gemm_when_lora_is_zero():
    M, N, K, r = 7, 9, 128, 4
    X = synth.bf16_normal(0, 1, (M, K))
    W = synth.bf16_normal(0, 2, (N, K), 0.02)
    A = synth.bf16_normal(0, 3, (r, K), 0.01)
    dY = synth.bf16_normal(0, 5, (M, N))
    Bz = np.zeros((N, r), np.uint16)
    Y, _ = oracle.linear_fwd(X, W, A, Bz, 2.0)
    np.testing.assert_allclose(Y, _f(X) @ _f(W).T, rtol=1e-12, atol=1e-12)
    dX, dA, dB = oracle.linear_bwd(dY, X, W, A, Bz, 2.0)
    np.testing.assert_allclose(dX, _f(dY) @ _f(W), rtol=1e-12, atol=1e-12)
    assert np.all(dA == 0)
    np.testing.assert_allclose(dB, 2.0 * _f(dY).T @ (_f(X) @ _f(A).T), rtol=1e-12, atol=1e-14)


def test_linear_reduces_to_lora_path_when_w_is_zero():
    M, N, K, r = 5, 6, 64, 3
    X = synth.bf16_normal(1, 1, (M, K))
    A = synth.bf16_normal(1, 3, (r, K), 0.01)
    B = synth.bf16_normal(1, 4, (N, r), 0.01)
    dY = synth.bf16_normal(1, 5, (M, N))
    W0 = np.zeros((N, K), np.uint16)
    s = 0.25
    Y, T0 = oracle.linear_fwd(X, W0, A, B, s)
    np.testing.assert_allclose(T0, _f(X) @ _f(A).T, rtol=1e-12, atol=1e-15)
    np.testing.assert_allclose(Y, s * (_f(X) @ _f(A).T) @ _f(B).T, rtol=1e-12, atol=1e-15)
    dX, dA, dB = oracle.linear_bwd(dY, X, W0, A, B, s)
    np.testing.assert_allclose(dX, s * (_f(dY) @ _f(B)) @ _f(A), rtol=1e-12, atol=1e-15)
    np.testing.assert_allclose(dA, s * (_f(dY) @ _f(B)).T @ _f(X), rtol=1e-12, atol=1e-15)


def test_linear_backward_matches_finite_differences():
    """Loss L = <dY, Y>.  Y is linear in each single entry of X, A and B, so
    a central difference with a step exact in bf16 gives the derivative
    up to fp64 rounding.  There is no dW (section 3.5)."""
    M, N, K, r, s = 3, 5, 64, 2, 2.0
    X = _grid_bf16(0, 1, (M, K))
    W = _grid_bf16(0, 2, (N, K))
    A = _grid_bf16(0, 3, (r, K))
    B = _grid_bf16(0, 4, (N, r))
    dY = _grid_bf16(0, 5, (M, N))
    h = 0.125
    dX, dA, dB = oracle.linear_bwd(dY, X, W, A, B, s)

    def loss(X_, A_, B_):
        Y, _ = oracle.linear_fwd(X_, W, A_, B_, s)
        return float(np.sum(Y * _f(dY)))

    rs = synth.rng(0, 9)
    for name, T, G in (("X", X, dX), ("A", A, dA), ("B", B, dB)):
        for _ in range(12):
            idx = tuple(int(rs.integers(0, d)) for d in T.shape)
            v = float(_f(np.array([T[idx]]))[0])
            Tp, Tm = T.copy(), T.copy()
            Tp[idx], Tm[idx] = _bits(v + h), _bits(v - h)
            args_p = {"X": X, "A": A, "B": B}
            args_m = dict(args_p)
            args_p[name], args_m[name] = Tp, Tm
            fd = (loss(args_p["X"], args_p["A"], args_p["B"]) -
                  loss(args_m["X"], args_m["A"], args_m["B"])) / (2 * h)
            assert abs(fd - G[idx]) <= 1e-9 * max(1.0, abs(G[idx])), (name, idx, fd, G[idx])


def test_linear_row_subset_and_threads_agree():
    M, N, K, r = 12, 10, 128, 4
    X = synth.bf16_normal(2, 1, (M, K))
    W = synth.bf16_normal(2, 2, (N, K), 0.02)
    A = synth.bf16_normal(2, 3, (r, K), 0.01)
    B = synth.bf16_normal(2, 4, (N, r), 0.01)
    dY = synth.bf16_normal(2, 5, (M, N))
    rows = np.array([11, 0, 5], np.int64)
    Y, _ = oracle.linear_fwd(X, W, A, B, 0.5)
    Ys, _ = oracle.linear_fwd(X, W, A, B, 0.5, rows=rows)
    np.testing.assert_array_equal(Ys, Y[rows])
    old = oracle.threads()
    try:
        oracle.set_threads(1)
        dX1, dA1, dB1 = oracle.linear_bwd(dY, X, W, A, B, 0.5)
        oracle.set_threads(5)
        dX5, dA5, dB5 = oracle.linear_bwd(dY, X, W, A, B, 0.5, rows=rows)
    finally:
        oracle.set_threads(old)
    np.testing.assert_array_equal(dX5, dX1[rows])
    np.testing.assert_array_equal(dA5, dA1)
    np.testing.assert_array_equal(dB5, dB1)


# ------------------------------------------------- eq. 1 / eq. 2 worked example

def test_int8_absmax_worked_example():
    """Section 3.1 eq. (1)-(2) on the pages' block [-5, 3, -2]."""
    g = _golden("int8_absmax_worked_example.txt")
    codes, c = oracle.int8_quant(np.float32(g["block"]))
    assert c == np.float32(g["c"][0])
    assert codes.tolist() == [int(v) for v in g["codes"]]
    deq = oracle.int8_dequant(codes, c)
    np.testing.assert_allclose(deq, g["dequant"], rtol=0, atol=2e-6)


def test_int8_blocks_follow_the_definition():
    """Block-wise eq. (1)/(2): every block gets c = RN32(127 / absmax) and
    codes round-half-away(RN32(c x)) -- checked against a numpy restatement
    element by element; the absmax element maps to +-127; |codes| <= 127;
    a zero block has c = 0, codes 0 and dequantizes to exact zeros; the
    round trip is within half a step (absmax / 254) plus fp32 rounding."""
    rng = np.random.default_rng(7)
    x = (rng.standard_normal(64 * 37 + 13) * 0.02).astype(np.float32)
    x[64 * 5:64 * 6] = 0.0                      # a zero block
    x[64 * 9 + 3] = 0.5                          # an outlier
    codes, c = oracle.int8_quant_blocks(x, 64)
    nb = -(-x.size // 64)
    assert c.size == nb
    for j in range(nb):
        blk = x[64 * j:64 * j + 64]
        a = np.float32(np.max(np.abs(blk)))
        if a == 0:
            assert c[j] == 0 and not codes[64 * j:64 * j + 64].any()
            continue
        cj = np.float32(np.float32(127.0) / a)
        assert c[j] == cj
        t = (cj * blk).astype(np.float32)   # RN32(c x)
        t64 = t.astype(np.float64)          # half away from zero, exactly, in fp64
        ref = np.sign(t64) * np.floor(np.abs(t64) + 0.5)
        np.testing.assert_array_equal(codes[64 * j:64 * j + blk.size].astype(np.float64), ref)
        k = int(np.argmax(np.abs(blk)))
        assert abs(int(codes[64 * j + k])) == 127
    assert np.abs(codes.astype(np.int32)).max() <= 127
    deq = oracle.int8_dequant_blocks(codes, c, 64)
    assert not deq[64 * 5:64 * 6].any()
    for j in range(nb):
        blk = x[64 * j:64 * j + 64]
        a = float(np.max(np.abs(blk)))
        err = np.abs(deq[64 * j:64 * j + blk.size].astype(np.float64) - blk)
        assert np.all(err <= a / 254 * (1 + 1e-5) + 1e-12)


# ------------------------------------------- the FP4 / Int4 comparison types

def test_e2m1_decode_matches_the_format():
    """OCP E2M1: sign, 2-bit exponent (bias 1), 1-bit mantissa; exponent 0 is
    subnormal.  The 16 patterns give +-{0, 0.5, 1, 1.5, 2, 3, 4, 6}."""
    import math
    mags = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]
    for b in range(16):
        v = oracle.e2m1_decode(b)
        assert abs(v) == mags[b & 7]
        assert (math.copysign(1.0, v) < 0) == (b >= 8)  # the sign bit, -0 included


def test_fp4_and_int4_tables():
    f = oracle.codebook("fp4")
    ref = np.array(sorted({s * m for s in (-1, 1) for m in (0, 0.5, 1, 1.5, 2, 3, 4, 6)}), np.float64) / 6.0
    assert ref.size == 15
    np.testing.assert_array_equal(f[:15], ref.astype(np.float32))
    assert f[15] == f[14] == 1.0 and f[0] == -1.0 and np.all(np.diff(f[:15]) > 0)
    i4 = oracle.codebook("int4")
    np.testing.assert_array_equal(i4[:15], (np.arange(-7, 8) / 7.0).astype(np.float32))
    assert i4[15] == i4[14] == 1.0 and np.all(i4[:15] == -i4[14::-1])


@pytest.mark.parametrize("qtype", ["fp4", "int4"])
def test_other_types_encode_by_brute_force(qtype):
    """Codes are the argmin over the type's table (ties to the lower index):
    the repeated top value is never chosen; block maxima map to the ends."""
    q = oracle.codebook(qtype)
    rng = np.random.default_rng(11)
    w = (rng.standard_normal(64 * 20 + 9) * 0.02).astype(np.float32)
    codes, c2, st = oracle.quantize_nf4(w, 64, qtype)
    assert st == 0
    allc = np.empty(w.size, np.int64)
    allc[0::2] = codes >> 4
    allc[1::2] = (codes & 15)[: w.size // 2]
    for j in range(c2.size):
        blk = w[64 * j:64 * j + 64]
        n = (blk / c2[j]).astype(np.float32)
        d = np.abs(n[:, None] - q[None, :]).astype(np.float32)
        np.testing.assert_array_equal(allc[64 * j:64 * j + blk.size], np.argmin(d, axis=1))
    assert not np.any(allc == 15)
