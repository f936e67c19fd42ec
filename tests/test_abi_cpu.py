"""Host-side checks of the C-ABI library that need no GPU: it loads, it
exports every entry point include/qlora.h declares, its host-computed NF4
codebook equals the oracle's bit for bit, and argument errors are caught on
the host before anything is launched."""
import ctypes
import os
import re

import numpy as np
import pytest

import oracle

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _header_functions():
    text = open(os.path.join(ROOT, "include", "qlora.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^\s*[A-Za-z_][\w\s\*]*?\b(qlora_\w+)\s*\(", text, flags=re.M)))


@pytest.fixture(scope="module")
def q():
    from bit_nf4_quantized_13_b200 import build
    build.build()
    import bit_nf4_quantized_13_b200 as mod
    return mod


def test_header_declares_the_five_calls():
    names = _header_functions()
    for n in ("qlora_nf4_codebook", "qlora_quantize_nf4_dq", "qlora_dequantize",
              "qlora_linear_fwd", "qlora_linear_bwd"):
        assert n in names


def test_library_exports_every_declared_symbol(q):
    raw = ctypes.CDLL(q.LIB_PATH)
    for n in _header_functions():
        assert hasattr(raw, n), n


def test_codebook_matches_oracle_bit_exact(q):
    got = q.qlora_nf4_codebook()
    ref = oracle.nf4_codebook()
    np.testing.assert_array_equal(got.view(np.uint32), ref.view(np.uint32))
    assert q.lib.qlora_nf4_codebook(None) == 1
    for name, qt in (("nf4", q.TYPE_NF4), ("fp4", q.TYPE_FP4), ("int4", q.TYPE_INT4)):
        np.testing.assert_array_equal(q.qlora_codebook(qt).view(np.uint32), oracle.codebook(name).view(np.uint32))


def test_workspace_sizes(q):
    assert q.qlora_quantize_workspace_size(0) == 2048 + 16
    assert q.qlora_quantize_workspace_size(64) == 2048 + 16 + 16
    assert q.qlora_quantize_workspace_size(4096 * 4096) == 2048 + 16 + 4 * 4096 * 4096 // 64
    assert q.qlora_linear_fwd_workspace_size(4096, 4096, 4096, 64) >= 4096 * 64 * 2
    assert q.qlora_linear_bwd_workspace_size(4096, 4096, 4096, 64) >= 2 * 4096 * 64 * 2
    assert q.qlora_linear_fwd_workspace_size(16, 100, 100, 8) == 0  # K % 64 != 0
    assert q.qlora_linear_group_fwd_workspace_size(4096, 3, 64) >= 4096 * 192 * 2
    assert q.qlora_linear_group_bwd_workspace_size(4096, 3, 64) >= 2 * 4096 * 192 * 2
    assert q.qlora_linear_group_fwd_workspace_size(16, 5, 8) == 0      # more than 4 linears
    assert q.qlora_linear_group_bwd_workspace_size(16, 2, 256) == 0    # G r > 256


def test_argument_validation_on_host(q):
    L = q.lib
    P = 1 << 20  # a 16-byte-aligned stand-in address; never dereferenced on these paths
    # quantize: block sizes, negative numel, NULL / misaligned pointers, workspace
    assert L.qlora_quantize_nf4_dq(P, 64, 32, 256, P, P, P, P, P, 4096, None, None) == 2
    assert L.qlora_quantize_nf4_dq(P, 64, 64, 128, P, P, P, P, P, 4096, None, None) == 2
    assert L.qlora_quantize_nf4_dq(P, -1, 64, 256, P, P, P, P, P, 4096, None, None) == 1
    assert L.qlora_quantize_nf4_dq(P, 0, 64, 256, None, None, None, None, None, 0, None, None) == 0
    assert L.qlora_quantize_nf4_dq(None, 64, 64, 256, P, P, P, P, P, 4096, None, None) == 1
    assert L.qlora_quantize_nf4_dq(P + 4, 64, 64, 256, P, P, P, P, P, 4096, None, None) == 1
    assert L.qlora_quantize_nf4_dq(P, 64, 64, 256, P, P, P, P, None, 0, None, None) == 3
    assert L.qlora_quantize_nf4_dq(P, 64, 64, 256, P, P, P, P, P, 100, None, None) == 3
    assert L.qlora_quantize_nf4_dq(P, 64, 64, 256, P, P, P, P, P, 4096, P + 2, None) == 1
    # dequant: dtype, block sizes
    assert L.qlora_dequantize(P, P, P, P, 64, 64, 256, P, 2, None) == 1
    assert L.qlora_dequantize(P, P, P, P, 64, 64, 64, P, 0, None) == 2
    assert L.qlora_dequantize(P, P, P, P, 0, 64, 256, None, 0, None) == 0
    # linear: K % 64, rank bounds, shapes, pointers, workspace
    f32 = ctypes.c_float
    assert L.qlora_linear_fwd(P, 16, 64, 100, P, P, P, P, P, P, 8, f32(1), P, P, P, 1 << 20, None) == 2
    assert L.qlora_linear_fwd(P, 16, 64, 128, P, P, P, P, P, P, 257, f32(1), P, P, P, 1 << 20, None) == 2
    assert L.qlora_linear_fwd(P, 16, 64, 128, P, P, P, P, P, P, 0, f32(1), P, P, P, 1 << 20, None) == 1
    assert L.qlora_linear_fwd(P, -1, 64, 128, P, P, P, P, P, P, 8, f32(1), P, P, P, 1 << 20, None) == 1
    assert L.qlora_linear_fwd(P, 16, 64, 128, P, P, P, P, None, P, 8, f32(1), P, P, P, 1 << 20, None) == 1
    assert L.qlora_linear_fwd(P, 16, 64, 128, P, P, P, P, P, P, 8, f32(1), P, None, None, 0, None) == 3
    assert L.qlora_linear_bwd(P, P, 16, 64, 128, P, P, P, P, P, P, 8, f32(1), None, P, P, P, None, 0,
                              None) == 3
    assert L.qlora_linear_bwd(P, P, 16, 64, 128, P, P, P, P, P, P, 8, f32(1), None, P, None, P, P,
                              1 << 20, None) == 1
    assert L.qlora_fp8_e4m3_encode(P, P, -1, None) == 1
    assert L.qlora_fp8_e4m3_encode(None, None, 0, None) == 0
    # Int8: block sizes, negative sizes, pointers
    assert L.qlora_int8_quantize(P, 64, 48, P, P, None, None) == 2
    assert L.qlora_int8_quantize(P, -1, 64, P, P, None, None) == 1
    assert L.qlora_int8_quantize(None, 64, 64, P, P, None, None) == 1
    assert L.qlora_int8_quantize(P, 0, 64, None, None, None, None) == 0
    assert L.qlora_int8_dequantize(P, P, 64, 512, P, None) == 2
    assert L.qlora_int8_dequantize(P, P, 64, 64, P + 8, None) == 1
    # the typed 4-bit entry points refuse unknown types
    assert L.qlora_quantize_4bit_dq(3, P, 64, 64, 256, P, P, P, P, P, 4096, None, None) == 1
    assert L.qlora_dequantize_4bit(-1, P, P, P, P, 64, 64, 256, P, 0, None) == 1
    assert L.qlora_linear_fwd_4bit(9, P, 16, 64, 128, P, P, P, P, P, P, 8, f32(1), P, P, P, 1 << 20, None) == 1
    assert L.qlora_linear_bwd_4bit(9, P, P, 16, 64, 128, P, P, P, P, P, P, 8, f32(1), None, P, P, P, P, 1 << 20,
                                   None) == 1
    # grouped linears: group size, total rank, weight descriptors, type
    W = (q._Weight4bit * 5)(*[q._Weight4bit(P, P, P, P, 256) for _ in range(5)])
    gf = L.qlora_linear_group_fwd
    assert gf(0, P, 0, 128, W, 3, P, P, 8, f32(1), P, None, None, 0, None) == 0   # M == 0: nothing to do
    assert gf(0, P, 0, 128, W, 5, P, P, 8, f32(1), P, None, None, 0, None) == 2   # G > 4
    assert gf(0, P, 0, 128, W, 0, P, P, 8, f32(1), P, None, None, 0, None) == 1   # G < 1
    assert gf(0, P, 0, 128, None, 2, P, P, 8, f32(1), P, None, None, 0, None) == 1
    assert gf(0, P, 0, 128, W, 3, P, P, 128, f32(1), P, None, None, 0, None) == 2  # G r > 256
    assert gf(0, P, 0, 128, W, 2, P, P, 12, f32(1), P, None, None, 0, None) == 2   # r % 8
    assert gf(0, P, 0, 100, W, 2, P, P, 8, f32(1), P, None, None, 0, None) == 2    # K % 64
    assert gf(9, P, 0, 128, W, 2, P, P, 8, f32(1), P, None, None, 0, None) == 1    # unknown type
    assert gf(0, P, 0, 128, W, 2, None, P, 8, f32(1), P, None, None, 0, None) == 1
    Wn = (q._Weight4bit * 2)(q._Weight4bit(P, P, P, P, 256), q._Weight4bit(P, None, P, P, 256))
    assert gf(0, P, 0, 128, Wn, 2, P, P, 8, f32(1), P, None, None, 0, None) == 1
    Wr = (q._Weight4bit * 2)(q._Weight4bit(P, P, P, P, 256), q._Weight4bit(P, P, P, P, 100))
    assert gf(0, P, 16, 128, Wr, 2, P, P, 8, f32(1), P, None, None, 0, None) == 2  # N_g % 256
    assert L.qlora_linear_group_bwd(0, P, P, 0, 128, W, 2, P, P, 8, f32(1), None, P, None, P, None, 0,
                                    None) == 1  # dA_cat NULL
    # the ceiling probes: word counts that are not whole 16-byte runs, NULL pointers
    assert L.qlora_debug_fill(P, 3, 0, None) == 1
    assert L.qlora_debug_fill(None, 4, 0, None) == 1
    assert L.qlora_debug_fill(P + 4, 4, 0, None) == 1
    assert L.qlora_debug_fill(None, 0, 0, None) == 0       # nothing to write, nothing launched
    assert L.qlora_debug_read(P, 4, 0, None, None) == 1    # no sink
    assert L.qlora_debug_read(P, -4, 0, P, None) == 1
    # the failure-detection self-test refuses limits outside (0, 1 s]
    assert L.qlora_debug_wait_timeout(0, None) == 1
    assert L.qlora_debug_wait_timeout(2_000_000_000, None) == 1
