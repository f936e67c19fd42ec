"""Shared test helpers: moving synthetic inputs to the GPU and the parity
tolerances for the bf16 GEMM outputs."""
import numpy as np

# Y, dX, dA, dB against the fp64 oracle: relative Frobenius error and
# max-abs error relative to the largest reference magnitude.
REL_FRO_TOL = 5e-3
MAX_ABS_TOL = 2e-2


def dev_f32(a):
    import torch
    return torch.from_numpy(np.ascontiguousarray(a, np.float32)).cuda()


def dev_bf16(bits):
    import torch
    t = torch.from_numpy(np.ascontiguousarray(bits, np.uint16).view(np.int16)).cuda()
    return t.view(torch.bfloat16)


def host_f64(t):
    return t.float().cpu().numpy().astype(np.float64)


def bits_of(t):
    """bf16 CUDA tensor -> numpy uint16 bit patterns."""
    import torch
    return t.view(torch.int16).cpu().numpy().view(np.uint16)


def check_close(got, ref, name=""):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    assert got.shape == ref.shape, (name, got.shape, ref.shape)
    assert np.all(np.isfinite(got)), name
    err = got - ref
    nref = np.linalg.norm(ref)
    rel = np.linalg.norm(err) / nref if nref > 0 else np.linalg.norm(err)
    mref = np.max(np.abs(ref)) if ref.size else 0.0
    mabs = np.max(np.abs(err)) if err.size else 0.0
    assert rel <= REL_FRO_TOL, f"{name}: relative Frobenius error {rel:.3e}"
    assert mabs <= MAX_ABS_TOL * max(mref, 1e-30), f"{name}: max abs error {mabs:.3e} vs max|ref| {mref:.3e}"
    return rel, mabs
