"""Test-side conversions between torch tensors and the oracle's numpy arrays,
and the float tolerance.  Shared by the GPU parity tests; holds none of the
method's arithmetic (the SwiGLU bound calls the oracle's SwiGLU)."""
import numpy as np
import torch

from oracle import formats as F


def bf16_np(t):
    """BF16 torch tensor (any device) -> float64 numpy array of its values."""
    return t.detach().to("cpu").to(torch.float32).numpy().astype(np.float64)


def bf16_torch(a, device="cuda"):
    """float64 numpy array of BF16-exact values -> BF16 torch tensor."""
    return torch.from_numpy(np.asarray(a, dtype=np.float32)).to(torch.bfloat16).to(device)


def u8_np(t):
    return t.detach().to("cpu").numpy().astype(np.uint8)


def unpack_codes(packed_t):
    return F.unpack_nibbles(u8_np(packed_t))


def assert_close_tol(got, ref, absdot, rel=1e-2, dot=1e-3, what=""):
    """Per-element |got - ref| <= rel*|ref| + dot*sum|a*b| (the float parity bar)."""
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    bound = rel * np.abs(ref) + dot * np.asarray(absdot, dtype=np.float64)
    err = np.abs(got - ref)
    bad = err > bound
    if bad.any():
        i = np.flatnonzero(bad.ravel())[:5]
        raise AssertionError(f"{what}: {bad.sum()} of {bad.size} elements out of tolerance; "
                             f"first: got {got.ravel()[i]}, ref {ref.ravel()[i]}, bound {bound.ravel()[i]}")


def assert_bits_equal(got, ref, what=""):
    got = np.asarray(got)
    ref = np.asarray(ref)
    assert got.shape == ref.shape, (what, got.shape, ref.shape)
    bad = got != ref
    if bad.any():
        i = np.flatnonzero(bad.ravel())[:8]
        raise AssertionError(f"{what}: {bad.sum()} of {bad.size} differ; first at {i}: got {got.ravel()[i]}, "
                             f"ref {ref.ravel()[i]}")


def f32_of(t):
    return t.detach().to("cpu").numpy().astype(np.float64)


def gate_up_interleave_index(F):
    """Row order of gate/up weights interleaved in blocks of 64: destination
    row 128 b + j holds gate row 64 b + j (j < 64) or up row F + 64 b + j - 64."""
    dst = np.arange(2 * F)
    b, j = dst // 128, dst % 128
    return np.where(j < 64, 64 * b + j, F + 64 * b + (j - 64))


def swiglu_carried(y_ref, absdot, F_):
    """The oracle's h = SwiGLU(bf16(y)) from its gate/up output y_ref [rows,
    2F] and a per-element bound on |h_gpu - h|: the GEMM tolerance of y
    (1e-2 |y| + 1e-3 sum|a b|) carried through SwiGLU to first order, plus
    one BF16 rounding of h."""
    from oracle import moe as M
    tol_y = 1e-2 * np.abs(y_ref) + 1e-3 * absdot
    g, u = y_ref[:, :F_], y_ref[:, F_:]
    sig = 1.0 / (1.0 + np.exp(-g))
    h_ref = M.swiglu(F.bf16_rne(y_ref.astype(np.float32)))
    dsilu = np.abs(sig * (1.0 + g * (1.0 - sig)))
    tol_h = dsilu * (np.abs(u) + tol_y[:, F_:]) * tol_y[:, :F_] + np.abs(g * sig) * tol_y[:, F_:] + \
        2.0 ** -7 * np.abs(h_ref) + 1e-30
    return h_ref, tol_h
