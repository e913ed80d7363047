"""CUDA router, permutation, gather, SwiGLU and combine against the CPU oracle
on the same seeded inputs: routing indices and permutations bit-exact, float
outputs within the tolerance."""
import numpy as np
import pytest
import torch

from oracle import formats as F
from oracle import moe as M
from oracle import nvfp4 as Q
from tests.helpers import (assert_bits_equal, assert_close_tol, bf16_np, bf16_torch, f32_of, u8_np)
from train_alignment_b200 import workloads as W

pytestmark = pytest.mark.gpu


def _logits(T, E, seed, kind="normal"):
    g = torch.Generator().manual_seed(seed)
    l = W.router_logits(T, E, kind, g, "cpu")
    if seed % 2 == 0:
        l = torch.round(l * 4) / 4          # many exact ties
    return l


@pytest.mark.parametrize("T,E,k", [(1, 8, 2), (333, 8, 2), (512, 128, 8), (1000, 64, 4), (77, 256, 8), (40, 5, 5)])
@pytest.mark.parametrize("renorm", [True, False])
def test_router_parity(cuda_lib, T, E, k, renorm):
    l = _logits(T, E, T + E + k, "zipf" if E >= 64 else "normal")
    idx, w = cuda_lib.moe_router_topk(l.cuda(), k, renorm)
    torch.cuda.synchronize()
    idx_ref, w_ref = M.router_topk(l.numpy().astype(np.float64), k, renorm)
    assert_bits_equal(f32_of(idx).astype(np.int64), idx_ref.astype(np.int64), "topk idx")
    assert np.allclose(f32_of(w), w_ref, rtol=2e-6, atol=1e-7)


@pytest.mark.parametrize("T,E,k", [(1, 4, 1), (300, 8, 2), (2048, 8, 2), (4096, 128, 8), (5000, 64, 4),
                                   (5000, 64, 8), (16384, 128, 8)])
def test_permute_parity(cuda_lib, T, E, k):
    l = _logits(T, E, 7 * T + E, "zipf")
    idx_ref, _ = M.router_topk(l.numpy().astype(np.float64), k)
    idx = torch.from_numpy(idx_ref.astype(np.int32)).cuda()
    off, row_of, src_of = cuda_lib.moe_permute(idx, E)
    torch.cuda.synchronize()
    off_ref, row_ref, src_ref = M.permute(idx_ref, E)
    assert_bits_equal(f32_of(off).astype(np.int64), off_ref.astype(np.int64), "expert_off")
    assert_bits_equal(f32_of(row_of).astype(np.int64), row_ref.astype(np.int64), "row_of")
    n = int(off_ref[-1])
    assert_bits_equal(f32_of(src_of)[:n].astype(np.int64), src_ref.astype(np.int64), "src_of")


def test_gather_parity(cuda_lib):
    T, E, k, K, nc = 300, 8, 2, 256, 16
    r = np.random.default_rng(3)
    x = F.bf16_rne(r.standard_normal((T, K)).astype(np.float32))
    c, s, g = Q.quantize(x)
    chan = Q.pad_channels(np.array([1, 9, 100]))
    resid = Q.residual_channels(x, c, s, g, chan)
    idx_ref, _ = M.router_topk(r.standard_normal((T, E)), k)
    off_ref, row_ref, src_ref = M.permute(idx_ref, E)
    cap = cuda_lib.moe_rows_capacity(T, k, E)
    src_full = np.full(cap, -7, dtype=np.int32)
    src_full[:len(src_ref)] = src_ref
    pc, ps, pr = cuda_lib.moe_gather(torch.from_numpy(src_full).cuda(), torch.from_numpy(off_ref).cuda(), E, cap,
                                     torch.from_numpy(F.pack_nibbles(c)).cuda(), torch.from_numpy(s).cuda(), K,
                                     bf16_torch(resid))
    torch.cuda.synchronize()
    n = int(off_ref[-1])
    assert_bits_equal(u8_np(pc)[:n], F.pack_nibbles(M.gather_rows(c, src_ref)), "codes")
    s_got = F.scales_from_tiled(u8_np(ps), cap, K // 16)[:n]
    assert_bits_equal(s_got, M.gather_rows(s, src_ref), "scales")
    assert_bits_equal(F.bf16_bits(bf16_np(pr)[:n]), F.bf16_bits(M.gather_rows(resid, src_ref)), "resid")


@pytest.mark.parametrize("T,E,k,K,nc", [(1, 4, 1, 64, 0), (300, 8, 2, 256, 16), (4096, 128, 8, 512, 32)])
def test_route_permute_composite(cuda_lib, T, E, k, K, nc):
    """quads_moe_route_permute (router + permutation + gather in one call)
    against the oracle's router_topk, permute and gather_rows: indices,
    offsets, rows, gathered codes, scales and residuals bit for bit, weights
    within float rounding."""
    r = np.random.default_rng(T + E + K)
    x = F.bf16_rne(r.standard_normal((T, K)).astype(np.float32))
    c, s, g = Q.quantize(x)
    chan = Q.pad_channels(np.sort(r.choice(K, max(nc - 5, 1), replace=False))) if nc else np.zeros(0, np.int32)
    resid = Q.residual_channels(x, c, s, g, chan) if nc else None
    l = _logits(T, E, 3 * T + E, "zipf" if E >= 64 else "normal")
    idx, w, off, row_of, src_of, pc, ps, pr = cuda_lib.moe_route_permute(
        l.cuda(), k, torch.from_numpy(F.pack_nibbles(c)).cuda(), torch.from_numpy(s).cuda(), K,
        bf16_torch(resid) if nc else None)
    torch.cuda.synchronize()
    assert cuda_lib.device_status() == cuda_lib.OK
    idx_ref, w_ref = M.router_topk(l.numpy().astype(np.float64), k)
    assert_bits_equal(f32_of(idx).astype(np.int64), idx_ref.astype(np.int64), "topk idx")
    assert np.allclose(f32_of(w), w_ref, rtol=2e-6, atol=1e-7)
    off_ref, row_ref, src_ref = M.permute(idx_ref, E)
    assert_bits_equal(f32_of(off).astype(np.int64), off_ref.astype(np.int64), "expert_off")
    assert_bits_equal(f32_of(row_of).astype(np.int64), row_ref.astype(np.int64), "row_of")
    n = int(off_ref[-1])
    assert_bits_equal(f32_of(src_of)[:n].astype(np.int64), src_ref.astype(np.int64), "src_of")
    assert_bits_equal(u8_np(pc)[:n], F.pack_nibbles(M.gather_rows(c, src_ref)), "gathered codes")
    cap = cuda_lib.moe_rows_capacity(T, k, E)
    assert_bits_equal(F.scales_from_tiled(u8_np(ps), cap, K // 16)[:n], M.gather_rows(s, src_ref), "gathered scales")
    if nc:
        assert_bits_equal(F.bf16_bits(bf16_np(pr)[:n]), F.bf16_bits(M.gather_rows(resid, src_ref)), "gathered resid")


@pytest.mark.parametrize("T,E,k,H", [(1, 4, 1, 64), (300, 8, 2, 1024), (4096, 64, 4, 2048)])
def test_gather_bf16_parity(cuda_lib, T, E, k, H):
    """BF16 rows gathered into expert order against the oracle's gather_rows:
    bit for bit, pad rows zero, rows past expert_off[E] untouched."""
    r = np.random.default_rng(T + E + H)
    x = F.bf16_rne(r.standard_normal((T, H)).astype(np.float32))
    idx_ref, _ = M.router_topk(r.standard_normal((T, E)), k)
    off_ref, row_ref, src_ref = M.permute(idx_ref, E)
    cap = cuda_lib.moe_rows_capacity(T, k, E)
    src_full = np.full(cap, -7, dtype=np.int32)
    src_full[:len(src_ref)] = src_ref
    out = torch.full((cap, H), float("nan"), dtype=torch.bfloat16, device="cuda")
    cuda_lib.moe_gather_bf16(torch.from_numpy(src_full).cuda(), torch.from_numpy(off_ref).cuda(), E, cap,
                             bf16_torch(x), out=out)
    torch.cuda.synchronize()
    n = int(off_ref[-1])
    got = bf16_np(out)
    assert_bits_equal(F.bf16_bits(got[:n]), F.bf16_bits(M.gather_rows(x, src_ref)), "gathered rows")
    assert np.all(np.isnan(got[n:])), "rows past expert_off[E] must be untouched"


def test_swiglu_parity(cuda_lib):
    E, F_ = 3, 256
    off = np.array([0, 128, 128, 384], dtype=np.int32)
    r = np.random.default_rng(4)
    y = F.bf16_rne((r.standard_normal((512, 2 * F_)) * 3).astype(np.float32))
    h, amax = cuda_lib.swiglu(bf16_torch(y), F_, torch.from_numpy(off).cuda(), E)
    torch.cuda.synchronize()
    n = int(off[-1])
    ref = M.swiglu(y[:n])
    got = bf16_np(h)[:n]
    assert_close_tol(got, ref, np.abs(ref), rel=1e-2, dot=0.0, what="swiglu")
    # per-expert amax is the max |h| of the device's own output, exactly
    a = f32_of(amax)
    assert a[1] == 0.0
    assert a[0] == np.max(np.abs(got[0:128])) and a[2] == np.max(np.abs(got[128:384]))


def test_combine_parity(cuda_lib):
    T, k, H = 500, 4, 1024
    r = np.random.default_rng(5)
    Y = F.bf16_rne(r.standard_normal((4096, H)).astype(np.float32))
    row_of = r.permutation(4096)[:T * k].astype(np.int32)
    w = r.random((T, k)).astype(np.float32)
    out = cuda_lib.moe_unpermute_combine(bf16_torch(Y), torch.from_numpy(row_of).cuda(),
                                         torch.from_numpy(w).cuda(), T, k, H)
    torch.cuda.synchronize()
    ref = M.combine(Y, row_of, w.astype(np.float64), k)
    absdot = M.combine(np.abs(Y), row_of, np.abs(w.astype(np.float64)), k)
    assert_close_tol(bf16_np(out), ref, absdot, what="combine")
