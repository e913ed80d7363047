"""CUDA quantizer, dequantizer, fake-quant, STE and channel calibration against
the CPU oracle on the same seeded inputs: codes, scales, per-tensor scales and
residuals bit-exact; float outputs bit-exact where the oracle's rounding is
the same single rounding."""
import numpy as np
import pytest
import torch

from oracle import formats as F
from oracle import nvfp4 as Q
from tests.helpers import (assert_bits_equal, bf16_np, bf16_torch, f32_of, gate_up_interleave_index, u8_np,
                           unpack_codes)
from train_alignment_b200 import workloads as W

pytestmark = pytest.mark.gpu


def _x(rows, K, seed, outliers=4, scale=20.0):
    r = np.random.default_rng(seed)
    x = r.standard_normal((rows, K)) * 10.0 ** r.uniform(-2, 2)
    ch = r.choice(K, min(outliers, K), replace=False)
    x[:, ch] *= scale
    return F.bf16_rne(x.astype(np.float32))


def _check_quant(lib, x, layout, amax=None, chan=None, group_off=None):
    rows, K = x.shape
    xt = bf16_torch(x)
    kw = dict(scale_layout=layout)
    ng = 1
    if group_off is not None:
        ng = len(group_off) - 1
        kw.update(group_off=torch.tensor(group_off, dtype=torch.int32, device="cuda"), n_groups=ng)
    if amax is not None:
        kw["amax_in"] = torch.tensor(np.atleast_1d(amax), dtype=torch.float32, device="cuda")
    if chan is not None:
        kw["chan"] = torch.tensor(chan, dtype=torch.int32, device="cuda")
    codes, scales, g, resid = lib.quantize_nvfp4(xt, **kw)
    torch.cuda.synchronize()
    if group_off is None:
        c_ref, s_ref, g_ref = Q.quantize(x, amax)
        g_ref = np.array([g_ref])
    else:
        c_ref, s_ref, g_ref = Q.quantize_grouped(x, group_off, None if amax is None else np.atleast_1d(amax))
    assert_bits_equal(f32_of(g).astype(np.float32), g_ref.astype(np.float32), "g")
    assert_bits_equal(unpack_codes(codes), c_ref, "codes")
    s_got = u8_np(scales)
    if layout == lib.SCALES_TILED:
        s_got = F.scales_from_tiled(s_got, rows, K // 16)
        # padding of the tiled layout is zero
        full = u8_np(scales)
        assert full.sum() == s_got.astype(np.int64).sum()
    else:
        s_got = s_got.reshape(rows, K // 16)
    assert_bits_equal(s_got, s_ref, "scales")
    if chan is not None:
        r_ref = Q.residual_channels(x, c_ref, s_ref, g_ref[0] if group_off is None else 0, chan) \
            if group_off is None else None
        if r_ref is not None:
            assert_bits_equal(F.bf16_bits(bf16_np(resid)), F.bf16_bits(r_ref), "resid")
    return codes, scales, g


@pytest.mark.parametrize("rows,K", [(1, 16), (37, 64), (200, 256), (1000, 1024), (130, 4096)])
@pytest.mark.parametrize("layout", [0, 1])
def test_quantize_parity(cuda_lib, rows, K, layout):
    x = _x(rows, K, rows * 31 + K)
    _check_quant(cuda_lib, x, layout)


def test_quantize_with_amax_and_channels(cuda_lib):
    x = _x(300, 512, 5, outliers=6, scale=30.0)
    chan = [3, 17, 40, 41, 200, 511] + [-1] * 10
    _check_quant(cuda_lib, x, 0, chan=chan)
    # calibrated amax smaller than the data max: saturation path
    _check_quant(cuda_lib, x, 1, amax=float(np.max(np.abs(x)) * 0.5), chan=chan)


def test_quantize_ties_and_special_values(cuda_lib):
    """g = 1 exactly (amax 2688) and a block with amax 6, so x * inv is x:
    every E2M1 midpoint is hit exactly, both signs, plus zeros and -0."""
    row = np.zeros((4, 64))
    row[0, :16] = [6, 0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5, -0.25, -0.75, -1.25, -1.75, -2.5, -3.5, -5, -0.0]
    row[0, 16:32] = 2688.0
    row[1, :16] = [6, 0.2, 0.3, 0.74, 0.76, 1.24, 1.26, 4.9, 5.1, 5.9, 6.0, -6.0, 0.0, -0.0, 1e-6, -1e-6]
    row[2, :] = 0.0
    row[3, 32:48] = -0.0
    x = F.bf16_rne(row.astype(np.float32))
    x[3, 32:48] = -0.0
    _check_quant(cuda_lib, x, 0)
    _check_quant(cuda_lib, x, 1)


def test_quantize_all_zero(cuda_lib):
    x = np.zeros((5, 32))
    _check_quant(cuda_lib, x, 0)


def test_quantize_grouped(cuda_lib):
    x = _x(700, 256, 9)
    off = [0, 128, 128, 384, 700]
    _check_quant(cuda_lib, x, 0, group_off=off)
    _check_quant(cuda_lib, x, 1, group_off=off)


def _every_block_max(tensor_amax, seed, binades=13):
    """Rows of 16-element blocks per group: one block for every BF16 value v in
    [A 2^-binades, A] as the block maximum (the other 15 elements below it,
    random signs), so that every block-scale ratio amax_b / fp32(6 g) that can
    round to a non-zero E4M3 code occurs."""
    r = np.random.default_rng(seed)
    blocks, off = [], [0]
    for A in tensor_amax:
        a_bits = int(F.bf16_bits(np.array([A], dtype=np.float32))[0])
        lo_bits = int(F.bf16_bits(np.array([A * 2.0 ** -binades], dtype=np.float32))[0])
        vals = F.bf16_from_bits(np.arange(lo_bits, a_bits + 1, dtype=np.uint16)).astype(np.float64)
        n = (len(vals) + 31) // 32 * 32                 # whole rows of 32 blocks
        vals = np.concatenate([vals, np.full(n - len(vals), A)])
        b = vals[:, None] * r.uniform(0, 1, (n, 16))
        b[np.arange(n), r.integers(0, 16, n)] = vals
        b *= r.choice([-1.0, 1.0], (n, 16))
        blocks.append(F.bf16_rne(b.astype(np.float32)).reshape(n // 32, 512))
        off.append(off[-1] + n // 32)
    return np.concatenate(blocks), off


@pytest.mark.parametrize("n_groups", [8, 40])
def test_quantize_every_block_scale(cuda_lib, n_groups):
    """Every BF16 block maximum over 13 binades below the tensor maximum, for
    tensor maxima from 2^-80 to 2^80 (the smallest ones below the range where
    the quantizer's quotient shortcut applies): codes and scales bit-exact
    against the oracle.  8 groups use the per-group scale table, 40 do not."""
    r = np.random.default_rng(100 + n_groups)
    A = F.bf16_rne((2.0 ** r.uniform(-80, 80, n_groups) * r.uniform(1, 2, n_groups)).astype(np.float32))
    A[:3] = F.bf16_rne(np.array([2.0 ** -70, 448.0, 1.0], dtype=np.float32))
    x, off = _every_block_max(A.astype(np.float64), n_groups)
    _check_quant(cuda_lib, x, 1, group_off=off)


def test_amax_strided_rows(cuda_lib):
    """Rows with a stride above K take the row kernel; contiguous rows the
    flat one: both give the exact max |x| per group."""
    x = _x(300, 256 + 64, 15)
    full = bf16_torch(x)
    view = full[:, :256]                      # row stride 320 elements
    off = [0, 7, 7, 300]
    t_off = torch.tensor(off, dtype=torch.int32, device="cuda")
    got_s = f32_of(cuda_lib.amax_bf16(view, t_off, 3))
    got_c = f32_of(cuda_lib.amax_bf16(view.contiguous(), t_off, 3))
    want = [np.max(np.abs(x[0:7, :256])), 0.0, np.max(np.abs(x[7:300, :256]))]
    assert_bits_equal(got_s, np.array(want), "amax strided")
    assert_bits_equal(got_c, np.array(want), "amax contiguous")


def test_amax_groups(cuda_lib):
    x = _x(500, 128, 10)
    off = [0, 100, 100, 500]
    got = f32_of(cuda_lib.amax_bf16(bf16_torch(x), torch.tensor(off, dtype=torch.int32, device="cuda"), 3))
    want = [np.max(np.abs(x[0:100])), 0.0, np.max(np.abs(x[100:500]))]
    assert_bits_equal(got, np.array(want), "amax")


def test_amax_ignores_rows_past_the_last_group(cuda_lib):
    """Rows at or past group_off[n] belong to no group: huge values there
    (the unused tail of an expert-ordered buffer) change no group's amax, in
    the strided and the contiguous kernel, and in the quantizer's own amax."""
    x = _x(384, 128, 21)
    x[300:] = 3.0e38
    off = torch.tensor([0, 100, 100, 300], dtype=torch.int32, device="cuda")
    full = bf16_torch(np.concatenate([x, np.zeros((384, 64))], axis=1))
    want = [np.max(np.abs(x[0:100])), 0.0, np.max(np.abs(x[100:300]))]
    assert_bits_equal(f32_of(cuda_lib.amax_bf16(bf16_torch(x), off, 3)), np.array(want), "amax contiguous")
    assert_bits_equal(f32_of(cuda_lib.amax_bf16(full[:, :128], off, 3)), np.array(want), "amax strided")
    _, _, g, _ = cuda_lib.quantize_nvfp4(bf16_torch(x), group_off=off, n_groups=3, scale_layout=cuda_lib.SCALES_TILED)
    g_ref = [Q.tensor_scale(a) for a in want]
    assert_bits_equal(f32_of(g).astype(np.float32), np.array(g_ref, dtype=np.float32), "g")


@pytest.mark.parametrize("layout", [0, 1])
def test_dequant_parity(cuda_lib, layout):
    x = _x(257, 512, 11)
    codes, scales, g = _check_quant(cuda_lib, x, layout)
    c_ref, s_ref, g_ref = Q.quantize(x)
    out32 = cuda_lib.dequant(codes, scales, layout, g, 257, 512, out_dtype=cuda_lib.OUT_F32)
    out16 = cuda_lib.dequant(codes, scales, layout, g, 257, 512, out_dtype=cuda_lib.OUT_BF16)
    ref32 = Q.dequant_f32(c_ref, s_ref, g_ref)
    assert_bits_equal(f32_of(out32).astype(np.float32), ref32.astype(np.float32), "deq f32")
    assert_bits_equal(F.bf16_bits(bf16_np(out16)), F.bf16_bits(F.bf16_rne(Q.dequant(c_ref, s_ref, g_ref))),
                      "deq bf16")


@pytest.mark.parametrize("fold", [True, False])
def test_fakequant_parity(cuda_lib, fold):
    r = np.random.default_rng(12)
    n_mat, rows, K = 3, 256, 192
    w = F.bf16_rne((r.standard_normal((n_mat, rows, K)) * 0.02 * (1 + np.arange(n_mat))[:, None, None])
                   .astype(np.float32))
    chan = [5, 77, 150, -1]
    wt = bf16_torch(w)
    ch = torch.tensor(chan, dtype=torch.int32, device="cuda")
    w_fq, codes, scales, g, w_chan = cuda_lib.fakequant_weight_ste(wt, fold_global=fold, chan=ch)
    w_fq2, _, _, _, w_raw = cuda_lib.fakequant_weight_ste(wt, fold_global=fold, chan=ch, chan_raw=True)
    torch.cuda.synchronize()
    s_all = F.scales_from_tiled(u8_np(scales), n_mat * rows, K // 16).reshape(n_mat, rows, K // 16)
    c_all = unpack_codes(codes)
    for m in range(n_mat):
        wf_ref, c_ref, s_ref, g_ref = Q.fakequant_weight(w[m], fold_global=fold)
        assert_bits_equal(F.bf16_bits(bf16_np(w_fq[m])), F.bf16_bits(wf_ref), f"w_fq[{m}]")
        assert_bits_equal(c_all[m], c_ref, f"codes[{m}]")
        assert_bits_equal(s_all[m], s_ref, f"scales[{m}]")
        assert np.float32(f32_of(g)[m]) == np.float32(g_ref)
        # the compensation operand is the folded dequantized weight column (or the raw column)
        deq = F.bf16_rne(F.f32(Q.dequant(c_ref, s_ref, g_ref)))
        for j, c in enumerate(chan):
            want = deq[:, c] if c >= 0 else np.zeros(rows)
            assert_bits_equal(F.bf16_bits(bf16_np(w_chan[m][:, j])), F.bf16_bits(want), "w_chan")
            want_raw = w[m][:, c] if c >= 0 else np.zeros(rows)
            assert_bits_equal(F.bf16_bits(bf16_np(w_raw[m][:, j])), F.bf16_bits(want_raw), "w_chan raw")
    # the rollout's quantizer gives the same grid on the same matrix
    c1, s1, g1, _ = cuda_lib.quantize_nvfp4(wt[1].contiguous(), scale_layout=cuda_lib.SCALES_TILED)
    torch.cuda.synchronize()
    assert_bits_equal(unpack_codes(c1), c_all[1], "rollout vs trainer codes")


@pytest.mark.parametrize("fold", [True, False])
def test_fakequant_gate_up_interleaved(cuda_lib, fold):
    """The gate/up variant: W_fq in the input order, the rollout's codes,
    scales and compensation columns in the 64-row interleaved gate/up order."""
    r = np.random.default_rng(13)
    n_mat, F_, K = 2, 192, 128
    rows = 2 * F_
    w = F.bf16_rne((r.standard_normal((n_mat, rows, K)) * 0.02).astype(np.float32))
    chan = [3, 64, 100, -1]
    wt = bf16_torch(w)
    ch = torch.tensor(chan, dtype=torch.int32, device="cuda")
    w_fq, codes, scales, g, w_chan = cuda_lib.fakequant_weight_ste(wt, fold_global=fold, chan=ch, gate_up=True)
    torch.cuda.synchronize()
    perm = gate_up_interleave_index(F_)
    s_all = F.scales_from_tiled(u8_np(scales), n_mat * rows, K // 16).reshape(n_mat, rows, K // 16)
    c_all = unpack_codes(codes)
    for m in range(n_mat):
        wf_ref, c_ref, s_ref, g_ref = Q.fakequant_weight(w[m], fold_global=fold)
        assert_bits_equal(F.bf16_bits(bf16_np(w_fq[m])), F.bf16_bits(wf_ref), f"w_fq[{m}]")
        assert_bits_equal(c_all[m], c_ref[perm], f"codes[{m}]")
        assert_bits_equal(s_all[m], s_ref[perm], f"scales[{m}]")
        assert np.float32(f32_of(g)[m]) == np.float32(g_ref)
        deq = F.bf16_rne(F.f32(Q.dequant(c_ref, s_ref, g_ref)))
        for j, c in enumerate(chan):
            want = deq[perm, c] if c >= 0 else np.zeros(rows)
            assert_bits_equal(F.bf16_bits(bf16_np(w_chan[m][:, j])), F.bf16_bits(want), "w_chan")


@pytest.mark.parametrize("accumulate", [False, True])
def test_ste_backward(cuda_lib, accumulate):
    r = np.random.default_rng(13)
    n = 1000 * 8 + 5
    a = F.bf16_rne(r.standard_normal(n).astype(np.float32))
    b = F.bf16_rne(r.standard_normal(n).astype(np.float32))
    gw = bf16_torch(b)
    out = cuda_lib.fakequant_weight_ste_backward(bf16_torch(a), gw, accumulate=accumulate)
    torch.cuda.synchronize()
    ref = Q.ste_backward(a, b if accumulate else None)
    assert_bits_equal(F.bf16_bits(bf16_np(out)), F.bf16_bits(ref), "ste")


def test_channel_scores_and_selection(cuda_lib):
    x = _x(600, 512, 14, outliers=8, scale=25.0)
    sc = cuda_lib.channel_scores(bf16_torch(x))
    torch.cuda.synchronize()
    ref = Q.channel_scores(x)
    got = f32_of(sc)
    assert np.allclose(got, ref, rtol=2e-5, atol=1e-30)
    n = 16
    sel = cuda_lib.select_channels(sc, n)
    torch.cuda.synchronize()
    sel_ref = Q.select_channels(ref, n)
    got_sel = f32_of(sel).astype(np.int64)
    assert np.all(np.diff(got_sel) > 0)
    # same set unless the boundary scores are within float32 summation error
    if set(got_sel) != set(sel_ref):
        kth = np.sort(ref)[::-1][n - 1]
        diff = set(got_sel) ^ set(sel_ref)
        assert all(abs(ref[c] - kth) <= 1e-4 * kth for c in diff)
    # the device selection is exact on the device's own scores
    assert_bits_equal(got_sel, Q.select_channels(got, n), "select on device scores")


def test_quantize_large_activation(cuda_lib):
    """Full-size activation of the 16384-token prefill layer (67M elements):
    sampled rows against the oracle, all rows' scales against the oracle's
    block-scale formula evaluated on the sampled blocks."""
    cfg = W.PREFILL_T16384
    x = W.activations(cfg.T, cfg.H, "student_t", 0, 1.0, torch.Generator(device="cuda").manual_seed(3), "cuda")
    codes, scales, g, _ = cuda_lib.quantize_nvfp4(x, scale_layout=cuda_lib.SCALES_LINEAR)
    torch.cuda.synchronize()
    amax = float(x.abs().max().float())
    r = np.random.default_rng(0)
    rows = np.sort(r.choice(cfg.T, 48, replace=False))
    xs = bf16_np(x[rows])
    g_ref = Q.tensor_scale(amax)
    c_ref, s_ref = Q.quantize_with_scale(xs, g_ref)
    assert np.float32(f32_of(g)[0]) == np.float32(g_ref)
    assert_bits_equal(unpack_codes(codes[rows]), c_ref, "codes (sampled rows)")
    assert_bits_equal(u8_np(scales).reshape(cfg.T, cfg.H // 16)[rows], s_ref, "scales (sampled rows)")
