"""The tcgen05 NVFP4 grouped GEMM with residual compensation against the CPU
oracle: per element |err| <= 1e-2 |ref| + 1e-3 sum|a b| (compensation terms
included).  Inputs (codes, scales, residuals, weights) come from the oracle's
quantizer on seeded BF16 data."""
import numpy as np
import pytest
import torch

from oracle import formats as F
from oracle import moe as M
from oracle import nvfp4 as Q
from tests.helpers import (assert_bits_equal, assert_close_tol, bf16_np, bf16_torch, f32_of, gate_up_interleave_index,
                           swiglu_carried, u8_np)
from train_alignment_b200 import workloads as W

pytestmark = pytest.mark.gpu


def _problem(counts, N, K, nc, seed, x_scale=1.0):
    """Expert-ordered activations with the given per-expert row counts,
    quantized by the oracle; weights per expert quantized by the oracle."""
    r = np.random.default_rng(seed)
    E = len(counts)
    padded = [-(-c // 128) * 128 for c in counts]
    off = np.concatenate([[0], np.cumsum(padded)]).astype(np.int32)
    R = int(off[-1])
    cap = R + 128                                    # spare rows past the last expert
    x = np.zeros((cap, K))
    for e in range(E):
        x[off[e]:off[e] + counts[e]] = r.standard_normal((counts[e], K)) * x_scale
    ch_out = r.choice(K, 3, replace=False)
    x[:, ch_out] *= 16
    x = F.bf16_rne(x.astype(np.float32))
    a_c, a_s, g_a = Q.quantize(x[:R])
    chan = Q.pad_channels(Q.select_channels(Q.channel_scores(x[:R]), nc - 5) if nc else np.zeros(0, int), 16) \
        if nc else None
    w = F.bf16_rne((r.standard_normal((E, N, K)) * 0.02).astype(np.float32))
    wq = [Q.quantize(w[e]) for e in range(E)]
    w_c = np.stack([q[0] for q in wq])
    w_s = np.stack([q[1] for q in wq])
    g_w = np.array([q[2] for q in wq])
    resid = wc = None
    if nc:
        resid = Q.residual_channels(x[:R], a_c, a_s, g_a, chan)
        wc = np.zeros((E, N, nc))
        for e in range(E):
            deq = F.bf16_rne(F.f32(Q.dequant(w_c[e], w_s[e], g_w[e])))
            for j, c in enumerate(chan):
                if c >= 0:
                    wc[e, :, j] = deq[:, c]
    return dict(E=E, N=N, K=K, nc=nc, off=off, cap=cap, R=R, a_c=a_c, a_s=a_s, g_a=g_a, w_c=w_c, w_s=w_s,
                g_w=g_w, resid=resid, wc=wc)


def _run_gpu(lib, p):
    E, N, K, cap, R = p["E"], p["N"], p["K"], p["cap"], p["R"]
    a_codes = np.zeros((cap, K // 2), np.uint8)
    a_codes[:R] = F.pack_nibbles(p["a_c"])
    a_scales = np.zeros((cap, K // 16), np.uint8)
    a_scales[:R] = p["a_s"]
    w_codes = F.pack_nibbles(p["w_c"])
    w_scales = F.scales_to_tiled(p["w_s"].reshape(E * N, K // 16))
    dev = "cuda"
    args = dict(
        a_codes=torch.from_numpy(a_codes).to(dev), a_scales=torch.from_numpy(F.scales_to_tiled(a_scales)).to(dev),
        g_a=torch.tensor([p["g_a"]], dtype=torch.float32, device=dev),
        w_codes=torch.from_numpy(np.ascontiguousarray(w_codes)).to(dev), w_scales=torch.from_numpy(w_scales).to(dev),
        g_w=torch.tensor(p["g_w"], dtype=torch.float32, device=dev),
        expert_off=torch.from_numpy(p["off"]).to(dev), E=E, rows_cap=cap, N=N, K=K)
    if p["nc"]:
        resid = np.zeros((cap, p["nc"]))
        resid[:R] = p["resid"]
        args["a_resid"] = bf16_torch(resid)
        args["w_resid"] = bf16_torch(p["wc"])
    y = torch.full((cap, N), float("nan"), dtype=torch.bfloat16, device=dev)
    lib.moe_grouped_gemm_nvfp4(y=y, **args)
    assert lib.device_status() == lib.OK
    torch.cuda.synchronize()
    return bf16_np(y)


def _oracle(p):
    return M.grouped_gemm(p["a_c"], p["a_s"], p["g_a"], p["w_c"], p["w_s"], p["g_w"], p["off"], p["resid"], p["wc"])


@pytest.mark.parametrize("counts,N,K,nc", [
    ([64], 128, 64, 0),                 # one tile, one MMA along K
    ([100], 128, 256, 0),               # one stage
    ([64], 512, 256, 16),               # the single-linear shape with compensation
    ([130, 0, 257], 256, 512, 32),      # empty expert, ragged experts, two stages
    ([128, 300], 128, 320, 16),         # partial last stage (K % 256 = 64)
    ([500, 20, 1000, 3], 384, 1024, 64),
    ([256], 128, 4096, 128),            # long K, widest compensation
])
def test_grouped_gemm_parity(cuda_lib, counts, N, K, nc):
    p = _problem(counts, N, K, nc, seed=sum(counts) + N + K + nc)
    got = _run_gpu(cuda_lib, p)
    ref, absdot = _oracle(p)
    R = p["R"]
    assert_close_tol(got[:R], ref, absdot, what="grouped gemm")
    assert np.all(np.isnan(got[R:])), "rows past expert_off[E] must be untouched"


def test_compensation_changes_output(cuda_lib):
    """The compensation term is really added: without it the result differs
    from the compensated one by R . Wc."""
    p = _problem([200, 90], 128, 256, 32, seed=99)
    y1 = _run_gpu(cuda_lib, p)
    p0 = dict(p, nc=0, resid=None, wc=None)
    y0 = _run_gpu(cuda_lib, p0)
    R = p["R"]
    corr = np.zeros((R, 128))
    for e in range(2):
        lo, hi = p["off"][e], p["off"][e + 1]
        corr[lo:hi] = p["resid"][lo:hi] @ p["wc"][e].T
    assert_close_tol(y1[:R] - y0[:R], corr, np.abs(y1[:R]) + np.abs(y0[:R]) + 1e-3, rel=1e-2, dot=1e-2,
                     what="compensation delta")


def test_grouped_gemm_bench_layer_shape(cuda_lib):
    """The gate/up GEMM of the 2048-token, 8-expert layer (N = 4096, K = 1024,
    32 compensation channels) in full, with the layer's routing."""
    cfg = W.MOE_T2048
    r = np.random.default_rng(7)
    l = W.router_logits(cfg.T, cfg.E, "normal", torch.Generator().manual_seed(1), "cpu").numpy()
    idx, _ = M.router_topk(l.astype(np.float64), cfg.k)
    counts = np.bincount(idx.ravel(), minlength=cfg.E).tolist()
    p = _problem(counts, 2 * cfg.F, cfg.H, cfg.n_chan, seed=5)
    got = _run_gpu(cuda_lib, p)
    ref, absdot = _oracle(p)
    assert_close_tol(got[:p["R"]], ref, absdot, what="gate/up gemm")


def _gpu_args(p, w_c, w_s, wc):
    E, N, K, cap, R = p["E"], p["N"], p["K"], p["cap"], p["R"]
    a_codes = np.zeros((cap, K // 2), np.uint8)
    a_codes[:R] = F.pack_nibbles(p["a_c"])
    a_scales = np.zeros((cap, K // 16), np.uint8)
    a_scales[:R] = p["a_s"]
    dev = "cuda"
    args = dict(
        a_codes=torch.from_numpy(a_codes).to(dev), a_scales=torch.from_numpy(F.scales_to_tiled(a_scales)).to(dev),
        g_a=torch.tensor([p["g_a"]], dtype=torch.float32, device=dev),
        w_codes=torch.from_numpy(np.ascontiguousarray(F.pack_nibbles(w_c))).to(dev),
        w_scales=torch.from_numpy(F.scales_to_tiled(w_s.reshape(E * N, K // 16))).to(dev),
        g_w=torch.tensor(p["g_w"], dtype=torch.float32, device=dev),
        expert_off=torch.from_numpy(p["off"]).to(dev), E=E, rows_cap=cap, K=K)
    if p["nc"]:
        resid = np.zeros((cap, p["nc"]))
        resid[:R] = p["resid"]
        args["a_resid"] = bf16_torch(resid)
        args["w_resid"] = bf16_torch(np.ascontiguousarray(wc))
    return args


def _swiglu_ref(p, F_):
    """The oracle's h = SwiGLU(bf16(y)) and a bound on |h_gpu - h|: the GEMM
    tolerance of y carried through SwiGLU, plus one BF16 rounding of h."""
    y_ref, absdot = _oracle(p)
    tol_y = 1e-2 * np.abs(y_ref) + 1e-3 * absdot
    g, u = y_ref[:, :F_], y_ref[:, F_:]
    sig = 1.0 / (1.0 + np.exp(-g))
    h_ref = M.swiglu(F.bf16_rne(y_ref.astype(np.float32)))
    dsilu = np.abs(sig * (1.0 + g * (1.0 - sig)))
    tol_h = dsilu * (np.abs(u) + tol_y[:, F_:]) * tol_y[:, :F_] + np.abs(g * sig) * tol_y[:, F_:] + \
        2.0 ** -7 * np.abs(h_ref) + 1e-30
    return h_ref, tol_h


@pytest.mark.parametrize("counts,F_,K,nc", [
    ([64], 64, 64, 0),                  # one tile: 64 gate + 64 up columns
    ([130, 0, 257], 128, 512, 32),      # empty expert, ragged experts
    ([500, 20, 1000, 3], 192, 1024, 64),
])
def test_grouped_gemm_swiglu_parity(cuda_lib, counts, F_, K, nc):
    """Gate/up GEMM with the SwiGLU in its epilogue, on weights in the 64-row
    interleaved gate/up order: h against the oracle's SwiGLU of the oracle's
    GEMM (tolerance propagated through SwiGLU), bit for bit against the plain
    GEMM followed by the SwiGLU kernel, and the per-expert amax exact."""
    p = _problem(counts, 2 * F_, K, nc, seed=3 * sum(counts) + F_ + K + nc)
    perm = gate_up_interleave_index(F_)
    wc_il = p["wc"][:, perm] if nc else None
    args = _gpu_args(p, p["w_c"][:, perm], p["w_s"][:, perm], wc_il)
    E, cap, R = p["E"], p["cap"], p["R"]
    h = torch.full((cap, F_), float("nan"), dtype=torch.bfloat16, device="cuda")
    h, amax = cuda_lib.moe_grouped_gemm_nvfp4_swiglu(F=F_, h=h, **args)
    torch.cuda.synchronize()
    assert cuda_lib.device_status() == cuda_lib.OK
    got = bf16_np(h)
    assert np.all(np.isnan(got[R:])), "rows past expert_off[E] must be untouched"
    # against the oracle: y within the GEMM tolerance, carried through SwiGLU
    h_ref, tol_h = _swiglu_ref(p, F_)
    err = np.abs(got[:R] - h_ref)
    assert np.all(err <= tol_h), f"{np.sum(err > tol_h)} of {err.size} h values outside the tolerance"
    # against the plain GEMM (same operands) + the SwiGLU kernel: identical bits
    y_il = torch.full((cap, 2 * F_), float("nan"), dtype=torch.bfloat16, device="cuda")
    cuda_lib.moe_grouped_gemm_nvfp4(N=2 * F_, y=y_il, **args)
    inv = np.argsort(perm)
    y_nat = y_il[:, torch.from_numpy(inv).cuda()].contiguous()
    h2, amax2 = cuda_lib.swiglu(y_nat, F_, args["expert_off"], E)
    torch.cuda.synchronize()
    assert_bits_equal(F.bf16_bits(got[:R]), F.bf16_bits(bf16_np(h2)[:R]), "fused vs separate SwiGLU")
    a = f32_of(amax)
    for e in range(E):
        lo, hi = p["off"][e], p["off"][e + 1]
        want = np.max(np.abs(got[lo:hi])) if hi > lo else 0.0
        assert a[e] == want, (e, a[e], want)
    assert_bits_equal(a.astype(np.float32), f32_of(amax2).astype(np.float32), "amax vs SwiGLU kernel")


@pytest.mark.parametrize("counts,F_,K,nc,nch,amax_scale", [
    ([64], 64, 64, 0, 0, 1.0),                 # one tile, no channels on either side
    ([130, 0, 257], 128, 512, 32, 16, 1.0),    # empty expert, ragged experts, h channels
    ([500, 20, 1000, 3], 192, 1024, 64, 32, 0.7),   # stale amax below the true max: saturating codes
    ([300, 40], 256, 256, 16, 48, 1.3),        # stale amax above it; channels in several 32-column chunks
])
def test_grouped_gemm_swiglu_quant(cuda_lib, counts, F_, K, nc, nch, amax_scale):
    """Gate/up GEMM with SwiGLU and the NVFP4 quantization of h in one
    epilogue: h, its codes, tiled scales, per-expert scales and channel
    residuals identical to the SwiGLU GEMM followed by quads_quantize_nvfp4
    with the same per-expert amax (given in advance, as delayed scaling
    does); the dequantized h against the oracle's quantization of the
    oracle's h within the GEMM tolerance carried through SwiGLU plus one
    NVFP4 step of each side."""
    p = _problem(counts, 2 * F_, K, nc, seed=5 * sum(counts) + F_ + K + nc + nch)
    perm = gate_up_interleave_index(F_)
    wc_il = p["wc"][:, perm] if nc else None
    args = _gpu_args(p, p["w_c"][:, perm], p["w_s"][:, perm], wc_il)
    E, cap, R = p["E"], p["cap"], p["R"]
    off = p["off"]
    # two-pass path: SwiGLU GEMM, then the quantizer with a given amax
    h_ref_gpu, amax_true = cuda_lib.moe_grouped_gemm_nvfp4_swiglu(F=F_, **args)
    amax_in = (amax_true * amax_scale).contiguous()
    r = np.random.default_rng(nch + F_)
    chan_h = None
    if nch:
        chan_h = torch.from_numpy(Q.pad_channels(np.sort(r.choice(F_, nch - 3, replace=False)), 16)).cuda()
    c2, s2, g2, r2 = cuda_lib.quantize_nvfp4(h_ref_gpu[:R], group_off=args["expert_off"], n_groups=E,
                                             amax_in=amax_in, scale_layout=cuda_lib.SCALES_TILED, chan=chan_h)
    # fused
    h = torch.full((cap, F_), float("nan"), dtype=torch.bfloat16, device="cuda")
    hc = torch.full((cap, F_ // 2), 0xAB, dtype=torch.uint8, device="cuda")
    c1, s1, r1, g1, amax1 = cuda_lib.moe_grouped_gemm_nvfp4_swiglu_quant(F=F_, amax_h_in=amax_in, chan_h=chan_h,
                                                                        h=h, h_codes=hc, **args)
    torch.cuda.synchronize()
    assert cuda_lib.device_status() == cuda_lib.OK
    assert_bits_equal(F.bf16_bits(bf16_np(h)[:R]), F.bf16_bits(bf16_np(h_ref_gpu)[:R]), "h")
    assert np.all(np.isnan(bf16_np(h)[R:])), "rows past expert_off[E] must be untouched"
    assert_bits_equal(u8_np(c1)[:R], u8_np(c2), "h codes")
    assert np.all(u8_np(c1)[R:] == 0xAB), "code rows past expert_off[E] must be untouched"
    nsb = cuda_lib.scales_bytes(R, F_, cuda_lib.SCALES_TILED)
    assert_bits_equal(u8_np(s1)[:nsb], u8_np(s2), "h scales")
    assert_bits_equal(f32_of(g1).astype(np.float32), f32_of(g2).astype(np.float32), "g_h")
    assert_bits_equal(f32_of(amax1).astype(np.float32), f32_of(amax_true).astype(np.float32), "amax_h_out")
    if nch:
        assert_bits_equal(F.bf16_bits(bf16_np(r1)[:R]), F.bf16_bits(bf16_np(r2)), "h residuals")
    # against the oracle: its h, quantized by its quantizer with the same amax.
    # |Q(a) - Q(b)| <= e(a) + e(b) + |a - b|, where one NVFP4 step moves a value
    # of a block with max m by at most max(S, m - 6 S) for the block scale
    # S <= m (1 + 2^-4) / 6 + g (E4M3 rounding, subnormal floor) and
    # 6 S >= min(m (1 - 2^-4), 2688 g) - 6 g (saturation at 448 when the given amax
    # is below the data's)
    h_or, tol_h = _swiglu_ref(p, F_)
    amax_or = f32_of(amax_in).astype(np.float64)
    qc, qs, qg = Q.quantize_grouped(h_or, off, amax=amax_or)
    deq_or = np.zeros_like(h_or)
    for e in range(E):
        if off[e + 1] > off[e]:
            deq_or[off[e]:off[e + 1]] = Q.dequant(qc[off[e]:off[e + 1]], qs[off[e]:off[e + 1]], qg[e])
    deq_gpu = f32_of(cuda_lib.dequant(c1, s1, cuda_lib.SCALES_TILED, g1, R, F_, group_off=args["expert_off"],
                                      n_groups=E, out_dtype=cuda_lib.OUT_F32))
    g_row = np.repeat(qg, np.diff(off))[:, None]
    m = (np.abs(h_or) + tol_h).reshape(R, F_ // 16, 16).max(axis=2)
    m = np.repeat(m, 16, axis=1)
    s_hi = m * (1 + 2.0 ** -4) / 6 + g_row
    e_step = np.maximum(s_hi, m - np.minimum(m * (1 - 2.0 ** -4), 2688.0 * g_row) + 6 * g_row)
    tol = 2 * e_step + tol_h + 1e-30
    err = np.abs(deq_gpu - deq_or)
    assert np.all(err <= tol), f"{np.sum(err > tol)} of {err.size} dequantized h values outside the tolerance"
    match = np.mean(F.unpack_nibbles(u8_np(c1)[:R]) == qc)
    assert match > 0.9, f"only {match:.3f} of the h codes match the oracle's"


@pytest.mark.parametrize("counts,N,K,nc,swiglu", [
    ([64], 128, 64, 64, False),                 # one tile, one main and one correction K block
    ([130, 0, 257], 256, 512, 128, False),      # empty expert, ragged experts, two correction blocks
    ([500, 20, 1000, 3], 384, 1024, 64, True),  # SwiGLU epilogue
    ([300, 40], 256, 320, 192, False),          # partial main stage, three correction blocks
])
def test_grouped_gemm_fp4_comp_parity(cuda_lib, counts, N, K, nc, swiglu):
    """The literal second quantization pass: residual channels and weight
    channel columns NVFP4-quantized on the device (per-expert residual scale
    from quads_moe_fp4_comp_amax) bit for bit against the oracle's operands,
    and the GEMM over the channel-extended reduction axis against the
    oracle's within the GEMM tolerance."""
    p = _problem(counts, N, K, nc, seed=7 * sum(counts) + N + K + nc)
    E, cap, R, off = p["E"], p["cap"], p["R"], p["off"]
    rc, rs, g_r, wcc, wcs, g_wc = M.fp4_compensation_operands(p["resid"], p["wc"], p["g_a"], p["g_w"], off)
    perm = gate_up_interleave_index(N // 2) if swiglu else np.arange(N)
    args = _gpu_args(p, p["w_c"][:, perm], p["w_s"][:, perm], p["wc"][:, perm])
    dev = "cuda"
    # device operand path
    wc_dev = args["w_resid"].reshape(E * N, nc)
    wcc_d, wcs_d, g_wc_d, _ = cuda_lib.quantize_nvfp4(wc_dev, n_groups=E, scale_layout=cuda_lib.SCALES_TILED)
    amax_r = cuda_lib.moe_fp4_comp_amax(args["g_a"], args["g_w"], g_wc_d, E)
    ra = torch.zeros((cap, nc), dtype=torch.bfloat16, device=dev)
    ra[:R] = bf16_torch(p["resid"])
    rc_d = torch.full((cap, nc // 2), 0, dtype=torch.uint8, device=dev)
    rs_d = torch.zeros(cuda_lib.scales_bytes(cap, nc, cuda_lib.SCALES_TILED), dtype=torch.uint8, device=dev)
    _, _, g_r_d, _ = cuda_lib.quantize_nvfp4(ra, group_off=args["expert_off"], n_groups=E, amax_in=amax_r,
                                             scale_layout=cuda_lib.SCALES_TILED, codes=rc_d, scales=rs_d)
    torch.cuda.synchronize()
    assert_bits_equal(f32_of(g_wc_d).astype(np.float32), g_wc.astype(np.float32), "g_wc")
    assert_bits_equal(f32_of(amax_r).astype(np.float32), M.fp4_comp_amax(p["g_a"], p["g_w"], g_wc).astype(np.float32),
                      "amax_r")
    assert_bits_equal(f32_of(g_r_d).astype(np.float32), g_r.astype(np.float32), "g_r")
    assert_bits_equal(u8_np(rc_d)[:R], F.pack_nibbles(rc), "residual codes")
    assert_bits_equal(F.scales_from_tiled(u8_np(rs_d), cap, nc // 16)[:R], rs, "residual scales")
    assert_bits_equal(u8_np(wcc_d).reshape(E, N, nc // 2), F.pack_nibbles(wcc[:, perm]), "weight-column codes")
    # the GEMM
    if swiglu:
        h, amax = cuda_lib.moe_grouped_gemm_nvfp4_fp4comp(
            args["a_codes"], args["a_scales"], args["g_a"], args["w_codes"], args["w_scales"], args["g_w"],
            args["expert_off"], E, cap, N, K, rc_d, rs_d, wcc_d, wcs_d, nc, swiglu=True)
    else:
        y = torch.full((cap, N), float("nan"), dtype=torch.bfloat16, device=dev)
        cuda_lib.moe_grouped_gemm_nvfp4_fp4comp(
            args["a_codes"], args["a_scales"], args["g_a"], args["w_codes"], args["w_scales"], args["g_w"],
            args["expert_off"], E, cap, N, K, rc_d, rs_d, wcc_d, wcs_d, nc, y=y)
    torch.cuda.synchronize()
    assert cuda_lib.device_status() == cuda_lib.OK
    ref, absdot = M.grouped_gemm_fp4_comp(p["a_c"], p["a_s"], p["g_a"], p["w_c"], p["w_s"], p["g_w"], off, rc, rs,
                                          wcc, wcs)
    if not swiglu:
        got = bf16_np(y)
        assert_close_tol(got[:R], ref, absdot, what="grouped gemm with FP4 correction")
        assert np.all(np.isnan(got[R:]))
    else:
        F_ = N // 2
        tol_y = 1e-2 * np.abs(ref) + 1e-3 * absdot
        g, u = ref[:, :F_], ref[:, F_:]
        sig = 1.0 / (1.0 + np.exp(-g))
        h_ref = M.swiglu(F.bf16_rne(ref.astype(np.float32)))
        dsilu = np.abs(sig * (1.0 + g * (1.0 - sig)))
        tol_h = dsilu * (np.abs(u) + tol_y[:, F_:]) * tol_y[:, :F_] + np.abs(g * sig) * tol_y[:, F_:] + \
            2.0 ** -7 * np.abs(h_ref) + 1e-30
        err = np.abs(bf16_np(h)[:R] - h_ref)
        assert np.all(err <= tol_h), f"{np.sum(err > tol_h)} of {err.size} h values outside the tolerance"


def _w4a16_problem(counts, N, K, seed):
    r = np.random.default_rng(seed)
    E = len(counts)
    padded = [-(-c // 128) * 128 for c in counts]
    off = np.concatenate([[0], np.cumsum(padded)]).astype(np.int32)
    R = int(off[-1])
    cap = R + 128
    x = np.zeros((cap, K))
    for e in range(E):
        x[off[e]:off[e] + counts[e]] = r.standard_normal((counts[e], K))
    x = F.bf16_rne(x.astype(np.float32))
    w = F.bf16_rne((r.standard_normal((E, N, K)) * 0.02).astype(np.float32))
    wq = [Q.quantize(w[e]) for e in range(E)]
    return dict(E=E, N=N, K=K, off=off, R=R, cap=cap, x=x, w=w, w_c=np.stack([q[0] for q in wq]),
                w_s=np.stack([q[1] for q in wq]), g_w=np.array([q[2] for q in wq]))


@pytest.mark.parametrize("counts,N,K", [
    ([64], 128, 64),                   # one tile, one stage
    ([130, 0, 257], 256, 512),         # empty expert, ragged experts
    ([500, 20, 1000, 3], 384, 1024),
    ([256], 128, 4096),                # long K
    ([300, 0, 40], 512, 256),          # 256-row weight tiles, an empty expert
    ([129], 256, 1024),                # 256-row weight tiles, one expert
])
def test_grouped_gemm_w4a16_parity(cuda_lib, counts, N, K):
    """The trainer-side W4A16 GEMM (BF16 activations, NVFP4 weights
    dequantized on chip) against the oracle within the GEMM tolerance, and
    against a plain PyTorch FP32 matmul of x with the device fake-quant's
    W_fq; rows past expert_off[E] untouched."""
    p = _w4a16_problem(counts, N, K, seed=sum(counts) + N + K)
    E, cap, R, off = p["E"], p["cap"], p["R"], p["off"]
    dev = "cuda"
    w_codes = torch.from_numpy(np.ascontiguousarray(F.pack_nibbles(p["w_c"]))).to(dev)
    w_scales = torch.from_numpy(F.scales_to_tiled(p["w_s"].reshape(E * N, K // 16))).to(dev)
    g_w = torch.tensor(p["g_w"], dtype=torch.float32, device=dev)
    x = bf16_torch(p["x"])
    y = torch.full((cap, N), float("nan"), dtype=torch.bfloat16, device=dev)
    cuda_lib.moe_grouped_gemm_w4a16(x, w_codes, w_scales, g_w, torch.from_numpy(off).to(dev), E, cap, N, K, y=y)
    torch.cuda.synchronize()
    assert cuda_lib.device_status() == cuda_lib.OK
    got = bf16_np(y)
    ref, absdot = M.grouped_gemm_w4a16(p["x"][:R], p["w_c"], p["w_s"], p["g_w"], off)
    assert_close_tol(got[:R], ref, absdot, what="W4A16 GEMM")
    assert np.all(np.isnan(got[R:]))
    # against PyTorch: the device fake-quant's W_fq, FP32 matmul, BF16 rounding
    w_fq = cuda_lib.fakequant_weight_ste(bf16_torch(p["w"]), want_codes=False)[0]
    for e in range(E):
        lo, hi = int(off[e]), int(off[e + 1])
        if hi == lo:
            continue
        yt = torch.matmul(x[lo:hi].float(), w_fq[e].float().t())
        err = (y[lo:hi].float() - yt).abs()
        bound = 2.0 ** -8 * yt.abs() + K * 2.0 ** -22 * torch.matmul(x[lo:hi].float().abs(), w_fq[e].float().abs().t())
        assert bool((err <= bound).all()), f"expert {e}: {int((err > bound).sum())} outside the FP32 bound"


@pytest.mark.parametrize("shape", [0, 1])
@pytest.mark.parametrize("counts,N,K,swiglu", [([300, 0, 40, 700], 512, 384, False), ([257, 1, 600], 768, 256, True)])
def test_grouped_gemm_w4a16_both_kernels(cuda_lib, shape, counts, N, K, swiglu):
    """Where N % 256 == 0 the W4A16 GEMM takes the weights-as-M kernel (W_fq
    converted into tensor memory, 128 weight rows by 256 rows per unit);
    tile shape 0 keeps the 128 x N kernel.  Both against the oracle."""
    prev = cuda_lib.gemm_set_tile_shape(shape)
    try:
        p = _w4a16_problem(counts, N, K, seed=3 * sum(counts) + N + K + shape)
        E, cap, R, off = p["E"], p["cap"], p["R"], p["off"]
        dev = "cuda"
        perm = gate_up_interleave_index(N // 2) if swiglu else np.arange(N)
        w_codes = torch.from_numpy(np.ascontiguousarray(F.pack_nibbles(p["w_c"][:, perm]))).to(dev)
        w_scales = torch.from_numpy(F.scales_to_tiled(p["w_s"][:, perm].reshape(E * N, K // 16))).to(dev)
        g_w = torch.tensor(p["g_w"], dtype=torch.float32, device=dev)
        x = bf16_torch(p["x"])
        offt = torch.from_numpy(off).to(dev)
        ref, absdot = M.grouped_gemm_w4a16(p["x"][:R], p["w_c"], p["w_s"], p["g_w"], off)
        if not swiglu:
            y = torch.full((cap, N), float("nan"), dtype=torch.bfloat16, device=dev)
            cuda_lib.moe_grouped_gemm_w4a16(x, w_codes, w_scales, g_w, offt, E, cap, N, K, y=y)
            torch.cuda.synchronize()
            assert cuda_lib.device_status() == cuda_lib.OK
            got = bf16_np(y)
            assert_close_tol(got[:R], ref, absdot, what=f"W4A16 GEMM (tile shape {shape})")
            assert np.all(np.isnan(got[R:]))
        else:
            h, amax = cuda_lib.moe_grouped_gemm_w4a16(x, w_codes, w_scales, g_w, offt, E, cap, N, K, swiglu=True)
            torch.cuda.synchronize()
            assert cuda_lib.device_status() == cuda_lib.OK
            F_ = N // 2
            h_ref, tol = swiglu_carried(ref, absdot, F_)
            got = bf16_np(h)[:R]
            err = np.abs(got - h_ref)
            assert np.all(err <= tol), f"{int(np.sum(err > tol))} h values outside the tolerance"
            a = f32_of(amax)
            for e in range(E):
                lo, hi = off[e], off[e + 1]
                assert a[e] == (np.max(np.abs(got[lo:hi])) if hi > lo else 0.0), e
    finally:
        cuda_lib.gemm_set_tile_shape(prev)


@pytest.mark.parametrize("counts,F_,K", [([64], 64, 64), ([500, 20, 1000, 3], 192, 1024),
                                         ([200, 0, 70], 256, 512), ([130], 128, 64)])
def test_grouped_gemm_w4a16_swiglu(cuda_lib, counts, F_, K):
    """The W4A16 GEMM with the SwiGLU epilogue on 64-row interleaved gate/up
    weights, bit for bit against the plain W4A16 GEMM followed by the SwiGLU
    kernel."""
    p = _w4a16_problem(counts, 2 * F_, K, seed=11 * sum(counts) + F_ + K)
    E, cap, R, off, N = p["E"], p["cap"], p["R"], p["off"], 2 * F_
    perm = gate_up_interleave_index(F_)
    dev = "cuda"
    w_codes = torch.from_numpy(np.ascontiguousarray(F.pack_nibbles(p["w_c"][:, perm]))).to(dev)
    w_scales = torch.from_numpy(F.scales_to_tiled(p["w_s"][:, perm].reshape(E * N, K // 16))).to(dev)
    g_w = torch.tensor(p["g_w"], dtype=torch.float32, device=dev)
    x = bf16_torch(p["x"])
    offt = torch.from_numpy(off).to(dev)
    h, amax = cuda_lib.moe_grouped_gemm_w4a16(x, w_codes, w_scales, g_w, offt, E, cap, N, K, swiglu=True)
    y_il = cuda_lib.moe_grouped_gemm_w4a16(x, w_codes, w_scales, g_w, offt, E, cap, N, K)
    y_nat = y_il[:, torch.from_numpy(np.argsort(perm)).cuda()].contiguous()
    h2, amax2 = cuda_lib.swiglu(y_nat, F_, offt, E)
    torch.cuda.synchronize()
    assert cuda_lib.device_status() == cuda_lib.OK
    assert_bits_equal(F.bf16_bits(bf16_np(h)[:R]), F.bf16_bits(bf16_np(h2)[:R]), "fused vs separate SwiGLU")
    assert_bits_equal(f32_of(amax).astype(np.float32), f32_of(amax2).astype(np.float32), "amax")
