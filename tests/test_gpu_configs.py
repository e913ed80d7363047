"""Each further layer configuration at its full size, in the launch
configuration the benchmark times (MoELayer.step, two streams, fused SwiGLU),
against the oracle.

Exact at full size, where the oracle computes everything quickly:
  - the per-tensor scale of X;
  - the routing and the permutation;
  - the mismatch count of the replay, for the decode shapes.
Sampled, with each sampled item computed by the oracle on its own:
  - X codes, scales and residuals of sampled rows;
  - the weights of two sampled experts (codes, scales, scale, W_fq, Wc);
  - every row of the busiest expert, stage by stage: the gate/up GEMM and
    SwiGLU against the oracle's (GEMM tolerance carried through SwiGLU, every
    element); the oracle's quantization of the GPU's h (the expert's scale,
    codes, scales and residuals, bit for bit); the oracle's down GEMM on the
    GPU's quantized h (every element within the tolerance);
  - the replayed X rows.
Property at full size: combine (out = sum_s w y_down[row_of]) on sampled
tokens, using the GPU's own tensors on both sides.

The 2048-token layer is covered in full by test_gpu_layer.py."""
import numpy as np
import pytest
import torch

from oracle import formats as F
from oracle import moe as M
from oracle import nvfp4 as Q
from oracle import trace as TR
from tests.helpers import (assert_bits_equal, assert_close_tol, bf16_np, f32_of, gate_up_interleave_index,
                           swiglu_carried, u8_np, unpack_codes)
from train_alignment_b200 import layer as L
from train_alignment_b200 import workloads as W

pytestmark = pytest.mark.gpu

NAMES = ["decode_t64_h2048_e128k8_f768", "decode_t512_h2048_e128k8_f768", "decode_t4096_h2048_e128k8_f768",
         "prefill_t16384_h4096_e128k8_f1536"]


@pytest.fixture(scope="module", params=NAMES)
def stepped(cuda_lib, request):
    cfg = W.CONFIGS[request.param]
    dev = "cuda"
    inp = W.moe_layer_inputs(cfg, seed=3, device=dev)
    layer = L.build_layer(cfg, inp, dev)
    x_train = W.engine_drift(inp["x"], 1e-2, seed=3, device=dev)
    _, g_gu, g_d = layer.grad_fq_buffers()
    g_gu.copy_(W.random_bf16(layer.w_gu.shape, 5, 1e-3, dev))
    g_d.copy_(W.random_bf16(layer.w_d.shape, 6, 1e-3, dev))
    layer.reset_counts()
    layer.step(inp["x"], inp["logits"], x_train, g_gu, g_d)
    torch.cuda.synchronize()
    assert cuda_lib.device_status() == cuda_lib.OK
    yield cfg, layer, inp, x_train, g_d
    del layer
    torch.cuda.empty_cache()


def _rows(n, count, seed):
    r = np.random.default_rng(seed)
    return np.unique(np.concatenate([[0, n - 1], r.choice(n, min(count, n), replace=False)]))


def test_input_quantization_routing_permutation(stepped):
    cfg, layer, inp, _, _ = stepped
    x = bf16_np(inp["x"])
    amax = float(np.max(np.abs(x)))
    gx = Q.tensor_scale(amax)
    assert np.float32(f32_of(layer.g_x)[0]) == np.float32(gx)
    rows = _rows(cfg.T, 24, 1)
    c_ref, s_ref = Q.quantize_with_scale(x[rows], gx)
    assert_bits_equal(unpack_codes(layer.x_codes)[rows], c_ref, "x codes")
    assert_bits_equal(u8_np(layer.x_scales).reshape(cfg.T, cfg.H // 16)[rows], s_ref, "x scales")
    chan_x = f32_of(layer.chan_x).astype(np.int64)
    r_ref = Q.residual_channels(x[rows], c_ref, s_ref, gx, chan_x)
    assert_bits_equal(F.bf16_bits(bf16_np(layer.x_resid)[rows]), F.bf16_bits(r_ref), "x resid")
    idx_ref, w_ref = M.router_topk(inp["logits"].cpu().numpy().astype(np.float64), cfg.k)
    assert_bits_equal(f32_of(layer.topk_idx).astype(np.int64), idx_ref.astype(np.int64), "topk idx")
    assert np.allclose(f32_of(layer.topk_w), w_ref, rtol=2e-6, atol=1e-7)
    off_ref, row_ref, src_ref = M.permute(idx_ref, cfg.E)
    assert_bits_equal(f32_of(layer.expert_off).astype(np.int64), off_ref.astype(np.int64), "expert_off")
    assert_bits_equal(f32_of(layer.row_of).astype(np.int64), row_ref.astype(np.int64), "row_of")
    n = int(off_ref[-1])
    assert_bits_equal(f32_of(layer.src_of)[:n].astype(np.int64), src_ref.astype(np.int64), "src_of")


def _expert_weights(layer, inp, e, F_):
    """The oracle's weight sync of expert e (gate/up and down) from the inputs."""
    wgu = bf16_np(inp["w_gu"][e])
    wd = bf16_np(inp["w_d"][e])
    chan_x = f32_of(layer.chan_x).astype(np.int64)
    chan_h = f32_of(layer.chan_h).astype(np.int64)
    out = {}
    for name, w, chan in (("gu", wgu, chan_x), ("d", wd, chan_h)):
        w_fq, c, s, g = Q.fakequant_weight(w, fold_global=True)
        wc = np.zeros((w.shape[0], len(chan)))
        ok = chan >= 0
        wc[:, ok] = w_fq[:, chan[ok]]
        out[name] = dict(w_fq=w_fq, codes=c, scales=s, g=g, wc=wc)
    return out


def _busiest_expert(layer):
    off = f32_of(layer.expert_off).astype(np.int64)
    return int(np.argmax(np.diff(off))), off


def test_weights_of_sampled_experts(stepped):
    cfg, layer, inp, _, _ = stepped
    e_big, _ = _busiest_expert(layer)
    perm = gate_up_interleave_index(cfg.F) if layer.fuse_swiglu else np.arange(2 * cfg.F)
    for e in sorted({0, e_big}):
        ref = _expert_weights(layer, inp, e, cfg.F)
        c = unpack_codes(layer.w_gu_codes[e])
        assert_bits_equal(c, ref["gu"]["codes"][perm], f"w_gu codes[{e}]")
        # expert e's rows are whole 128-row bands of the tiled layout: a contiguous byte range
        band = cfg.H // 16 // 4 * 512 * (2 * cfg.F // 128)
        seg = u8_np(layer.w_gu_scales[e * band:(e + 1) * band])
        assert_bits_equal(F.scales_from_tiled(seg, 2 * cfg.F, cfg.H // 16), ref["gu"]["scales"][perm],
                          f"w_gu scales[{e}]")
        assert np.float32(f32_of(layer.g_w_gu)[e]) == np.float32(ref["gu"]["g"])
        assert_bits_equal(F.bf16_bits(bf16_np(layer.w_gu_fq[e])), F.bf16_bits(ref["gu"]["w_fq"]), f"w_gu_fq[{e}]")
        assert_bits_equal(F.bf16_bits(bf16_np(layer.wc_gu[e])), F.bf16_bits(ref["gu"]["wc"][perm]), f"wc_gu[{e}]")
        assert_bits_equal(unpack_codes(layer.w_d_codes[e]), ref["d"]["codes"], f"w_d codes[{e}]")
        assert np.float32(f32_of(layer.g_w_d)[e]) == np.float32(ref["d"]["g"])
        assert_bits_equal(F.bf16_bits(bf16_np(layer.wc_d[e])), F.bf16_bits(ref["d"]["wc"]), f"wc_d[{e}]")


def test_one_expert_through_both_gemms(stepped):
    """Every row of the busiest expert, each stage against the oracle fed the
    GPU's output of the stage before: gate/up GEMM + SwiGLU (from the
    layer's inputs), the expert's NVFP4 h (from the GPU's h) and the down
    GEMM (from the GPU's quantized h)."""
    cfg, layer, inp, _, _ = stepped
    e, off = _busiest_expert(layer)
    lo, hi = int(off[e]), int(off[e + 1])
    idx_ref, _ = M.router_topk(inp["logits"].cpu().numpy().astype(np.float64), cfg.k)
    off_ref, row_ref, src_ref = M.permute(idx_ref, cfg.E)
    toks = src_ref[lo:hi]
    real = toks >= 0
    lo_r, hi_r = lo, lo + int(np.sum(real))          # padding rows follow the expert's real rows
    toks = toks[real]
    x = bf16_np(inp["x"])
    gx = Q.tensor_scale(float(np.max(np.abs(x))))
    chan_x = f32_of(layer.chan_x).astype(np.int64)
    chan_h = f32_of(layer.chan_h).astype(np.int64)
    cx, sx = Q.quantize_with_scale(x[toks], gx)
    rx = Q.residual_channels(x[toks], cx, sx, gx, chan_x)
    wts = _expert_weights(layer, inp, e, cfg.F)
    one = np.array([0, len(toks)])
    gu = wts["gu"]
    y1, absdot1 = M.grouped_gemm(cx, sx, gx, gu["codes"][None], gu["scales"][None], np.array([gu["g"]]), one, rx,
                                 gu["wc"][None])
    # gate/up GEMM + SwiGLU: every element within the GEMM tolerance carried through SwiGLU
    h_ref, tol_h = swiglu_carried(y1, absdot1, cfg.F)
    h_seg = bf16_np(layer.h)[lo:hi]
    err = np.abs(h_seg[:hi_r - lo] - h_ref)
    assert np.all(err <= tol_h), f"{np.sum(err > tol_h)} of {err.size} h values outside the tolerance"
    assert np.all(h_seg[hi_r - lo:] == 0), "padding rows of h"
    # the expert's NVFP4 h, from the GPU's h: scale, codes, tiled scales, residuals bit for bit
    gh_got = float(f32_of(layer.g_h)[e])
    gh_ref = Q.tensor_scale(float(np.max(np.abs(h_seg))))
    assert np.float32(gh_got) == np.float32(gh_ref), (gh_got, gh_ref)
    ch, sh = Q.quantize_with_scale(h_seg, gh_ref)
    codes = unpack_codes(layer.h_codes)[lo:hi]
    assert_bits_equal(codes, ch, "h codes")
    band = cfg.F // 16 // 4 * 512                    # tiled-scale bytes of one 128-row band
    seg = u8_np(layer.h_scales[lo // 128 * band:hi // 128 * band])
    scales = F.scales_from_tiled(seg, hi - lo, cfg.F // 16)
    assert_bits_equal(scales, sh, "h scales")
    resid = bf16_np(layer.h_resid)[lo:hi]
    rh = Q.residual_channels(h_seg, ch, sh, gh_ref, chan_h)
    assert_bits_equal(F.bf16_bits(resid), F.bf16_bits(rh), "h residuals")
    # down GEMM on the GPU's quantized h: every element within the tolerance
    d = wts["d"]
    y2, absdot2 = M.grouped_gemm(codes, scales, gh_got, d["codes"][None], d["scales"][None], np.array([d["g"]]),
                                 np.array([0, hi - lo]), resid, d["wc"][None])
    assert_close_tol(bf16_np(layer.y_d)[lo:hi], y2, absdot2, what=f"down GEMM of expert {e}")


def test_combine_property(stepped):
    cfg, layer, _, _, _ = stepped
    toks = _rows(cfg.T, 32, 2)
    y = bf16_np(layer.y_d)
    row_of = f32_of(layer.row_of).astype(np.int64).reshape(cfg.T, cfg.k)
    w = f32_of(layer.topk_w)
    ref = np.stack([np.sum(w[t][:, None] * y[row_of[t]], axis=0) for t in toks])
    got = bf16_np(layer.out)[toks]
    absdot = np.stack([np.sum(np.abs(w[t][:, None] * y[row_of[t]]), axis=0) for t in toks])
    assert np.all(np.abs(got - ref) <= 2 ** -7 * np.abs(ref) + 1e-6 * absdot + 1e-30)


def test_replay(stepped):
    cfg, layer, inp, x_train, _ = stepped
    assert int(layer.status.item()) == 0 and int(layer.status_h.item()) == 0
    x = bf16_np(inp["x"])
    gx = Q.tensor_scale(float(np.max(np.abs(x))))
    chan_x = f32_of(layer.chan_x).astype(np.int64)
    rows = _rows(cfg.T, 24, 3)
    cx, sx = Q.quantize_with_scale(x[rows], gx)
    rx = Q.residual_channels(x[rows], cx, sx, gx, chan_x)
    rec = TR.export_tensor(cx, sx, gx, chan=chan_x, resid=rx)
    x_hat, _, _ = TR.replay_tensor(rec)
    assert_bits_equal(F.bf16_bits(bf16_np(layer.x_hat)[rows]), F.bf16_bits(x_hat), "x_hat")
    if cfg.T * cfg.H <= 1 << 23:            # the full mismatch count where the oracle is quick
        c_all, s_all = Q.quantize_with_scale(x, gx)
        r_all = Q.residual_channels(x, c_all, s_all, gx, chan_x)
        _, cm, sm = TR.replay_tensor(TR.export_tensor(c_all, s_all, gx, chan=chan_x, resid=r_all), bf16_np(x_train))
        assert f32_of(layer.counts).astype(np.int64).tolist() == [cm, sm]


def test_ste_down_gradient(stepped):
    """One step into a zero master gradient leaves the incoming gradient."""
    _, layer, _, _, g_d = stepped
    assert_bits_equal(F.bf16_bits(bf16_np(layer.grad_d)), F.bf16_bits(bf16_np(g_d)), "grad_d")
