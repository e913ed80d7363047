"""One full step of the 2048-token, 8-expert layer (hidden 1024, ffn 2048,
32 + 32 compensation channels) on the GPU against the oracle on the same
seeded inputs, stage by stage.

Bit-exact: input quantization, residuals, routing, permutation, weight
fake-quant / rollout weights / compensation columns, replayed operand and
mismatch counts.  Float, on every element: the gate/up GEMM within the
tolerance, and each later stage against the oracle fed the GPU's output of
the stage before it: SwiGLU of the GPU's gate/up output, the NVFP4
quantization of the GPU's h (bit-exact), the down GEMM on the GPU's
quantized h, the combine of the GPU's down output.  Where h comes out of the
gate/up GEMM's epilogue (y is never stored) h is checked against the
oracle's own GEMM with the tolerance carried through SwiGLU."""
import numpy as np
import pytest
import torch

from oracle import formats as F
from oracle import layer as OL
from oracle import moe as M
from oracle import nvfp4 as Q
from tests.helpers import (assert_bits_equal, assert_close_tol, bf16_np, f32_of, gate_up_interleave_index,
                           swiglu_carried, u8_np, unpack_codes)
from train_alignment_b200 import layer as L
from train_alignment_b200 import workloads as W

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", params=[True, False], ids=["fused_swiglu", "separate_swiglu"])
def run(cuda_lib, request):
    cfg = W.MOE_T2048
    inp = W.moe_layer_inputs(cfg, seed=0, device="cpu")
    r = np.random.default_rng(0)
    chan_x = Q.pad_channels(np.sort(r.choice(cfg.H, cfg.n_chan - 3, replace=False)))
    chan_h = Q.pad_channels(np.sort(r.choice(cfg.F, cfg.n_chan_f - 7, replace=False)))
    x_train = W.engine_drift(inp["x"], 1e-2, seed=0)
    dev = "cuda"
    layer = L.MoELayer(cfg, inp["w_gu"].to(dev), inp["w_d"].to(dev), torch.from_numpy(chan_x),
                       torch.from_numpy(chan_h), dev, fuse_swiglu=request.param)
    _, g_gu, g_d = layer.grad_fq_buffers()
    g_gu.copy_(W.random_bf16(layer.w_gu.shape, 1, 1e-3, dev))
    g_d.copy_(W.random_bf16(layer.w_d.shape, 2, 1e-3, dev))
    layer.reset_counts()
    layer.step(inp["x"].to(dev), inp["logits"].to(dev), x_train.to(dev), g_gu, g_d)
    assert cuda_lib.device_status() == cuda_lib.OK
    torch.cuda.synchronize()
    ref = OL.step(bf16_np(inp["x"]), inp["logits"].numpy().astype(np.float64), bf16_np(x_train),
                  bf16_np(inp["w_gu"]), bf16_np(inp["w_d"]), chan_x, chan_h, cfg.k,
                  grad_gu_fq=bf16_np(g_gu), grad_gu=np.zeros(tuple(layer.w_gu.shape)))
    ref["grad_d"] = bf16_np(g_d)          # accumulated onto a zero master gradient: itself
    return cfg, layer, ref


def test_weights(run):
    cfg, layer, ref = run
    E, F2, H = cfg.E, 2 * cfg.F, cfg.H
    # the rollout's gate/up weights are in the interleaved order when SwiGLU is fused
    perm = gate_up_interleave_index(cfg.F) if layer.fuse_swiglu else np.arange(F2)
    assert_bits_equal(unpack_codes(layer.w_gu_codes), ref["wgu"]["codes"][:, perm], "w_gu codes")
    s = F.scales_from_tiled(u8_np(layer.w_gu_scales), E * F2, H // 16).reshape(E, F2, H // 16)
    assert_bits_equal(s, ref["wgu"]["scales"][:, perm], "w_gu scales")
    assert_bits_equal(f32_of(layer.g_w_gu).astype(np.float32), ref["wgu"]["g"].astype(np.float32), "g_w")
    assert_bits_equal(F.bf16_bits(bf16_np(layer.w_gu_fq)), F.bf16_bits(ref["wgu"]["w_fq"]), "w_gu_fq")
    assert_bits_equal(F.bf16_bits(bf16_np(layer.wc_gu)), F.bf16_bits(ref["wgu"]["wc"][:, perm]), "wc_gu")
    assert_bits_equal(unpack_codes(layer.w_d_codes), ref["wd"]["codes"], "w_d codes")
    assert_bits_equal(F.bf16_bits(bf16_np(layer.wc_d)), F.bf16_bits(ref["wd"]["wc"]), "wc_d")


def test_rollout_input_and_routing(run):
    cfg, layer, ref = run
    f = ref["fwd"]
    assert_bits_equal(unpack_codes(layer.x_codes), f["cx"], "x codes")
    assert_bits_equal(u8_np(layer.x_scales).reshape(cfg.T, cfg.H // 16), f["sx"], "x scales")
    assert np.float32(f32_of(layer.g_x)[0]) == np.float32(f["gx"])
    assert_bits_equal(F.bf16_bits(bf16_np(layer.x_resid)), F.bf16_bits(f["rx"]), "x resid")
    assert_bits_equal(f32_of(layer.topk_idx).astype(np.int64), f["idx"].astype(np.int64), "topk idx")
    assert np.allclose(f32_of(layer.topk_w), f["w"], rtol=2e-6)
    assert_bits_equal(f32_of(layer.expert_off).astype(np.int64), f["off"].astype(np.int64), "expert_off")
    assert_bits_equal(f32_of(layer.row_of).astype(np.int64), f["row_of"].astype(np.int64), "row_of")


def test_gate_up_gemm(run):
    cfg, layer, ref = run
    if layer.fuse_swiglu:
        pytest.skip("y is not stored when SwiGLU runs in the GEMM epilogue (h is checked instead)")
    f = ref["fwd"]
    n = int(f["off"][-1])
    assert_close_tol(bf16_np(layer.y_gu)[:n], f["y1"], f["absdot1"], what="gate/up GEMM")


def test_h(run):
    """SwiGLU: against the oracle's SwiGLU of the GPU's stored gate/up output
    (separate pass), or of the oracle's own gate/up output with the GEMM
    tolerance carried through (fused epilogue); every element."""
    cfg, layer, ref = run
    f = ref["fwd"]
    n = int(f["off"][-1])
    h = bf16_np(layer.h)[:n]
    if layer.fuse_swiglu:
        h_ref, tol = swiglu_carried(f["y1"], f["absdot1"], cfg.F)
    else:
        y = bf16_np(layer.y_gu)[:n]
        h_ref = M.swiglu(y)
        tol = 1e-2 * np.abs(h_ref) + 1e-3 * np.abs(y[:, :cfg.F] / (1.0 + np.exp(-y[:, :cfg.F])) * y[:, cfg.F:])
    err = np.abs(h - h_ref)
    assert np.all(err <= tol), f"{np.sum(err > tol)} of {err.size} h values outside the tolerance"


def _gpu_quantized_h(layer, cfg, n):
    """The GPU's NVFP4 h of rows [0, n): codes, linear scales, per-expert
    scale, channel residuals."""
    codes = unpack_codes(layer.h_codes)[:n]
    scales = F.scales_from_tiled(u8_np(layer.h_scales), n, cfg.F // 16)
    resid = bf16_np(layer.h_resid)[:n]
    return codes, scales, f32_of(layer.g_h).astype(np.float32).astype(np.float64), resid


def test_h_quantization(run):
    """The oracle's per-expert NVFP4 quantization of the GPU's h (amax of each
    expert's rows, codes, scales, residuals on the ffn channel set): bit for
    bit."""
    cfg, layer, ref = run
    f = ref["fwd"]
    n = int(f["off"][-1])
    h = bf16_np(layer.h)[:n]
    codes, scales, g_h, resid = _gpu_quantized_h(layer, cfg, n)
    c_ref, s_ref, g_ref = Q.quantize_grouped(h, f["off"])
    assert_bits_equal(g_h.astype(np.float32), g_ref.astype(np.float32), "g_h")
    assert_bits_equal(codes, c_ref, "h codes")
    assert_bits_equal(scales, s_ref, "h scales")
    chan_h = f32_of(layer.chan_h).astype(np.int64)
    r_ref = np.zeros_like(resid)
    for e in range(cfg.E):
        lo, hi = int(f["off"][e]), int(f["off"][e + 1])
        if hi > lo:
            r_ref[lo:hi] = Q.residual_channels(h[lo:hi], c_ref[lo:hi], s_ref[lo:hi], g_ref[e], chan_h)
    assert_bits_equal(F.bf16_bits(resid), F.bf16_bits(r_ref), "h residuals")


def test_down_gemm(run):
    """The oracle's down GEMM fed the GPU's quantized h: every element within
    the tolerance."""
    cfg, layer, ref = run
    f = ref["fwd"]
    n = int(f["off"][-1])
    codes, scales, g_h, resid = _gpu_quantized_h(layer, cfg, n)
    wd = ref["wd"]
    y2, absdot2 = M.grouped_gemm(codes, scales, g_h, wd["codes"], wd["scales"], wd["g"], f["off"], resid, wd["wc"])
    assert_close_tol(bf16_np(layer.y_d)[:n], y2, absdot2, what="down GEMM")


def test_combine(run):
    """The oracle's combine of the GPU's down output with the GPU's routing
    weights: every element within the tolerance (sum |w y| as the scale)."""
    cfg, layer, ref = run
    y = bf16_np(layer.y_d)
    w = f32_of(layer.topk_w)
    row_of = f32_of(layer.row_of).astype(np.int64)
    out_ref = M.combine(y, row_of, w, cfg.k)
    rows = row_of.reshape(cfg.T, cfg.k)
    absdot = sum(np.abs(w[:, s:s + 1] * y[rows[:, s]]) for s in range(cfg.k))
    assert_close_tol(bf16_np(layer.out), out_ref, absdot, what="combine")


def test_output_against_oracle_end_to_end(run):
    """Report: the layer output against the oracle's own end-to-end result.
    Past the first BF16 GEMM output the two can round an intermediate to
    neighbouring values, which can flip an NVFP4 code of h; the flip rate is
    printed, and the outputs must agree in norm."""
    cfg, layer, ref = run
    f = ref["fwd"]
    n = int(f["off"][-1])
    flips = np.mean(unpack_codes(layer.h_codes)[:n] != f["ch"])
    out = bf16_np(layer.out)
    rel = np.linalg.norm(out - f["out"]) / np.linalg.norm(f["out"])
    print(f"h code flips against the oracle's own h: {flips:.2e}; output relative distance {rel:.2e}")
    assert rel < 1e-2, rel


def test_replay(run):
    cfg, layer, ref = run
    assert int(layer.status.item()) == 0 and int(layer.status_h.item()) == 0
    assert_bits_equal(F.bf16_bits(bf16_np(layer.x_hat)), F.bf16_bits(ref["x_hat"]), "x_hat")
    assert f32_of(layer.counts).astype(np.int64).tolist() == [ref["code_mismatches"], ref["scale_mismatches"]]


def test_ste(run):
    cfg, layer, ref = run
    assert_bits_equal(F.bf16_bits(bf16_np(layer.grad_gu)), F.bf16_bits(ref["grad"]), "grad_gu")
    assert_bits_equal(F.bf16_bits(bf16_np(layer.grad_d)), F.bf16_bits(ref["grad_d"]), "grad_d")


def test_fused_requant_layer_matches_two_pass(cuda_lib):
    """The layer with h's NVFP4 quantization in the gate/up GEMM epilogue
    (delayed scaling: the per-expert scale comes from the amax held from the
    step before) against the two-pass layer, on the same batch twice.  With
    the held amax equal to this batch's own, the fused layer's h codes,
    scales, residuals, per-expert scales, TRACE record and output are the
    two-pass layer's, bit for bit; its amax_h is this step's exact amax."""
    cfg = W.MOE_T2048
    inp = W.moe_layer_inputs(cfg, seed=1, device="cpu")
    r = np.random.default_rng(1)
    chan_x = torch.from_numpy(Q.pad_channels(np.sort(r.choice(cfg.H, cfg.n_chan - 3, replace=False))))
    chan_h = torch.from_numpy(Q.pad_channels(np.sort(r.choice(cfg.F, cfg.n_chan_f - 7, replace=False))))
    dev = "cuda"
    x, logits = inp["x"].to(dev), inp["logits"].to(dev)
    x_train = W.engine_drift(inp["x"], 1e-2, seed=1).to(dev)
    two = L.MoELayer(cfg, inp["w_gu"].to(dev), inp["w_d"].to(dev), chan_x, chan_h, dev)
    _, g_gu, g_d = two.grad_fq_buffers()
    g_gu.zero_()
    g_d.zero_()
    two.reset_counts()
    two.step(x, logits, x_train, g_gu, g_d)
    torch.cuda.synchronize()
    fused = L.MoELayer(cfg, inp["w_gu"].to(dev), inp["w_d"].to(dev), chan_x, chan_h, dev, fuse_requant=True,
                       amax_h_init=two.amax_h.clone())
    for step in range(2):
        fused.reset_counts()
        fused.step(x, logits, x_train, g_gu, g_d)
        torch.cuda.synchronize()
        assert cuda_lib.device_status() == cuda_lib.OK
        R = int(two.expert_off[-1].item())
        assert_bits_equal(u8_np(fused.h_codes)[:R], u8_np(two.h_codes)[:R], f"h codes, step {step}")
        nsb = cuda_lib.scales_bytes(R, cfg.F, cuda_lib.SCALES_TILED)
        assert_bits_equal(u8_np(fused.h_scales)[:nsb], u8_np(two.h_scales)[:nsb], f"h scales, step {step}")
        assert_bits_equal(F.bf16_bits(bf16_np(fused.h_resid)[:R]), F.bf16_bits(bf16_np(two.h_resid)[:R]),
                          f"h residuals, step {step}")
        assert_bits_equal(f32_of(fused.g_h).astype(np.float32), f32_of(two.g_h).astype(np.float32), "g_h")
        assert_bits_equal(f32_of(fused.amax_h).astype(np.float32), f32_of(two.amax_h).astype(np.float32), "amax_h")
        assert_bits_equal(F.bf16_bits(bf16_np(fused.out)), F.bf16_bits(bf16_np(two.out)), f"output, step {step}")
        assert_bits_equal(u8_np(fused.record), u8_np(two.record), f"TRACE record, step {step}")
        assert_bits_equal(f32_of(fused.counts).astype(np.int64), f32_of(two.counts).astype(np.int64), "counts")


def test_fp4_compensation_layer(cuda_lib):
    """The layer with the literal second quantization pass (residual and
    weight channel columns NVFP4-quantized, one FP4 product) next to the
    BF16-compensated layer and an uncompensated one, on the same batch: the
    FP4 correction keeps the output close to the BF16-corrected one and
    removes most of the uncompensated layer's distance to it."""
    cfg = W.MOE_T2048
    inp = W.moe_layer_inputs(cfg, seed=2, device="cpu")
    dev = "cuda"
    x, logits = inp["x"].to(dev), inp["logits"].to(dev)
    chan_x = L.calibrate_channels(x, cfg.n_chan)
    r = np.random.default_rng(2)
    chan_h = torch.from_numpy(Q.pad_channels(np.sort(r.choice(cfg.F, cfg.n_chan_f - 7, replace=False)))).to(dev)
    none = torch.full((16,), -1, dtype=torch.int32, device=dev)
    outs = {}
    for name, cx, ch, comp in [("bf16", chan_x, chan_h, "bf16"), ("fp4", chan_x, chan_h, "fp4"),
                               ("none", none, none, "bf16")]:
        layer = L.MoELayer(cfg, inp["w_gu"].to(dev), inp["w_d"].to(dev), cx, ch, dev, comp=comp)
        layer.weight_sync()
        outs[name] = layer.rollout_forward(x, logits).float().clone()
        torch.cuda.synchronize()
        assert cuda_lib.device_status() == cuda_lib.OK
        if comp == "fp4":
            assert layer.nc_x % 64 == 0 and layer.nc_h % 64 == 0
        del layer
    ref = outs["bf16"]
    d_fp4 = torch.linalg.vector_norm(outs["fp4"] - ref, dim=1) / torch.linalg.vector_norm(ref, dim=1)
    d_none = torch.linalg.vector_norm(outs["none"] - ref, dim=1) / torch.linalg.vector_norm(ref, dim=1)
    print(f"distance to the BF16-compensated output: FP4 correction median {d_fp4.median():.4f}, "
          f"none {d_none.median():.4f}")
    assert torch.isfinite(outs["fp4"]).all()
    assert d_fp4.median() < 0.5 * d_none.median()
