"""The operations that join layers into a stack (router projection, residual
connection) against the CPU oracle."""
import numpy as np
import pytest
import torch

from oracle import formats as F
from oracle import moe as M
from oracle import nvfp4 as Q
from oracle import stack as S
from tests.helpers import assert_bits_equal, bf16_np, bf16_torch, f32_of
from train_alignment_b200 import stack as ST
from train_alignment_b200 import workloads as W

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("T,H,E", [(1, 16, 1), (100, 2048, 64), (257, 96, 130), (4096, 2048, 64)])
def test_router_logits(cuda_lib, T, H, E):
    r = np.random.default_rng(T + H + E)
    x = F.bf16_rne(r.standard_normal((T, H)).astype(np.float32))
    w = (r.standard_normal((H, E)) / np.sqrt(H)).astype(np.float32)
    got = f32_of(cuda_lib.router_logits(bf16_torch(x), torch.from_numpy(w).cuda()))
    torch.cuda.synchronize()
    ref, absdot = S.router_logits(x, w.astype(np.float64))
    # an FP32 FMA chain over H terms: |err| <= H 2^-24 sum|x w| (plus the final rounding)
    bound = (H + 1) * 2.0 ** -24 * absdot + 1e-30
    assert np.all(np.abs(got - ref) <= bound)


@pytest.mark.parametrize("n", [8, 1000, 1 << 20])
def test_residual_add(cuda_lib, n):
    r = np.random.default_rng(n)
    x = F.bf16_rne((r.standard_normal(n) * 10.0 ** r.uniform(-3, 3, n)).astype(np.float32))
    y = F.bf16_rne((r.standard_normal(n) * 10.0 ** r.uniform(-3, 3, n)).astype(np.float32))
    xt = bf16_torch(x)
    got = cuda_lib.residual_add(xt, bf16_torch(y))
    cuda_lib.residual_add(xt, bf16_torch(y), out=xt)            # in place
    torch.cuda.synchronize()
    ref = S.residual_add(x, y)
    assert_bits_equal(F.bf16_bits(bf16_np(got)), F.bf16_bits(ref), "residual add")
    assert_bits_equal(F.bf16_bits(bf16_np(xt)), F.bf16_bits(ref), "residual add in place")


def test_stack_alignment_pass(cuda_lib):
    """The 8-layer stack (hidden 2048, 64 experts top-4, ffn 1024, 4096 tokens;
    the last 4 layers recorded and replayed): one alignment pass runs, layer
    0's routing agrees with the oracle's wherever the k-th and (k+1)-th
    logits are further apart than the logits' rounding bound, every recorded
    layer's record replays its own rollout input with zero mismatches, and
    the per-token gap between the two sides is reported (unpinned)."""
    cfg = W.CONFIGS["stack8_t4096_h2048_e64k4_f1024"]
    st = ST.LayerStack(cfg, seed=0, device="cuda")
    gap, cm, sm = st.alignment_pass(drift=1e-3)
    torch.cuda.synchronize()
    assert cuda_lib.device_status() == cuda_lib.OK
    g = gap.cpu().numpy()
    assert np.all(np.isfinite(g)) and g.shape == (cfg.T,)
    print(f"per-token gap: median {np.median(g):.4f}, p90 {np.percentile(g, 90):.4f}, max {g.max():.4f}; "
          f"replayed-layer mismatches: codes {cm}, scales {sm}")
    # layer 0 routing against the oracle's logits on the same synthetic input
    x0 = bf16_np(st.x0)
    lg, absdot = S.router_logits(x0, st.w_r[0].cpu().numpy().astype(np.float64))
    idx_ref, _ = M.router_topk(lg, cfg.k)
    bound = (cfg.H + 1) * 2.0 ** -24 * absdot
    srt = np.sort(lg, axis=1)[:, ::-1]
    b_at = np.take_along_axis(bound, np.argsort(-lg, axis=1), axis=1)
    clear = (srt[:, cfg.k - 1] - srt[:, cfg.k]) > (b_at[:, cfg.k - 1] + b_at[:, cfg.k])
    assert clear.mean() > 0.9                # the bound is a worst case; most tokens are unambiguous
    got = f32_of(st.layers[0].topk_idx).astype(np.int64)
    assert_bits_equal(got[clear], idx_ref[clear].astype(np.int64), "layer-0 routing")
    # each record replays its own rollout input exactly
    for l in range(cfg.layers - st.recorded, cfg.layers):
        layer = st.layers[l]
        layer.reset_counts()
        layer.trainer_replay(st.x_roll[l], layer_id=l)
        torch.cuda.synchronize()
        assert int(layer.status.item()) == 0
        assert f32_of(layer.counts).astype(np.int64).tolist() == [0, 0], l


@pytest.mark.parametrize("rows,K", [(2048, 1024), (77, 512), (1, 64)])
def test_activation_fakequant_matches_oracle(cuda_lib, rows, K):
    """The symmetric W4A4 trainer's activation fake-quant (one per-tensor
    scale, the device fake-quant kernel on a single matrix) against the
    oracle's, bit for bit; the straight-through backward passes the gradient
    through unchanged."""
    r = np.random.default_rng(rows + K)
    x = F.bf16_rne((r.standard_normal((rows, K)) * np.exp(r.standard_normal((1, K)))).astype(np.float32))
    xt = bf16_torch(x)
    x_fq, _, _, g, _ = cuda_lib.fakequant_weight_ste(xt.unsqueeze(0), want_codes=False)
    gy = W.random_bf16((rows, K), 3, 1.0, "cuda")
    gx = cuda_lib.fakequant_weight_ste_backward(gy)
    torch.cuda.synchronize()
    ref, _, _, g_ref = Q.fakequant_weight(x)
    assert_bits_equal(F.bf16_bits(bf16_np(x_fq[0])), F.bf16_bits(ref), "x_fq")
    assert np.float32(f32_of(g)[0]) == np.float32(g_ref)
    assert_bits_equal(F.bf16_bits(bf16_np(gx)), F.bf16_bits(bf16_np(gy)), "STE backward")


def test_stack_w4a4_trainer_gap(cuda_lib):
    """The symmetric W4A4 QAT trainer (activations fake-quantized too, no
    compensation, no replay) on the same 8-layer stack and rollout: the pass
    runs and its per-token gap is reported next to the replayed trainer's
    (a diagnostic; the pages' claim is about training, which is not run)."""
    cfg = W.CONFIGS["stack8_t4096_h2048_e64k4_f1024"]
    st = ST.LayerStack(cfg, seed=0, device="cuda")
    gap_q, _, _ = st.alignment_pass(drift=1e-3)
    gap_w4, cm, sm = st.alignment_pass(drift=1e-3, w4a4=True)
    torch.cuda.synchronize()
    assert cuda_lib.device_status() == cuda_lib.OK
    gq, gw = gap_q.cpu().numpy(), gap_w4.cpu().numpy()
    assert np.all(np.isfinite(gw)) and (cm, sm) == (0, 0)
    print(f"per-token gap, replayed trainer: median {np.median(gq):.4f}; W4A4 QAT trainer: median "
          f"{np.median(gw):.4f}, p90 {np.percentile(gw, 90):.4f}")


def test_stack_trainer_w4a16_matches_library(cuda_lib):
    """The stack's trainer side on the W4A16 kernels (NVFP4 weight codes
    dequantized on chip) against the same trainer on per-expert BF16 library
    matmuls with the stored W_fq: the two differ only in FP32 accumulation
    order and the rounding of intermediate BF16 values, so their outputs
    agree to a small relative distance per token."""
    cfg = W.CONFIGS["stack8_t4096_h2048_e64k4_f1024"]
    st = ST.LayerStack(cfg, seed=0, device="cuda")
    st.rollout(st.x0)
    x0_t = W.engine_drift(st.x0, 1e-3, seed=0, device="cuda")
    y_w4, cm, sm = st.trainer(x0_t)
    y_w4 = y_w4.float().clone()
    st.trainer_gemm = "library"
    y_lib, cm2, sm2 = st.trainer(x0_t)
    torch.cuda.synchronize()
    assert cuda_lib.device_status() == cuda_lib.OK
    # the replayed layers count the trainer's own rounding of inputs that the
    # earlier (non-replayed) layers computed, so the counts differ a little
    assert abs(cm - cm2) <= 1e-3 * max(cm, cm2) and abs(sm - sm2) <= 1e-3 * max(sm, sm2)
    d = torch.linalg.vector_norm(y_w4 - y_lib.float(), dim=1) / torch.linalg.vector_norm(y_lib.float(), dim=1)
    print(f"W4A16 vs library trainer: per-token relative distance median {d.median():.2e}, max {d.max():.2e}")
    assert d.median() < 1e-2


def test_stack_w4a4_trainer_kernels_match_library(cuda_lib):
    """The W4A4 ablation's trainer on the device kernels (fake-quant of x,
    BF16 gather, W4A16 gate/up + SwiGLU, per-expert quantize and dequantize
    of h, W4A16 down, combine) against the same trainer on per-expert BF16
    library matmuls with the stored W_fq: they differ in FP32 accumulation
    order and intermediate BF16 roundings, which can move an NVFP4 code of h,
    so their outputs agree to a small relative distance per token."""
    cfg = W.CONFIGS["stack8_t4096_h2048_e64k4_f1024"]
    st = ST.LayerStack(cfg, seed=0, device="cuda")
    st.rollout(st.x0)
    x0_t = W.engine_drift(st.x0, 1e-3, seed=0, device="cuda")
    y_k, cm, sm = st.trainer(x0_t, w4a4=True)
    y_k = y_k.float().clone()
    st.trainer_gemm = "library"
    y_lib, _, _ = st.trainer(x0_t, w4a4=True)
    torch.cuda.synchronize()
    assert cuda_lib.device_status() == cuda_lib.OK
    assert (cm, sm) == (0, 0)
    d = torch.linalg.vector_norm(y_k - y_lib.float(), dim=1) / torch.linalg.vector_norm(y_lib.float(), dim=1)
    print(f"W4A4 trainer, kernels vs library: per-token relative distance median {d.median():.2e}, "
          f"max {d.max():.2e}")
    assert d.median() < 2e-2
