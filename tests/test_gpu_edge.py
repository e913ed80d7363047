"""Empty and degenerate inputs on the GPU path: zero-size calls succeed and
leave their outputs untouched; a routing that sends no row to any expert runs
the grouped GEMM over zero tiles; a one-token, one-expert, top-1 layer runs
the whole step and matches the oracle's composition."""
import numpy as np
import pytest
import torch

from oracle import layer as OL
from oracle import nvfp4 as Q
from tests.helpers import assert_bits_equal, bf16_np, f32_of, unpack_codes
from train_alignment_b200 import layer as L
from train_alignment_b200 import workloads as W

pytestmark = pytest.mark.gpu


def test_zero_size_calls(cuda_lib):
    dev = "cuda"
    E, k, H = 4, 2, 64
    x = torch.empty((0, H), dtype=torch.bfloat16, device=dev)
    amax = cuda_lib.amax_bf16(x)
    one = torch.ones(1, dtype=torch.float32, device=dev)
    codes, scales, g, _ = cuda_lib.quantize_nvfp4(x, amax_in=one)
    assert codes.numel() == 0
    logits = torch.empty((0, E), dtype=torch.float32, device=dev)
    idx, w = cuda_lib.moe_router_topk(logits, k)
    off, row_of, src_of = cuda_lib.moe_permute(idx, E)
    torch.cuda.synchronize()
    assert f32_of(off).tolist() == [0] * (E + 1)
    bits = cuda_lib.trace_direction_bits(x, codes, scales, cuda_lib.SCALES_LINEAR, one)
    y = torch.empty((0, H), dtype=torch.bfloat16, device=dev)
    out = cuda_lib.moe_unpermute_combine(y, row_of, w, 0, k, H)
    torch.cuda.synchronize()
    assert cuda_lib.device_status() == cuda_lib.OK
    assert out.numel() == 0 and bits.numel() == 0 and float(amax.item()) == 0.0


def test_gemm_with_no_routed_rows(cuda_lib):
    """Every expert segment empty: the persistent grid finds zero tiles and
    writes nothing (the output keeps its NaN fill)."""
    dev = "cuda"
    E, N, K, cap = 3, 128, 128, 256
    a_codes = torch.zeros((cap, K // 2), dtype=torch.uint8, device=dev)
    a_scales = torch.zeros(cuda_lib.scales_bytes(cap, K, cuda_lib.SCALES_TILED), dtype=torch.uint8, device=dev)
    w_codes = torch.zeros((E, N, K // 2), dtype=torch.uint8, device=dev)
    w_scales = torch.zeros(cuda_lib.scales_bytes(E * N, K, cuda_lib.SCALES_TILED), dtype=torch.uint8, device=dev)
    g = torch.ones(E, dtype=torch.float32, device=dev)
    off = torch.zeros(E + 1, dtype=torch.int32, device=dev)
    y = torch.full((cap, N), float("nan"), dtype=torch.bfloat16, device=dev)
    cuda_lib.moe_grouped_gemm_nvfp4(a_codes, a_scales, g[:1], w_codes, w_scales, g, off, E, cap, N, K, y=y)
    xb = torch.zeros((cap, K), dtype=torch.bfloat16, device=dev)
    y2 = torch.full((cap, N), float("nan"), dtype=torch.bfloat16, device=dev)
    cuda_lib.moe_grouped_gemm_w4a16(xb, w_codes, w_scales, g, off, E, cap, N, K, y=y2)
    torch.cuda.synchronize()
    assert cuda_lib.device_status() == cuda_lib.OK
    assert torch.isnan(y.float()).all() and torch.isnan(y2.float()).all()


def test_one_token_one_expert_layer(cuda_lib):
    """T = 1, E = 1, k = 1, hidden 128 (the GEMM's smallest output width), ffn
    64: the whole step (weight sync,
    rollout, record, replay, STE) against the oracle: input codes, routing
    and replayed operand bit-exact, output within 2 % (L2)."""
    cfg = W.MoEConfig("tiny_t1_h128_e1k1_f64", T=1, H=128, E=1, k=1, F=64, n_chan=16, n_chan_f=16)
    inp = W.moe_layer_inputs(cfg, seed=5, device="cpu")
    r = np.random.default_rng(5)
    chan_x = Q.pad_channels(np.sort(r.choice(cfg.H, 5, replace=False)))
    chan_h = Q.pad_channels(np.sort(r.choice(cfg.F, 4, replace=False)))
    x_train = W.engine_drift(inp["x"], 1e-2, seed=5)
    dev = "cuda"
    layer = L.MoELayer(cfg, inp["w_gu"].to(dev), inp["w_d"].to(dev), torch.from_numpy(chan_x),
                       torch.from_numpy(chan_h), dev)
    _, g_gu, g_d = layer.grad_fq_buffers()
    g_gu.zero_()
    g_d.zero_()
    layer.reset_counts()
    layer.step(inp["x"].to(dev), inp["logits"].to(dev), x_train.to(dev), g_gu, g_d)
    torch.cuda.synchronize()
    assert cuda_lib.device_status() == cuda_lib.OK
    ref = OL.step(bf16_np(inp["x"]), inp["logits"].numpy().astype(np.float64), bf16_np(x_train),
                  bf16_np(inp["w_gu"]), bf16_np(inp["w_d"]), chan_x, chan_h, cfg.k)
    f = ref["fwd"]
    assert_bits_equal(unpack_codes(layer.x_codes), f["cx"], "x codes")
    assert f32_of(layer.topk_idx).astype(np.int64).tolist() == f["idx"].astype(np.int64).tolist()
    assert f32_of(layer.expert_off).astype(np.int64).tolist() == f["off"].astype(np.int64).tolist()
    assert int(layer.status.item()) == 0 and int(layer.status_h.item()) == 0
    out = bf16_np(layer.out)
    rel = np.linalg.norm(out - f["out"]) / np.linalg.norm(f["out"])
    assert rel < 2e-2, rel
