"""The library's SM budget (quads_set_sm_budget): the STE backward on its
bulk-copy kernel (one CTA per budgeted SM) and the persistent grouped GEMMs
on fewer CTAs than tiles give the same bits as without a budget, and the STE
matches the oracle.  The overlapped layer step splits the GPU this way."""
import numpy as np
import pytest
import torch

from oracle import formats as F
from oracle import nvfp4 as Q
from tests.helpers import assert_bits_equal, bf16_np, bf16_torch
from tests.test_gpu_gemm import _gpu_args, _problem

pytestmark = pytest.mark.gpu


@pytest.fixture
def budget(cuda_lib):
    prev = cuda_lib.set_sm_budget(0)
    yield cuda_lib
    cuda_lib.set_sm_budget(prev)


@pytest.mark.parametrize("n,sms", [
    (5, 3),                        # the tail kernel alone
    (8 * 1000 + 5, 3),             # one partial chunk and a tail
    (8 * 2048 * 7 + 8 * 100, 3),   # several chunks per CTA, a partial last one
    (8 * 2048 * 40 + 3, 16),       # more chunks than ring stages per CTA
])
@pytest.mark.parametrize("accumulate", [False, True])
def test_ste_backward_budget(budget, n, sms, accumulate):
    lib = budget
    r = np.random.default_rng(n + sms)
    a = F.bf16_rne(r.standard_normal(n).astype(np.float32))
    b = F.bf16_rne(r.standard_normal(n).astype(np.float32))
    lib.set_sm_budget(sms)
    out = lib.fakequant_weight_ste_backward(bf16_torch(a), bf16_torch(b), accumulate=accumulate)
    torch.cuda.synchronize()
    lib.set_sm_budget(0)
    assert lib.device_status() == lib.OK, lib.last_error()
    ref = Q.ste_backward(a, b if accumulate else None)
    assert_bits_equal(F.bf16_bits(bf16_np(out)), F.bf16_bits(ref), "ste under an SM budget")


@pytest.mark.parametrize("shape", [0, 1, 2])
@pytest.mark.parametrize("swiglu", [False, True])
def test_gemm_budget_same_bits(budget, shape, swiglu):
    """Fewer CTAs than tiles (every CTA loops over several): the same output
    bits as the grid sized to the device."""
    lib = budget
    prev_shape = lib.gemm_set_tile_shape(shape)
    prev_dec = lib.gemm_set_decode_rows(0)
    try:
        p = _problem([300, 0, 129, 517, 64], 1024, 512, 32, seed=77)
        args = _gpu_args(p, p["w_c"], p["w_s"], p["wc"])
        outs = []
        for sms in (0, 6):
            lib.set_sm_budget(sms)
            if swiglu:
                h = torch.full((p["cap"], 512), float("nan"), dtype=torch.bfloat16, device="cuda")
                h, _ = lib.moe_grouped_gemm_nvfp4_swiglu(F=512, h=h, **args)
                y = h
            else:
                y = torch.full((p["cap"], 1024), float("nan"), dtype=torch.bfloat16, device="cuda")
                lib.moe_grouped_gemm_nvfp4(N=1024, y=y, **args)
            torch.cuda.synchronize()
            assert lib.device_status() == lib.OK, lib.last_error()
            outs.append(F.bf16_bits(bf16_np(y)[:p["R"]]))
        lib.set_sm_budget(0)
        assert_bits_equal(outs[1], outs[0], f"grouped gemm (tile shape {shape}) under an SM budget")
    finally:
        lib.gemm_set_tile_shape(prev_shape)
        lib.gemm_set_decode_rows(prev_dec)


def test_budget_switch(cuda_lib):
    prev = cuda_lib.set_sm_budget(10)
    assert cuda_lib.set_sm_budget(prev) == 10
    with pytest.raises(cuda_lib.QuadsError):
        cuda_lib.set_sm_budget(-1)


def test_layer_step_split_matches_unsplit(budget):
    """The overlapped layer step with the STE on its own SMs beside the GEMMs
    gives the same outputs, records, replayed operands, mismatch counts and
    master gradients, bit for bit, as the step with every kernel on all SMs."""
    from train_alignment_b200 import layer as L
    from train_alignment_b200 import workloads as W
    cfg = W.MOE_T2048
    dev = torch.device("cuda")
    inp = W.moe_layer_inputs(cfg, seed=3, device=dev)
    x_train = W.engine_drift(inp["x"], 1e-2, seed=3, device=dev)
    results = []
    for side in (0, 40):
        layer = L.build_layer(cfg, inp, dev, side_sms=side)
        _, g_gu, g_d = layer.grad_fq_buffers()
        g_gu.copy_(W.random_bf16(layer.w_gu.shape, 5, 1e-3, dev))
        g_d.copy_(W.random_bf16(layer.w_d.shape, 6, 1e-3, dev))
        layer.grad_all.zero_()
        layer.reset_counts()
        out = layer.step(inp["x"], inp["logits"], x_train, g_gu, g_d)
        torch.cuda.synchronize()
        assert budget.device_status() == budget.OK, budget.last_error()
        assert budget.set_sm_budget(0) == 0, "the step leaves no budget behind"
        n_rows = int(layer.expert_off[-1].item())       # h past the last expert's rows is never written
        results.append({k: v.detach().clone() for k, v in (("out", out), ("h", layer.h[:n_rows]),
                                                           ("counts", layer.counts), ("grad", layer.grad_all),
                                                           ("record", layer.record))})
    for k in results[0]:
        a, b = results[0][k], results[1][k]
        assert torch.equal(a.view(torch.uint8) if a.dtype != torch.int64 else a,
                           b.view(torch.uint8) if b.dtype != torch.int64 else b), k
