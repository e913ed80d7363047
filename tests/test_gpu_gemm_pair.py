"""The FP4 grouped GEMM on its wide output tiles -- 128 x 256 on one CTA and
256 x 256 on a pair of CTAs (tcgen05 cta_group::2), both with the BF16
correction accumulated as (R / G) . Wc -- against the CPU oracle, per
element within 1e-2 |ref| + 1e-3 sum|a b|, and against the 128 x 128 kernel
on the same operands.  In the pair, segments with an odd number of 128-row
blocks end in a pair whose second half is not the expert's: those rows, and
rows past the last expert, stay untouched."""
import numpy as np
import pytest
import torch

from oracle import formats as F
from oracle import nvfp4 as Q
from tests.helpers import assert_bits_equal, assert_close_tol, bf16_np, f32_of, gate_up_interleave_index
from tests.test_gpu_gemm import _gpu_args, _oracle, _problem, _swiglu_ref

pytestmark = pytest.mark.gpu


@pytest.fixture(params=[1, 2], ids=["128x256", "pair_256x256"])
def pair_tiles(cuda_lib, request):
    prev = cuda_lib.gemm_set_tile_shape(request.param)
    prev_dec = cuda_lib.gemm_set_decode_rows(0)         # these shapes, not the decode tiles
    cuda_lib.shape = request.param
    yield cuda_lib
    cuda_lib.gemm_set_tile_shape(prev)
    cuda_lib.gemm_set_decode_rows(prev_dec)


def _plain(lib, p, pair):
    lib.gemm_set_tile_shape(lib.shape if pair else 0)
    args = _gpu_args(p, p["w_c"], p["w_s"], p["wc"])
    y = torch.full((p["cap"], p["N"]), float("nan"), dtype=torch.bfloat16, device="cuda")
    lib.moe_grouped_gemm_nvfp4(N=p["N"], y=y, **args)
    torch.cuda.synchronize()
    assert lib.device_status() == lib.OK, lib.last_error()
    return bf16_np(y)


@pytest.mark.parametrize("counts,N,K,nc", [
    ([64], 256, 64, 0),                     # one pair, second half not the expert's, one MMA along K
    ([256], 256, 256, 16),                  # one full pair, one stage, one correction stage
    ([130, 0, 257], 512, 512, 32),          # empty expert; 2 and 3 row blocks (a half pair)
    ([500, 20, 1000, 3], 256, 1024, 64),
    ([383, 129], 256, 320, 128),            # partial last stage, widest correction (two stages)
    ([1000] * 6, 1024, 1024, 32),           # several tiles per cluster
])
def test_pair_parity(pair_tiles, counts, N, K, nc):
    p = _problem(counts, N, K, nc, seed=3 * sum(counts) + N + K + nc)
    got = _plain(pair_tiles, p, True)
    ref, absdot = _oracle(p)
    R = p["R"]
    assert_close_tol(got[:R], ref, absdot, what="pair-tile grouped gemm")
    assert np.all(np.isnan(got[R:])), "rows past expert_off[E] must be untouched"
    single = _plain(pair_tiles, p, False)
    assert_close_tol(single[:R], ref, absdot, what="128 x 128 grouped gemm")
    pair_tiles.gemm_set_tile_shape(pair_tiles.shape)


def test_pair_zero_input_gives_zero(pair_tiles):
    """An all-zero activation tensor (g_a = 0, zero residuals): the folded
    correction R / G is taken as zero and every output is 0."""
    p = _problem([200, 77], 256, 256, 16, seed=5)
    p = dict(p, a_c=np.zeros_like(p["a_c"]), a_s=np.zeros_like(p["a_s"]), g_a=0.0, resid=np.zeros_like(p["resid"]))
    got = _plain(pair_tiles, p, True)
    assert np.all(got[:p["R"]] == 0.0)


@pytest.mark.parametrize("counts,F_,K,nc", [
    ([64], 128, 64, 0),
    ([130, 0, 257], 256, 512, 32),
    ([500, 20, 1000, 3], 384, 1024, 64),
])
def test_pair_swiglu(pair_tiles, counts, F_, K, nc):
    """The SwiGLU epilogue on pair tiles: h against the oracle (GEMM tolerance
    carried through SwiGLU), bit for bit against the pair-tile plain GEMM
    followed by the SwiGLU kernel, per-expert amax exact."""
    lib = pair_tiles
    p = _problem(counts, 2 * F_, K, nc, seed=7 * sum(counts) + F_ + K + nc)
    perm = gate_up_interleave_index(F_)
    args = _gpu_args(p, p["w_c"][:, perm], p["w_s"][:, perm], p["wc"][:, perm] if nc else None)
    E, cap, R = p["E"], p["cap"], p["R"]
    h = torch.full((cap, F_), float("nan"), dtype=torch.bfloat16, device="cuda")
    h, amax = lib.moe_grouped_gemm_nvfp4_swiglu(F=F_, h=h, **args)
    torch.cuda.synchronize()
    assert lib.device_status() == lib.OK
    got = bf16_np(h)
    assert np.all(np.isnan(got[R:]))
    h_ref, tol_h = _swiglu_ref(p, F_)
    err = np.abs(got[:R] - h_ref)
    assert np.all(err <= tol_h), f"{np.sum(err > tol_h)} of {err.size} h values outside the tolerance"
    y_il = torch.full((cap, 2 * F_), float("nan"), dtype=torch.bfloat16, device="cuda")
    lib.moe_grouped_gemm_nvfp4(N=2 * F_, y=y_il, **args)
    inv = np.argsort(perm)
    h2, amax2 = lib.swiglu(y_il[:, torch.from_numpy(inv).cuda()].contiguous(), F_, args["expert_off"], E)
    torch.cuda.synchronize()
    assert_bits_equal(F.bf16_bits(got[:R]), F.bf16_bits(bf16_np(h2)[:R]), "fused vs separate SwiGLU")
    a = f32_of(amax)
    for e in range(E):
        lo, hi = p["off"][e], p["off"][e + 1]
        assert a[e] == (np.max(np.abs(got[lo:hi])) if hi > lo else 0.0)


def test_pair_swiglu_quant(pair_tiles):
    """The quantizing SwiGLU epilogue on pair tiles: h's NVFP4 codes, scales,
    per-expert scales and residuals equal the pair-tile SwiGLU GEMM followed
    by the quantizer with the same amax, bit for bit."""
    lib = pair_tiles
    counts, F_, K, nc, nch = [300, 40, 700], 256, 512, 16, 48
    p = _problem(counts, 2 * F_, K, nc, seed=11)
    perm = gate_up_interleave_index(F_)
    args = _gpu_args(p, p["w_c"][:, perm], p["w_s"][:, perm], p["wc"][:, perm])
    E, cap, R = p["E"], p["cap"], p["R"]
    h_two, amax_true = lib.moe_grouped_gemm_nvfp4_swiglu(F=F_, **args)
    amax_in = (amax_true * 1.1).contiguous()
    chan_h = torch.from_numpy(Q.pad_channels(np.sort(np.random.default_rng(1).choice(F_, nch, replace=False)))).cuda()
    c2, s2, g2, r2 = lib.quantize_nvfp4(h_two[:R], group_off=args["expert_off"], n_groups=E, amax_in=amax_in,
                                        scale_layout=lib.SCALES_TILED, chan=chan_h)
    h = torch.full((cap, F_), float("nan"), dtype=torch.bfloat16, device="cuda")
    c1, s1, r1, g1, amax1 = lib.moe_grouped_gemm_nvfp4_swiglu_quant(F=F_, amax_h_in=amax_in, chan_h=chan_h, h=h,
                                                                   **args)
    torch.cuda.synchronize()
    assert lib.device_status() == lib.OK
    assert_bits_equal(F.bf16_bits(bf16_np(h)[:R]), F.bf16_bits(bf16_np(h_two)[:R]), "h")
    nsb = lib.scales_bytes(R, F_, lib.SCALES_TILED)
    assert_bits_equal(c1.cpu().numpy()[:R], c2.cpu().numpy()[:R], "h codes")
    assert_bits_equal(s1.cpu().numpy()[:nsb], s2.cpu().numpy()[:nsb], "h scales")
    assert_bits_equal(f32_of(g1).astype(np.float32), f32_of(g2).astype(np.float32), "g_h")
    assert_bits_equal(f32_of(amax1).astype(np.float32), f32_of(amax_true).astype(np.float32), "amax_h_out")
    assert_bits_equal(F.bf16_bits(bf16_np(r1)[:R]), F.bf16_bits(bf16_np(r2)[:R]), "h residuals")
