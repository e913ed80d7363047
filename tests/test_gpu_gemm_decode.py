"""The FP4 grouped GEMM on its decode tiles -- the weights as the MMA's M
operand, 256 weight rows by up to 128 of an expert's rows per tile, the
BF16 correction accumulated as (R / G) . Wc -- against the CPU oracle, per
element within 1e-2 |ref| + 1e-3 sum|a b|.  Row blocks of an expert past
its first 128 rows, experts without rows, a partial last K stage and both
correction widths are covered; rows past the last expert stay untouched."""
import numpy as np
import pytest
import torch

from oracle import formats as F
from tests.helpers import assert_bits_equal, assert_close_tol, bf16_np, f32_of, gate_up_interleave_index
from tests.test_gpu_gemm import _gpu_args, _oracle, _problem, _swiglu_ref

pytestmark = pytest.mark.gpu


@pytest.fixture
def decode_tiles(cuda_lib):
    prev = cuda_lib.gemm_set_decode_rows(1 << 30)        # every eligible GEMM takes the decode tiles
    yield cuda_lib
    cuda_lib.gemm_set_decode_rows(prev)


def _plain(lib, p, decode):
    prev = lib.gemm_set_decode_rows((1 << 30) if decode else 0)
    try:
        args = _gpu_args(p, p["w_c"], p["w_s"], p["wc"])
        y = torch.full((p["cap"], p["N"]), float("nan"), dtype=torch.bfloat16, device="cuda")
        lib.moe_grouped_gemm_nvfp4(N=p["N"], y=y, **args)
        torch.cuda.synchronize()
        assert lib.device_status() == lib.OK, lib.last_error()
    finally:
        lib.gemm_set_decode_rows(prev)
    return bf16_np(y)


@pytest.mark.parametrize("counts,N,K,nc", [
    ([1], 256, 64, 0),                          # one row, one MMA along K
    ([5, 0, 17, 33], 512, 256, 16),             # few rows, an empty expert, one stage
    ([100, 1, 0, 30, 64, 128, 129, 7], 256, 512, 32),   # 128 and 129 rows: one and two row blocks
    ([300, 20, 3], 512, 320, 64),               # three row blocks; partial last stage (K % 256 = 64)
    ([40, 2], 256, 2048, 128),                  # long K, widest correction (two stages)
    ([33, 31, 32, 1, 0, 96], 768, 1024, 64),    # three weight blocks per expert
])
def test_decode_parity(cuda_lib, counts, N, K, nc):
    p = _problem(counts, N, K, nc, seed=5 * sum(counts) + N + K + nc)
    got = _plain(cuda_lib, p, True)
    ref, absdot = _oracle(p)
    R = p["R"]
    assert_close_tol(got[:R], ref, absdot, what="decode-tile grouped gemm")
    assert np.all(np.isnan(got[R:])), "rows past expert_off[E] must be untouched"
    other = _plain(cuda_lib, p, False)
    assert_close_tol(other[:R], ref, absdot, what="grouped gemm without decode tiles")


def test_decode_zero_input_gives_zero(decode_tiles):
    """An all-zero activation tensor (g_a = 0, zero residuals): the folded
    correction R / G is taken as zero and every output is 0."""
    p = _problem([20, 77], 256, 256, 16, seed=5)
    p = dict(p, a_c=np.zeros_like(p["a_c"]), a_s=np.zeros_like(p["a_s"]), g_a=0.0, resid=np.zeros_like(p["resid"]))
    got = _plain(decode_tiles, p, True)
    assert np.all(got[:p["R"]] == 0.0)


@pytest.mark.parametrize("counts,F_,K,nc", [
    ([1], 128, 64, 0),
    ([5, 0, 130, 2], 256, 512, 32),
    ([300, 20, 3, 64], 384, 1024, 64),
])
def test_decode_swiglu(decode_tiles, counts, F_, K, nc):
    """The SwiGLU epilogue on decode tiles (half 0 the gate rows, half 1 the
    matching up rows): h against the oracle (GEMM tolerance carried through
    SwiGLU), bit for bit against the decode-tile plain GEMM followed by the
    SwiGLU kernel, and the per-expert amax exact."""
    lib = decode_tiles
    p = _problem(counts, 2 * F_, K, nc, seed=9 * sum(counts) + F_ + K + nc)
    perm = gate_up_interleave_index(F_)
    args = _gpu_args(p, p["w_c"][:, perm], p["w_s"][:, perm], p["wc"][:, perm] if nc else None)
    E, cap, R = p["E"], p["cap"], p["R"]
    h = torch.full((cap, F_), float("nan"), dtype=torch.bfloat16, device="cuda")
    h, amax = lib.moe_grouped_gemm_nvfp4_swiglu(F=F_, h=h, **args)
    torch.cuda.synchronize()
    assert lib.device_status() == lib.OK, lib.last_error()
    got = bf16_np(h)
    assert np.all(np.isnan(got[R:])), "rows past expert_off[E] must be untouched"
    h_ref, tol_h = _swiglu_ref(p, F_)
    err = np.abs(got[:R] - h_ref)
    assert np.all(err <= tol_h), f"{np.sum(err > tol_h)} of {err.size} h values outside the tolerance"
    y_il = torch.full((cap, 2 * F_), float("nan"), dtype=torch.bfloat16, device="cuda")
    lib.moe_grouped_gemm_nvfp4(N=2 * F_, y=y_il, **args)
    inv = np.argsort(perm)
    h2, _ = lib.swiglu(y_il[:, torch.from_numpy(inv).cuda()].contiguous(), F_, args["expert_off"], E)
    torch.cuda.synchronize()
    assert_bits_equal(F.bf16_bits(got[:R]), F.bf16_bits(bf16_np(h2)[:R]), "fused vs separate SwiGLU")
    a = f32_of(amax)
    for e in range(E):
        lo, hi = p["off"][e], p["off"][e + 1]
        assert a[e] == (np.max(np.abs(got[lo:hi])) if hi > lo else 0.0), e


def test_decode_rows_switch(cuda_lib):
    """The switch returns the previous value and refuses a negative one."""
    prev = cuda_lib.gemm_set_decode_rows(7)
    assert cuda_lib.gemm_set_decode_rows(prev) == 7
    with pytest.raises(cuda_lib.QuadsError):
        cuda_lib.gemm_set_decode_rows(-1)
