"""The operations that join layers into a stack (router projection, residual
connection) against the CPU oracle."""
import numpy as np
import pytest
import torch

from oracle import formats as F
from oracle import stack as S
from tests.helpers import assert_bits_equal, bf16_np, bf16_torch, f32_of

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
