"""The allocation-free quantizer, quads_quantize_nvfp4_noalloc.

It exists for callers that cannot give the library device memory beyond
their inputs and outputs -- code whose GPU memory is all owned by another
allocator, plugin interfaces with no way to pass a workspace, loops that
cannot afford an allocation -- and keeps its only scratch (one amax per row
group) in a small device array that lives as long as the library.

Checked here through the C ABI: two calls in a row give exactly what the
workspace-taking quads_quantize_nvfp4 gives (codes, scales, per-tensor
scales and residuals bit for bit), the second one with a smaller amax than
the first so that scratch left over from the first call would show, and
requests beyond the scratch's size are refused before any launch.  This file
is collected last so that a failure here leaves every other test run.
"""

import numpy as np
import pytest
import torch

from train_alignment_b200 import binding as B

pytestmark = pytest.mark.gpu


def _reference(x, chan, group_off, n_groups, layout):
    return B.quantize_nvfp4(x, group_off=group_off, n_groups=n_groups, scale_layout=layout, chan=chan)


def _noalloc(lib, x, chan, group_off, n_groups, layout):
    rows, K = x.shape
    dev = x.device
    n_chan = 0 if chan is None else chan.numel()
    codes = torch.empty((rows, K // 2), dtype=torch.uint8, device=dev)
    scales = torch.empty((B.scales_bytes(rows, K, layout),), dtype=torch.uint8, device=dev)
    g = torch.empty((n_groups,), dtype=torch.float32, device=dev)
    resid = torch.empty((rows, n_chan), dtype=torch.bfloat16, device=dev) if n_chan else None
    rc = lib.quads_quantize_nvfp4_noalloc(
        B._p(x), rows, K, K, B._p(group_off), n_groups, None, B._p(codes), B._p(scales), layout, B._p(g),
        B._p(chan), n_chan, B._p(resid), B._s())
    assert rc == B.OK, lib.quads_last_error().decode()
    return codes, scales, g, resid


def _same(a, b):
    for u, v in zip(a, b):
        if u is None:
            assert v is None
            continue
        assert torch.equal(u.view(torch.uint8) if u.dtype != torch.float32 else u,
                           v.view(torch.uint8) if v.dtype != torch.float32 else v)


def test_two_calls_match_the_workspace_quantizer(cuda_lib):
    lib = B.load()
    gen = torch.Generator(device="cuda").manual_seed(11)
    chan = torch.tensor([5, 40, 41, 300] + [-1] * 12, dtype=torch.int32, device="cuda")
    # first call: large values, one group, linear scales, with residual channels
    x1 = (torch.randn(333, 512, generator=gen, device="cuda") * 50).to(torch.bfloat16)
    got1 = _noalloc(lib, x1, chan, None, 1, B.SCALES_LINEAR)
    ref1 = _reference(x1, chan, None, 1, B.SCALES_LINEAR)
    torch.cuda.synchronize()
    _same(got1, ref1)
    # second call right after: smaller values, three row groups, tiled scales
    x2 = torch.randn(640, 512, generator=gen, device="cuda").to(torch.bfloat16)
    off = torch.tensor([0, 128, 384, 640], dtype=torch.int32, device="cuda")
    got2 = _noalloc(lib, x2, chan, off, 3, B.SCALES_TILED)
    ref2 = _reference(x2, chan, off, 3, B.SCALES_TILED)
    torch.cuda.synchronize()
    _same(got2, ref2)
    assert float(got2[2].max()) < float(got1[2][0]) / 10


def test_too_many_groups_is_refused(cuda_lib):
    lib = B.load()
    x = torch.zeros((2050, 16), dtype=torch.bfloat16, device="cuda")
    before = lib.quads_launch_count()
    rc = lib.quads_quantize_nvfp4_noalloc(B._p(x), 2050, 16, 16, None, 1025, None, B._p(x), B._p(x), 0, B._p(x),
                                          None, 0, None, B._s())
    assert rc == B.ERR_UNSUPPORTED_SHAPE
    msg = lib.quads_last_error().decode()
    assert "allocation-free quantizer supports at most 1024 row groups" in msg, msg
    assert lib.quads_launch_count() == before
