"""The C-ABI library without a GPU: it loads, exports every function that
include/quads.h declares, rejects invalid arguments on the host before any
launch, and lays TRACE records out as documented."""
import ctypes
import os
import re
import subprocess

import pytest

from train_alignment_b200 import binding as B

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "quads.h")


def _declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
    names = re.findall(r"^\s*(?:const\s+)?[A-Za-z_][A-Za-z0-9_]*\s*\**\s+\**\s*((?:quads|trace)_[A-Za-z0-9_]+)\s*\(",
                       text, flags=re.M)
    return sorted(set(names))


@pytest.fixture(scope="module")
def lib():
    from train_alignment_b200 import build
    build.build()
    return B.load()


def test_header_declares_the_path():
    names = _declared_functions()
    for required in ["quads_quantize_nvfp4", "quads_dequant", "quads_moe_route_permute",
                     "quads_moe_grouped_gemm_nvfp4", "quads_fakequant_weight_ste",
                     "trace_export_qrecord", "trace_replay_qrecord"]:
        assert required in names


def test_every_declared_symbol_is_exported(lib):
    out = subprocess.run(["nm", "-D", "--defined-only", B._LIB_PATH], capture_output=True, text=True).stdout
    exported = set(re.findall(r" T ((?:quads|trace)_\w+)", out))
    declared = set(_declared_functions())
    assert declared - exported == set()
    assert declared == set(B.exported_symbols())


def test_binding_signatures_cover_header(lib):
    for name in _declared_functions():
        assert getattr(lib, name).argtypes is not None or name in ("quads_last_error",)


def test_abi_version(lib):
    assert lib.quads_abi_version() == 1


def test_scales_bytes(lib):
    assert lib.quads_scales_bytes(64, 256, B.SCALES_LINEAR) == 64 * 16
    assert lib.quads_scales_bytes(64, 256, B.SCALES_TILED) == 128 * 16
    assert lib.quads_scales_bytes(130, 64 * 3, B.SCALES_TILED) == 256 * 12
    assert lib.quads_scales_bytes(10, 17, B.SCALES_LINEAR) == 0


def test_rows_capacity(lib):
    # sum over experts of ceil128(count) <= ceil(T*k/128)*128 + 128*E
    for T, k, E in [(2048, 2, 8), (64, 8, 128), (1, 1, 1)]:
        cap = lib.quads_moe_rows_capacity(T, k, E)
        assert cap % 128 == 0 and cap >= T * k + 127 * E


@pytest.mark.parametrize("call", [
    lambda l: l.quads_quantize_nvfp4(None, 4, 24, 24, None, 1, None, None, None, 0, None, None, 0, None, None, 0,
                                     None),
    lambda l: l.quads_quantize_nvfp4(None, 4, 32, 16, None, 1, None, None, None, 0, None, None, 0, None, None, 0,
                                     None),
    lambda l: l.quads_moe_router_topk(None, 4, 300, 2, 1, None, None, None),
    lambda l: l.quads_moe_router_topk(None, 4, 8, 9, 1, None, None, None),
    lambda l: l.quads_moe_grouped_gemm_nvfp4(None, None, None, 0, None, None, None, None, 8, 256, 100, 256, None,
                                             None, 0, None, None),
    lambda l: l.quads_moe_grouped_gemm_nvfp4(None, None, None, 0, None, None, None, None, 8, 256, 128, 96, None,
                                             None, 0, None, None),
    lambda l: l.quads_moe_grouped_gemm_nvfp4(None, None, None, 0, None, None, None, None, 8, 256, 128, 128, None,
                                             None, 24, None, None),
    lambda l: l.quads_fakequant_weight_ste(None, 0, 128, 64, None, 1, None, None, None, None, None, 0, 0, None, None, 0,
                                           None),
    lambda l: l.quads_swiglu(None, 128, 12, None, 4, None, None, None),
    lambda l: l.quads_moe_unpermute_combine(None, None, None, 4, 2, 12, None, None),
    lambda l: l.quads_select_channels(None, 20000, 4, None, None),
    lambda l: l.trace_replay_qrecord(None, 0, 0, 0, 4, 16, None, None, None, None, None),
    # N not a multiple of the weight tile
    lambda l: l.quads_moe_grouped_gemm_w4a16(None, None, None, None, None, 8, 256, 100, 256, None, None),
    # F not a multiple of 64
    lambda l: l.quads_moe_grouped_gemm_w4a16_swiglu(None, None, None, None, None, 8, 256, 96, 256, None, None, None),
    # no experts
    lambda l: l.quads_moe_fp4_comp_amax(None, 0, None, None, 0, None, None),
    # correction operands missing
    lambda l: l.quads_moe_grouped_gemm_nvfp4_fp4comp(None, None, None, 0, None, None, None, None, 8, 256, 256, 128,
                                                     None, None, None, None, 32, None, None),
    # K not a multiple of 16
    lambda l: l.trace_direction_bits(None, 4, 24, None, None, 0, None, None, 1, None, None),
    # rows without scales
    lambda l: l.trace_replay_direction(None, None, 0, None, None, 1, 4, 32, None, None, 0, None, None, None, None,
                                       None),
    lambda l: l.quads_copy_f32(None, None, -1, None),
    # a negative SM budget
    lambda l: l.quads_set_sm_budget(-1),
])
def test_invalid_arguments_are_rejected_on_the_host(lib, call):
    rc = call(lib)
    assert rc in (B.ERR_INVALID_ARG, B.ERR_UNSUPPORTED_SHAPE, B.ERR_BAD_RECORD)
    assert lib.quads_last_error().decode() != ""


def test_trace_record_layout(lib):
    src = (B.TraceQTensorSrc * 2)()
    s0 = src[0]
    s0.rows, s0.K, s0.n_groups, s0.n_chan, s0.scale_layout, s0.present = 100, 64, 1, 16, B.SCALES_LINEAR, 1
    s1 = src[1]
    s1.rows, s1.K, s1.n_groups, s1.n_chan, s1.scale_layout, s1.present = 384, 128, 3, 0, B.SCALES_TILED, 1
    hdr = B.TraceQRecordHeader()
    n = lib.trace_qrecord_layout(7, 50, 2, ctypes.cast(src, ctypes.c_void_p), 2, ctypes.byref(hdr))
    assert n == hdr.total_bytes and n % 256 == 0
    assert hdr.magic == 0x31434552 and hdr.version == 1 and hdr.layer_id == 7 and hdr.k == 2 and hdr.T == 50
    d0, d1 = hdr.t[0], hdr.t[1]
    assert d0.codes_bytes == 100 * 32 and d0.scales_bytes == 100 * 4
    assert d1.codes_bytes == 384 * 64 and d1.scales_bytes == 384 * 8
    secs = [(d0.codes_off, d0.codes_bytes), (d0.scales_off, d0.scales_bytes), (d0.g_off, 4),
            (d0.chan_off, 64), (d0.resid_off, 100 * 16 * 2), (d1.codes_off, d1.codes_bytes),
            (d1.scales_off, d1.scales_bytes), (d1.g_off, 12), (d1.group_off_off, 16), (hdr.topk_idx_off, 400)]
    secs.sort()
    assert secs[0][0] >= ctypes.sizeof(B.TraceQRecordHeader)
    for (o, b), (o2, _) in zip(secs, secs[1:]):
        assert o % 256 == 0 and o + b <= o2
    assert secs[-1][0] + secs[-1][1] <= n
    # invalid description
    s0.K = 24
    assert lib.trace_qrecord_layout(7, 50, 2, ctypes.cast(src, ctypes.c_void_p), 2, ctypes.byref(hdr)) == 0


def test_missing_library_fails_loudly(monkeypatch, tmp_path):
    """Without the built library every op raises: there is no CPU fallback."""
    import torch
    monkeypatch.setattr(B, "_lib", None)
    monkeypatch.setattr(B, "_LIB_PATH", str(tmp_path / "libquads.so"))
    with pytest.raises(RuntimeError, match="missing"):
        B.load()
    # a host tensor is refused too, rather than computed on the CPU
    with pytest.raises(ValueError, match="CUDA"):
        B.amax_bf16(torch.zeros((4, 16), dtype=torch.bfloat16))


def test_sm_budget_switch(lib):
    """The SM budget is host state: set, read back, restored (no launch)."""
    prev = lib.quads_set_sm_budget(37)
    assert lib.quads_set_sm_budget(prev) == 37
    assert lib.quads_set_sm_budget(prev) == prev
