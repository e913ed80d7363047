"""Thin ctypes binding of libquads.so (the C ABI in include/quads.h).

Argument marshalling only: every function passes torch tensors' device
pointers, sizes and the current CUDA stream to the library and raises
QuadsError on a non-zero status.  Output tensors are allocated with torch
when the caller does not pass them.  There is no fallback: if the library is
missing, load() raises.
"""
import ctypes
import os

import torch

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libquads.so")
_lib = None

OK = 0
ERR_INVALID_ARG = -1
ERR_UNSUPPORTED_SHAPE = -2
ERR_CUDA = -3
ERR_TIMEOUT = -4
ERR_BAD_RECORD = -5
SCALES_LINEAR = 0
SCALES_TILED = 1
OUT_BF16 = 0
OUT_F32 = 1
TRACE_MAX_TENSORS = 2

c_i64, c_i32, c_sz, c_vp, c_u64 = ctypes.c_int64, ctypes.c_int, ctypes.c_size_t, ctypes.c_void_p, ctypes.c_uint64


class QuadsError(RuntimeError):
    def __init__(self, code, where, msg):
        super().__init__(f"{where} failed with status {code}: {msg}")
        self.code = code


class TraceQTensorDesc(ctypes.Structure):
    _fields_ = [("rows", c_i64), ("K", c_i64), ("n_groups", ctypes.c_int32), ("n_chan", ctypes.c_int32),
                ("scale_layout", ctypes.c_int32), ("present", ctypes.c_int32),
                ("codes_off", c_u64), ("scales_off", c_u64), ("g_off", c_u64), ("group_off_off", c_u64),
                ("chan_off", c_u64), ("resid_off", c_u64), ("codes_bytes", c_u64), ("scales_bytes", c_u64)]


class TraceQRecordHeader(ctypes.Structure):
    _fields_ = [("magic", ctypes.c_uint32), ("version", ctypes.c_uint32), ("layer_id", ctypes.c_int32),
                ("k", ctypes.c_int32), ("T", c_i64), ("total_bytes", c_u64), ("topk_idx_off", c_u64),
                ("t", TraceQTensorDesc * TRACE_MAX_TENSORS)]


class TraceQTensorSrc(ctypes.Structure):
    _fields_ = [("rows", c_i64), ("K", c_i64), ("n_groups", ctypes.c_int32), ("n_chan", ctypes.c_int32),
                ("scale_layout", ctypes.c_int32), ("present", ctypes.c_int32),
                ("codes", c_vp), ("scales", c_vp), ("g", c_vp), ("group_off", c_vp), ("chan", c_vp),
                ("resid", c_vp)]


_SIGS = {
    "quads_last_error": (ctypes.c_char_p, []),
    "quads_abi_version": (c_i32, []),
    "quads_launch_count": (c_u64, []),
    "quads_device_status": (c_i32, [c_vp]),
    "quads_selftest_bounded_wait": (c_i32, [c_u64, c_vp]),
    "quads_gemm_set_tile_shape": (c_i32, [c_i32]),
    "quads_gemm_set_decode_rows": (c_i32, [c_i32]),
    "quads_set_sm_budget": (c_i32, [c_i32]),
    "quads_scales_bytes": (c_sz, [c_i64, c_i64, c_i32]),
    "quads_amax_bf16": (c_i32, [c_vp, c_i64, c_i64, c_i64, c_vp, c_i32, c_vp, c_vp]),
    "quads_quantize_workspace_bytes": (c_sz, [c_i32]),
    "quads_quantize_nvfp4": (c_i32, [c_vp, c_i64, c_i64, c_i64, c_vp, c_i32, c_vp, c_vp, c_vp, c_i32, c_vp,
                                     c_vp, c_i32, c_vp, c_vp, c_sz, c_vp]),
    "quads_quantize_nvfp4_noalloc": (c_i32, [c_vp, c_i64, c_i64, c_i64, c_vp, c_i32, c_vp, c_vp, c_vp, c_i32,
                                             c_vp, c_vp, c_i32, c_vp, c_vp]),
    "quads_dequant": (c_i32, [c_vp, c_vp, c_i32, c_vp, c_vp, c_i32, c_i64, c_i64, c_vp, c_i32, c_vp]),
    "quads_channel_scores_workspace_bytes": (c_sz, [c_i64, c_i64]),
    "quads_channel_scores": (c_i32, [c_vp, c_i64, c_i64, c_vp, c_vp, c_vp, c_sz, c_vp]),
    "quads_select_channels": (c_i32, [c_vp, c_i64, c_i32, c_vp, c_vp]),
    "quads_moe_router_topk": (c_i32, [c_vp, c_i64, c_i32, c_i32, c_i32, c_vp, c_vp, c_vp]),
    "quads_moe_rows_capacity": (c_i64, [c_i64, c_i32, c_i32]),
    "quads_moe_permute_workspace_bytes": (c_sz, [c_i64, c_i32, c_i32]),
    "quads_moe_permute": (c_i32, [c_vp, c_i64, c_i32, c_i32, c_vp, c_vp, c_vp, c_vp, c_sz, c_vp]),
    "quads_moe_gather": (c_i32, [c_vp, c_vp, c_i32, c_i64, c_vp, c_vp, c_i64, c_vp, c_i32, c_vp, c_vp, c_vp,
                                 c_vp]),
    "quads_moe_gather_bf16": (c_i32, [c_vp, c_vp, c_i32, c_i64, c_vp, c_i64, c_vp, c_vp]),
    "quads_moe_route_permute": (c_i32, [c_vp, c_i64, c_i32, c_i32, c_i32, c_vp, c_vp, c_vp, c_vp, c_vp, c_i64,
                                        c_vp, c_vp, c_i64, c_vp, c_i32, c_vp, c_vp, c_vp, c_vp, c_sz, c_vp]),
    "quads_moe_grouped_gemm_nvfp4": (c_i32, [c_vp, c_vp, c_vp, c_i32, c_vp, c_vp, c_vp, c_vp, c_i32, c_i64, c_i64,
                                             c_i64, c_vp, c_vp, c_i32, c_vp, c_vp]),
    "quads_moe_grouped_gemm_nvfp4_swiglu": (c_i32, [c_vp, c_vp, c_vp, c_i32, c_vp, c_vp, c_vp, c_vp, c_i32, c_i64,
                                                    c_i64, c_i64, c_vp, c_vp, c_i32, c_vp, c_vp, c_vp]),
    "quads_moe_grouped_gemm_nvfp4_swiglu_quant": (c_i32, [c_vp, c_vp, c_vp, c_i32, c_vp, c_vp, c_vp, c_vp, c_i32,
                                                          c_i64, c_i64, c_i64, c_vp, c_vp, c_i32, c_vp, c_vp, c_i32,
                                                          c_vp, c_vp, c_vp, c_vp, c_vp, c_vp, c_vp]),
    "quads_moe_grouped_gemm_nvfp4_fp4comp": (c_i32, [c_vp, c_vp, c_vp, c_i32, c_vp, c_vp, c_vp, c_vp, c_i32, c_i64,
                                                     c_i64, c_i64, c_vp, c_vp, c_vp, c_vp, c_i64, c_vp, c_vp]),
    "quads_moe_grouped_gemm_nvfp4_swiglu_fp4comp": (c_i32, [c_vp, c_vp, c_vp, c_i32, c_vp, c_vp, c_vp, c_vp, c_i32,
                                                            c_i64, c_i64, c_i64, c_vp, c_vp, c_vp, c_vp, c_i64, c_vp,
                                                            c_vp, c_vp]),
    "quads_moe_fp4_comp_amax": (c_i32, [c_vp, c_i32, c_vp, c_vp, c_i32, c_vp, c_vp]),
    "quads_copy_f32": (c_i32, [c_vp, c_vp, c_i64, c_vp]),
    "quads_moe_grouped_gemm_w4a16": (c_i32, [c_vp, c_vp, c_vp, c_vp, c_vp, c_i32, c_i64, c_i64, c_i64, c_vp, c_vp]),
    "quads_moe_grouped_gemm_w4a16_swiglu": (c_i32, [c_vp, c_vp, c_vp, c_vp, c_vp, c_i32, c_i64, c_i64, c_i64, c_vp,
                                                    c_vp, c_vp]),
    "quads_swiglu": (c_i32, [c_vp, c_i64, c_i64, c_vp, c_i32, c_vp, c_vp, c_vp]),
    "quads_moe_unpermute_combine": (c_i32, [c_vp, c_vp, c_vp, c_i64, c_i32, c_i64, c_vp, c_vp]),
    "quads_fakequant_weight_ste": (c_i32, [c_vp, c_i64, c_i64, c_i64, c_vp, c_i32, c_vp, c_vp, c_vp, c_vp, c_vp, c_i32,
                                           c_i32, c_vp, c_vp, c_sz, c_vp]),
    "quads_fakequant_weight_ste_gate_up": (c_i32, [c_vp, c_i64, c_i64, c_i64, c_vp, c_i32, c_vp, c_vp, c_vp, c_vp,
                                                   c_vp, c_i32, c_i32, c_vp, c_vp, c_sz, c_vp]),
    "quads_fakequant_weight_ste_backward": (c_i32, [c_vp, c_vp, c_i64, c_i32, c_vp]),
    "quads_router_logits": (c_i32, [c_vp, c_i64, c_i64, c_vp, c_i32, c_vp, c_vp]),
    "quads_residual_add": (c_i32, [c_vp, c_vp, c_i64, c_vp, c_vp]),
    "trace_qrecord_layout": (c_sz, [c_i32, c_i64, c_i32, c_vp, c_i32, c_vp]),
    "trace_export_qrecord": (c_i32, [c_i32, c_i64, c_i32, c_vp, c_vp, c_i32, c_vp, c_sz, c_vp]),
    "trace_replay_qrecord": (c_i32, [c_vp, c_sz, c_i32, c_i32, c_i64, c_i64, c_vp, c_vp, c_vp, c_vp, c_vp]),
    "trace_direction_bits": (c_i32, [c_vp, c_i64, c_i64, c_vp, c_vp, c_i32, c_vp, c_vp, c_i32, c_vp, c_vp]),
    "trace_replay_direction": (c_i32, [c_vp, c_vp, c_i32, c_vp, c_vp, c_i32, c_i64, c_i64, c_vp, c_vp, c_i32, c_vp,
                                       c_vp, c_vp, c_vp, c_vp]),
}


def load(path=None):
    """Load libquads.so (raises if it is missing; there is no fallback)."""
    global _lib
    if _lib is not None:
        return _lib
    p = path or _LIB_PATH
    if not os.path.exists(p):
        raise RuntimeError(f"{p} is missing: build it with `python -m train_alignment_b200.build`")
    lib = ctypes.CDLL(p)
    for name, (res, args) in _SIGS.items():
        f = getattr(lib, name)
        f.restype = res
        f.argtypes = args
    _lib = lib
    return lib


def exported_symbols():
    return list(_SIGS)


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _s():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _check(rc, where):
    if rc != OK:
        raise QuadsError(rc, where, load().quads_last_error().decode())


def _dev(t, dtype, name):
    if t is None:
        return
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _bits(t):
    """BF16 tensors travel as their uint16 bit patterns."""
    return t


def _empty(shape, dtype, device):
    return torch.empty(shape, dtype=dtype, device=device)


# ------------------------------------------------------------------ status


def last_error():
    return load().quads_last_error().decode()


def launch_count():
    return int(load().quads_launch_count())


def device_status():
    return int(load().quads_device_status(_s()))


def selftest_bounded_wait(timeout_ns):
    _check(load().quads_selftest_bounded_wait(int(timeout_ns), _s()), "quads_selftest_bounded_wait")


TILE_128x128, TILE_128x256, TILE_PAIR_256x256 = 0, 1, 2


def gemm_set_tile_shape(shape):
    """Output tile of the FP4 grouped GEMMs (0: 128 x 128, 1: 128 x 256,
    2: 256 x 256 on a CTA pair); returns the previous shape."""
    prev = int(load().quads_gemm_set_tile_shape(int(shape)))
    if prev < 0:
        _check(prev, "quads_gemm_set_tile_shape")
    return prev


def gemm_set_decode_rows(rows):
    """Average rows per expert at or below which the FP4 grouped GEMMs take
    the decode tiles (weights as the MMA's M operand); 0: never.  Returns
    the previous value."""
    prev = int(load().quads_gemm_set_decode_rows(int(rows)))
    if prev < 0:
        _check(prev, "quads_gemm_set_decode_rows")
    return prev


def set_sm_budget(n):
    """SMs that the persistent GEMMs and the STE backward launched afterwards
    may use (0: all).  Returns the previous budget."""
    prev = int(load().quads_set_sm_budget(int(n)))
    if prev < 0:
        _check(prev, "quads_set_sm_budget")
    return prev


def scales_bytes(rows, K, layout):
    return int(load().quads_scales_bytes(rows, K, layout))


# ---------------------------------------------------------------- quantize


def quantize_workspace_bytes(n_groups):
    return int(load().quads_quantize_workspace_bytes(n_groups))


def _rows_view(x, name):
    """A BF16 matrix whose rows may be strided (row stride = ld elements)."""
    if not x.is_cuda or x.dtype != torch.bfloat16 or x.dim() != 2 or x.stride(1) != 1:
        raise ValueError(f"{name} must be a CUDA bfloat16 matrix with unit column stride")
    return x.shape[0], x.shape[1], x.stride(0)


def amax_bf16(x, group_off=None, n_groups=1, out=None):
    rows, K, ld = _rows_view(x, "x")
    out = out if out is not None else _empty((n_groups,), torch.float32, x.device)
    _check(load().quads_amax_bf16(_p(x), rows, K, ld, _p(group_off), n_groups, _p(out), _s()), "quads_amax_bf16")
    return out


def quantize_nvfp4(x, *, group_off=None, n_groups=1, amax_in=None, scale_layout=SCALES_LINEAR, chan=None,
                   codes=None, scales=None, g_out=None, resid_out=None, ws=None):
    """Returns (codes [rows, K/2] u8, scales u8, g [n_groups] f32, resid [rows, n_chan] bf16 or None)."""
    _dev(x, torch.bfloat16, "x")
    rows, K = x.shape
    dev = x.device
    n_chan = 0 if chan is None else int(chan.numel())
    codes = codes if codes is not None else _empty((rows, K // 2), torch.uint8, dev)
    scales = scales if scales is not None else _empty((scales_bytes(rows, K, scale_layout),), torch.uint8, dev)
    g_out = g_out if g_out is not None else _empty((n_groups,), torch.float32, dev)
    if n_chan and resid_out is None:
        resid_out = _empty((rows, n_chan), torch.bfloat16, dev)
    if amax_in is None and ws is None:
        ws = _empty((quantize_workspace_bytes(n_groups),), torch.uint8, dev)
    _check(load().quads_quantize_nvfp4(
        _p(x), rows, K, K, _p(group_off), n_groups, _p(amax_in), _p(codes), _p(scales), scale_layout, _p(g_out),
        _p(chan), n_chan, _p(resid_out) if n_chan else None, _p(ws), 0 if ws is None else ws.numel(), _s()),
        "quads_quantize_nvfp4")
    return codes, scales, g_out, (resid_out if n_chan else None)


def dequant(codes, scales, scale_layout, g, rows, K, group_off=None, n_groups=1, out_dtype=OUT_BF16, out=None):
    dt = torch.bfloat16 if out_dtype == OUT_BF16 else torch.float32
    out = out if out is not None else _empty((rows, K), dt, codes.device)
    _check(load().quads_dequant(_p(codes), _p(scales), scale_layout, _p(g), _p(group_off), n_groups, rows, K,
                                _p(out), out_dtype, _s()), "quads_dequant")
    return out


def channel_scores(x, amax_in=None):
    _dev(x, torch.bfloat16, "x")
    rows, K = x.shape
    ws = _empty((int(load().quads_channel_scores_workspace_bytes(rows, K)),), torch.uint8, x.device)
    out = _empty((K,), torch.float32, x.device)
    _check(load().quads_channel_scores(_p(x), rows, K, _p(amax_in), _p(out), _p(ws), ws.numel(), _s()),
           "quads_channel_scores")
    return out


def select_channels(scores, n_sel):
    out = _empty((n_sel,), torch.int32, scores.device)
    _check(load().quads_select_channels(_p(scores), scores.numel(), n_sel, _p(out), _s()), "quads_select_channels")
    return out


# --------------------------------------------------------------------- MoE


def moe_rows_capacity(T, k, E):
    return int(load().quads_moe_rows_capacity(T, k, E))


def moe_permute_workspace_bytes(T, k, E):
    return int(load().quads_moe_permute_workspace_bytes(T, k, E))


def moe_router_topk(logits, k, renorm=True, idx=None, w=None):
    _dev(logits, torch.float32, "logits")
    T, E = logits.shape
    idx = idx if idx is not None else _empty((T, k), torch.int32, logits.device)
    w = w if w is not None else _empty((T, k), torch.float32, logits.device)
    _check(load().quads_moe_router_topk(_p(logits), T, E, k, 1 if renorm else 0, _p(idx), _p(w), _s()),
           "quads_moe_router_topk")
    return idx, w


def moe_permute(topk_idx, E, expert_off=None, row_of=None, src_of=None, ws=None):
    _dev(topk_idx, torch.int32, "topk_idx")
    T, k = topk_idx.shape
    dev = topk_idx.device
    cap = moe_rows_capacity(T, k, E)
    expert_off = expert_off if expert_off is not None else _empty((E + 1,), torch.int32, dev)
    row_of = row_of if row_of is not None else _empty((T * k,), torch.int32, dev)
    src_of = src_of if src_of is not None else _empty((cap,), torch.int32, dev)
    ws = ws if ws is not None else _empty((moe_permute_workspace_bytes(T, k, E),), torch.uint8, dev)
    _check(load().quads_moe_permute(_p(topk_idx), T, k, E, _p(expert_off), _p(row_of), _p(src_of), _p(ws),
                                    ws.numel(), _s()), "quads_moe_permute")
    return expert_off, row_of, src_of


def moe_gather(src_of, expert_off, E, rows_cap, a_codes, a_scales, K, a_resid=None, pa_codes=None,
               pa_scales=None, pa_resid=None):
    dev = a_codes.device
    n_chan = 0 if a_resid is None else a_resid.shape[1]
    pa_codes = pa_codes if pa_codes is not None else _empty((rows_cap, K // 2), torch.uint8, dev)
    pa_scales = pa_scales if pa_scales is not None else _empty((scales_bytes(rows_cap, K, SCALES_TILED),),
                                                               torch.uint8, dev)
    if n_chan and pa_resid is None:
        pa_resid = _empty((rows_cap, n_chan), torch.bfloat16, dev)
    _check(load().quads_moe_gather(_p(src_of), _p(expert_off), E, rows_cap, _p(a_codes), _p(a_scales), K,
                                   _p(a_resid), n_chan, _p(pa_codes), _p(pa_scales),
                                   _p(pa_resid) if n_chan else None, _s()), "quads_moe_gather")
    return pa_codes, pa_scales, (pa_resid if n_chan else None)


def moe_gather_bf16(src_of, expert_off, E, rows_cap, x, out=None):
    """BF16 rows of x in expert order (pad rows zero): [rows_cap, H]."""
    _dev(x, torch.bfloat16, "x")
    H = x.shape[1]
    out = out if out is not None else _empty((rows_cap, H), torch.bfloat16, x.device)
    _check(load().quads_moe_gather_bf16(_p(src_of), _p(expert_off), E, rows_cap, _p(x), H, _p(out), _s()),
           "quads_moe_gather_bf16")
    return out


def moe_route_permute(logits, k, a_codes, a_scales, K, a_resid=None, renorm=True):
    """Router top-k, permutation and gather in one call (quads_moe_route_permute).
    Returns (topk_idx, topk_w, expert_off, row_of, src_of, pa_codes, pa_scales,
    pa_resid)."""
    _dev(logits, torch.float32, "logits")
    T, E = logits.shape
    dev = logits.device
    cap = moe_rows_capacity(T, k, E)
    n_chan = 0 if a_resid is None else a_resid.shape[1]
    idx, w = _empty((T, k), torch.int32, dev), _empty((T, k), torch.float32, dev)
    off, row_of, src_of = _empty((E + 1,), torch.int32, dev), _empty((T * k,), torch.int32, dev), \
        _empty((cap,), torch.int32, dev)
    pa_codes = _empty((cap, K // 2), torch.uint8, dev)
    pa_scales = _empty((scales_bytes(cap, K, SCALES_TILED),), torch.uint8, dev)
    pa_resid = _empty((cap, n_chan), torch.bfloat16, dev) if n_chan else None
    ws = _empty((moe_permute_workspace_bytes(T, k, E),), torch.uint8, dev)
    _check(load().quads_moe_route_permute(_p(logits), T, E, k, 1 if renorm else 0, _p(idx), _p(w), _p(off),
                                          _p(row_of), _p(src_of), cap, _p(a_codes), _p(a_scales), K,
                                          _p(a_resid) if n_chan else None, n_chan, _p(pa_codes), _p(pa_scales),
                                          _p(pa_resid) if n_chan else None, _p(ws), ws.numel(), _s()),
           "quads_moe_route_permute")
    return idx, w, off, row_of, src_of, pa_codes, pa_scales, pa_resid


def moe_grouped_gemm_nvfp4(a_codes, a_scales, g_a, w_codes, w_scales, g_w, expert_off, E, rows_cap, N, K,
                           a_resid=None, w_resid=None, y=None):
    n_chan = 0 if a_resid is None else a_resid.shape[1]
    y = y if y is not None else _empty((rows_cap, N), torch.bfloat16, a_codes.device)
    per_expert = 1 if g_a.numel() == E and E > 1 else 0
    _check(load().quads_moe_grouped_gemm_nvfp4(
        _p(a_codes), _p(a_scales), _p(g_a), per_expert, _p(w_codes), _p(w_scales), _p(g_w), _p(expert_off), E,
        rows_cap, N, K, _p(a_resid), _p(w_resid), n_chan, _p(y), _s()), "quads_moe_grouped_gemm_nvfp4")
    return y


def moe_grouped_gemm_nvfp4_swiglu(a_codes, a_scales, g_a, w_codes, w_scales, g_w, expert_off, E, rows_cap, F, K,
                                  a_resid=None, w_resid=None, h=None, amax=None, want_amax=True):
    """Gate/up GEMM with SwiGLU fused; W rows in the 64-row interleaved
    gate/up order.  Returns (h [rows_cap, F], per-expert amax or None)."""
    n_chan = 0 if a_resid is None else a_resid.shape[1]
    h = h if h is not None else _empty((rows_cap, F), torch.bfloat16, a_codes.device)
    if want_amax and amax is None:
        amax = _empty((E,), torch.float32, a_codes.device)
    per_expert = 1 if g_a.numel() == E and E > 1 else 0
    _check(load().quads_moe_grouped_gemm_nvfp4_swiglu(
        _p(a_codes), _p(a_scales), _p(g_a), per_expert, _p(w_codes), _p(w_scales), _p(g_w), _p(expert_off), E,
        rows_cap, F, K, _p(a_resid), _p(w_resid), n_chan, _p(h), _p(amax) if want_amax else None, _s()),
        "quads_moe_grouped_gemm_nvfp4_swiglu")
    return h, (amax if want_amax else None)


def moe_grouped_gemm_nvfp4_swiglu_quant(a_codes, a_scales, g_a, w_codes, w_scales, g_w, expert_off, E, rows_cap, F,
                                        K, amax_h_in, chan_h=None, a_resid=None, w_resid=None, h_codes=None,
                                        h_scales=None, h_resid=None, g_h=None, amax_h_out=None, h=None):
    """Gate/up GEMM + SwiGLU + NVFP4 quantization of h (per-expert scale from
    amax_h_in).  Returns (h_codes, h_scales, h_resid or None, g_h, amax_h_out)."""
    dev = a_codes.device
    n_chan = 0 if a_resid is None else a_resid.shape[1]
    n_chan_h = 0 if chan_h is None else int(chan_h.numel())
    h_codes = h_codes if h_codes is not None else _empty((rows_cap, F // 2), torch.uint8, dev)
    h_scales = h_scales if h_scales is not None else _empty((scales_bytes(rows_cap, F, SCALES_TILED),), torch.uint8,
                                                            dev)
    if n_chan_h and h_resid is None:
        h_resid = _empty((rows_cap, n_chan_h), torch.bfloat16, dev)
    g_h = g_h if g_h is not None else _empty((E,), torch.float32, dev)
    amax_h_out = amax_h_out if amax_h_out is not None else _empty((E,), torch.float32, dev)
    per_expert = 1 if g_a.numel() == E and E > 1 else 0
    _check(load().quads_moe_grouped_gemm_nvfp4_swiglu_quant(
        _p(a_codes), _p(a_scales), _p(g_a), per_expert, _p(w_codes), _p(w_scales), _p(g_w), _p(expert_off), E,
        rows_cap, F, K, _p(a_resid), _p(w_resid), n_chan, _p(amax_h_in), _p(chan_h), n_chan_h, _p(h_codes),
        _p(h_scales), _p(h_resid) if n_chan_h else None, _p(g_h), _p(amax_h_out), _p(h), _s()),
        "quads_moe_grouped_gemm_nvfp4_swiglu_quant")
    return h_codes, h_scales, (h_resid if n_chan_h else None), g_h, amax_h_out


def moe_grouped_gemm_nvfp4_fp4comp(a_codes, a_scales, g_a, w_codes, w_scales, g_w, expert_off, E, rows_cap, N, K,
                                   r_codes, r_scales, wc_codes, wc_scales, Kc, y=None, swiglu=False, amax=None):
    """Grouped GEMM with the FP4 residual correction; swiglu=True gives
    (h [rows_cap, N/2], amax) with N = 2F, else y [rows_cap, N]."""
    dev = a_codes.device
    per_expert = 1 if g_a.numel() == E and E > 1 else 0
    if swiglu:
        F = N // 2
        y = y if y is not None else _empty((rows_cap, F), torch.bfloat16, dev)
        amax = amax if amax is not None else _empty((E,), torch.float32, dev)
        _check(load().quads_moe_grouped_gemm_nvfp4_swiglu_fp4comp(
            _p(a_codes), _p(a_scales), _p(g_a), per_expert, _p(w_codes), _p(w_scales), _p(g_w), _p(expert_off), E,
            rows_cap, F, K, _p(r_codes), _p(r_scales), _p(wc_codes), _p(wc_scales), Kc, _p(y), _p(amax), _s()),
            "quads_moe_grouped_gemm_nvfp4_swiglu_fp4comp")
        return y, amax
    y = y if y is not None else _empty((rows_cap, N), torch.bfloat16, dev)
    _check(load().quads_moe_grouped_gemm_nvfp4_fp4comp(
        _p(a_codes), _p(a_scales), _p(g_a), per_expert, _p(w_codes), _p(w_scales), _p(g_w), _p(expert_off), E,
        rows_cap, N, K, _p(r_codes), _p(r_scales), _p(wc_codes), _p(wc_scales), Kc, _p(y), _s()),
        "quads_moe_grouped_gemm_nvfp4_fp4comp")
    return y


def moe_grouped_gemm_w4a16(x, w_codes, w_scales, g_w, expert_off, E, rows_cap, N, K, y=None, swiglu=False,
                           amax=None):
    """Trainer GEMM: BF16 x [rows_cap, K] times the fake-quantized weights
    given as NVFP4 codes/scales.  swiglu=True returns (h, amax) with N = 2F."""
    _dev(x, torch.bfloat16, "x")
    dev = x.device
    if swiglu:
        F = N // 2
        y = y if y is not None else _empty((rows_cap, F), torch.bfloat16, dev)
        amax = amax if amax is not None else _empty((E,), torch.float32, dev)
        _check(load().quads_moe_grouped_gemm_w4a16_swiglu(_p(x), _p(w_codes), _p(w_scales), _p(g_w), _p(expert_off),
                                                          E, rows_cap, F, K, _p(y), _p(amax), _s()),
               "quads_moe_grouped_gemm_w4a16_swiglu")
        return y, amax
    y = y if y is not None else _empty((rows_cap, N), torch.bfloat16, dev)
    _check(load().quads_moe_grouped_gemm_w4a16(_p(x), _p(w_codes), _p(w_scales), _p(g_w), _p(expert_off), E,
                                               rows_cap, N, K, _p(y), _s()), "quads_moe_grouped_gemm_w4a16")
    return y


def moe_fp4_comp_amax(g_a, g_w, g_wc, E, out=None):
    out = out if out is not None else _empty((E,), torch.float32, g_w.device)
    per_expert = 1 if g_a.numel() == E and E > 1 else 0
    _check(load().quads_moe_fp4_comp_amax(_p(g_a), per_expert, _p(g_w), _p(g_wc), E, _p(out), _s()),
           "quads_moe_fp4_comp_amax")
    return out


def swiglu(y, F, expert_off, E, h=None, amax=None, want_amax=True):
    rows_cap = y.shape[0]
    h = h if h is not None else _empty((rows_cap, F), torch.bfloat16, y.device)
    if want_amax and amax is None:
        amax = _empty((E,), torch.float32, y.device)
    _check(load().quads_swiglu(_p(y), rows_cap, F, _p(expert_off), E, _p(h), _p(amax) if want_amax else None,
                               _s()), "quads_swiglu")
    return h, (amax if want_amax else None)


def moe_unpermute_combine(y, row_of, topk_w, T, k, H, out=None):
    out = out if out is not None else _empty((T, H), torch.bfloat16, y.device)
    _check(load().quads_moe_unpermute_combine(_p(y), _p(row_of), _p(topk_w), T, k, H, _p(out), _s()),
           "quads_moe_unpermute_combine")
    return out


# ------------------------------------------------------------ fake-quant


def fakequant_weight_ste(w, fold_global=True, chan=None, chan_raw=False, want_codes=True, w_fq=None, codes=None,
                         scales=None, g_out=None, w_chan=None, ws=None, amax_in=None, gate_up=False, want_wfq=True):
    """w: [n_mat, rows, K] bf16.  Returns (w_fq, codes, scales, g, w_chan).
    gate_up=True: codes, scales and w_chan in the 64-row gate/up interleaved
    order of quads_fakequant_weight_ste_gate_up."""
    _dev(w, torch.bfloat16, "w")
    n_mat, rows, K = w.shape
    dev = w.device
    n_chan = 0 if chan is None else int(chan.numel())
    layout = SCALES_TILED if rows % 128 == 0 else SCALES_LINEAR
    if want_wfq:
        w_fq = w_fq if w_fq is not None else _empty((n_mat, rows, K), torch.bfloat16, dev)
    else:
        w_fq = None
    if want_codes:
        codes = codes if codes is not None else _empty((n_mat, rows, K // 2), torch.uint8, dev)
        scales = scales if scales is not None else _empty((scales_bytes(n_mat * rows, K, layout),), torch.uint8,
                                                          dev)
    g_out = g_out if g_out is not None else _empty((n_mat,), torch.float32, dev)
    if n_chan and w_chan is None:
        w_chan = _empty((n_mat, rows, n_chan), torch.bfloat16, dev)
    if amax_in is None and ws is None:
        ws = _empty((quantize_workspace_bytes(n_mat),), torch.uint8, dev)
    name = "quads_fakequant_weight_ste_gate_up" if gate_up else "quads_fakequant_weight_ste"
    _check(getattr(load(), name)(
        _p(w), n_mat, rows, K, _p(amax_in), 1 if fold_global else 0, _p(w_fq), _p(codes) if want_codes else None,
        _p(scales) if want_codes else None, _p(g_out), _p(chan), n_chan, 1 if chan_raw else 0,
        _p(w_chan) if n_chan else None, _p(ws), 0 if ws is None else ws.numel(), _s()), name)
    return w_fq, (codes if want_codes else None), (scales if want_codes else None), g_out, \
        (w_chan if n_chan else None)


def fakequant_weight_ste_backward(grad_wfq, grad_w=None, accumulate=False):
    grad_w = grad_w if grad_w is not None else torch.empty_like(grad_wfq)
    _check(load().quads_fakequant_weight_ste_backward(_p(grad_wfq), _p(grad_w), grad_wfq.numel(),
                                                      1 if accumulate else 0, _s()),
           "quads_fakequant_weight_ste_backward")
    return grad_w


# ---------------------------------------------------------------- TRACE


def qtensor_src(codes, scales, g, rows, K, scale_layout, group_off=None, chan=None, resid=None):
    """Description of one recorded tensor (keeps the tensors alive via ._keep)."""
    s = TraceQTensorSrc()
    s.rows, s.K = rows, K
    s.n_groups = int(g.numel())
    s.n_chan = 0 if chan is None else int(chan.numel())
    s.scale_layout = scale_layout
    s.present = 1
    s.codes, s.scales, s.g = codes.data_ptr(), scales.data_ptr(), g.data_ptr()
    s.group_off = group_off.data_ptr() if (group_off is not None and s.n_groups > 1) else None
    s.chan = chan.data_ptr() if s.n_chan else None
    s.resid = resid.data_ptr() if s.n_chan else None
    s._keep = (codes, scales, g, group_off, chan, resid)
    return s


def qtensor_shape(rows, K, scale_layout, n_groups=1, n_chan=0):
    """A record slot described by its sizes only (for trace_qrecord_layout)."""
    s = TraceQTensorSrc()
    s.rows, s.K, s.n_groups, s.n_chan, s.scale_layout, s.present = rows, K, n_groups, n_chan, scale_layout, 1
    return s


def record_views(record, hdr, which):
    """Views of slot `which` of a record laid out by trace_qrecord_layout:
    codes, scales (u8), g (f32), group_off and chan (i32), resid (bf16), each
    None when the slot has no such section."""
    d = hdr.t[which]

    def sec(off, nbytes, dtype):
        return record[off:off + nbytes].view(dtype)

    ng, nc, rows = int(d.n_groups), int(d.n_chan), int(d.rows)
    return {
        "codes": sec(d.codes_off, d.codes_bytes, torch.uint8),
        "scales": sec(d.scales_off, d.scales_bytes, torch.uint8),
        "g": sec(d.g_off, 4 * ng, torch.float32),
        "group_off": sec(d.group_off_off, 4 * (ng + 1), torch.int32) if ng > 1 else None,
        "chan": sec(d.chan_off, 4 * nc, torch.int32) if nc else None,
        "resid": sec(d.resid_off, 2 * nc * rows, torch.bfloat16) if nc else None,
    }


def _src_array(tensors):
    arr = (TraceQTensorSrc * TRACE_MAX_TENSORS)()
    for i, t in enumerate(tensors):
        if t is not None:
            arr[i] = t
    return arr


def trace_qrecord_layout(layer_id, T, k, tensors):
    hdr = TraceQRecordHeader()
    arr = _src_array(tensors)
    n = int(load().trace_qrecord_layout(layer_id, T, k, ctypes.cast(arr, c_vp), len(tensors), ctypes.byref(hdr)))
    if n == 0:
        raise QuadsError(ERR_INVALID_ARG, "trace_qrecord_layout", "invalid record description")
    return n, hdr


def trace_export_qrecord(layer_id, T, k, topk_idx, tensors, record=None):
    n, _ = trace_qrecord_layout(layer_id, T, k, tensors)
    dev = torch.device("cuda", torch.cuda.current_device())
    record = record if record is not None else _empty((n,), torch.uint8, dev)
    arr = _src_array(tensors)
    _check(load().trace_export_qrecord(layer_id, T, k, _p(topk_idx), ctypes.cast(arr, c_vp), len(tensors),
                                       _p(record), record.numel(), _s()), "trace_export_qrecord")
    return record


def trace_replay_qrecord(record, layer_id, which, rows, K, x_train=None, x_hat=None, counts=None, status=None):
    dev = record.device
    x_hat = x_hat if x_hat is not None else _empty((rows, K), torch.bfloat16, dev)
    if x_train is not None and counts is None:
        counts = torch.zeros(2, dtype=torch.int64, device=dev)
    status = status if status is not None else _empty((1,), torch.int32, dev)
    _check(load().trace_replay_qrecord(_p(record), record.numel(), layer_id, which, rows, K, _p(x_train),
                                       _p(x_hat), _p(counts), _p(status), _s()), "trace_replay_qrecord")
    return x_hat, counts, status


# ------------------------------------------------------------ layer stacking


def trace_direction_bits(x, codes, scales, scale_layout, g, group_off=None, n_groups=1, bits=None):
    """One rounding-direction bit per element of the rollout's quantization
    of x: returns bits [rows, K/8] u8."""
    _dev(x, torch.bfloat16, "x")
    rows, K = x.shape
    bits = bits if bits is not None else _empty((rows, K // 8), torch.uint8, x.device)
    _check(load().trace_direction_bits(_p(x), rows, K, _p(codes), _p(scales), scale_layout, _p(g), _p(group_off),
                                       n_groups, _p(bits), _s()), "trace_direction_bits")
    return bits


def trace_replay_direction(bits, scales, scale_layout, g, x_train, group_off=None, n_groups=1, chan=None,
                           resid=None, x_hat=None, codes_out=None, corrections=None):
    """The trainer's rounding of x_train guided by the recorded directions.
    Returns (x_hat, codes_out or None, corrections or None)."""
    _dev(x_train, torch.bfloat16, "x_train")
    rows, K = x_train.shape
    n_chan = 0 if chan is None else int(chan.numel())
    x_hat = x_hat if x_hat is not None else _empty((rows, K), torch.bfloat16, x_train.device)
    _check(load().trace_replay_direction(_p(bits), _p(scales), scale_layout, _p(g), _p(group_off), n_groups, rows, K,
                                         _p(x_train), _p(chan), n_chan, _p(resid) if n_chan else None, _p(x_hat),
                                         _p(codes_out), _p(corrections), _s()), "trace_replay_direction")
    return x_hat, codes_out, corrections


def copy_f32(src, dst):
    _check(load().quads_copy_f32(_p(src), _p(dst), src.numel(), _s()), "quads_copy_f32")
    return dst


def router_logits(x, w_r, out=None):
    """logits [T, E] f32 = x [T, H] bf16 . w_r [H, E] f32."""
    _dev(x, torch.bfloat16, "x")
    _dev(w_r, torch.float32, "w_r")
    T, H = x.shape
    E = w_r.shape[1]
    out = out if out is not None else _empty((T, E), torch.float32, x.device)
    _check(load().quads_router_logits(_p(x), T, H, _p(w_r), E, _p(out), _s()), "quads_router_logits")
    return out


def residual_add(x, y, out=None):
    """out = bf16(x + y), elementwise (out may be x)."""
    _dev(x, torch.bfloat16, "x")
    _dev(y, torch.bfloat16, "y")
    out = out if out is not None else torch.empty_like(x)
    _check(load().quads_residual_add(_p(x), _p(y), x.numel(), _p(out), _s()), "quads_residual_add")
    return out
