"""Plant plausible mistakes in the CPU oracle (monkeypatched, CPU only) and
check that at least one pin catches each of them."""
import numpy as np
import pytest

import inspect
import textwrap

from oracle import formats as F
from oracle import layer as OL
from oracle import moe as M
from oracle import nvfp4 as Q
from oracle import stack as ST
from oracle import trace as TR
from tests import oracle_pins as P


def _e2m1_ties_up(v):
    v = np.asarray(v, dtype=np.float64)
    a = np.abs(v)
    lv = F.E2M1_LEVELS
    lo = np.clip(np.searchsorted(lv, a, side="right") - 1, 0, 7)
    hi = np.minimum(lo + 1, 7)
    up = (lv[hi] - a) <= (a - lv[lo])
    idx = np.where(a >= 6, 7, lo + up)
    return ((np.signbit(v).astype(np.int64) << 3) | idx).astype(np.uint8)


# the unmutated functions, taken before any test patches them (a mutation
# that called the patched name would only recurse)
_orig_e2m1_code = F.e2m1_rne_code
_orig_e4m3_code = F.e4m3_rn_satfinite_code


def _e2m1_no_sign(v):
    return _orig_e2m1_code(np.abs(np.asarray(v, dtype=np.float64)))


def _e4m3_truncate(t):
    t = np.minimum(np.asarray(t, dtype=np.float64), 448.0)
    with np.errstate(divide="ignore"):
        e = np.maximum(np.floor(np.log2(np.where(t > 0, t, 1.0))), -6.0)
    q = np.exp2(e - 3.0)
    return _orig_e4m3_code(np.floor(t / q) * q)


def _tensor_scale_wrong(amax):
    return F.f32(np.float64(amax) / (6.0 * 256.0))


_orig_gemm = M.grouped_gemm


def _gemm_no_comp(a_codes, a_scales, g_a, w_codes, w_scales, g_w, off, resid=None, wc=None):
    return _orig_gemm(a_codes, a_scales, g_a, w_codes, w_scales, g_w, off)


def _gemm_no_gw(a_codes, a_scales, g_a, w_codes, w_scales, g_w, off, resid=None, wc=None):
    return _orig_gemm(a_codes, a_scales, g_a, w_codes, w_scales, np.ones_like(np.asarray(g_w)),
                      off, resid, wc)


def _router_ties_high(logits, k, renorm=True):
    l = np.asarray(logits, dtype=np.float64)
    E = l.shape[1]
    idx, w = M.__dict__["_orig_router"](l[:, ::-1], k, renorm)
    return (E - 1 - idx).astype(np.int32), w


_orig_permute = M.permute


def _permute_reversed(idx, E):
    off, row_of, src_of = _orig_permute(idx, E)
    flat = np.asarray(idx).reshape(-1)
    row2 = row_of.copy()
    for e in range(E):
        sel = np.flatnonzero(flat == e)
        row2[sel] = row_of[sel][::-1]
    src2 = np.full_like(src_of, -1)
    k = np.asarray(idx).shape[1]
    src2[row2] = np.arange(len(flat)) // k
    return off, row2, src2


def _combine_transposed(y, row_of, w, k):
    T = np.asarray(w).shape[0]
    r = np.asarray(row_of).reshape(T, k).T.reshape(-1)[:T * k]
    return M.__dict__["_orig_combine"](y, r.reshape(-1), w, k)


def _resid_sign(x, codes, scales, g):
    return F.f32(Q.dequant_f32(codes, scales, g) - np.asarray(x, dtype=np.float64))


def _bf16_truncate(v):
    u = np.asarray(v, dtype=np.float32).view(np.uint32)
    return ((u >> np.uint32(16)) << np.uint32(16)).view(np.float32).astype(np.float64)


def _swiglu_wrong(y):
    y = np.asarray(y, dtype=np.float64)
    Fh = y.shape[1] // 2
    g, u = y[:, :Fh], y[:, Fh:]
    return u / (1.0 + np.exp(-u)) * g


def _pack_swapped(codes):
    c = np.asarray(codes, dtype=np.uint8)
    return (c[..., 1::2] | (c[..., 0::2] << 4)).astype(np.uint8)


def _select_ties_high(scores, n):
    s = np.asarray(scores, dtype=np.float64)
    order = np.lexsort((-np.arange(len(s)), -s))
    return np.sort(order[:n]).astype(np.int32)


def _div_instead_of_recip(x, g):
    # divides by 2*S: a wrong element scale (dropped factor)
    x = np.asarray(x, dtype=np.float64)
    codes, s = Q.__dict__["_orig_qws"](x * 0.5, g)
    return codes, s


def _floor_level_left(a):
    # an off-by-one at exact grid points: the level strictly below a
    from oracle import formats as FF
    return np.clip(np.searchsorted(FF.E2M1_LEVELS, a, side="left") - 1, 0, 7)


def _guided_ignores_bit(bits, scales, g_rows, x_train, chan=None, resid=None):
    return TR.__dict__["_orig_replay_dir"](np.zeros_like(bits), scales, g_rows, x_train, chan, resid)


def _comp_amax_uses_gw(g_a, g_w, g_wc):
    # the ratio taken against the wrong per-tensor scale
    return M.__dict__["_orig_comp_amax"](g_a, g_w, np.asarray(g_w, dtype=np.float64) * 4.0)


def _w4a16_unfolded(x, w_codes, w_scales, g_w, expert_off):
    # the per-expert scale dropped from W_fq
    return M.__dict__["_orig_w4a16"](x, w_codes, w_scales, np.ones(len(g_w)), expert_off)


def _residual_add_no_bf16(x, y):
    # the BF16 rounding of the sum dropped
    return F.f32(np.asarray(x, dtype=np.float64) + np.asarray(y, dtype=np.float64))


def _router_logits_abs(x, w_r):
    # the magnitude product used for the logits themselves
    x = np.asarray(x, dtype=np.float64)
    w = np.asarray(w_r, dtype=np.float64)
    return np.abs(x) @ np.abs(w), np.abs(x) @ np.abs(w)


def _ste_overwrites(grad_wfq, grad_w=None):
    # the existing gradient dropped instead of accumulated
    return np.asarray(grad_wfq, dtype=np.float64).copy()


def _replay_drops_residual(rec, x_train=None):
    # the recorded residual channels not added back
    return TR.__dict__["_orig_replay"](dict(rec, resid=None), x_train)


def _replay_counts_codes_only(rec, x_train=None):
    # scale mismatches never counted
    x_hat, cm, sm = TR.__dict__["_orig_replay"](rec, x_train)
    return x_hat, cm, (None if sm is None else 0)


def _dequant_unit_drops_scale(codes, scales):
    # the E4M3 block scale left out of the dequantized value
    return F.e2m1_value(np.asarray(codes))


def _source_mutation(func, old, new):
    """A copy of `func` with one source fragment replaced, compiled in the
    function's own module namespace (so the planted slip sits exactly where
    it would in the oracle's code)."""
    src = textwrap.dedent(inspect.getsource(func))
    assert src.count(old) == 1, (func.__name__, old)
    ns = {}
    exec(compile(src.replace(old, new), f"<mutated {func.__name__}>", "exec"), func.__globals__, ns)
    return ns[func.__name__]


# slips in the layer composition: h's residuals taken with one scale for all
# experts instead of the expert's own; the gate/up channel set used for the
# down weights' compensation columns; the gate/up output fed to SwiGLU before
# its BF16 storage rounding
_layer_h_resid_one_scale = _source_mutation(OL.rollout_forward, "sh[lo:hi], gh[e], chan_h)",
                                            "sh[lo:hi], gh.max(), chan_h)")
_layer_down_wc_chan_x = _source_mutation(OL.step, "wd = weight_sync(w_d, chan_h)", "wd = weight_sync(w_d, chan_x)")
_layer_no_bf16_before_swiglu = _source_mutation(OL.rollout_forward, "M.swiglu(y1b)", "M.swiglu(y1)")


def _gap_over_rollout_norm(y_rollout, y_trainer):
    a = np.asarray(y_rollout, dtype=np.float64)
    b = np.asarray(y_trainer, dtype=np.float64)
    return np.linalg.norm(a - b, axis=1) / np.maximum(np.linalg.norm(a, axis=1), 1e-30)


def _gap_squared(y_rollout, y_trainer):
    a = np.asarray(y_rollout, dtype=np.float64)
    b = np.asarray(y_trainer, dtype=np.float64)
    return np.sum((a - b) ** 2, axis=1) / np.maximum(np.sum(b * b, axis=1), 1e-30)


MUTATIONS = {
    "e2m1_ties_away": [(F, "e2m1_rne_code", _e2m1_ties_up), (Q, "e2m1_rne_code", _e2m1_ties_up)],
    "e2m1_drops_sign": [(F, "e2m1_rne_code", _e2m1_no_sign), (Q, "e2m1_rne_code", _e2m1_no_sign)],
    "e4m3_truncates": [(F, "e4m3_rn_satfinite_code", _e4m3_truncate),
                       (Q, "e4m3_rn_satfinite_code", _e4m3_truncate)],
    "tensor_scale_constant": [(Q, "tensor_scale", _tensor_scale_wrong)],
    "gemm_drops_compensation": [(M, "grouped_gemm", _gemm_no_comp)],
    "gemm_drops_weight_scale": [(M, "grouped_gemm", _gemm_no_gw)],
    "router_ties_to_high_index": [(M, "_orig_router", M.router_topk), (M, "router_topk", _router_ties_high)],
    "permute_unstable": [(M, "permute", _permute_reversed)],
    "combine_slot_index": [(M, "_orig_combine", M.combine), (M, "combine", _combine_transposed)],
    "residual_sign": [(Q, "residual_f32", _resid_sign)],
    "bf16_truncates": [(F, "bf16_rne", _bf16_truncate), (Q, "bf16_rne", _bf16_truncate)],
    "swiglu_gate_up_swapped": [(M, "swiglu", _swiglu_wrong)],
    "nibble_order": [(F, "pack_nibbles", _pack_swapped)],
    "channel_ties_to_high_index": [(Q, "select_channels", _select_ties_high)],
    "w4a16_drops_weight_scale": [(M, "_orig_w4a16", M.grouped_gemm_w4a16), (M, "grouped_gemm_w4a16", _w4a16_unfolded)],
    "residual_add_keeps_fp32": [(ST, "residual_add", _residual_add_no_bf16)],
    "router_logits_magnitudes": [(ST, "router_logits", _router_logits_abs)],
    "fp4_comp_wrong_scale": [(M, "_orig_comp_amax", M.fp4_comp_amax), (M, "fp4_comp_amax", _comp_amax_uses_gw)],
    "direction_floor_off_by_one": [(TR, "_floor_level_index", _floor_level_left)],
    "direction_bit_ignored": [(TR, "_orig_replay_dir", TR.replay_direction),
                              (TR, "replay_direction", _guided_ignores_bit)],
    "element_scale_dropped_factor": [(Q, "_orig_qws", Q.quantize_with_scale),
                                     (Q, "quantize_with_scale", _div_instead_of_recip)],
    "ste_overwrites_gradient": [(Q, "ste_backward", _ste_overwrites)],
    "replay_drops_residual": [(TR, "_orig_replay", TR.replay_tensor), (TR, "replay_tensor", _replay_drops_residual)],
    "replay_skips_scale_count": [(TR, "_orig_replay", TR.replay_tensor),
                                 (TR, "replay_tensor", _replay_counts_codes_only)],
    "permute_pads_to_64": [(M, "PAD", 64)],
    "dequant_drops_block_scale": [(Q, "dequant_unit", _dequant_unit_drops_scale)],
    "layer_h_residual_one_scale": [(OL, "rollout_forward", _layer_h_resid_one_scale)],
    "layer_down_wc_from_gate_up_channels": [(OL, "step", _layer_down_wc_chan_x)],
    "layer_swiglu_before_bf16_storage": [(OL, "rollout_forward", _layer_no_bf16_before_swiglu)],
    "gap_over_rollout_norm": [(M, "per_token_gap", _gap_over_rollout_norm)],
    "gap_squared_norms": [(M, "per_token_gap", _gap_squared)],
}


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_mutation_is_caught(name, monkeypatch):
    for mod, attr, fn in MUTATIONS[name]:
        monkeypatch.setattr(mod, attr, fn, raising=False)
    failures = []
    for pin in P.ALL_PINS:
        try:
            pin()
        except AssertionError:
            failures.append(pin.__name__)
    assert failures, f"mutation {name} failed no pin's assertion"
