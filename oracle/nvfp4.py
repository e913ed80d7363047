"""NVFP4 quantization, dequantization, residual channels, calibration and
weight fake-quantization with a straight-through backward.

Oracle module (test infrastructure only, see ``oracle/__init__``).

Method statements followed:
* [TRACE] "Fonctionnement, côté ingénierie": FP4 formats scale by blocks --
  a small group of values shares one scale factor and each value keeps four
  bits; for every value the rounding direction (up or down on the grid) is
  a discrete choice.
* [format]: blocks are 16 consecutive elements along the reduction axis K,
  the block scale is E4M3, and one FP32 per-tensor scale g sits above them.
  The per-tensor scale is a *decode* scale: value = e2m1 * e4m3 * g.
* [QUADS-fr §2.2.B] / [QUADS-es §2.2.B]: the rollout finds the input
  channels where the FP4 error is largest ("high-residual" channels, a binary
  mask of the top channels by residual magnitude) and adds a correction for
  them to the quantized output.  The residual r = x - deq(q(x)) on those
  channels is that correction's operand.
* [QUADS-fr §2.1], [QUADS-fr §2.2.A]: weights are replicated, so the trainer
  applies the same quantize-dequantize path to its weights (asymmetric
  W4A16 QAT: weights fake-quantized to NVFP4, activations stay BF16, the
  optimizer updates BF16 master weights, every forward sees the rollout's
  discretized weights).  The backward through the fake-quant is the
  straight-through estimator (identity).

Readings where the pages are silent:
* g = fp32(amax / (6 * 448)), so that the largest block scale lands on 448.
* Block scale: d = fp32(6 * g); t = fp32(a_b / d); s_b = E4M3_RN_satfinite(t).
* Element codes: S = fp32(val(s_b) * g); inv = fp32(1 / S);
  q_i = E2M1_RNE(fp32(x_i * inv)).  If S == 0 (an all-zero tensor, or a block
  far below the tensor maximum) every code of the block is a signed zero.
* The residual is computed in float32 and stored as BF16:
  r = bf16(fp32(x - fp32(val(q) * val(s_b) * g))).
"""
import numpy as np

from .formats import (NVFP4_RANGE, bf16_rne, e2m1_rne_code, e2m1_value,
                      e4m3_rn_satfinite_code, e4m3_value, f32)

BLOCK = 16


def tensor_scale(amax):
    """Per-tensor decode scale g = fp32(amax / 2688) for an FP32 amax."""
    return f32(np.float64(amax) / NVFP4_RANGE)


def quantize_with_scale(x, g):
    """Quantize a [rows, K] array (BF16-exact values) with a given per-tensor
    decode scale g.  Returns (codes [rows, K] uint8, scales [rows, K/16]
    uint8 E4M3 codes).  K must be a multiple of 16."""
    x = np.asarray(x, dtype=np.float64)
    rows, K = x.shape
    if K % BLOCK:
        raise ValueError("K must be a multiple of 16")
    g = float(g)
    xb = x.reshape(rows, K // BLOCK, BLOCK)
    a_b = np.max(np.abs(xb), axis=2)
    if g == 0.0:
        s_code = np.zeros(a_b.shape, dtype=np.uint8)
    else:
        d = f32(6.0 * g)
        t = f32(a_b / d)
        s_code = e4m3_rn_satfinite_code(t)
    S = f32(e4m3_value(s_code) * g)
    safe = np.where(S > 0, S, 1.0)
    inv = f32(1.0 / safe)
    y = f32(xb * inv[:, :, None])
    codes = e2m1_rne_code(y)
    zero_blk = (S == 0)[:, :, None]
    signed_zero = (np.signbit(xb).astype(np.uint8) << 3)
    codes = np.where(zero_blk, signed_zero, codes).astype(np.uint8)
    return codes.reshape(rows, K), s_code


def quantize(x, amax=None):
    """NVFP4-quantize one tensor.  amax=None uses max|x| (exact); otherwise a
    calibrated FP32 amax.  Returns (codes, scales, g)."""
    x = np.asarray(x, dtype=np.float64)
    a_t = float(np.max(np.abs(x))) if amax is None else float(f32(amax))
    g = float(tensor_scale(a_t))
    codes, scales = quantize_with_scale(x, g)
    return codes, scales, g


def quantize_grouped(x, group_off, amax=None):
    """Quantize row groups [group_off[i], group_off[i+1]) with one per-tensor
    scale each (used for the expert-ordered SwiGLU output h, one scale per
    expert).  amax: None or an array with one FP32 amax per group.
    Returns (codes, scales, g[n_groups])."""
    x = np.asarray(x, dtype=np.float64)
    n = len(group_off) - 1
    codes = np.zeros(x.shape, dtype=np.uint8)
    scales = np.zeros((x.shape[0], x.shape[1] // BLOCK), dtype=np.uint8)
    gs = np.zeros(n, dtype=np.float64)
    for i in range(n):
        lo, hi = int(group_off[i]), int(group_off[i + 1])
        seg = x[lo:hi]
        if amax is None:
            a_t = float(np.max(np.abs(seg))) if hi > lo else 0.0
        else:
            a_t = float(f32(amax[i]))
        gs[i] = tensor_scale(a_t)
        if hi > lo:
            codes[lo:hi], scales[lo:hi] = quantize_with_scale(seg, gs[i])
    return codes, scales, gs


def dequant_unit(codes, scales):
    """val(q) * val(s_b): the dequantized value without the per-tensor scale.
    Exact in float64 (and in float32 / BF16: at most 6 significant bits)."""
    codes = np.asarray(codes)
    rows, K = codes.shape
    sv = e4m3_value(scales)
    return e2m1_value(codes) * np.repeat(sv, BLOCK, axis=1)[:, :K]


def dequant(codes, scales, g):
    """deq(q) = val(q) * val(s_b) * g, exact in float64."""
    return dequant_unit(codes, scales) * float(g)


def dequant_f32(codes, scales, g):
    """deq(q) rounded once to float32 (what a float32 consumer sees)."""
    return f32(dequant(codes, scales, g))


def residual_f32(x, codes, scales, g):
    """r = fp32(x - fp32(deq)) for every element."""
    return f32(np.asarray(x, dtype=np.float64) - dequant_f32(codes, scales, g))


def residual_channels(x, codes, scales, g, chan):
    """BF16 residual on the selected channels: [rows, len(chan)], entries of
    chan that are negative are padding and give 0."""
    r = bf16_rne(residual_f32(x, codes, scales, g))
    chan = np.asarray(chan, dtype=np.int64)
    out = np.zeros((r.shape[0], len(chan)), dtype=np.float64)
    ok = chan >= 0
    out[:, ok] = r[:, chan[ok]]
    return out


def channel_scores(x, amax=None):
    """Calibration score per input channel: sum over rows of |r| with the
    float32 residual r of the tensor's own quantization ([QUADS-fr §2.2.B]
    ranks channels by residual magnitude; the sum over a calibration batch is
    this oracle's reading of "magnitude")."""
    codes, scales, g = quantize(x, amax)
    r = residual_f32(x, codes, scales, g)
    return np.sum(np.abs(r), axis=0)


def select_channels(scores, n_sel):
    """Top n_sel channels by score (ties: lower index first), returned in
    ascending channel order."""
    scores = np.asarray(scores, dtype=np.float64)
    order = np.lexsort((np.arange(len(scores)), -scores))
    return np.sort(order[:n_sel]).astype(np.int32)


def pad_channels(chan, multiple=16):
    """Pad a channel list with -1 entries to a multiple of ``multiple``."""
    chan = np.asarray(chan, dtype=np.int32)
    n = -(-len(chan) // multiple) * multiple
    out = np.full(n, -1, dtype=np.int32)
    out[:len(chan)] = chan
    return out


def fakequant_weight(w, fold_global=True):
    """Trainer-side weight fake-quant on the rollout's grid [QUADS-fr §2.2.A].

    fold_global=True: W_fq = bf16(val(q) * val(s_b) * g).
    fold_global=False: W_fq = val(q) * val(s_b) (exact in BF16), g separate.
    Returns (w_fq float64 of BF16-exact values, codes, scales, g)."""
    codes, scales, g = quantize(w)
    if fold_global:
        w_fq = bf16_rne(f32(dequant(codes, scales, g)))
    else:
        w_fq = dequant_unit(codes, scales)
    return w_fq, codes, scales, g


def ste_backward(grad_wfq, grad_w=None):
    """Straight-through estimator: dL/dW = dL/dW_fq.  With an existing
    gradient buffer the result is accumulated: bf16(fp32(grad_w + grad_wfq))."""
    g = np.asarray(grad_wfq, dtype=np.float64)
    if grad_w is None:
        return g.copy()
    return bf16_rne(f32(np.asarray(grad_w, dtype=np.float64) + g))
