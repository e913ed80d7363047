"""Rollout quantization record (export) and trainer replay.

Oracle module (test infrastructure only, see ``oracle/__init__``).

Method statements followed:
* [TRACE] "L'idée centrale de TRACE": the rollout side's quantization
  results guide the trainer's rounding -- the trainer reproduces the rounding
  that the rollout engine actually did, so that both paths agree; a compact
  cache keeps the mantissa and the scale factors of the deep layers only.
* [TRACE] "Fonctionnement, côté ingénierie": the rollout quantizes and
  records the result; the trainer reads that record during its forward pass
  and uses it to choose the rounding.
* [TRACE] "Impact pour les développeurs": the inference engine exports its
  quantization results and the training framework consumes them.

Readings where the pages are silent:
* What is recorded for one quantized tensor: the 4-bit codes, the E4M3 block
  scales, the FP32 per-tensor scale(s), the BF16 residual on the
  compensation channels, and, per layer, the router's top-k expert indices.
* What the trainer computes from it: x_hat = bf16(fp32(deq(record)) + r) on
  the compensation channels and bf16(deq(record)) elsewhere -- the operand
  the rollout's compensated GEMM effectively multiplied -- and, as a
  diagnostic, how many codes and block scales its own quantization of
  x_train (with the recorded per-tensor scale) would have chosen
  differently.
"""
import numpy as np

from .formats import bf16_rne, f32
from .nvfp4 import BLOCK, dequant_f32, quantize_with_scale


def export_tensor(codes, scales, g, group_off=None, chan=None, resid=None):
    """One recorded tensor: a plain copy of what the rollout quantizer made."""
    rec = {
        "codes": np.array(codes, dtype=np.uint8, copy=True),
        "scales": np.array(scales, dtype=np.uint8, copy=True),
        "g": np.atleast_1d(np.array(g, dtype=np.float64, copy=True)),
        "group_off": None if group_off is None else np.array(group_off, dtype=np.int64),
        "chan": None if chan is None else np.array(chan, dtype=np.int32),
        "resid": None if resid is None else np.array(resid, dtype=np.float64),
    }
    return rec


def row_scales(rec):
    """Per-row per-tensor decode scale of a recorded tensor."""
    rows = rec["codes"].shape[0]
    if rec["group_off"] is None:
        return np.full(rows, float(rec["g"][0]))
    off = rec["group_off"]
    out = np.zeros(rows)
    for i in range(len(off) - 1):
        out[int(off[i]):int(off[i + 1])] = rec["g"][i]
    return out


def replay_tensor(rec, x_train=None):
    """Trainer-side replay of one recorded tensor.

    Returns (x_hat float64 BF16-exact [rows, K], code_mismatches,
    scale_mismatches); the counts are None when x_train is None."""
    codes, scales = rec["codes"], rec["scales"]
    rows, K = codes.shape
    if rec["group_off"] is None:
        bounds = [(0, rows, float(rec["g"][0]))]
    else:
        off = rec["group_off"]
        bounds = [(int(off[i]), int(off[i + 1]), float(rec["g"][i])) for i in range(len(off) - 1)]
    deq32 = np.zeros((rows, K))
    for lo, hi, g in bounds:
        if hi > lo:
            deq32[lo:hi] = dequant_f32(codes[lo:hi], scales[lo:hi], g)
    xh = deq32.copy()
    chan = rec["chan"]
    if chan is not None and rec["resid"] is not None:
        for j, c in enumerate(chan):
            if c >= 0:
                xh[:, c] = f32(deq32[:, c] + rec["resid"][:, j])
    x_hat = bf16_rne(xh)
    if x_train is None:
        return x_hat, None, None
    x_train = np.asarray(x_train, dtype=np.float64)
    cm = 0
    sm = 0
    for lo, hi, g in bounds:
        if hi > lo:
            c2, s2 = quantize_with_scale(x_train[lo:hi], g)
            cm += int(np.count_nonzero(c2 != codes[lo:hi]))
            sm += int(np.count_nonzero(s2 != scales[lo:hi]))
    return x_hat, cm, sm


def n_blocks(rec):
    return rec["codes"].shape[0] * rec["codes"].shape[1] // BLOCK


# ------------------------------------------- compact rounding-direction record
#
# [TRACE] "Fonctionnement, côté ingénierie": on a block-scaled FP4 grid the
# rounding of each value is a discrete choice, up to the grid point above or
# down to the one below, and the trainer uses the rollout's record to make
# the same choice.  [TRACE] "L'idée centrale": the cache keeps the mantissa
# and the scale factors selectively to save memory.
#
# Reading: the compact record keeps, per element, one
# bit -- the rounding direction the rollout took -- in place of the 4-bit
# code, with the block scales and per-tensor scales unchanged.  For an
# element with scaled value y = fp32(x * fp32(1/S)):
#   floor level: the largest E2M1 level <= |y| (6 at and above 6);
#   bit = 1 if the rollout's code magnitude is above that level (rounded up),
#         0 if it equals it (rounded down, or y on the grid, or saturated).
# The trainer, with its own y_t (same recorded S), takes the level at or
# below |y_t| plus the recorded bit (capped at 6), with y_t's sign.  Where
# both sides' values fall between the same two grid levels this is exactly
# the rollout's code; elsewhere it is a neighbour of the trainer's own value.
# Blocks with S == 0 record 0 and replay signed zeros, as the quantizer does.


def _block_inv(scales, g_rows, K):
    """Per-element S and fp32(1/S) (1 where S == 0) from block scales and
    per-row decode scales."""
    from .formats import e4m3_value
    S = f32(e4m3_value(scales) * np.asarray(g_rows, dtype=np.float64)[:, None])
    S = np.repeat(S, BLOCK, axis=1)[:, :K]
    inv = f32(1.0 / np.where(S > 0, S, 1.0))
    return S, inv


def _floor_level_index(a):
    """Index (0..7) of the largest E2M1 level <= a, for a >= 0."""
    from .formats import E2M1_LEVELS
    return np.clip(np.searchsorted(E2M1_LEVELS, a, side="right") - 1, 0, 7)


def direction_bits(x, codes, scales, g_rows):
    """The rollout's rounding direction per element (uint8 0/1, [rows, K])."""
    x = np.asarray(x, dtype=np.float64)
    rows, K = x.shape
    S, inv = _block_inv(scales, g_rows, K)
    y = f32(x * inv)
    lvl = _floor_level_index(np.abs(y))
    up = (np.asarray(codes, dtype=np.int64) & 7) > lvl
    return np.where(S > 0, up, False).astype(np.uint8)


def replay_direction(bits, scales, g_rows, x_train, chan=None, resid=None):
    """Trainer-side replay of a compact record.  Returns (codes [rows, K]
    uint8, x_hat float64 BF16-exact, corrections): corrections counts the
    elements whose guided code differs from the trainer's own nearest-even
    rounding with the same scale."""
    from .formats import e2m1_rne_code
    x_t = np.asarray(x_train, dtype=np.float64)
    rows, K = x_t.shape
    S, inv = _block_inv(scales, g_rows, K)
    y = f32(x_t * inv)
    lvl = np.minimum(_floor_level_index(np.abs(y)) + np.asarray(bits, dtype=np.int64), 7)
    lvl = np.where(S > 0, lvl, 0)
    sign = np.where(S > 0, np.signbit(y), np.signbit(x_t)).astype(np.int64)
    codes = ((sign << 3) | lvl).astype(np.uint8)
    own = np.where(S > 0, e2m1_rne_code(y) & 7, 0)
    corrections = int(np.count_nonzero(own != lvl))
    deq32 = np.zeros((rows, K))
    g = np.asarray(g_rows, dtype=np.float64)
    for r in range(rows):
        deq32[r] = dequant_f32(codes[r:r + 1], scales[r:r + 1], g[r])[0]
    xh = deq32.copy()
    if chan is not None and resid is not None:
        for j, c in enumerate(chan):
            if c >= 0:
                xh[:, c] = f32(deq32[:, c] + np.asarray(resid, dtype=np.float64)[:, j])
    return codes, bf16_rne(xh), corrections


def pack_bits(bits):
    """[rows, K] 0/1 -> [rows, K/8] bytes, element 8j + i in bit i of byte j."""
    b = np.asarray(bits, dtype=np.uint8)
    rows, K = b.shape
    return np.packbits(b.reshape(rows, K // 8, 8), axis=2, bitorder="little").reshape(rows, K // 8)
