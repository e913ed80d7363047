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

Readings where the pages are silent (each also listed in the design doc):
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
