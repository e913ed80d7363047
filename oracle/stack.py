"""The operations that join MoE layers into a stack, in float64.

Oracle module (test infrastructure only, see ``oracle/__init__``).  The pages
describe the MoE layer, not the model around it.  The stack is the plainest
one the rest supports: x_{l+1} = x_l + MoE_l(x_l), router logits_l = x_l W_r[l].
"""
import numpy as np

from .formats import bf16_rne, f32


def router_logits(x, w_r):
    """logits [T, E] = x [T, H] . w_r [H, E], exact in float64 (the kernel
    accumulates in FP32).  Returns (logits, sum |x w| per output: the
    tolerance's scale)."""
    x = np.asarray(x, dtype=np.float64)
    w = np.asarray(w_r, dtype=np.float64)
    return x @ w, np.abs(x) @ np.abs(w)


def residual_add(x, y):
    """bf16(fp32(x + y)): the sum of two BF16 values is exact in float64,
    then one FP32 rounding and one BF16 rounding."""
    return bf16_rne(f32(np.asarray(x, dtype=np.float64) + np.asarray(y, dtype=np.float64)))
