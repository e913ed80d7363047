"""Mixture-of-Experts expert layer: router top-k, token permutation, the
NVFP4 grouped expert GEMM with residual compensation, SwiGLU, combine.

Oracle module (test infrastructure only, see ``oracle/__init__``).

Method statements followed:
* [QUADS-fr §1] / [QUADS-es §1]: the rollout runs MoE layers with native
  NVFP4 W4A4 GEMMs (4-bit weights, 4-bit activations).
* [QUADS-fr §2.2.B] / [QUADS-es §2.2.B]: on the high-residual channels a
  correction term is computed and added to the quantized output, keeping the
  W4A4 GEMM for the bulk of the work.  Here: Y = g_a g_w (deq_unit(A) .
  deq_unit(W)^T) + R . Wc^T with R the BF16 residual on the channel set C
  and Wc the weight columns of C (an operand: by default the dequantized
  weights, so that selecting every channel gives exactly X . deq(W)^T).
* [TRACE] "Fonctionnement, côté ingénierie": the router's choice of experts
  is discrete, so small numeric differences can change which experts run.

Readings where the pages are silent:
* Router: experts ordered by (logit descending, index ascending), first k
  taken; weights are the softmax over the k selected logits (renorm=True) or
  the full softmax restricted to them (renorm=False).
* Permutation: stable counting sort of the (token, slot) pairs by expert in
  increasing token*k + slot order; each expert's segment is padded to a
  multiple of 128 rows (the tensor-core tile height); pad rows are zero.
* SwiGLU: the gate/up GEMM output row is [gate (F) | up (F)];
  h = silu(gate) * up, silu(v) = v / (1 + exp(-v)).
* Combine: y_t = sum over slots s = 0..k-1 of w[t, s] * Y[row_of[t, s]].
"""
import numpy as np

from .formats import bf16_rne, f32
from .nvfp4 import dequant_unit

PAD = 128


def router_topk(logits, k, renorm=True):
    """Returns (idx [T, k] int32, w [T, k] float64)."""
    l = np.asarray(logits, dtype=np.float64)
    T, E = l.shape
    order = np.argsort(-l, axis=1, kind="stable")      # stable: lower index first on ties
    idx = order[:, :k].astype(np.int32)
    sel = np.take_along_axis(l, idx, axis=1)
    if renorm:
        z = np.exp(sel - sel.max(axis=1, keepdims=True))
        w = z / z.sum(axis=1, keepdims=True)
    else:
        zall = np.exp(l - l.max(axis=1, keepdims=True))
        w = np.take_along_axis(zall, idx, axis=1) / zall.sum(axis=1, keepdims=True)
    return idx, w


def permute(idx, E):
    """Stable counting sort of the flattened (token, slot) pairs by expert.

    Returns (expert_off [E+1] int32, 128-padded; row_of [T*k] int32, the
    expert-ordered row of pair i = t*k + s; src_of [expert_off[E]] int32,
    the token of each expert-ordered row or -1 for a pad row)."""
    flat = np.asarray(idx, dtype=np.int64).reshape(-1)
    k = np.asarray(idx).shape[1]
    counts = np.bincount(flat, minlength=E)
    padded = -(-counts // PAD) * PAD
    off = np.concatenate([[0], np.cumsum(padded)]).astype(np.int32)
    order = np.argsort(flat, kind="stable")            # pairs grouped by expert, in pair order
    first_of = np.concatenate([[0], np.cumsum(counts)])[:-1]
    rank = np.arange(len(flat)) - first_of[flat[order]]
    row_of = np.empty(len(flat), dtype=np.int32)
    row_of[order] = off[flat[order]] + rank
    src_of = np.full(int(off[-1]), -1, dtype=np.int32)
    src_of[row_of] = (np.arange(len(flat)) // k).astype(np.int32)
    return off, row_of, src_of


def gather_rows(a, src_of):
    """Rows of a in expert order; pad rows (src -1) are zero."""
    a = np.asarray(a)
    out = np.zeros((len(src_of),) + a.shape[1:], dtype=a.dtype)
    ok = np.asarray(src_of) >= 0
    out[ok] = a[np.asarray(src_of)[ok]]
    return out


def expert_of_rows(expert_off):
    """Expert index of every row [0, expert_off[-1])."""
    off = np.asarray(expert_off, dtype=np.int64)
    return np.repeat(np.arange(len(off) - 1), np.diff(off))


def grouped_gemm(a_codes, a_scales, g_a, w_codes, w_scales, g_w, expert_off,
                 resid=None, wc=None):
    """For every expert e and its rows [off[e], off[e+1]):
        Y = g_a[e] * g_w[e] * deq_unit(A) . deq_unit(W_e)^T + R . Wc_e^T
    in float64.  a_* are [R, K] codes / [R, K/16] scales (unpacked),
    w_* are [E, N, K] / [E, N, K/16]; g_a is a scalar or [E]; resid is
    [R, nc] (BF16-exact values) and wc [E, N, nc].

    Returns (Y [R, N], absdot [R, N]) where absdot is sum |a*b| over every
    product term, compensation included (the tolerance's scale)."""
    off = np.asarray(expert_off, dtype=np.int64)
    E = len(off) - 1
    g_a = np.broadcast_to(np.asarray(g_a, dtype=np.float64), (E,))
    R = int(off[-1])
    N = np.asarray(w_codes).shape[1]
    Y = np.zeros((R, N))
    absdot = np.zeros((R, N))
    for e in range(E):
        lo, hi = int(off[e]), int(off[e + 1])
        if hi == lo:
            continue
        A = dequant_unit(a_codes[lo:hi], a_scales[lo:hi])
        W = dequant_unit(w_codes[e], w_scales[e])
        G = g_a[e] * float(g_w[e])
        Y[lo:hi] = G * (A @ W.T)
        absdot[lo:hi] = abs(G) * (np.abs(A) @ np.abs(W).T)
        if resid is not None and wc is not None and np.asarray(resid).shape[1] > 0:
            Rr = np.asarray(resid, dtype=np.float64)[lo:hi]
            Wc = np.asarray(wc, dtype=np.float64)[e]
            Y[lo:hi] += Rr @ Wc.T
            absdot[lo:hi] += np.abs(Rr) @ np.abs(Wc).T
    return Y, absdot


def swiglu(y):
    """h = silu(gate) * up with y = [gate | up] along the last axis, float64."""
    y = np.asarray(y, dtype=np.float64)
    F = y.shape[1] // 2
    gate, up = y[:, :F], y[:, F:]
    return gate / (1.0 + np.exp(-gate)) * up


def combine(y, row_of, w, k):
    """y_t = sum_s w[t, s] * Y[row_of[t*k + s]], slots in order, float64."""
    y = np.asarray(y, dtype=np.float64)
    w = np.asarray(w, dtype=np.float64)
    T = w.shape[0]
    rows = np.asarray(row_of).reshape(T, k)
    out = np.zeros((T, y.shape[1]))
    for s in range(k):
        out += w[:, s:s + 1] * y[rows[:, s]]
    return out


def per_token_gap(y_rollout, y_trainer):
    """Per-token L2 distance between two layer outputs, relative to the
    trainer output's norm (a reported diagnostic: no page fixes its value)."""
    a = np.asarray(y_rollout, dtype=np.float64)
    b = np.asarray(y_trainer, dtype=np.float64)
    return np.linalg.norm(a - b, axis=1) / np.maximum(np.linalg.norm(b, axis=1), 1e-30)


def bf16_out(v):
    """Round float64 results to BF16 via float32 (as a BF16 store does)."""
    return bf16_rne(f32(v))


# ------------------------------------------- literal second quantization pass
#
# [QUADS-fr §2.2.B] / [QUADS-es §2.2.B] describe the compensation as a second
# quantization pass over the high-residual channels whose correction is added
# to the quantized output.  Here the residual R and the weight columns Wc are
# themselves NVFP4-quantized and multiplied on the FP4 path.
#
# Reading: Wc_e is quantized per expert with its own
# amax (decode scale g_wc[e]); R is quantized per expert segment with the
# decode scale derived from amax_r[e] = fp32(fp32(G_e / g_wc[e]) * 2688),
# G_e = fp32(g_a g_w[e]), so that g_r g_wc equals G_e up to one rounding and
# the correction shares the main product's per-tensor scale.  The block
# scales of R carry its magnitude.  The layer output is then
#   Y = G_e (deq_unit(A) . deq_unit(W_e)^T + deq_unit(q(R)) . deq_unit(q(Wc_e))^T),
# one FP4 product over the channel-extended reduction axis.


def fp4_comp_amax(g_a, g_w, g_wc):
    """amax_r[e] = fp32(fp32(fp32(g_a g_w[e]) / g_wc[e]) * 2688), 0 where
    g_wc[e] == 0."""
    g_w = np.asarray(g_w, dtype=np.float64)
    g_wc = np.asarray(g_wc, dtype=np.float64)
    G = f32(np.broadcast_to(np.asarray(g_a, dtype=np.float64), g_w.shape) * g_w)
    ratio = np.where(g_wc > 0, f32(G / np.where(g_wc > 0, g_wc, 1.0)), 0.0)
    return f32(ratio * 2688.0)


def fp4_compensation_operands(resid, wc, g_a, g_w, expert_off):
    """NVFP4 operands of the FP4 correction: q(Wc_e) per expert (own amax)
    and q(R) per expert segment with amax_r.  resid [R, nc] and wc [E, N, nc]
    are BF16-exact values (nc a multiple of 16).  Returns (r_codes, r_scales,
    g_r [E], wc_codes [E, N, nc], wc_scales [E, N, nc/16], g_wc [E])."""
    from .nvfp4 import quantize, quantize_grouped
    wc = np.asarray(wc, dtype=np.float64)
    E = wc.shape[0]
    q = [quantize(wc[e]) for e in range(E)]
    wc_codes = np.stack([t[0] for t in q])
    wc_scales = np.stack([t[1] for t in q])
    g_wc = np.array([t[2] for t in q])
    amax_r = fp4_comp_amax(g_a, g_w, g_wc)
    r_codes, r_scales, g_r = quantize_grouped(resid, expert_off, amax=amax_r)
    return r_codes, r_scales, g_r, wc_codes, wc_scales, g_wc


def grouped_gemm_fp4_comp(a_codes, a_scales, g_a, w_codes, w_scales, g_w, expert_off, r_codes, r_scales,
                          wc_codes, wc_scales):
    """Y = G_e (A . W_e^T + q(R) . q(Wc_e)^T) on the NVFP4 values: the
    grouped GEMM over the reduction axis extended by the channel columns.
    Returns (Y, absdot) as grouped_gemm does."""
    a_c = np.concatenate([np.asarray(a_codes), np.asarray(r_codes)], axis=1)
    a_s = np.concatenate([np.asarray(a_scales), np.asarray(r_scales)], axis=1)
    w_c = np.concatenate([np.asarray(w_codes), np.asarray(wc_codes)], axis=2)
    w_s = np.concatenate([np.asarray(w_scales), np.asarray(wc_scales)], axis=2)
    return grouped_gemm(a_c, a_s, g_a, w_c, w_s, g_w, expert_off)


# ------------------------------------------------ trainer-side W4A16 GEMM
#
# [QUADS-fr §2.2.A]: the trainer keeps BF16 activations and multiplies them
# by its fake-quantized weights W_fq = bf16(deq(q(W))), the rollout's grid.
# Given the weights as their NVFP4 codes, scales and per-expert scale:
#   Y[r] = X[r] . W_fq[e]^T for every row r of expert e's segment,
# with W_fq = bf16(fp32(val(q) val(s) g_w[e])) (the folded fake-quant).


def grouped_gemm_w4a16(x, w_codes, w_scales, g_w, expert_off):
    """Returns (Y [R, N] float64, absdot [R, N]) for BF16-exact x [R, K]."""
    from .nvfp4 import dequant
    x = np.asarray(x, dtype=np.float64)
    off = np.asarray(expert_off, dtype=np.int64)
    E = len(off) - 1
    R = int(off[-1])
    N = np.asarray(w_codes).shape[1]
    Y = np.zeros((R, N))
    absdot = np.zeros((R, N))
    for e in range(E):
        lo, hi = int(off[e]), int(off[e + 1])
        if hi == lo:
            continue
        w_fq = bf16_rne(f32(dequant(w_codes[e], w_scales[e], float(g_w[e]))))
        Y[lo:hi] = x[lo:hi] @ w_fq.T
        absdot[lo:hi] = np.abs(x[lo:hi]) @ np.abs(w_fq).T
    return Y, absdot
