"""One MoE expert layer on both sides, composed from the oracle's steps, with
BF16 storage at the same points as the CUDA path (the gate/up output, h and
the layer output are BF16 tensors there).

Oracle module (test infrastructure only, see ``oracle/__init__``).
Follows [QUADS-fr §1, §2.2.A, §2.2.B] and [TRACE] as the step modules do.
"""
import numpy as np

from . import moe as M
from . import nvfp4 as Q
from . import trace as TR
from .formats import bf16_rne, f32


def weight_sync(w, chan):
    """Per expert: fake-quantized W (BF16), codes, scales, g and the
    compensation columns (BF16 dequantized weight at the channels)."""
    E = w.shape[0]
    out = {"w_fq": [], "codes": [], "scales": [], "g": np.zeros(E), "wc": []}
    for e in range(E):
        w_fq, c, s, g = Q.fakequant_weight(w[e], fold_global=True)
        out["w_fq"].append(w_fq)
        out["codes"].append(c)
        out["scales"].append(s)
        out["g"][e] = g
        wc = np.zeros((w.shape[1], len(chan)))
        ok = np.asarray(chan) >= 0
        wc[:, ok] = w_fq[:, np.asarray(chan)[ok]]
        out["wc"].append(wc)
    for key in ("w_fq", "codes", "scales", "wc"):
        out[key] = np.stack(out[key])
    return out


def rollout_forward(x, logits, wgu, wd, chan_x, chan_h, k, renorm=True):
    """Returns a dict with every intermediate and the layer output (float64
    arrays of BF16-exact values where the CUDA path stores BF16)."""
    E = wgu["codes"].shape[0]
    F = wgu["codes"].shape[1] // 2
    cx, sx, gx = Q.quantize(x)
    rx = Q.residual_channels(x, cx, sx, gx, chan_x)
    idx, w = M.router_topk(logits, k, renorm)
    off, row_of, src_of = M.permute(idx, E)
    ac, as_, ar = M.gather_rows(cx, src_of), M.gather_rows(sx, src_of), M.gather_rows(rx, src_of)
    y1, absdot1 = M.grouped_gemm(ac, as_, gx, wgu["codes"], wgu["scales"], wgu["g"], off, ar, wgu["wc"])
    y1b = bf16_rne(f32(y1))
    h = bf16_rne(f32(M.swiglu(y1b)))
    ch, sh, gh = Q.quantize_grouped(h, off)
    rh = np.zeros((h.shape[0], len(chan_h)))
    for e in range(E):
        lo, hi = int(off[e]), int(off[e + 1])
        if hi > lo:
            rh[lo:hi] = Q.residual_channels(h[lo:hi], ch[lo:hi], sh[lo:hi], gh[e], chan_h)
    y2, absdot2 = M.grouped_gemm(ch, sh, gh, wd["codes"], wd["scales"], wd["g"], off, rh, wd["wc"])
    y2b = bf16_rne(f32(y2))
    out = M.combine(y2b, row_of, w, k)
    return dict(cx=cx, sx=sx, gx=gx, rx=rx, idx=idx, w=w, off=off, row_of=row_of, src_of=src_of, y1=y1,
                absdot1=absdot1, h=h, ch=ch, sh=sh, gh=gh, rh=rh, y2=y2, absdot2=absdot2, out=out, F=F)


def trainer_replay(fwd, x_train, chan_x, chan_h):
    rec_x = TR.export_tensor(fwd["cx"], fwd["sx"], fwd["gx"], chan=chan_x, resid=fwd["rx"])
    rec_h = TR.export_tensor(fwd["ch"], fwd["sh"], fwd["gh"], group_off=fwd["off"], chan=chan_h, resid=fwd["rh"])
    x_hat, cm, sm = TR.replay_tensor(rec_x, x_train)
    h_hat, _, _ = TR.replay_tensor(rec_h)
    return x_hat, h_hat, cm, sm


def step(x, logits, x_train, w_gu, w_d, chan_x, chan_h, k, grad_gu_fq=None, grad_gu=None):
    """One pass of the whole path (weight sync, rollout forward, record,
    replay, straight-through backward) over one batch."""
    wgu = weight_sync(w_gu, chan_x)
    wd = weight_sync(w_d, chan_h)
    fwd = rollout_forward(x, logits, wgu, wd, chan_x, chan_h, k)
    x_hat, h_hat, cm, sm = trainer_replay(fwd, x_train, chan_x, chan_h)
    g = None
    if grad_gu_fq is not None:
        g = Q.ste_backward(grad_gu_fq, grad_gu)
    return dict(fwd=fwd, x_hat=x_hat, h_hat=h_hat, code_mismatches=cm, scale_mismatches=sm, grad=g,
                wgu=wgu, wd=wd)
