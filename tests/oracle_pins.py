"""Pins of the CPU oracle: checks against brute force, library routines, closed
forms and invariants -- never against the oracle itself.

Each ``pin_*`` raises AssertionError on failure.  ``test_oracle_pins.py`` runs
them; ``test_oracle_mutations.py`` plants plausible mistakes in the oracle
and checks that some pin catches each one.
"""
import itertools

import numpy as np
import torch

from oracle import formats as F
from oracle import moe as M
from oracle import nvfp4 as Q
from oracle import stack as ST
from oracle import trace as TR

RNG = np.random.default_rng(12345)

# ---------------------------------------------------------------- formats


def _bf16_grid(lo, hi):
    """Every BF16 value in [lo, hi] (lo >= 0), as float64."""
    bits = np.arange(0, 0x7F80, dtype=np.uint16)
    v = F.bf16_from_bits(bits)
    return v[(v >= lo) & (v <= hi)]


def _f32_neighbours(v):
    v32 = np.asarray(v, dtype=np.float32)
    return np.concatenate([v32, np.nextafter(v32, np.float32(np.inf)),
                           np.nextafter(v32, np.float32(-np.inf))]).astype(np.float64)


def pin_e2m1_levels():
    """Eight non-negative levels per sign ([QUADS-fr §1]) with the E2M1 layout
    1 sign, 2 exponent (bias 1), 1 mantissa bit ([format]), built bit by bit."""
    vals = []
    for code in range(8):
        e, m = code >> 1, code & 1
        vals.append(m * 0.5 if e == 0 else (1 + m / 2) * 2.0 ** (e - 1))
    assert len(set(vals)) == 8
    assert np.array_equal(F.e2m1_value(np.arange(8)), np.array(vals))
    assert np.array_equal(F.e2m1_value(np.arange(8, 16)), -np.array(vals))


def pin_e2m1_rounding_bruteforce():
    """Nearest level by exhaustive distance, ties to the even code, saturation
    at 6, sign kept: every BF16 value in [-8, 8] plus the float32 neighbours
    of every level and every midpoint."""
    lv = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])
    mids = (lv[1:] + lv[:-1]) / 2
    pos = np.concatenate([_bf16_grid(0.0, 8.0), _f32_neighbours(lv), _f32_neighbours(mids),
                          _f32_neighbours(np.array([6.0, 7.0, 7.5, 8.0]))])
    pos = pos[pos >= 0]
    vals = np.concatenate([pos, -pos])
    got = F.e2m1_rne_code(vals)
    for v, c in zip(vals, got):
        a = abs(v)
        if a >= 6.0:
            best = 7
        else:
            d = np.abs(lv - a)
            cand = np.flatnonzero(d == d.min())
            best = int(cand[0]) if len(cand) == 1 else int([i for i in cand if i % 2 == 0][0])
        want = (8 if np.signbit(v) else 0) | best
        assert int(c) == want, (v, int(c), want)


def pin_e2m1_worked_ties():
    table = {0.25: 0, 0.75: 2, 1.25: 2, 1.75: 4, 2.5: 4, 3.5: 6, 5.0: 6, 6.5: 7,
             100.0: 7, 0.2: 0, 0.3: 1, -0.1: 8, -0.0: 8, -5.5: 15}
    for v, c in table.items():
        assert int(F.e2m1_rne_code(np.array([v]))[0]) == c, (v, c)


def pin_e4m3_values_vs_torch():
    codes = torch.arange(256, dtype=torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = F.e4m3_value(np.arange(256))
    assert np.array_equal(np.isnan(ref), np.isnan(got))
    ok = ~np.isnan(ref)
    assert np.array_equal(ref[ok], got[ok])


def pin_e4m3_rounding_vs_torch():
    """Round to nearest even with saturation at 448, against torch's
    float8_e4m3fn cast of the value clamped to 448 (torch's cast rounds to
    nearest even and does not saturate)."""
    tv = F.e4m3_value(np.arange(0, 127))               # non-negative finite codes
    mids = (tv[1:] + tv[:-1]) / 2
    vals = np.concatenate([_bf16_grid(0.0, 480.0), _f32_neighbours(tv), _f32_neighbours(mids),
                           RNG.uniform(0, 500, 20000), RNG.uniform(0, 2 ** -6, 5000),
                           np.array([0.0, 2 ** -10, 2 ** -9, 1e-30, 448.0, 464.0, 1e9])])
    vals = np.asarray(vals, dtype=np.float32).astype(np.float64)
    vals = vals[vals >= 0]
    ref = torch.from_numpy(np.minimum(vals, 448.0).astype(np.float32)).to(
        torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = F.e4m3_rn_satfinite_code(vals)
    bad = np.flatnonzero(ref != got)
    assert bad.size == 0, (vals[bad[:5]], ref[bad[:5]], got[bad[:5]])


def pin_bf16_vs_torch():
    v = np.concatenate([RNG.standard_normal(50000) * 10.0 ** RNG.integers(-8, 8, 50000),
                        # exact ties: 8 kept bits then a lone 1 in bit 15
                        F.bf16_from_bits(RNG.integers(0, 0x7F00, 2000, dtype=np.uint16))
                        * (1 + 2.0 ** -8)])
    v32 = v.astype(np.float32)
    ref = torch.from_numpy(v32).to(torch.bfloat16).to(torch.float64).numpy()
    assert np.array_equal(F.bf16_rne(v32), ref)


def pin_f32_vs_numpy_float32_ops():
    """fp64-then-round emulation equals native float32 arithmetic (IEEE)."""
    a = RNG.standard_normal(20000).astype(np.float32)
    b = (RNG.standard_normal(20000) + 3).astype(np.float32)
    A, B = a.astype(np.float64), b.astype(np.float64)
    assert np.array_equal(F.f32(A * B), (a * b).astype(np.float64))
    assert np.array_equal(F.f32(A / B), (a / b).astype(np.float64))
    assert np.array_equal(F.f32(A - B), (a - b).astype(np.float64))
    assert np.array_equal(F.f32(1.0 / B), (np.float32(1) / b).astype(np.float64))


def pin_nibble_packing():
    codes = np.array([[0x1, 0x2, 0xF, 0x8]], dtype=np.uint8)
    assert F.pack_nibbles(codes).tolist() == [[0x21, 0x8F]]
    c = RNG.integers(0, 16, (7, 32)).astype(np.uint8)
    assert np.array_equal(F.unpack_nibbles(F.pack_nibbles(c)), c)


def pin_scale_tiling():
    """The tiled scale layout: a bijection; each 512-byte tile holds rows
    [128i, 128i+128) x scale columns [4j, 4j+4); the 16 bytes at 16*r hold
    rows r, r+32, r+64, r+96 (4 scales each)."""
    rows, cols = 256, 12
    s = np.arange(rows * cols, dtype=np.int64).reshape(rows, cols)
    tiled_pos = F.scale_tile_offset(*np.meshgrid(np.arange(rows), np.arange(cols), indexing="ij"), cols // 4)
    assert len(np.unique(tiled_pos)) == rows * cols and tiled_pos.max() == rows * cols - 1
    flat = np.empty(rows * cols, dtype=np.int64)
    flat[tiled_pos] = s
    for ti in range(2):
        for tj in range(3):
            tile = flat[(ti * 3 + tj) * 512:(ti * 3 + tj + 1) * 512]
            for r in range(32):
                chunk = tile[16 * r:16 * r + 16].reshape(4, 4)
                for q in range(4):
                    assert np.array_equal(chunk[q], s[128 * ti + r + 32 * q, 4 * tj:4 * tj + 4])
    small = RNG.integers(0, 256, (70, 6)).astype(np.uint8)
    assert np.array_equal(F.scales_from_tiled(F.scales_to_tiled(small), 70, 6), small)


# ---------------------------------------------------------------- quantizer


def _act(rows, K, seed, outliers=3, scale=20.0):
    r = np.random.default_rng(seed)
    x = r.standard_normal((rows, K))
    ch = r.choice(K, outliers, replace=False)
    x[:, ch] *= scale
    return F.bf16_rne(x.astype(np.float32))


def pin_quantize_constant_block():
    """A block of equal values v that holds the tensor maximum is coded as
    all +-6 with scale 448, and dequantizes to v (up to float32 rounding of g)."""
    for v in [1.0, 3.5, 0.0078125, 1000.0, 2.0 ** -20]:
        x = np.full((1, 32), v)
        x[0, 16:] = -v / 3
        codes, scales, g = Q.quantize(x)
        assert g == float(np.float32(np.float32(v) / np.float32(2688.0)))
        assert scales[0, 0] == 0x7E                       # 448
        assert np.all(codes[0, :16] == 7)
        deq = Q.dequant(codes, scales, g)
        assert abs(deq[0, 0] - v) <= 2 ** -22 * v


def pin_quantize_all_zero():
    x = np.zeros((3, 48))
    codes, scales, g = Q.quantize(x)
    assert g == 0.0 and not scales.any() and not codes.any()
    xn = -x
    codes, _, _ = Q.quantize(xn)
    assert np.all(codes == 8)                            # signed zeros keep the sign


def pin_quantize_tiny_block():
    """A block far below the tensor max gets scale 0 and all-zero codes; its
    residual is the input itself."""
    x = np.zeros((1, 32))
    x[0, :16] = 1000.0
    x[0, 16:] = 1e-6 * np.linspace(-1, 1, 16)
    codes, scales, g = Q.quantize(x)
    assert scales[0, 1] == 0
    assert np.all(F.e2m1_value(codes[0, 16:]) == 0)
    r = Q.residual_f32(x, codes, scales, g)
    assert np.array_equal(r[0, 16:], F.f32(x[0, 16:]))


def pin_quantize_error_bound():
    """|x * inv - val(q)| <= half the local E2M1 step for unsaturated elements
    (closed-form grid spacing: 0.5 below 2, 1 in [2, 4), 2 in [4, 6])."""
    x = _act(64, 256, 1)
    codes, scales, g = Q.quantize(x)
    S = F.f32(F.e4m3_value(scales) * g)
    inv = F.f32(1.0 / S)
    y = F.f32(x.reshape(64, 16, 16) * inv[:, :, None]).reshape(64, 256)
    q = F.e2m1_value(codes)
    ay = np.abs(y)
    half = np.where(ay < 2, 0.25, np.where(ay < 4, 0.5, 1.0))
    unsat = ay <= 6.0
    assert np.all(np.abs(y - q)[unsat] <= half[unsat])
    assert np.all(q[~unsat] == np.sign(y[~unsat]) * 6.0)


def pin_quantize_block_scale_definition():
    """Block scale lands where the block max maps to the top of the E2M1 range:
    val(s_b) is within E4M3's relative spacing (1/8) of amax_b / (6 g)."""
    x = _act(32, 512, 2)
    codes, scales, g = Q.quantize(x)
    a_b = np.abs(x.reshape(32, 32, 16)).max(axis=2)
    t = a_b / (6 * g)
    sv = F.e4m3_value(scales)
    ok = t >= 2 ** -6
    assert np.all(np.abs(sv[ok] - t[ok]) <= t[ok] / 16 + 1e-12)
    # the block maximum codes to +-6 (or 4 only at the exact midpoint 5)
    mx = np.abs(F.e2m1_value(codes)).reshape(32, 32, 16).max(axis=2)
    assert np.all(mx[ok] == 6.0)


def pin_quantize_idempotent():
    x = _act(48, 128, 3)
    c1, s1, g1 = Q.quantize(x)
    d = Q.dequant(c1, s1, g1)
    c2, s2, g2 = Q.quantize(d)
    assert g1 == g2 and np.array_equal(s1, s2) and np.array_equal(c1, c2)


def pin_quantize_bruteforce_tiny():
    """Tiny tensors against a per-element loop that follows the definition
    with scalar Python floats rounded through numpy.float32."""
    r = np.random.default_rng(4)
    for trial in range(20):
        x = F.bf16_rne((r.standard_normal((2, 32)) * 10.0 ** r.integers(-3, 3)).astype(np.float32))
        codes, scales, g = Q.quantize(x)
        f = np.float32
        amax = f(max(abs(v) for v in x.ravel()))
        gg = f(amax / f(2688.0))
        assert float(gg) == g
        for i in range(2):
            for b in range(2):
                blk = x[i, 16 * b:16 * b + 16]
                ab = f(max(abs(v) for v in blk))
                t = f(ab / f(f(6.0) * gg)) if gg > 0 else f(0.0)
                # nearest E4M3 by exhaustive search over the 127 finite codes
                tv = F.e4m3_value(np.arange(127))
                d = np.abs(tv - min(float(t), 448.0))
                cand = np.flatnonzero(d == d.min())
                sc = int(cand[0]) if len(cand) == 1 else int([c for c in cand if c % 2 == 0][0])
                assert scales[i, b] == sc, (trial, i, b, scales[i, b], sc)
                S = f(f(tv[sc]) * gg)
                for j in range(16):
                    v = blk[j]
                    if S == 0:
                        want = 8 if np.signbit(v) else 0
                    else:
                        yy = f(f(v) * f(f(1.0) / S))
                        lv = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])
                        a = min(abs(float(yy)), 6.0)
                        dd = np.abs(lv - a)
                        cc = np.flatnonzero(dd == dd.min())
                        idx = int(cc[0]) if len(cc) == 1 else int([c for c in cc if c % 2 == 0][0])
                        want = (8 if np.signbit(yy) else 0) | idx
                    assert codes[i, 16 * b + j] == want


def pin_grouped_quantize_matches_separate():
    x = _act(300, 64, 5)
    off = np.array([0, 128, 128, 300])
    c, s, g = Q.quantize_grouped(x, off)
    for i in range(3):
        lo, hi = off[i], off[i + 1]
        if hi > lo:
            c1, s1, g1 = Q.quantize(x[lo:hi])
            assert g[i] == g1 and np.array_equal(c[lo:hi], c1) and np.array_equal(s[lo:hi], s1)
        else:
            assert g[i] == 0.0


def pin_residual_definition():
    x = _act(16, 64, 6)
    c, s, g = Q.quantize(x)
    chan = np.array([3, 17, 40, -1])
    r = Q.residual_channels(x, c, s, g, chan)
    for i in range(16):
        for j, ch in enumerate(chan):
            if ch < 0:
                assert r[i, j] == 0
                continue
            f = np.float32
            dq = f(f(F.e2m1_value(c[i, ch]) * F.e4m3_value(s[i, ch // 16])) * f(g))
            rr = f(f(x[i, ch]) - dq)
            want = torch.tensor(float(rr), dtype=torch.float32).to(torch.bfloat16).item()
            assert r[i, j] == want


def pin_channel_selection():
    x = _act(64, 128, 7, outliers=4, scale=30.0)
    sc = Q.channel_scores(x)
    c, s, g = Q.quantize(x)
    deq = Q.dequant_f32(c, s, g)
    brute = [sum(abs(float(np.float32(np.float32(x[i, j]) - np.float32(deq[i, j])))) for i in range(64))
             for j in range(128)]
    assert np.allclose(sc, brute, rtol=1e-12, atol=0)
    sel = Q.select_channels(sc, 8)
    want = sorted(sorted(range(128), key=lambda j: (-brute[j], j))[:8])
    assert sel.tolist() == want
    tied = Q.select_channels(np.array([1.0, 2.0, 2.0, 2.0, 0.5]), 2)
    assert tied.tolist() == [1, 2]


def pin_fakequant_grid():
    """Weight fake-quant lands on the rollout's grid: the unit form is exact
    E2M1 x E4M3 products and re-quantizes to the same codes and scales; the
    folded form is the BF16 rounding of those products times g."""
    w = F.bf16_rne((np.random.default_rng(8).standard_normal((32, 64)) * 0.02).astype(np.float32))
    wu, c, s, g = Q.fakequant_weight(w, fold_global=False)
    c2, s2, g2 = Q.quantize(wu)
    assert np.array_equal(c, c2) and np.array_equal(s, s2) and g2 == 1.0
    wf, c3, s3, g3 = Q.fakequant_weight(w, fold_global=True)
    ref = torch.from_numpy((wu * g).astype(np.float32)).to(torch.bfloat16).to(torch.float64).numpy()
    assert np.array_equal(wf, ref)


def pin_ste():
    a = F.bf16_rne(RNG.standard_normal(1000).astype(np.float32))
    b = F.bf16_rne(RNG.standard_normal(1000).astype(np.float32))
    assert np.array_equal(Q.ste_backward(a), a)
    ref = (torch.from_numpy(a.astype(np.float32)).to(torch.bfloat16)
           + torch.from_numpy(b.astype(np.float32)).to(torch.bfloat16)).to(torch.float64).numpy()
    assert np.array_equal(Q.ste_backward(a, grad_w=b), ref)


# ---------------------------------------------------------------- MoE


def pin_router_bruteforce():
    r = np.random.default_rng(9)
    for E, k in [(8, 2), (16, 4), (5, 5)]:
        l = np.round(r.standard_normal((50, E)) * 2) / 2          # many ties
        l = l.astype(np.float32).astype(np.float64)
        idx, w = M.router_topk(l, k)
        for t in range(50):
            want = sorted(range(E), key=lambda e: (-l[t, e], e))[:k]
            assert idx[t].tolist() == want
            ex = [np.exp(l[t, e]) for e in want]
            assert np.allclose(w[t], np.array(ex) / sum(ex), rtol=1e-13)
        if k == E:
            from scipy.special import softmax
            assert np.allclose(np.sort(w, axis=1), np.sort(softmax(l, axis=1), axis=1), rtol=1e-12)
        _, w2 = M.router_topk(l, k, renorm=False)
        from scipy.special import softmax
        full = softmax(l, axis=1)
        assert np.allclose(w2, np.take_along_axis(full, idx, axis=1), rtol=1e-12)


def pin_permute_bruteforce():
    r = np.random.default_rng(10)
    for T, E, k in [(37, 5, 2), (300, 8, 3), (1, 4, 1)]:
        idx = np.stack([r.choice(E, k, replace=False) for _ in range(T)]).astype(np.int32)
        off, row_of, src_of = M.permute(idx, E)
        pos = 0
        for e in range(E):
            assert off[e] == pos
            pairs = [(t, s) for t in range(T) for s in range(k) if idx[t, s] == e]
            for j, (t, s) in enumerate(pairs):
                assert row_of[t * k + s] == pos + j
                assert src_of[pos + j] == t
            n = len(pairs)
            padded = (n + 127) // 128 * 128
            assert np.all(src_of[pos + n:pos + padded] == -1)
            pos += padded
        assert off[E] == pos


def _tiny_quantized(rows, K, seed, E=None):
    r = np.random.default_rng(seed)
    shape = (rows, K) if E is None else (E, rows, K)
    codes = r.integers(0, 16, shape).astype(np.uint8)
    scales = r.integers(0, 0x7F, shape[:-1] + (K // 16,)).astype(np.uint8)
    return codes, scales


def pin_gemm_bruteforce():
    """Quadruple loop over experts, rows, columns and K on tiny inputs."""
    E, K, N, nc = 3, 32, 5, 2
    off = np.array([0, 2, 2, 5])
    ac, as_ = _tiny_quantized(5, K, 11)
    wc_, ws_ = _tiny_quantized(N, K, 12, E=E)
    g_a = np.array([0.5, 2.0, 0.25])
    g_w = np.array([1.5, 3.0, 0.125])
    r = np.random.default_rng(13)
    resid = r.standard_normal((5, nc))
    wcomp = r.standard_normal((E, N, nc))
    Y, absdot = M.grouped_gemm(ac, as_, g_a, wc_, ws_, g_w, off, resid, wcomp)
    ev = lambda c: float(F.e2m1_value(c))
    sv = lambda s: float(F.e4m3_value(s))
    for e in range(E):
        for i in range(off[e], off[e + 1]):
            for n in range(N):
                acc = 0.0
                aacc = 0.0
                for kk in range(K):
                    a = ev(ac[i, kk]) * sv(as_[i, kk // 16]) * g_a[e]
                    b = ev(wc_[e, n, kk]) * sv(ws_[e, n, kk // 16]) * g_w[e]
                    acc += a * b
                    aacc += abs(a * b)
                for j in range(nc):
                    acc += resid[i, j] * wcomp[e, n, j]
                    aacc += abs(resid[i, j] * wcomp[e, n, j])
                assert abs(Y[i, n] - acc) <= 1e-12 * (1 + aacc)
                assert abs(absdot[i, n] - aacc) <= 1e-12 * (1 + aacc)


def pin_compensation_all_channels_exact():
    """Selecting every channel with the exact residual and Wc = deq(W) gives
    X . deq(W)^T exactly: the compensation adds back all of X - deq(X)."""
    x = _act(40, 64, 14)
    w = F.bf16_rne((np.random.default_rng(15).standard_normal((24, 64)) * 0.02).astype(np.float32))
    cx, sx, gx = Q.quantize(x)
    cw, sw, gw = Q.quantize(w)
    dw = Q.dequant(cw, sw, gw)
    resid = x - Q.dequant(cx, sx, gx)
    off = np.array([0, 40])
    Y, _ = M.grouped_gemm(cx, sx, gx, cw[None], sw[None], np.array([gw]), off, resid, dw[None])
    assert np.allclose(Y, x @ dw.T, rtol=1e-12, atol=1e-12)
    # without compensation: the plain W4A4 product
    Y0, _ = M.grouped_gemm(cx, sx, gx, cw[None], sw[None], np.array([gw]), off)
    assert np.allclose(Y0, Q.dequant(cx, sx, gx) @ dw.T, rtol=1e-12, atol=1e-12)


def pin_swiglu():
    from scipy.special import expit
    y = np.random.default_rng(16).standard_normal((7, 10)) * 4
    h = M.swiglu(y)
    assert np.allclose(h, y[:, :5] * expit(y[:, :5]) * y[:, 5:], rtol=1e-13)
    assert M.swiglu(np.array([[0.0, 3.0]]))[0, 0] == 0.0


def pin_combine():
    r = np.random.default_rng(17)
    T, k, H = 9, 3, 4
    Y = r.standard_normal((40, H))
    row_of = r.permutation(40)[:T * k]
    w = r.random((T, k))
    out = M.combine(Y, row_of, w, k)
    for t in range(T):
        want = sum(w[t, s] * Y[row_of[t * k + s]] for s in range(k))
        assert np.allclose(out[t], want, rtol=1e-14)


# ---------------------------------------------------------------- trace


def pin_replay_roundtrip():
    """Replaying the rollout's own input with the recorded scale reproduces its
    rounding exactly (zero mismatches); the replayed operand with every
    channel compensated is the input up to one BF16 rounding of r."""
    x = _act(64, 64, 18)
    c, s, g = Q.quantize(x)
    chan = np.arange(64)
    resid = Q.residual_channels(x, c, s, g, chan)
    rec = TR.export_tensor(c, s, g, chan=chan, resid=resid)
    x_hat, cm, sm = TR.replay_tensor(rec, x)
    assert cm == 0 and sm == 0
    assert np.array_equal(rec["codes"], c)
    deq = Q.dequant_f32(c, s, g)
    r_exact = F.f32(x - deq)
    assert np.all(np.abs(x_hat - x) <= np.abs(r_exact) * 2 ** -8 + np.abs(x) * 2 ** -8)
    rec0 = TR.export_tensor(c, s, g)
    x0, _, _ = TR.replay_tensor(rec0)
    assert np.array_equal(x0, F.bf16_rne(deq))


def pin_replay_counts_drift():
    x = _act(64, 64, 19)
    c, s, g = Q.quantize(x)
    rec = TR.export_tensor(c, s, g)
    x2 = x.copy()
    x2[0, 0] = -x2[0, 0] if x2[0, 0] != 0 else 1.0          # flips the sign bit of one code
    _, cm, sm = TR.replay_tensor(rec, x2)
    assert cm >= 1
    c2, s2 = Q.quantize_with_scale(x2, g)
    assert cm == int(np.count_nonzero(c2 != c)) and sm == int(np.count_nonzero(s2 != s))
    # halving one block of the trainer's input halves its block maximum: the
    # block's E4M3 scale moves (its codes need not), so exactly one scale
    # mismatch is counted when the halved scale stays a normal E4M3 value
    x3 = x.copy()
    x3[1, 16:32] = x3[1, 16:32] * 0.5
    _, _, sm3 = TR.replay_tensor(rec, x3)
    assert s[1, 1] >= 16 and sm3 == 1, (s[1, 1], sm3)


def _unit_scale_block(vals):
    """One row of 32 values (two blocks) with block scales 1 and decode scale
    1, so the scaled value y equals x."""
    x = np.zeros((1, 32))
    x[0, :len(vals)] = vals
    s1 = F.e4m3_rn_satfinite_code(np.array([[1.0, 1.0]]))
    assert np.all(F.e4m3_value(s1) == 1.0)
    return x, s1.astype(np.uint8), np.array([1.0])


def pin_direction_worked_values():
    """Rounding directions worked by hand on the E2M1 grid (0, .5, 1, 1.5, 2,
    3, 4, 6) with S = 1: nearest level, ties to the even code, saturation at
    6 counts as rounding down; values on the grid round down."""
    cases = [(0.0, 0), (0.25, 0), (0.3, 1), (0.75, 1), (1.0, 0), (1.25, 0), (1.3, 1), (2.5, 0), (2.6, 1),
             (3.5, 1), (5.0, 0), (5.5, 1), (6.0, 0), (7.0, 0), (-3.5, 1), (-0.2, 0), (-1.75, 1)]
    x, s1, g = _unit_scale_block([v for v, _ in cases])
    codes = F.e2m1_rne_code(x)
    bits = TR.direction_bits(x, codes, s1, g)
    assert bits[0, :len(cases)].tolist() == [b for _, b in cases]
    # the trainer's guided choice, worked by hand: (y_t, recorded bit) -> level
    guided = [(3.49, 1, 4.0, True), (3.6, 0, 3.0, True), (3.6, 1, 4.0, False), (0.1, 1, 0.5, True),
              (6.5, 1, 6.0, False), (-2.2, 1, -3.0, True), (1.0, 1, 1.5, True)]
    xt, _, _ = _unit_scale_block([v for v, _, _, _ in guided])
    b = np.zeros((1, 32), dtype=np.uint8)
    b[0, :len(guided)] = [bit for _, bit, _, _ in guided]
    c, x_hat, corr = TR.replay_direction(b, s1, g, xt)
    assert F.e2m1_value(c[0, :len(guided)]).tolist() == [lv for _, _, lv, _ in guided]
    assert corr == sum(1 for _, _, _, fixed in guided if fixed)
    assert np.array_equal(x_hat[0, :len(guided)], [lv for _, _, lv, _ in guided])


def pin_direction_replay_reproduces_rounding():
    """With the trainer's input equal to the rollout's, the compact record
    replays the quantizer's codes exactly (zero corrections), including
    signed zeros, saturated blocks and all-zero blocks, and its x_hat equals
    the full record's replay."""
    x = _act(48, 64, 31)
    x[3, :16] = 0.0
    x[4, :16] = -0.0
    x[5, 16:32] = 1e-30
    c, s, g = Q.quantize(x)
    bits = TR.direction_bits(x, c, s, np.full(48, g))
    c2, x_hat, corr = TR.replay_direction(bits, s, np.full(48, g), x)
    assert np.array_equal(c2, c) and corr == 0
    chan = np.array([5, 17, 40, -1])
    resid = Q.residual_channels(x, c, s, g, chan)
    _, xh_c, _ = TR.replay_direction(bits, s, np.full(48, g), x, chan, resid)
    xr, _, _ = TR.replay_tensor(TR.export_tensor(c, s, g, chan=chan, resid=resid))
    assert np.array_equal(xh_c, xr)


def pin_direction_guided_is_a_neighbour():
    """Brute force on a drifted input: each guided magnitude is the level at
    or below the trainer's |y_t| or the next one up, and it equals the
    rollout's code wherever both values lie between the same two levels."""
    x = _act(32, 64, 32)
    c, s, g = Q.quantize(x)
    xt = F.bf16_rne(F.f32(x * (1 + 0.05 * RNG.standard_normal(x.shape))))
    bits = TR.direction_bits(x, c, s, np.full(32, g))
    c2, _, _ = TR.replay_direction(bits, s, np.full(32, g), xt)
    S = np.repeat(F.f32(F.e4m3_value(s) * g), 16, axis=1)
    yt = F.f32(xt * F.f32(1.0 / np.where(S > 0, S, 1.0)))
    yr = F.f32(x * F.f32(1.0 / np.where(S > 0, S, 1.0)))
    lv = F.E2M1_LEVELS
    for i, j in itertools.product(range(32), range(64)):
        if S[i, j] == 0:
            continue
        fl_t = max(k for k in range(8) if lv[k] <= abs(yt[i, j]))
        fl_r = max(k for k in range(8) if lv[k] <= abs(yr[i, j]))
        assert (c2[i, j] & 7) in (fl_t, min(fl_t + 1, 7))
        if fl_t == fl_r and np.signbit(yt[i, j]) == np.signbit(yr[i, j]):
            assert c2[i, j] == c[i, j], (i, j)


def pin_fp4_compensation_close_to_bf16():
    """The FP4 correction against the BF16 one it stands for, with every
    channel selected and Wc = deq(W): the BF16-compensated output is exactly
    X . deq(W)^T (a closed form), and the FP4-compensated output stays within
    the NVFP4 errors of R and Wc: |sum r wc - sum q(r) q(wc)| <=
    sum |r - q(r)| |wc| + |q(r)| |wc - q(wc)|, with each element error at most
    its block's max times 1/6 (half the widest level gap over the scale) plus
    the E4M3 rounding of the scale.  It also removes most of the plain W4A4
    error."""
    r = np.random.default_rng(41)
    K, N, rows = 64, 32, 40
    x = F.bf16_rne((r.standard_normal((rows, K)) * np.exp(r.standard_normal((1, K)))).astype(np.float32))
    w = F.bf16_rne((r.standard_normal((1, N, K)) * 0.05).astype(np.float32))
    a_c, a_s, g_a = Q.quantize(x)
    w_c, w_s, g_w = Q.quantize(w[0])
    chan = np.arange(K)
    resid = Q.residual_channels(x, a_c, a_s, g_a, chan)
    wdeq = F.bf16_rne(F.f32(Q.dequant(w_c, w_s, g_w)))
    off = np.array([0, rows])
    exact = x @ Q.dequant(w_c, w_s, g_w).T
    y_plain, _ = M.grouped_gemm(a_c, a_s, g_a, w_c[None], w_s[None], [g_w], off)
    rc, rs, g_r, wcc, wcs, g_wc = M.fp4_compensation_operands(resid, wdeq[None], g_a, [g_w], off)
    assert abs(g_r[0] * g_wc[0] / (g_a * g_w) - 1) < 2.0 ** -22
    y4, _ = M.grouped_gemm_fp4_comp(a_c, a_s, g_a, w_c[None], w_s[None], [g_w], off, rc, rs, wcc, wcs)
    qr = Q.dequant(rc, rs, g_r[0])
    qwc = Q.dequant(wcc[0], wcs[0], g_wc[0])
    def elem_err(v):
        m = np.repeat(np.abs(v).reshape(v.shape[0], -1, 16).max(axis=2), 16, axis=1)
        return m / 6.0 * (1 + 2.0 ** -3) + 1e-300
    bound = elem_err(resid) @ np.abs(wdeq).T + np.abs(qr) @ elem_err(wdeq).T
    # the BF16 rounding of the stored residual is inside r itself; the G_e vs
    # g_r g_wc rounding is a relative 2^-22 of the correction
    assert np.all(np.abs(y4 - exact) <= bound * (1 + 2.0 ** -20) + 1e-12 * np.abs(exact).max()
                  + np.abs(resid - F.f32(x - Q.dequant(a_c, a_s, g_a))) @ np.abs(wdeq).T)
    assert np.mean(np.abs(y4 - exact)) < 0.5 * np.mean(np.abs(y_plain - exact))
    # a zero residual contributes nothing
    z = M.fp4_compensation_operands(np.zeros_like(resid), wdeq[None], g_a, [g_w], off)
    y0, _ = M.grouped_gemm_fp4_comp(a_c, a_s, g_a, w_c[None], w_s[None], [g_w], off, z[0], z[1], z[3], z[4])
    assert np.array_equal(y0, y_plain)


def pin_w4a16_gemm_is_fakequant_matmul():
    """The trainer's W4A16 GEMM on the NVFP4 weights is the BF16 matmul of x
    with the pinned weight fake-quant, per expert (torch float64 matmul as
    the library routine); empty experts give no rows."""
    r = np.random.default_rng(43)
    E, N, K = 3, 16, 64
    w = F.bf16_rne((r.standard_normal((E, N, K)) * np.array([0.01, 1.0, 30.0])[:, None, None]).astype(np.float32))
    q = [Q.fakequant_weight(w[e]) for e in range(E)]
    off = np.array([0, 5, 5, 12])
    x = F.bf16_rne(r.standard_normal((12, K)).astype(np.float32))
    y, absdot = M.grouped_gemm_w4a16(x, np.stack([t[1] for t in q]), np.stack([t[2] for t in q]),
                                     [t[3] for t in q], off)
    for e in range(E):
        lo, hi = off[e], off[e + 1]
        ref = torch.matmul(torch.from_numpy(x[lo:hi]), torch.from_numpy(q[e][0]).T).numpy()
        assert np.allclose(y[lo:hi], ref, rtol=0, atol=1e-12 * max(1.0, np.abs(ref).max(initial=0)))
        assert np.all(absdot[lo:hi] >= np.abs(y[lo:hi]))


# ------------------------------------------------------------------ stack


def pin_router_logits_selects_rows():
    """One-hot inputs select rows of W_r; a sum of one-hot rows sums them."""
    H, E = 24, 7
    w = RNG.standard_normal((H, E))
    eye = np.eye(H)
    got, absdot = ST.router_logits(eye, w)
    assert np.array_equal(got, w) and np.array_equal(absdot, np.abs(w))
    two = np.zeros((1, H))
    two[0, [2, 5]] = [1.0, -2.0]
    got, _ = ST.router_logits(two, w)
    assert np.array_equal(got[0], w[2] - 2.0 * w[5])


def pin_router_logits_matches_torch():
    """Against torch's float64 matmul on random inputs."""
    x = RNG.standard_normal((13, 40))
    w = RNG.standard_normal((40, 9))
    got, _ = ST.router_logits(x, w)
    ref = (torch.from_numpy(x) @ torch.from_numpy(w)).numpy()
    assert np.allclose(got, ref, rtol=1e-12, atol=1e-12)


def pin_residual_add_against_torch_rounding():
    """bf16(fp32(x + y)) against torch's FP32 add and BF16 cast, including
    sums that fall on BF16 midpoints and cancellations."""
    x = F.bf16_rne(RNG.standard_normal(4000).astype(np.float32) * 8)
    y = F.bf16_rne(RNG.standard_normal(4000).astype(np.float32) / 64)
    y[:100] = -x[:100]                                   # exact cancellation
    y[100:200] = x[100:200] * 2.0 ** -8                  # midpoint-sized increments
    got = ST.residual_add(x, y)
    ref = (torch.from_numpy(x.astype(np.float32)) + torch.from_numpy(y.astype(np.float32))).to(torch.bfloat16)
    assert np.array_equal(got, ref.to(torch.float64).numpy())


def _golden_blocks(name):
    """Parse a tests/golden fixture: a `levels` line and `block` sections."""
    import os
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", name)
    levels, blocks, cur = None, [], None
    with open(path, encoding="utf-8") as f:
        for line in f:
            line = line.split("#", 1)[0].split()
            if not line:
                continue
            key, vals = line[0], line[1:]
            if key == "levels":
                levels = [float(v) for v in vals]
            elif key == "block":
                cur = {"name": vals[0]}
                blocks.append(cur)
            else:
                cur[key] = [float(v) for v in vals]
    return levels, blocks


def pin_golden_worked_blocks():
    """Hand-worked NVFP4 blocks (tests/golden/nvfp4_worked_blocks.txt, from
    the format's definition; [QUADS-fr §1] for the 8 levels per sign and
    [TRACE] Fonctionnement for rounding to a neighbouring grid point): the
    oracle's level set, block scale codes and element codes, signed zeros
    included."""
    levels, blocks = _golden_blocks("nvfp4_worked_blocks.txt")
    assert len(levels) == 8 and np.array_equal(F.E2M1_LEVELS, np.array(levels))
    assert len(blocks) == 4
    for b in blocks:
        x = np.array(b["x"], dtype=np.float64)[None]
        assert np.array_equal(F.bf16_rne(x), x) and np.array_equal(np.signbit(F.bf16_rne(x)), np.signbit(x))
        codes, scales = Q.quantize_with_scale(x, b["g"][0])
        assert int(scales[0, 0]) == int(b["scale"][0]), (b["name"], scales)
        assert codes[0].astype(int).tolist() == [int(c) for c in b["codes"]], (b["name"], codes)
        if "tensor_amax" in b:
            assert float(Q.tensor_scale(b["tensor_amax"][0])) == b["g"][0]


# ---------------------------------------------------------------- one layer


def _unit_values(codes, scales):
    """val(q) * val(s_b) element by element (the scale of element j is the
    one of block j // 16)."""
    rows, K = codes.shape
    out = np.zeros((rows, K))
    for i in range(rows):
        for j in range(K):
            out[i, j] = float(F.e2m1_value(codes[i, j])) * float(F.e4m3_value(scales[i, j // 16]))
    return out


def _layer_by_token(x, logits, x_train, w_gu, w_d, chan_x, chan_h, k):
    """One MoE layer on both sides recomputed token by token from the
    definitions, with none of the oracle's composition: quantize x with its
    own tensor scale; for each token its top-k experts by (logit desc, index
    asc) and the softmax over them; per selected expert the dequantized
    product with that expert's fake-quantized gate/up weights (own tensor
    scale) plus the BF16 residual of x on C times the BF16 W_fq columns of C;
    BF16 storage of that output; SwiGLU in FP64 stored as BF16; h quantized
    with the scale of its expert's rows (max over every row routed there);
    the down product with the residual of h on C_F times the down W_fq
    columns of C_F; BF16 storage; the weighted sum over the slots in order.
    The trainer side: x_hat = bf16(deq) with bf16(fp32(deq + r)) on C, and
    the counts of codes and scales that x_train's own rounding (same scale)
    changes.  Returns a dict of float64 arrays."""
    T, H = x.shape
    E, F2 = w_gu.shape[0], w_gu.shape[1]
    Fh = F2 // 2
    bf = lambda v: float(F.bf16_rne(F.f32(np.array([v])))[0])

    def fq(w):
        g = float(Q.tensor_scale(np.max(np.abs(w))))
        c, s = Q.quantize_with_scale(w, g)
        unit = _unit_values(c, s)
        return unit, g, F.bf16_rne(F.f32(unit * g))

    wg = [fq(w_gu[e]) for e in range(E)]
    wdn = [fq(w_d[e]) for e in range(E)]
    gx = float(Q.tensor_scale(np.max(np.abs(x))))
    cx, sx = Q.quantize_with_scale(x, gx)
    ux = _unit_values(cx, sx)
    r_x = {}
    for t in range(T):
        for c in chan_x:
            if c >= 0:
                r_x[t, c] = bf(x[t, c] - float(F.f32(ux[t, c] * gx)))
    sel, wts, h_of = {}, {}, {}
    for t in range(T):
        order = sorted(range(E), key=lambda e: (-logits[t, e], e))[:k]
        z = [np.exp(logits[t, e] - logits[t, order[0]]) for e in order]
        sel[t], wts[t] = order, [v / sum(z) for v in z]
        for s, e in enumerate(order):
            unit_w, gw, wfq = wg[e]
            y1 = np.zeros(F2)
            for n in range(F2):
                acc = gx * gw * float(np.dot(ux[t], unit_w[n]))
                for c in chan_x:
                    if c >= 0:
                        acc += r_x[t, c] * wfq[n, c]
                y1[n] = bf(acc)
            h = np.array([bf(y1[j] / (1.0 + np.exp(-y1[j])) * y1[Fh + j]) for j in range(Fh)])
            h_of[t, s] = h
    g_h = np.zeros(E)
    for e in range(E):
        rows = [h_of[t, s] for t in range(T) for s in range(k) if sel[t][s] == e]
        g_h[e] = float(Q.tensor_scale(max(np.max(np.abs(r)) for r in rows))) if rows else 0.0
    out = np.zeros((T, H))
    h_hat = {}
    for t in range(T):
        for s, e in enumerate(sel[t]):
            h = h_of[t, s]
            ch, sh = Q.quantize_with_scale(h[None], g_h[e])
            uh = _unit_values(ch, sh)[0]
            r_h = {c: bf(h[c] - float(F.f32(uh[c] * g_h[e]))) for c in chan_h if c >= 0}
            unit_w, gw, wfq = wdn[e]
            y2 = np.zeros(H)
            for n in range(H):
                acc = g_h[e] * gw * float(np.dot(uh, unit_w[n]))
                for c, r in r_h.items():
                    acc += r * wfq[n, c]
                y2[n] = bf(acc)
            out[t] += wts[t][s] * y2
            hh = np.array([bf(uh[j] * g_h[e]) for j in range(Fh)])
            for c, r in r_h.items():
                hh[c] = bf(float(F.f32(uh[c] * g_h[e])) + r)
            h_hat[t, s] = hh
    x_hat = np.array([[bf(ux[t, j] * gx) for j in range(H)] for t in range(T)])
    for (t, c), r in r_x.items():
        x_hat[t, c] = bf(float(F.f32(ux[t, c] * gx)) + r)
    ct, st = Q.quantize_with_scale(x_train, gx)
    return dict(out=out, h=h_of, h_hat=h_hat, g_h=g_h, x_hat=x_hat, sel=sel,
                code_mismatches=int(np.count_nonzero(ct != cx)), scale_mismatches=int(np.count_nonzero(st != sx)))


def pin_layer_composition_per_token():
    """The oracle's layer composition (weight sync, rollout forward, record,
    replay) against a token-by-token recomputation from the definitions on a
    tiny layer (T = 8, H = F = 32, E = 3, k = 2): routing, every stored h
    row, the per-expert scale of h, the layer output, the replayed x and h
    and the mismatch counts of a drifted trainer input.  [QUADS-fr §2.2.B]
    (compensation on the high-residual channels of each GEMM input),
    [QUADS-fr §2.2.A] (fake-quantized weights on the rollout's grid), [TRACE]
    Fonctionnement (the recorded rounding replayed by the trainer)."""
    from oracle import layer as OL
    T, H, Fh, E, k = 8, 32, 32, 3, 2
    r = np.random.default_rng(77)
    x = F.bf16_rne(F.f32(r.standard_normal((T, H))))
    x[:, 5] *= 16.0
    logits = F.f32(r.standard_normal((T, E)))
    logits[0, 1] = logits[0, 2]                                       # a tie: lower index first
    w_gu = F.bf16_rne(F.f32(r.standard_normal((E, 2 * Fh, H)) * 0.5))
    w_d = F.bf16_rne(F.f32(r.standard_normal((E, H, Fh)) * 0.5))
    w_d[2] *= 8.0                                                     # experts' h scales differ
    x_train = F.bf16_rne(F.f32(x + 0.05 * r.standard_normal((T, H))))
    chan_x = Q.pad_channels(np.array([1, 5, 20]))
    chan_h = Q.pad_channels(np.array([0, 7, 30]))
    ref = _layer_by_token(x, logits, x_train, w_gu, w_d, chan_x, chan_h, k)
    got = OL.step(x, logits, x_train, w_gu, w_d, chan_x, chan_h, k)
    f = got["fwd"]
    assert [list(map(int, f["idx"][t])) for t in range(T)] == [ref["sel"][t] for t in range(T)]
    for t in range(T):
        for s in range(k):
            row = int(f["row_of"][t * k + s])
            assert np.array_equal(f["h"][row], ref["h"][t, s]), ("h", t, s)
            assert np.array_equal(got["h_hat"][row], ref["h_hat"][t, s]), ("h_hat", t, s)
    assert np.array_equal(f["gh"], ref["g_h"]), (f["gh"], ref["g_h"])
    assert len(set(ref["g_h"].tolist())) == E
    assert np.allclose(f["out"], ref["out"], rtol=1e-12, atol=1e-12), np.max(np.abs(f["out"] - ref["out"]))
    assert np.array_equal(got["x_hat"], ref["x_hat"])
    assert (got["code_mismatches"], got["scale_mismatches"]) == (ref["code_mismatches"], ref["scale_mismatches"])
    assert ref["code_mismatches"] > 0


def pin_gather_rows_loop():
    r = np.random.default_rng(78)
    a = r.integers(0, 255, (9, 6)).astype(np.uint8)
    src = np.array([3, -1, 0, 8, -1, 3, 5])
    g = M.gather_rows(a, src)
    for i, s in enumerate(src):
        assert np.array_equal(g[i], a[s] if s >= 0 else np.zeros(6, np.uint8))


def pin_pack_bits_loop():
    r = np.random.default_rng(79)
    b = r.integers(0, 2, (3, 64)).astype(np.uint8)
    p = TR.pack_bits(b)
    for i in range(3):
        for j in range(8):
            assert int(p[i, j]) == sum(int(b[i, 8 * j + q]) << q for q in range(8))


def pin_per_token_gap_closed_forms():
    """The relative per-token distance ||y_r - y_t|| / ||y_t|| on rows built
    to have a known answer: equal rows, scaled rows, an orthogonal step (a
    3-4-5 triangle), and the trainer output as the denominator."""
    r = np.random.default_rng(80)
    yt = r.standard_normal((5, 16))
    assert np.all(M.per_token_gap(yt, yt) == 0.0)
    c = np.array([0.5, -0.25, 2.0, 1e-3, -1.0])
    assert np.allclose(M.per_token_gap(yt * (1.0 + c)[:, None], yt), np.abs(c), rtol=1e-12, atol=0.0)
    yt2 = np.zeros((3, 4))
    yt2[:, 0] = 4.0
    yr2 = yt2.copy()
    yr2[:, 1] = 3.0
    assert np.allclose(M.per_token_gap(yr2, yt2), 0.75, rtol=1e-15, atol=0.0)
    assert np.allclose(M.per_token_gap(yt2, yr2), 0.6, rtol=1e-15, atol=0.0)
    # a token whose two outputs are both zero has no gap
    z = np.zeros((1, 8))
    assert M.per_token_gap(z, z)[0] == 0.0


ALL_PINS = [v for k, v in sorted(globals().items()) if k.startswith("pin_")]
