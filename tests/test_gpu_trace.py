"""TRACE record export and trainer replay against the CPU oracle (replayed
operand bit-exact, mismatch counts exact), record validation, and the
bounded-wait timeout path (a barrier nothing completes)."""
import numpy as np
import pytest
import torch

from oracle import formats as F
from oracle import moe as M
from oracle import nvfp4 as Q
from oracle import trace as TR
from tests.helpers import assert_bits_equal, bf16_np, bf16_torch, f32_of

pytestmark = pytest.mark.gpu


def _setup(seed=0, T=300, K=256, E=4, k=2, F_=128):
    r = np.random.default_rng(seed)
    x = r.standard_normal((T, K))
    x[:, [3, 50]] *= 20
    x = F.bf16_rne(x.astype(np.float32))
    chan = Q.pad_channels(np.array([3, 50, 51]))
    c, s, g = Q.quantize(x)
    resid = Q.residual_channels(x, c, s, g, chan)
    idx, _ = M.router_topk(r.standard_normal((T, E)), k)
    off, _, _ = M.permute(idx, E)
    R = int(off[-1])
    h = F.bf16_rne((r.standard_normal((R, F_)) * 0.5).astype(np.float32))
    ch, sh, gh = Q.quantize_grouped(h, off)
    chan_h = Q.pad_channels(np.array([7]))
    return dict(x=x, chan=chan, c=c, s=s, g=g, resid=resid, idx=idx, off=off, R=R, h=h, ch=ch, sh=sh, gh=gh,
                chan_h=chan_h, T=T, K=K, E=E, k=k, F=F_)


def _export(lib, d, layer_id=5):
    dev = "cuda"
    t0 = lib.qtensor_src(torch.from_numpy(F.pack_nibbles(d["c"])).to(dev), torch.from_numpy(d["s"]).to(dev),
                         torch.tensor([d["g"]], dtype=torch.float32, device=dev), d["T"], d["K"], lib.SCALES_LINEAR,
                         chan=torch.from_numpy(d["chan"]).to(dev), resid=bf16_torch(d["resid"]))
    resid_h = np.zeros((d["R"], len(d["chan_h"])))             # h's residual slot: zeros (BF16)
    t1 = lib.qtensor_src(torch.from_numpy(F.pack_nibbles(d["ch"])).to(dev),
                         torch.from_numpy(F.scales_to_tiled(d["sh"])).to(dev),
                         torch.tensor(d["gh"], dtype=torch.float32, device=dev), d["R"], d["F"], lib.SCALES_TILED,
                         group_off=torch.from_numpy(d["off"]).to(dev), chan=torch.from_numpy(d["chan_h"]).to(dev),
                         resid=bf16_torch(resid_h))
    idx = torch.from_numpy(d["idx"].astype(np.int32)).to(dev)
    rec = lib.trace_export_qrecord(layer_id, d["T"], d["k"], idx, [t0, t1])
    torch.cuda.synchronize()
    return rec, resid_h


def test_export_replay_roundtrip(cuda_lib):
    d = _setup()
    rec, resid_h = _export(cuda_lib, d)
    # the rollout's own input replays with zero mismatches
    x_hat, counts, status = cuda_lib.trace_replay_qrecord(rec, 5, 0, d["T"], d["K"], x_train=bf16_torch(d["x"]))
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    assert f32_of(counts).tolist() == [0, 0]
    r0 = TR.export_tensor(d["c"], d["s"], d["g"], chan=d["chan"], resid=d["resid"])
    xh_ref, _, _ = TR.replay_tensor(r0)
    assert_bits_equal(F.bf16_bits(bf16_np(x_hat)), F.bf16_bits(xh_ref), "x_hat")
    # expert-ordered h with one scale per expert, tiled scales
    h_hat, _, status = cuda_lib.trace_replay_qrecord(rec, 5, 1, d["R"], d["F"])
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    r1 = TR.export_tensor(d["ch"], d["sh"], d["gh"], group_off=d["off"], chan=d["chan_h"], resid=resid_h)
    hh_ref, _, _ = TR.replay_tensor(r1)
    assert_bits_equal(F.bf16_bits(bf16_np(h_hat)), F.bf16_bits(hh_ref), "h_hat")
    # the routing section holds the exported top-k indices
    raw = rec.cpu().numpy()
    # locate the index section through the device-written header
    off_idx = int(np.frombuffer(raw[:64].tobytes(), dtype=np.uint64)[4])
    got_idx = np.frombuffer(raw[off_idx:off_idx + 4 * d["T"] * d["k"]].tobytes(), dtype=np.int32)
    assert_bits_equal(got_idx, d["idx"].astype(np.int32).ravel(), "topk idx section")


def test_replay_counts_drift(cuda_lib):
    d = _setup(seed=1)
    rec, _ = _export(cuda_lib, d, layer_id=6)
    r = np.random.default_rng(2)
    x_train = F.bf16_rne((d["x"] + r.standard_normal(d["x"].shape) * 1e-2).astype(np.float32))
    _, counts, status = cuda_lib.trace_replay_qrecord(rec, 6, 0, d["T"], d["K"], x_train=bf16_torch(x_train))
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    r0 = TR.export_tensor(d["c"], d["s"], d["g"], chan=d["chan"], resid=d["resid"])
    _, cm, sm = TR.replay_tensor(r0, x_train)
    assert cm > 0
    assert f32_of(counts).astype(np.int64).tolist() == [cm, sm]


def test_bad_record_is_rejected(cuda_lib):
    d = _setup(seed=2)
    rec, _ = _export(cuda_lib, d, layer_id=7)
    x_hat = torch.full((d["T"], d["K"]), 7.0, dtype=torch.bfloat16, device="cuda")
    # wrong layer id
    _, _, status = cuda_lib.trace_replay_qrecord(rec, 8, 0, d["T"], d["K"], x_hat=x_hat)
    torch.cuda.synchronize()
    assert int(status.item()) == cuda_lib.ERR_BAD_RECORD
    assert torch.all(x_hat == 7.0)
    # wrong shape
    _, _, status = cuda_lib.trace_replay_qrecord(rec, 7, 0, d["T"] - 1, d["K"])
    torch.cuda.synchronize()
    assert int(status.item()) == cuda_lib.ERR_BAD_RECORD
    # corrupted magic
    bad = rec.clone()
    bad[0] ^= 0xFF
    _, _, status = cuda_lib.trace_replay_qrecord(bad, 7, 0, d["T"], d["K"], x_hat=x_hat)
    torch.cuda.synchronize()
    assert int(status.item()) == cuda_lib.ERR_BAD_RECORD
    # truncated record: the header claims more bytes than the buffer holds
    short = rec[:rec.numel() - 256].clone()
    _, _, status = cuda_lib.trace_replay_qrecord(short, 7, 0, d["T"], d["K"], x_hat=x_hat)
    torch.cuda.synchronize()
    assert int(status.item()) == cuda_lib.ERR_BAD_RECORD
    assert torch.all(x_hat == 7.0)


def test_bounded_wait_times_out_and_context_survives(cuda_lib):
    assert cuda_lib.device_status() == cuda_lib.OK
    cuda_lib.selftest_bounded_wait(2_000_000)          # 2 ms on a barrier nothing completes
    assert cuda_lib.device_status() == cuda_lib.ERR_TIMEOUT
    assert cuda_lib.device_status() == cuda_lib.OK     # cleared
    # the context is still usable
    x = torch.ones(16, 32, dtype=torch.bfloat16, device="cuda")
    codes, scales, g, _ = cuda_lib.quantize_nvfp4(x)
    torch.cuda.synchronize()
    assert float(g.item()) == np.float32(1.0 / 2688.0)


# ------------------------------------------- compact rounding-direction record


def _direction_case(rows, K, groups, n_chan, tiled, seed, drift=0.05):
    """Rollout input x (outlier channels, a zero block, a negative-zero
    block), quantized by the oracle (per group when groups is given), the
    trainer's drifted copy, and a channel set."""
    r = np.random.default_rng(seed)
    x = r.standard_normal((rows, K)) * np.exp(0.5 * r.standard_normal((1, K)))
    x[:, r.choice(K, 2, replace=False)] *= 30
    if rows > 2:
        x[1, :16] = 0.0
        x[2, 16:32] = -0.0
    x = F.bf16_rne(x.astype(np.float32))
    if groups is None:
        off = np.array([0, rows])
        c, s, g = Q.quantize(x)
        gs = np.array([g])
    else:
        off = np.asarray(groups)
        c, s, gs = Q.quantize_grouped(x[:off[-1]], off)
        c = np.concatenate([c, np.zeros((rows - off[-1], K), np.uint8)])
        s = np.concatenate([s, np.zeros((rows - off[-1], K // 16), np.uint8)])
    g_rows = np.zeros(rows)
    for i in range(len(off) - 1):
        g_rows[off[i]:off[i + 1]] = gs[i]
    xt = F.bf16_rne(F.f32(x * (1 + drift * r.standard_normal(x.shape))))
    chan = Q.pad_channels(np.sort(r.choice(K, n_chan - 3, replace=False))) if n_chan else None
    resid = None
    if n_chan:
        resid = np.zeros((rows, len(chan)))
        for i in range(len(off) - 1):
            lo, hi = off[i], off[i + 1]
            if hi > lo:
                resid[lo:hi] = Q.residual_channels(x[lo:hi], c[lo:hi], s[lo:hi], gs[i], chan)
    return dict(x=x, xt=xt, c=c, s=s, gs=gs, g_rows=g_rows, off=off, R=int(off[-1]), chan=chan, resid=resid,
                tiled=tiled, grouped=groups is not None)


def _gpu_direction(lib, d):
    dev = "cuda"
    rows, K = d["x"].shape
    layout = lib.SCALES_TILED if d["tiled"] else lib.SCALES_LINEAR
    scales = F.scales_to_tiled(d["s"]) if d["tiled"] else d["s"]
    sc = torch.from_numpy(np.ascontiguousarray(scales)).to(dev)
    g = torch.tensor(d["gs"], dtype=torch.float32, device=dev)
    goff = torch.from_numpy(d["off"].astype(np.int32)).to(dev) if d["grouped"] else None
    n = len(d["gs"])
    bits = torch.full((rows, K // 8), 0xA5, dtype=torch.uint8, device=dev)
    cuda_lib_bits = lib.trace_direction_bits(bf16_torch(d["x"]), torch.from_numpy(F.pack_nibbles(d["c"])).to(dev),
                                             sc, layout, g, group_off=goff, n_groups=n, bits=bits)
    codes = torch.full((rows, K // 2), 0xA5, dtype=torch.uint8, device=dev)
    corr = torch.zeros(1, dtype=torch.int64, device=dev)
    x_hat = torch.full((rows, K), float("nan"), dtype=torch.bfloat16, device=dev)
    chan = torch.from_numpy(d["chan"]).to(dev) if d["chan"] is not None else None
    resid = bf16_torch(d["resid"]) if d["chan"] is not None else None
    lib.trace_replay_direction(cuda_lib_bits, sc, layout, g, bf16_torch(d["xt"]), group_off=goff, n_groups=n,
                               chan=chan, resid=resid, x_hat=x_hat, codes_out=codes, corrections=corr)
    torch.cuda.synchronize()
    assert lib.device_status() == lib.OK
    return cuda_lib_bits.cpu().numpy(), codes.cpu().numpy(), bf16_np(x_hat), int(corr.item())


@pytest.mark.parametrize("rows,K,groups,n_chan,tiled", [
    (64, 64, None, 0, False),                          # one pass, one group
    (333, 1040, None, 32, False),                      # ragged rows, 65 blocks: a partial third pass
    (768, 512, [0, 128, 128, 384, 640], 16, True),     # expert-ordered h: an empty expert, padding rows past the last
    (2048, 1024, None, 32, False),                     # the 2048-token layer input, full size
])
def test_direction_record_parity(cuda_lib, rows, K, groups, n_chan, tiled):
    """The compact record's bits bit for bit against the oracle's, and the
    trainer's guided codes, replayed operand and correction count against
    the oracle's replay of the same bits; rows past the last group are left
    untouched."""
    d = _direction_case(rows, K, groups, n_chan, tiled, seed=rows + K)
    bits, codes, x_hat, corr = _gpu_direction(cuda_lib, d)
    R = d["R"]
    b_ref = TR.direction_bits(d["x"][:R], d["c"][:R], d["s"][:R], d["g_rows"][:R])
    assert_bits_equal(bits[:R], TR.pack_bits(b_ref), "direction bits")
    assert np.all(bits[R:] == 0xA5), "rows past the last group must be untouched"
    c_ref, xh_ref, corr_ref = TR.replay_direction(b_ref, d["s"][:R], d["g_rows"][:R], d["xt"][:R],
                                                  d["chan"], d["resid"][:R] if d["resid"] is not None else None)
    assert_bits_equal(codes[:R], F.pack_nibbles(c_ref), "guided codes")
    assert_bits_equal(F.bf16_bits(x_hat[:R]), F.bf16_bits(xh_ref), "x_hat")
    assert corr == corr_ref
    assert np.all(np.isnan(x_hat[R:]))
    # the rollout's own input replays its codes exactly
    d0 = dict(d, xt=d["x"])
    _, codes0, _, corr0 = _gpu_direction(cuda_lib, d0)
    assert_bits_equal(codes0[:R], F.pack_nibbles(d["c"][:R]), "self-replay codes")
    assert corr0 == 0
