"""Benchmark of the NVFP4 MoE train/rollout alignment path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--workload NAME]

One step = one pass of the whole path over one batch of the default
workload, the large prefill MoE layer (16384 tokens, hidden 4096, 128
experts top-8 with Zipf(1.1)-skewed router logits, SwiGLU ffn 1536,
Student-t(3) channel scales, 128 + 128 compensation channels): weight sync
(amax + fake-quant of both expert weight tensors, which also writes the
rollout's NVFP4 weights and compensation columns), the rollout forward (amax
+ quantize x with residual channels, router top-k, permutation, gather,
grouped NVFP4 gate/up GEMM with compensation and the SwiGLU epilogue with
per-expert amax, per-expert quantize of h with residual channels, grouped
down GEMM with compensation, combine), the TRACE record export, the trainer
replay of both recorded tensors against the trainer's activation, and the
straight-through backward accumulated into both master gradients.
--workload moe_t2048_h1024_e8k2_f2048 runs the 2048-token, 8-expert layer.

value = FLOPs of the two grouped GEMMs (FP4 products + BF16 compensation,
algorithmic: routed rows only) per step, summed over ranks, / max-over-ranks
step time: step-level throughput.  The `gemm` block gives the grouped GEMMs'
own kernel throughput and its fraction of the dense FP4 peak, which this
run measures on its own GPU with the library's block-scaled NVFP4 GEMM.
Multi-GPU runs are data-parallel replicas (each rank its own batch, no
collective on the path): weak scaling.

--impl reference times the CPU oracle (float64 numpy) on a bounded sample of
the same workload (a slice of the tokens and of the ffn width, sized so that
the whole run takes about two minutes) on the host cores; under torchrun
only rank 0 runs it.
"""
import argparse
import datetime
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "NVFP4 MoE grouped-GEMM TFLOPS (% FP4 peak); quantize/replay GB/s (% HBM)"
UNIT = "TFLOP/s"
DEFAULT_WORKLOAD = "prefill_t16384_h4096_e128k8_f1536"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
FP4_OVER_BF16 = 4.0          # nominal dense ratio (9 / 2.25 PFLOP/s): used only if the FP4 measurement fails
FP4_PEAK_N = 8192            # the library FP4 GEMM is timed at N x N x N
L2_FLUSH_BYTES = 256 << 20


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-sweep", action="store_true", help="skip the standalone quantize/replay size sweep")
    ap.add_argument("--no-secondary", action="store_true",
                    help="skip the other workloads (single linear, 2048-token layer step, 8-layer alignment pass)")
    ap.add_argument("--serial", action="store_true", help="run the step on one stream (no weight-side overlap)")
    ap.add_argument("--comp", choices=["bf16", "fp4"], default="bf16",
                    help="compensation: BF16 R . Wc (default) or the NVFP4 second pass")
    ap.add_argument("--trainer-w4a16", action="store_true",
                    help="the trainer's GEMMs read the NVFP4 codes (W4A16 kernels), so W_fq is not written")
    ap.add_argument("--fuse-requant", action="store_true",
                    help="quantize h in the gate/up GEMM epilogue with the previous step's amax (delayed scaling)")
    return ap.parse_args()


def dist_env():
    return int(os.environ.get("RANK", 0)), int(os.environ.get("WORLD_SIZE", 1)), int(os.environ.get("LOCAL_RANK", 0))


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# Which source files build each kernel of the step; a DRAM-traffic figure
# recorded from an ncu capture is reported only while the hash of these
# files still equals the one recorded with it.
KERNEL_SOURCES = {
    "quantize.cu": ("amax_w", "fakequant_w_gate_up", "fakequant_w_down", "amax_x", "quantize_x", "quantize_h",
                    "quantize_wc_gate_up", "quantize_wc_down", "quantize_r", "quantize_rh"),
    "ste_backward.cu": ("ste_backward",),
    "grouped_gemm.cu": ("gemm_gate_up", "gemm_gate_up_swiglu", "gemm_gate_up_swiglu_quant",
                        "gemm_gate_up_swiglu_fp4comp", "gemm_down", "gemm_down_fp4comp"),
    "moe_route.cu": ("router_topk", "permute", "gather", "swiglu", "combine"),
    "trace_record.cu": ("export", "replay_x", "replay_h"),
}


def source_hash(kernel):
    import hashlib
    csrc = os.path.join(ROOT, "train_alignment_b200", "csrc")
    for src, names in KERNEL_SOURCES.items():
        if kernel in names:
            h = hashlib.sha256()
            for f in (src, "common.cuh"):
                with open(os.path.join(csrc, f), "rb") as fh:
                    h.update(fh.read())
            return h.hexdigest()[:12]
    return None


def recorded_traffic(workload, kernel):
    """DRAM bytes (read + write) per launch of `kernel` from the table in
    profiles/traffic.md, or None when there is no row or the kernel's sources
    changed since the capture."""
    path = os.path.join(ROOT, "profiles", "traffic.md")
    if not os.path.exists(path):
        return None
    want = source_hash(kernel)
    with open(path) as f:
        for line in f:
            cells = [c.strip().strip("`") for c in line.strip().strip("|").split("|")]
            if len(cells) < 6 or cells[0] != workload or cells[1] != kernel:
                continue
            try:
                rd, wr = float(cells[2]), float(cells[3])
            except ValueError:
                continue
            return rd + wr if cells[5] == want else None
    return None


# --------------------------------------------------------------- accounting


def max_over_ranks(v, world, device=None):
    """The slowest rank's value (every rank takes part; NCCL or gloo)."""
    if world == 1:
        return float(v)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(v)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_tflops(flops_per_rank, world, ms):
    """Aggregate throughput: every rank's work over the slowest rank's time."""
    return world * flops_per_rank / (ms * 1e-3) / 1e12


def gemm_flops(cfg, counts=None):
    """Algorithmic FLOPs of both grouped GEMMs for T*k routed rows."""
    R = cfg.T * cfg.k
    fp4 = 2 * R * (2 * cfg.F) * cfg.H + 2 * R * cfg.H * cfg.F
    comp = 2 * R * (2 * cfg.F) * cfg.n_chan + 2 * R * cfg.H * cfg.n_chan_f
    return fp4, comp


def kernel_work(cfg, rpad, wfq=True):
    """Algorithmic bytes (HBM) or FLOPs per launch of every kernel in a step,
    and which roofline bounds it."""
    import ctypes
    from train_alignment_b200 import binding as B
    T, H, E, k, F = cfg.T, cfg.H, cfg.E, cfg.k, cfg.F
    nc, ncf = cfg.n_chan, cfg.n_chan_f
    R = T * k
    wgu = E * 2 * F * H
    wd = E * H * F
    q = 0.5 + 1.0 / 16                      # codes + scales per element
    w = {
        "amax_w": ("hbm", 2.0 * (wgu + wd)),
        "fakequant_w_gate_up": ("hbm", wgu * (2 + (2 if wfq else 0) + q) + E * 2 * F * nc * 2),
        "fakequant_w_down": ("hbm", wd * (2 + (2 if wfq else 0) + q) + E * H * ncf * 2),
        "amax_x": ("hbm", 2.0 * T * H),
        "quantize_x": ("hbm", T * H * (2 + q) + T * nc * 2),
        "router_topk": ("hbm", T * E * 4 + R * 8),
        "permute": ("hbm", R * 4 * 3),
        "gather": ("hbm", (R + T) * (H * q + nc * 2)),
        "gemm_gate_up": ("tensor", 2.0 * R * 2 * F * H + 2.0 * R * 2 * F * nc),
        "gemm_gate_up_swiglu": ("tensor", 2.0 * R * 2 * F * H + 2.0 * R * 2 * F * nc),
        "gemm_gate_up_swiglu_quant": ("tensor", 2.0 * R * 2 * F * H + 2.0 * R * 2 * F * nc),
        "gemm_gate_up_swiglu_fp4comp": ("tensor", 2.0 * R * 2 * F * H + 2.0 * R * 2 * F * nc),
        "gemm_down_fp4comp": ("tensor", 2.0 * R * H * F + 2.0 * R * H * ncf),
        "quantize_wc_gate_up": ("hbm", E * 2 * F * nc * (2 + q)),
        "quantize_wc_down": ("hbm", E * H * ncf * (2 + q)),
        "quantize_r": ("hbm", rpad * nc * (2 + q)),
        "quantize_rh": ("hbm", rpad * ncf * (2 + q)),
        "swiglu": ("hbm", rpad * (2 * F * 2 + F * 2)),
        "quantize_h": ("hbm", rpad * F * (2 + q) + rpad * ncf * 2),
        "gemm_down": ("tensor", 2.0 * R * H * F + 2.0 * R * H * ncf),
        "combine": ("hbm", R * H * 2 + T * H * 2),
        # the step's producers write every recorded section into the record in
        # place, so its export copies no section: it writes the header alone
        "export": ("latency", float(ctypes.sizeof(B.TraceQRecordHeader))),
        "replay_x": ("hbm", T * H * (q + 2 + 2)),
        "replay_h": ("hbm", rpad * F * (q + 2)),
        "ste_backward": ("hbm", (wgu + wd) * 6.0),
    }
    return w


# ------------------------------------------------------------ FP4 peak


def fp4_library_peak(dev, n=FP4_PEAK_N, reps=20, sustain_s=2.0):
    """The dense FP4 tensor peak of this GPU, measured: the library's
    block-scaled NVFP4 GEMM (torch.nn.functional.scaled_mm with E2M1 operands
    and one E4M3 scale per 16 elements, i.e. cuBLASLt) at n x n x n on random
    codes, CUDA events around back-to-back launches.  `burst`: `reps`
    launches after five warm-up ones (the figure for kernels timed alone);
    `sustained`: launches for about `sustain_s` seconds, under the power
    cap."""
    import torch
    import torch.nn.functional as Fn
    from torch.nn.functional import ScalingType, SwizzleType
    gen = torch.Generator(device=dev).manual_seed(4)
    a = torch.randint(0, 256, (n, n // 2), dtype=torch.uint8, device=dev, generator=gen).view(torch.float4_e2m1fn_x2)
    b = torch.randint(0, 256, (n, n // 2), dtype=torch.uint8, device=dev, generator=gen).view(torch.float4_e2m1fn_x2)
    one = 0x38                                           # E4M3 code of 1.0
    sa = torch.full((n * (n // 16),), one, dtype=torch.uint8, device=dev).view(torch.float8_e4m3fn)
    sb = torch.full((n * (n // 16),), one, dtype=torch.uint8, device=dev).view(torch.float8_e4m3fn)

    def gemm():
        return Fn.scaled_mm(a, b.t(), [sa], [ScalingType.BlockWise1x16], [sb], [ScalingType.BlockWise1x16],
                            swizzle_a=[SwizzleType.SWIZZLE_32_4_4], swizzle_b=[SwizzleType.SWIZZLE_32_4_4],
                            output_dtype=torch.bfloat16)

    def timed(count):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(count):
            gemm()
        e1.record()
        e1.synchronize()
        return e0.elapsed_time(e1) / count

    for _ in range(5):
        gemm()
    torch.cuda.synchronize()
    flop = 2.0 * n * n * n
    ms_b = timed(reps)
    ms_s = timed(max(reps, int(sustain_s / (ms_b * 1e-3))))
    del a, b, sa, sb
    return {"burst_tflops": flop / (ms_b * 1e-3) / 1e12, "sustained_tflops": flop / (ms_s * 1e-3) / 1e12,
            "burst_ms": ms_b, "sustained_ms": ms_s, "shape": f"{n}x{n}x{n}",
            "library": "torch.nn.functional.scaled_mm, NVFP4 operands with E4M3 block scales (cuBLASLt)"}


# ------------------------------------------------------ quantize / replay sweep

SWEEP_LOG2 = (20, 22, 24, 26, 28, 30)       # BF16 elements, rows of 4096


def quantize_replay_sweep(dev, hbm_gbs, reps=10):
    """Standalone NVFP4 quantize (amax given: 2 B in, 0.5625 B out per element)
    and TRACE replay with the mismatch count (0.5625 B record + 2 B x_train in,
    2 B x_hat out) on [n / 4096, 4096] BF16 activations with Student-t (nu = 3)
    channel scales.  L2 is flushed before every timed launch; sizes up to 2^24
    elements fit in L2 nonetheless."""
    import torch
    from train_alignment_b200 import binding as B
    from train_alignment_b200 import workloads as W
    out = []
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    for lg in SWEEP_LOG2:
        n = 1 << lg
        rows, K = n // 4096, 4096
        gen = torch.Generator(device=dev).manual_seed(lg)
        x = W.activations(rows, K, "student_t", 0, 1.0, gen, dev)
        amax = B.amax_bf16(x)
        codes = torch.empty(rows, K // 2, dtype=torch.uint8, device=dev)
        scales = torch.empty(B.scales_bytes(rows, K, B.SCALES_LINEAR), dtype=torch.uint8, device=dev)
        g = torch.empty(1, dtype=torch.float32, device=dev)
        q = lambda: B.quantize_nvfp4(x, amax_in=amax, codes=codes, scales=scales, g_out=g)

        def timed(fn):
            return _timed_flushed(fn, flush, reps)

        tq = timed(q)
        src = [B.qtensor_src(codes, scales, g, rows, K, B.SCALES_LINEAR)]
        record = B.trace_export_qrecord(0, rows, 0, None, src)
        x_hat = torch.empty_like(x)
        counts = torch.zeros(2, dtype=torch.int64, device=dev)
        status = torch.empty(1, dtype=torch.int32, device=dev)
        r = lambda: B.trace_replay_qrecord(record, 0, 0, rows, K, x_train=x, x_hat=x_hat, counts=counts,
                                           status=status)
        tr = timed(r)
        torch.cuda.synchronize()
        assert int(status.item()) == 0 and int(counts[0].item()) == 0, "replay of the rollout's own input"
        # compact record: direction bits from x and its codes (2 + 0.5 + 1/16 B in,
        # 1/8 B out), guided replay (1/8 + 1/16 + 2 B in, 2 B out)
        bits = torch.empty(rows, K // 8, dtype=torch.uint8, device=dev)
        td = timed(lambda: B.trace_direction_bits(x, codes, scales, B.SCALES_LINEAR, g, bits=bits))
        corr = torch.zeros(1, dtype=torch.int64, device=dev)
        tg = timed(lambda: B.trace_replay_direction(bits, scales, B.SCALES_LINEAR, g, x, x_hat=x_hat,
                                                    corrections=corr))
        torch.cuda.synchronize()
        assert int(corr.item()) == 0, "guided replay of the rollout's own input"
        gq = n * (2 + 0.5625) / (tq * 1e-3) / 1e9
        gr = n * (0.5625 + 2 + 2) / (tr * 1e-3) / 1e9
        gd = n * (2 + 0.5625 + 0.125) / (td * 1e-3) / 1e9
        gg = n * (0.125 + 0.0625 + 2 + 2) / (tg * 1e-3) / 1e9
        out.append({"elements": n, "quantize_us": tq * 1e3, "quantize_gbs": gq, "quantize_frac": gq / hbm_gbs,
                    "replay_us": tr * 1e3, "replay_gbs": gr, "replay_frac": gr / hbm_gbs,
                    "direction_bits_us": td * 1e3, "direction_bits_frac": gd / hbm_gbs,
                    "direction_replay_us": tg * 1e3, "direction_replay_frac": gg / hbm_gbs})
        del x, codes, scales, record, x_hat, bits
        torch.cuda.empty_cache()
    return out


def trainer_gemm_timing(layer, dev, peaks, reps=20):
    """The trainer's gate/up projection on the layer's expert-ordered rows:
    the W4A16 kernel (BF16 activations, the NVFP4 weights dequantized on
    chip, SwiGLU epilogue) against the BF16 library matmul of the same rows
    with the stored W_fq (one per expert) it replaces.  L2 flushed before
    each timed launch."""
    import torch
    from train_alignment_b200 import binding as B
    cfg = layer.cfg
    E, F, H = cfg.E, cfg.F, cfg.H
    off = layer.expert_off.tolist()
    rpad = off[-1]
    gen = torch.Generator(device=dev).manual_seed(7)
    x = torch.randn(layer.cap, H, generator=gen, device=dev).to(torch.bfloat16)
    h = torch.empty(layer.cap, F, dtype=torch.bfloat16, device=dev)
    amax = torch.empty(E, dtype=torch.float32, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)

    def timed(fn):
        return _timed_flushed(fn, flush, reps)

    t_w4 = None
    if layer.fuse_swiglu:           # the rollout's gate/up codes are in the interleaved order SwiGLU needs
        t_w4 = timed(lambda: B.moe_grouped_gemm_w4a16(x, layer.w_gu_codes, layer.w_gu_scales, layer.g_w_gu,
                                                      layer.expert_off, E, layer.cap, 2 * F, H, y=h, swiglu=True,
                                                      amax=amax))
    y = torch.empty(layer.cap, 2 * F, dtype=torch.bfloat16, device=dev)

    def lib():
        for e in range(E):
            if off[e + 1] > off[e]:
                torch.matmul(x[off[e]:off[e + 1]], layer.w_gu_fq[e].t(), out=y[off[e]:off[e + 1]])
    t_lib = timed(lib)
    rows = cfg.T * cfg.k
    flops = 2.0 * rows * 2 * F * H
    out = {"shape": f"{rows} routed rows ({rpad} padded) x {2 * F} x {H}, {E} experts",
           "library_bf16_us": t_lib * 1e3, "library_bf16_tflops": flops / (t_lib * 1e-3) / 1e12,
           "peak_bf16_tflops": peaks["bf16_tflops"]}
    if t_w4 is not None:
        out.update({"w4a16_swiglu_us": t_w4 * 1e3, "w4a16_tflops": flops / (t_w4 * 1e-3) / 1e12,
                    "w4a16_frac_bf16": flops / (t_w4 * 1e-3) / 1e12 / peaks["bf16_tflops"]})
    return out


def _timed_flushed(fn, flush, reps=20):
    """Median device time (ms) of the launches fn() makes, L2 flushed (a
    write of a buffer larger than L2, then a read of it) before each.  The flush, two timing
    events and fn are captured once in a CUDA graph (the events as external
    event nodes, re-recorded at every replay), so the interval is the
    kernels' own time as they run inside a step's graph: neither the host
    work of preparing the launches (tensor maps, argument checks, the Python
    binding) nor the graph's launch latency falls inside it, either of which
    would dominate a kernel of tens of microseconds."""
    import torch
    fn()
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    e0 = torch.cuda.Event(enable_timing=True, external=True)
    e1 = torch.cuda.Event(enable_timing=True, external=True)
    words = flush.view(torch.int32)
    acc = torch.empty((), dtype=torch.int32, device=flush.device)
    with torch.cuda.graph(graph):
        flush.zero_()
        # then a read of the same buffer: its dirty lines are written back
        # here rather than during the timed kernel, which finds only clean,
        # unrelated lines in L2
        torch.sum(words, dim=0, out=acc)
        e0.record()
        fn()
        e1.record()
    ts = []
    for _ in range(reps + 1):
        graph.replay()
        torch.cuda.synchronize()
        ts.append(e0.elapsed_time(e1))
    del graph
    ts = sorted(ts[1:])
    return ts[len(ts) // 2]


def _gemm_calls(layer, comp=True):
    """The layer's two grouped GEMMs on its current operands (after a
    rollout): gate/up with the SwiGLU epilogue, and down."""
    from train_alignment_b200 import binding as B
    cfg = layer.cfg
    E, H, F = cfg.E, cfg.H, cfg.F
    gu = lambda: B.moe_grouped_gemm_nvfp4_swiglu(
        layer.pa_codes, layer.pa_scales, layer.g_x, layer.w_gu_codes, layer.w_gu_scales, layer.g_w_gu,
        layer.expert_off, E, layer.cap, F, H, layer.pa_resid if comp else None, layer.wc_gu if comp else None,
        h=layer.h, amax=layer.amax_h)
    dn = lambda: B.moe_grouped_gemm_nvfp4(
        layer.h_codes, layer.h_scales, layer.g_h, layer.w_d_codes, layer.w_d_scales, layer.g_w_d, layer.expert_off,
        E, layer.cap, H, F, layer.h_resid if comp else None, layer.wc_d if comp else None, y=layer.y_d)
    return gu, dn


def secondary_workloads(dev, peaks, fp4_peak, steps=20):
    """The other workloads, each timed on its own after the headline (L2
    flushed before each timed run): the single NVFP4 linear (64 x 256 x 512,
    8 compensation channels: quantize x + the GEMM, the weights quantized
    once beforehand), one step of the 2048-token layer (the whole path, one
    CUDA graph per step, as the headline step), and one train/rollout
    alignment pass of the 8-layer stack (rollout of all 8 layers with the
    last 4 recorded, then the trainer with those 4 replayed), host-launched,
    with its per-token output gap (a measured value that no page fixes)."""
    import torch
    from train_alignment_b200 import binding as B
    from train_alignment_b200 import layer as L
    from train_alignment_b200 import stack as ST
    from train_alignment_b200 import workloads as W
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    out = {}
    # single NVFP4 linear
    lc = W.LINEAR_64x256x512
    li = W.linear_inputs(lc, seed=0, device=dev)
    xt = torch.zeros(128, lc.K, dtype=torch.bfloat16, device=dev)
    xt[:lc.M] = li["x"]
    chan = torch.full((16,), -1, dtype=torch.int32, device=dev)   # 8 channels, padded to the GEMM's 16
    chan[:lc.n_chan] = B.select_channels(B.channel_scores(xt[:lc.M]), lc.n_chan)
    _, w_codes, w_scales, g_w, w_chan = B.fakequant_weight_ste(li["w"][None].contiguous(), chan=chan)
    off = torch.tensor([0, 128], dtype=torch.int32, device=dev)
    amax = torch.empty(1, dtype=torch.float32, device=dev)
    codes = torch.empty(128, lc.K // 2, dtype=torch.uint8, device=dev)
    scales = torch.empty(B.scales_bytes(128, lc.K, B.SCALES_TILED), dtype=torch.uint8, device=dev)
    g = torch.empty(1, dtype=torch.float32, device=dev)
    resid = torch.empty(128, chan.numel(), dtype=torch.bfloat16, device=dev)
    y = torch.empty(128, lc.N, dtype=torch.bfloat16, device=dev)

    def linear():
        B.amax_bf16(xt, out=amax)
        B.quantize_nvfp4(xt, amax_in=amax, scale_layout=B.SCALES_TILED, chan=chan, codes=codes, scales=scales,
                         g_out=g, resid_out=resid)
        B.moe_grouped_gemm_nvfp4(codes, scales, g, w_codes, w_scales, g_w, off, 1, 128, lc.N, lc.K, resid, w_chan,
                                 y=y)
    t = _timed_flushed(linear, flush) * 1e3
    flop = 2.0 * lc.M * lc.N * (lc.K + lc.n_chan)
    out[lc.name] = {"us": t, "TFLOP/s": flop / (t * 1e-6) / 1e12, "launches": 3,
                    "what": "amax + quantize x (codes, tiled scales, 8 residual channels) + the grouped GEMM"}
    assert B.device_status() == B.OK, B.last_error()
    # one step of the 2048-token layer
    cfg = W.CONFIGS["moe_t2048_h1024_e8k2_f2048"]
    inp = W.moe_layer_inputs(cfg, seed=0, device=dev)
    ly = L.build_layer(cfg, inp, dev)
    x_train = W.engine_drift(inp["x"], 1e-2, seed=0, device=dev)
    _, g_gu, g_d = ly.grad_fq_buffers()
    g_gu.copy_(W.random_bf16(ly.w_gu.shape, 100, 1e-3, dev))
    g_d.copy_(W.random_bf16(ly.w_d.shape, 200, 1e-3, dev))
    step = lambda: ly.step(inp["x"], inp["logits"], x_train, g_gu, g_d)
    for _ in range(3):
        step()
    ms = _timed_flushed(step, flush, steps)
    fp4, comp = gemm_flops(cfg)
    out[cfg.name] = {"ms_per_step": ms, "TFLOP/s": (fp4 + comp) / (ms * 1e-3) / 1e12,
                     "what": "the whole step (rollout layer, TRACE export, trainer replay, weight fake-quant and "
                             "STE backward), one CUDA graph"}
    assert B.device_status() == B.OK, B.last_error()
    del ly, inp, x_train, g_gu, g_d
    torch.cuda.empty_cache()
    # the 8-layer alignment pass
    scfg = W.CONFIGS["stack8_t4096_h2048_e64k4_f1024"]
    st = ST.LayerStack(scfg, seed=0, device=dev)
    st.alignment_pass(drift=1e-3)
    torch.cuda.synchronize()
    ts = []
    for _ in range(3):
        flush.zero_()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        gap, cm, sm = st.alignment_pass(drift=1e-3)
        e1.record()
        e1.synchronize()
        ts.append(e0.elapsed_time(e1))
    assert B.device_status() == B.OK, B.last_error()
    gp = gap.float()
    out[scfg.name] = {"ms_per_pass": statistics.median(ts), "tokens_per_s": scfg.T / (statistics.median(ts) * 1e-3),
                      "per_token_gap": {"median": float(gp.median()), "p90": float(gp.quantile(0.9)),
                                        "max": float(gp.max()), "fixed_by_pages": False},
                      "replayed_layer_mismatches": {"codes": int(cm), "scales": int(sm)},
                      "what": "rollout of 8 layers (last 4 recorded) + trainer with the 4 records replayed; "
                              "host-launched, events around the pass"}
    del st
    torch.cuda.empty_cache()
    return out


def gemm_side_measurements(layer, dev, peaks, fp4_peak=None):
    """(1) The compensation's cost: the step layer's two grouped GEMMs with
    and without the BF16 correction on the same operands.  (2) Decode
    shapes (2048 hidden, 128 experts top-8, ffn 768, T = 64 and 512), measured
    as weight-stream bandwidth: the NVFP4 weight bytes (codes, scales and the
    BF16 Wc columns) of every expert that received rows, over the GEMM time,
    on the tiles the library picks (the decode tiles, weights as the MMA's M
    operand) and on the 128 x 256 tiles.  (3) The same layer at T = 4096,
    near the ridge, also as FP4 TFLOP/s against the measured FP4 peak.  L2
    flushed before each timed launch."""
    import torch
    from train_alignment_b200 import layer as L
    from train_alignment_b200 import workloads as W
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    out = {}
    gu, dn = _gemm_calls(layer, True)
    gu0, dn0 = _gemm_calls(layer, False)
    t = {k: _timed_flushed(f, flush) * 1e3 for k, f in (("gate_up", gu), ("down", dn), ("gate_up_nocomp", gu0),
                                                         ("down_nocomp", dn0))}
    tot, tot0 = t["gate_up"] + t["down"], t["gate_up_nocomp"] + t["down_nocomp"]
    out["compensation"] = {"us_with": tot, "us_without": tot0, "overhead_frac": tot / tot0 - 1.0,
                           "gate_up_us": [t["gate_up"], t["gate_up_nocomp"]], "down_us": [t["down"], t["down_nocomp"]]}
    dec = []
    from train_alignment_b200 import binding as B
    for T in (64, 512, 4096):
        cfg = W.decode_config(T)
        inp = W.moe_layer_inputs(cfg, seed=0, device=dev)
        ly = L.build_layer(cfg, inp, dev)
        ly.weight_sync()
        ly.rollout_forward(inp["x"], inp["logits"])
        torch.cuda.synchronize()
        off = ly.expert_off.tolist()
        used = sum(1 for e in range(cfg.E) if off[e + 1] > off[e])
        q = 0.5 + 1.0 / 16
        wb_g = used * 2 * cfg.F * (cfg.H * q + ly.nc_x * 2)
        wb_d = used * cfg.H * (cfg.F * q + ly.nc_h * 2)
        row = {"workload": cfg.name, "experts_with_rows": used, "weight_bytes": wb_g + wb_d}
        # the library's own choice (decode tiles at these sizes), then the
        # 128 x 256 tiles on the same operands for comparison
        for key, rows in (("", None), ("tiles_128x256_", 0)):
            prev = B.gemm_set_decode_rows(rows) if rows is not None else None
            g, d = _gemm_calls(ly, True)
            tg, td = _timed_flushed(g, flush) * 1e3, _timed_flushed(d, flush) * 1e3
            if prev is not None:
                B.gemm_set_decode_rows(prev)
            gbs = (wb_g + wb_d) / ((tg + td) * 1e-6) / 1e9
            row.update({key + "gate_up_us": tg, key + "down_us": td, key + "weight_stream_gbs": gbs,
                        key + "frac_hbm": gbs / peaks["hbm_gbs"]})
            if T >= 4096:
                fl = sum(gemm_flops(cfg))
                row.update({key + "TFLOP/s": fl / ((tg + td) * 1e-6) / 1e12})
                if fp4_peak:
                    row[key + "frac_fp4"] = fl / ((tg + td) * 1e-6) / 1e12 / fp4_peak
        dec.append(row)
        del ly, inp
        torch.cuda.empty_cache()
    out["decode"] = dec
    return out


# ------------------------------------------------------------------- clocks


class ClockSampler:
    """nvidia-smi samples of this GPU's SM clock and throttle reasons."""

    FIELDS = ("uuid,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, uuid):
        self.uuid = uuid
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                                          "-lms", "200"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL,
                                         text=True)
        except (OSError, ValueError):
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            if self.uuid and self.uuid not in parts[0]:
                continue
            try:
                sm.append(float(parts[1]))
                mx.append(float(parts[2]))
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "samples": len(sm), "reasons": sorted(reasons)}


# -------------------------------------------------------------------- oracle


class OracleSample:
    """Bounded CPU sample of the workload for the oracle: a fraction `frac` of
    every part of one step.  The rollout forward and record replay run on a
    slice of the layer: T_s of the tokens (the workload's own x and router
    logits) over the first F_s of the ffn columns of every expert, with
    T_s * F_s about frac * T * F.  The weight sync and straight-through
    backward run on frac of the weight rows, taken from the same slice.
    Slicing the ffn width as well as the tokens keeps small samples small:
    the forward dequantizes every expert's weights once per call, whatever
    the number of tokens.  Only the slice's weights are drawn (BF16
    ~ N(0, 0.02) from their own seeded generator, so their values are not
    the GPU run's): the full expert weights of the large layers do not fit
    the host's memory in float64.  Inputs and the slice's NVFP4 weights
    (which the forward needs) are prepared in set_fraction, outside the
    timing."""

    def __init__(self, cfg, seed=0, frac=1.0):
        import numpy as np
        from oracle import layer as OL
        from oracle import nvfp4 as Q
        from train_alignment_b200 import workloads as W
        self.OL, self.Q, self.W, self.cfg, self.np = OL, Q, W, cfg, np
        inp = W.moe_layer_inputs(cfg, seed=seed, device="cpu", with_weights=False)
        self.x = inp["x"].float().numpy().astype(np.float64)
        self.logits = inp["logits"].numpy().astype(np.float64)
        self.seed = seed
        r = np.random.default_rng(seed)
        self.chan_x = Q.pad_channels(np.sort(r.choice(cfg.H, cfg.n_chan, replace=False)))
        self.F_s = None
        self.set_fraction(frac)

    def _slice_weights(self, F_s):
        """NVFP4 weights and ffn channel set of the first F_s ffn columns."""
        np, cfg, Q, OL = self.np, self.cfg, self.Q, self.OL
        ws = self.W.expert_weight_slice(cfg, F_s, seed=self.seed)
        self.w_gu = ws["w_gu"].float().numpy().astype(np.float64)
        self.w_d = ws["w_d"].float().numpy().astype(np.float64)
        r = np.random.default_rng(self.seed + 1)
        self.chan_h_s = Q.pad_channels(np.sort(r.choice(F_s, min(cfg.n_chan_f, F_s // 2), replace=False)))
        self.wgu_all = OL.weight_sync(self.w_gu, self.chan_x)
        self.wd_all = OL.weight_sync(self.w_d, self.chan_h_s)
        self.F_s = F_s

    def set_fraction(self, frac):
        np, cfg = self.np, self.cfg
        self.frac = frac
        F_s = min(cfg.F, max(16, int(round(cfg.F * np.sqrt(frac) / 16)) * 16))
        if F_s != self.F_s:
            self._slice_weights(F_s)
        self.T_s = max(1, min(cfg.T, int(round(cfg.T * frac * cfg.F / F_s))))
        self.rows_gu = min(cfg.E * 2 * F_s, max(16, int(round(cfg.E * 2 * cfg.F * frac))))
        self.rows_d = min(cfg.E * cfg.H, max(16, int(round(cfg.E * cfg.H * frac))))
        R = self.T_s * cfg.k
        n_cx = int((self.chan_x >= 0).sum())
        n_ch = int((self.chan_h_s >= 0).sum())
        self.flops = 2 * R * 2 * F_s * cfg.H + 2 * R * cfg.H * F_s + 2 * R * 2 * F_s * n_cx + 2 * R * cfg.H * n_ch
        self.desc = (f"oracle (float64 numpy) on {cfg.name}: forward and replay of {self.T_s} of {cfg.T} tokens "
                     f"over the first {F_s} of {cfg.F} ffn columns of all {cfg.E} experts ({n_cx} + {n_ch} "
                     f"compensation channels), weight sync + STE backward of {self.rows_gu} of "
                     f"{cfg.E * 2 * cfg.F} gate/up and {self.rows_d} of {cfg.E * cfg.H} down weight rows per step; "
                     f"the slice's weights drawn on the host with the layer's distribution")

    def run(self):
        OL, Q = self.OL, self.Q
        H, F_s = self.cfg.H, self.F_s
        wgu = self.w_gu.reshape(-1, H)[:self.rows_gu][None]
        wd = self.w_d.reshape(-1, F_s)[:self.rows_d][None]
        t0 = time.perf_counter()
        OL.weight_sync(wgu, self.chan_x)
        OL.weight_sync(wd, self.chan_h_s)
        fwd = OL.rollout_forward(self.x[:self.T_s], self.logits[:self.T_s], self.wgu_all, self.wd_all,
                                 self.chan_x, self.chan_h_s, self.cfg.k)
        OL.trainer_replay(fwd, self.x[:self.T_s], self.chan_x, self.chan_h_s)
        Q.ste_backward(wgu, wgu)
        Q.ste_backward(wd, wd)
        return time.perf_counter() - t0

    def fit(self, seconds, start=1.0 / 64, probes=8):
        """Pick the fraction whose step takes about `seconds`: a few probe
        runs, each rescaling the fraction by budget / time (the time is not
        proportional to the fraction, so one probe does not suffice); the
        largest probed fraction within the budget, else the smallest."""
        frac, tried = start, []
        for _ in range(probes):
            self.set_fraction(frac)
            t = self.run()
            tried.append((frac, t))
            nxt = min(1.0, max(1e-7, frac * seconds / max(t, 1e-6)))
            if 0.7 * seconds <= t <= 1.3 * seconds or nxt == frac:
                break
            frac = nxt
        fit = [f for f, t in tried if t <= 1.3 * seconds]
        self.set_fraction(max(fit) if fit else min(f for f, _ in tried))
        return self.frac


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [d.get("num_threads", 1) for d in threadpool_info() if d.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:  # noqa: BLE001
        return 1


def run_reference(args):
    rank, world, _ = dist_env()
    if rank != 0:
        return 0
    from train_alignment_b200 import workloads as W
    cfg = W.CONFIGS[args.workload]
    # size each step so that warm-up + timed steps take about 100 s
    sample = OracleSample(cfg, seed=0, frac=1.0 / 4096)
    sample.fit(100.0 / max(1, args.steps + args.warmup))
    for _ in range(args.warmup):
        sample.run()
    times = [sample.run() for _ in range(args.steps)]
    flops, desc = sample.flops, sample.desc
    ms = 1e3 * sum(times) / len(times)
    value = flops / (ms * 1e-3) / 1e12
    cores = blas_threads()
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": cfg.name, "T": cfg.T, "H": cfg.H, "E": cfg.E, "k": cfg.k, "F": cfg.F,
                       "n_chan": cfg.n_chan, "n_chan_f": cfg.n_chan_f, "sample": desc},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": desc},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
            "gpu_launches": 0}
    print(json.dumps(line), flush=True)
    return 0


# -------------------------------------------------------------------- ours


def run_ours(args):
    import torch
    import torch.distributed as dist

    from train_alignment_b200 import binding as B
    from train_alignment_b200 import layer as L
    from train_alignment_b200 import workloads as W

    rank, world, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300), device_id=dev)
    B.load()
    cfg = W.CONFIGS[args.workload]
    inp = W.moe_layer_inputs(cfg, seed=rank, device=dev)
    layer = L.build_layer(cfg, inp, dev, overlap=not args.serial, fuse_requant=args.fuse_requant, comp=args.comp,
                          materialize_wfq=not args.trainer_w4a16)
    x, logits = inp["x"], inp["logits"]
    x_train = W.engine_drift(x, 1e-2, seed=rank, device=dev)
    g_all, g_gu, g_d = layer.grad_fq_buffers()          # both weight gradients in one allocation
    g_gu.copy_(W.random_bf16(layer.w_gu.shape, 100 + rank, 1e-3, dev))
    g_d.copy_(W.random_bf16(layer.w_d.shape, 200 + rank, 1e-3, dev))
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)

    def barrier():
        if world > 1:
            dist.barrier()

    for _ in range(max(args.warmup, 3)):
        flush.zero_()
        n0 = B.launch_count()
        layer.step(x, logits, x_train, g_gu, g_d)
        launches_per_step = B.launch_count() - n0
    torch.cuda.synchronize()
    assert B.device_status() == B.OK, B.last_error()
    rpad = int(layer.expert_off[-1].item())

    # one step captured as a CUDA graph (stage events inside the graph)
    timing_mode = "cuda-graph"
    graph, gtimer = None, L.StageTimer(True, external=True)
    try:
        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            layer.step(x, logits, x_train, g_gu, g_d)
        torch.cuda.current_stream().wait_stream(side)
        torch.cuda.synchronize()
        # per-kernel breakdown: the step on one stream (kernels measured one at
        # a time, in step order) with an event between every two kernels
        overlap = layer.overlap
        layer.overlap = False
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            layer.step(x, logits, x_train, g_gu, g_d, timer=gtimer)
        layer.overlap = overlap
        graph_plain = torch.cuda.CUDAGraph()            # the step alone
        with torch.cuda.graph(graph_plain):
            layer.step(x, logits, x_train, g_gu, g_d)
        for _ in range(3):
            flush.zero_()
            graph.replay()
            graph_plain.replay()
        torch.cuda.synchronize()
        gtimer.durations_ms()
    except Exception as exc:  # noqa: BLE001 -- fall back to stream launches
        graph = None
        timing_mode = f"stream launches ({type(exc).__name__} in graph capture: {str(exc)[:120]})"
        torch.cuda.synchronize()

    uuid = None
    try:
        uuid = str(torch.cuda.get_device_properties(dev).uuid)
    except Exception:  # noqa: BLE001
        pass
    clocks = ClockSampler(uuid)
    clocks.start()
    time.sleep(0.3)
    barrier()
    torch.cuda.synchronize()
    launches0 = B.launch_count()
    # timed region: exactly K steps, each the whole path, events around each step
    step_ms = []
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    for i in range(args.steps):
        flush.zero_()                                   # L2 flush, outside the events
        ev[i][0].record()
        if graph is not None:
            graph_plain.replay()
        else:
            layer.step(x, logits, x_train, g_gu, g_d)
        ev[i][1].record()
    torch.cuda.synchronize()
    step_ms = [a.elapsed_time(b) for a, b in ev]
    barrier()
    launches = B.launch_count() - launches0
    if graph is not None:                               # graph replays bypass the host-side counter
        launches = args.steps * launches_per_step
    clk = clocks.stop()
    assert B.device_status() == B.OK, B.last_error()
    ms = sum(step_ms) / len(step_ms)
    # per-kernel breakdown: the same K steps again with an event between every two kernels
    per_kernel, inst_ms = {}, []
    for _ in range(args.steps):
        flush.zero_()
        if graph is not None:
            graph.replay()
            torch.cuda.synchronize()
            t = gtimer
        else:
            t = L.StageTimer(True)
            layer.step(x, logits, x_train, g_gu, g_d, timer=t)
            t.marks[-1][1].synchronize()
        inst_ms.append(t.marks[0][1].elapsed_time(t.marks[-1][1]))
        for name, v in t.durations_ms().items():
            per_kernel[name] = per_kernel.get(name, 0.0) + v / args.steps
    assert B.device_status() == B.OK, B.last_error()
    ms = max_over_ranks(ms, world, dev)
    fp4, comp = gemm_flops(cfg)
    value = whole_job_tflops(fp4 + comp, world, ms)

    # the dense FP4 peak of this GPU, measured with the library's NVFP4 GEMM
    try:
        fp4_meas = fp4_library_peak(dev)
        fp4_peak, fp4_src = fp4_meas["burst_tflops"], "measured on this GPU: library NVFP4 GEMM, burst"
    except Exception as exc:  # noqa: BLE001 -- the nominal ratio, said so in the line
        fp4_meas = {"error": f"{type(exc).__name__}: {str(exc)[:160]}"}
        fp4_peak, fp4_src = None, None

    # roofline of the dominant kernel: its own launches timed by two events
    # around it alone, in the one-stream step, over args.steps replays
    peaks, peak_src = load_peaks()
    if fp4_peak is None:
        fp4_peak = peaks["bf16_tflops"] * FP4_OVER_BF16
        fp4_src = f"{peak_src} bf16 burst x {FP4_OVER_BF16:g} (nominal ratio; the FP4 measurement failed)"
    work = kernel_work(cfg, rpad, wfq=not args.trainer_w4a16)
    dom = max(per_kernel, key=per_kernel.get)
    bound, amount = work[dom]
    dur = per_kernel[dom] * 1e-3
    dom_source = "events between every two kernels"
    if graph is not None:
        order = [n for n, _ in gtimer.marks]
        prev = order[order.index(dom) - 1]
        dtimer = L.StageTimer(True, external=True, only={prev, dom})
        layer.overlap = False
        graph_dom = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph_dom):
            layer.step(x, logits, x_train, g_gu, g_d, timer=dtimer)
        layer.overlap = overlap
        dsum = 0.0
        for i in range(args.steps + 3):
            flush.zero_()
            graph_dom.replay()
            torch.cuda.synchronize()
            if i >= 3:
                dsum += dtimer.durations_ms()[dom]
        dur = dsum / args.steps * 1e-3
        dom_source = "two events around the kernel alone (one-stream step)"
        del graph_dom
    assert B.device_status() == B.OK, B.last_error()
    if bound == "hbm":
        achieved, peak, unit = amount / dur / 1e9, peaks["hbm_gbs"], "GB/s"
    else:
        achieved, peak, unit = amount / dur / 1e12, fp4_peak, "TFLOP/s"
    kernels = {}
    for name, dms in per_kernel.items():
        b, a = work.get(name, ("hbm", 0.0))
        if b == "latency":
            kernels[name] = {"ms": dms, "bytes": a, "bound": "launch latency"}
        elif b == "hbm":
            kernels[name] = {"ms": dms, "GB/s": a / (dms * 1e-3) / 1e9, "frac_hbm": a / (dms * 1e-3) / 1e9 /
                             peaks["hbm_gbs"]}
        else:
            tf = a / (dms * 1e-3) / 1e12
            kernels[name] = {"ms": dms, "TFLOP/s": tf, "frac_fp4": tf / fp4_peak}
    traffic = recorded_traffic(cfg.name, dom)
    # the grouped GEMMs' own throughput: each launch timed alone by the events
    # around it in the one-stream step (the per-kernel breakdown above)
    gemm_names = [n for n in per_kernel if work.get(n, ("hbm",))[0] == "tensor"]
    g_ms = sum(per_kernel[n] for n in gemm_names)
    g_flop = sum(work[n][1] for n in gemm_names)
    gemm = {"kernels": {n: kernels[n] for n in gemm_names}, "ms": g_ms, "TFLOP/s": g_flop / (g_ms * 1e-3) / 1e12,
            "frac_fp4": g_flop / (g_ms * 1e-3) / 1e12 / fp4_peak, "fp4_peak_tflops": fp4_peak,
            # the same against the library GEMM held for seconds under the power cap
            "frac_fp4_of_sustained": (g_flop / (g_ms * 1e-3) / 1e12 / fp4_meas["sustained_tflops"]
                                      if fp4_meas and fp4_meas.get("sustained_tflops") else None),
            "fp4_peak_source": fp4_src, "fp4_peak_measurement": fp4_meas,
            "flops": "2 x routed rows x N x K per GEMM (FP4) + 2 x routed rows x N x channels (BF16 correction); "
                     "padding rows excluded",
            "timed_by": "events around each GEMM launch alone, one-stream step graph, L2 flushed before each step"}

    # end to end through the public API with host buffers
    e2e = None
    if not args.no_e2e:
        # End to end through the layer API with host buffers, pipelined the way
        # a serving loop runs it: step i's inputs are copied in from pinned host
        # memory on one copy stream while step i - 1 computes, and its output
        # and counters go back on another (two input and output buffer sets,
        # one CUDA graph of the step per set).  The timed region holds every
        # step's host-to-device and device-to-host copies; no L2 flush between
        # steps (each step streams ~0.7 GB, several times the L2).
        nb = 2
        x_h, l_h, xt_h = x.cpu().pin_memory(), logits.cpu().pin_memory(), x_train.cpu().pin_memory()
        ins = [(torch.empty_like(x), torch.empty_like(logits), torch.empty_like(x_train)) for _ in range(nb)]
        out_st = [torch.empty_like(layer.out) for _ in range(nb)]
        cnt_st = [torch.empty_like(layer.counts) for _ in range(nb)]
        out_h = [torch.empty(tuple(layer.out.shape), dtype=torch.bfloat16).pin_memory() for _ in range(nb)]
        cnt_h = [torch.empty(2, dtype=torch.int64).pin_memory() for _ in range(nb)]
        for b in range(nb):
            for d, h in zip(ins[b], (x_h, l_h, xt_h)):
                d.copy_(h)
        graphs = []
        if graph is not None:
            for b in range(nb):
                gph = torch.cuda.CUDAGraph()
                with torch.cuda.graph(gph):
                    layer.step(*ins[b], g_gu, g_d)
                graphs.append(gph)
        torch.cuda.synchronize()
        main = torch.cuda.current_stream()
        cs_in, cs_out = torch.cuda.Stream(), torch.cuda.Stream()
        ev_in = [torch.cuda.Event() for _ in range(nb)]
        ev_done = [torch.cuda.Event() for _ in range(nb)]
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        for i in range(args.warmup + args.steps):
            b = i % nb
            if i == args.warmup:
                torch.cuda.synchronize()
                barrier()
                t0.record(cs_in)
            if i >= nb:
                cs_in.wait_event(ev_done[b])             # step i - 2 has finished with this input set
            with torch.cuda.stream(cs_in):
                for d, h in zip(ins[b], (x_h, l_h, xt_h)):
                    d.copy_(h, non_blocking=True)
            ev_in[b].record(cs_in)
            main.wait_event(ev_in[b])
            if graphs:
                graphs[b].replay()
            else:
                layer.step(*ins[b], g_gu, g_d)
            out_st[b].copy_(layer.out)
            cnt_st[b].copy_(layer.counts)
            ev_done[b].record(main)
            cs_out.wait_event(ev_done[b])
            with torch.cuda.stream(cs_out):
                out_h[b].copy_(out_st[b], non_blocking=True)
                cnt_h[b].copy_(cnt_st[b], non_blocking=True)
        t1.record(cs_out)
        t1.synchronize()
        e_ms = max_over_ranks(t0.elapsed_time(t1) / args.steps, world, dev)
        del graphs
        assert B.device_status() == B.OK, B.last_error()
        h2d = x.numel() * 2 + logits.numel() * 4 + x_train.numel() * 2
        d2h = layer.out.numel() * 2 + 16
        e2e = {"value": whole_job_tflops(fp4 + comp, world, e_ms), "unit": UNIT, "ms_per_step": e_ms,
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
               "pipeline": "inputs of step i copied in while step i - 1 computes; outputs copied out on a second "
                           "copy stream; one CUDA graph of the step per buffer set"}

    sweep = None
    if not args.no_sweep:
        sweep = quantize_replay_sweep(dev, peaks["hbm_gbs"])
    trainer = trainer_gemm_timing(layer, dev, peaks) if not args.no_sweep else None
    gemm_side = (gemm_side_measurements(layer, dev, peaks, fp4_peak) if not args.no_sweep and layer.comp == "bf16"
                 else None)
    secondary = None
    if not args.no_secondary and world == 1:
        try:
            secondary = secondary_workloads(dev, peaks, fp4_peak)
        except Exception as exc:  # noqa: BLE001 -- reported, the headline stands
            secondary = {"error": f"{type(exc).__name__}: {str(exc)[:200]}"}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        # a bounded sample, about 10 s of host work on 8 cores: the whole step of
        # the 2048-token layer, 1/256 of the prefill layer's
        sample = OracleSample(cfg, seed=0, frac=1.0 if cfg.T * cfg.H * cfg.F <= 2 ** 33 else 1.0 / 256)
        dt, flops, desc = sample.run(), sample.flops, sample.desc
        cpu = {"value": flops / dt / 1e12, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
               "sample": desc + f"; {dt:.1f} s", "seconds": dt, "fraction_of_step": sample.frac}

    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return 0
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": max(args.warmup, 3), "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "nvfp4(e2m1+e4m3)/bf16", "data": "synthetic",
        "config": {"workload": cfg.name, "T": cfg.T, "H": cfg.H, "E": cfg.E, "k": cfg.k, "F": cfg.F,
                   "n_chan": cfg.n_chan, "n_chan_f": cfg.n_chan_f, "rows_padded": rpad,
                   "parallelism": f"dp{world} (replicas, no collective)",
                   "schedule": ("one stream" if args.serial else
                                "three streams (weight side overlapped" +
                                (f"; STE on {layer.side_sms} SMs beside the GEMMs on {layer.gemm_sms})"
                                 if layer.side_sms else ")")) +
                               ("; h quantized in the gate/up GEMM epilogue (delayed amax)" if args.fuse_requant
                                else "") +
                               ("; FP4 compensation (NVFP4 residual x NVFP4 weight columns)" if args.comp == "fp4"
                                else "") +
                               ("; trainer on W4A16 GEMMs (W_fq not written)" if args.trainer_w4a16 else ""),
                   "l2": "flushed between steps (256 MiB memset outside the timed events)",
                   "gemm_flops_per_step": fp4 + comp},
        "roofline": {"kernel": dom, "bound": bound, "achieved": achieved, "peak": peak, "unit": unit,
                     "frac": achieved / peak, "traffic": traffic, "duration_ms": dur * 1e3, "timed_by": dom_source,
                     "peak_source": fp4_src if bound == "tensor" else f"{peak_src} HBM copy"},
        "gemm": gemm,
        "kernels": kernels,
        "kernels_timed_by": "one-stream step graph, a CUDA event between every two kernels",
        "clocks": clk,
        "e2e": e2e,
        "gpu_launches": launches,
        "timing": timing_mode,
        "instrumented_ms_per_step": sum(inst_ms) / len(inst_ms),
        "quantize_replay_sweep": sweep,
        "trainer_gemm": trainer,
        "gemm_side": gemm_side,
        "secondary_workloads": secondary,
        "cpu_baseline": cpu,
    }
    print(json.dumps(line), flush=True)
    return 0


def main():
    args = parse()
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
