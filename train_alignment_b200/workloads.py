"""Seeded synthetic inputs shaped like the pages' MoE rollout workloads.

This module holds no arithmetic of the method: it only draws random numbers
(torch generators, seeded) and rounds them to BF16.  Both the CUDA path and
the CPU oracle are fed from it.

The pages' own workloads (a 25B-parameter MoE with 2.8B active parameters,
trained with GRPO on maths and code prompts; [QUADS-fr §4]) are not
available, so these synthetic tensors stand in for them:

* activations X: BF16 ~ N(0, 1) with a few outlier channels scaled up (the
  "high-residual" channels of [QUADS-fr §2.2.B]), or with heavy-tailed
  per-channel scales |Student-t(3)|;
* router logits: N(0, 1), or N(0, 1) + log p with Zipf(1.1) expert
  popularity p under a seeded permutation of the experts;
* expert weights: BF16 ~ N(0, 0.02), gate/up stored [E, 2F, H] (rows =
  output features, K = H contiguous), down stored [E, H, F].
"""
from dataclasses import dataclass
import math

import torch


@dataclass(frozen=True)
class MoEConfig:
    name: str
    T: int                 # tokens
    H: int                 # hidden size
    E: int                 # experts
    k: int                 # experts per token
    F: int                 # expert FFN size (SwiGLU: gate/up has 2F rows)
    n_chan: int            # compensation channels of the gate/up input
    n_chan_f: int          # compensation channels of the down input
    x_kind: str = "outlier"          # "outlier" | "student_t"
    n_outlier: int = 0
    outlier_scale: float = 1.0
    logit_kind: str = "normal"       # "normal" | "zipf"
    layers: int = 1
    description: str = ""


@dataclass(frozen=True)
class LinearConfig:
    name: str
    M: int
    K: int
    N: int
    n_chan: int
    n_outlier: int
    outlier_scale: float
    description: str = ""


LINEAR_64x256x512 = LinearConfig(
    "linear_m64_k256_n512", 64, 256, 512, 8, 4, 20.0,
    "single NVFP4 linear: X 64x256 N(0,1) with 4 outlier channels x20, "
    "W 256x512 N(0,0.02), compensation on the 8 highest-residual channels")

MOE_T2048 = MoEConfig(
    "moe_t2048_h1024_e8k2_f2048", T=2048, H=1024, E=8, k=2, F=2048,
    n_chan=32, n_chan_f=32, x_kind="outlier", n_outlier=5, outlier_scale=16.0,
    logit_kind="normal",
    description="one MoE FFN layer: 2048 tokens, hidden 1024, 8 experts top-2, "
                "SwiGLU ffn 2048, 0.5% outlier channels x16, 32 compensation channels")


def decode_config(T):
    return MoEConfig(
        f"decode_t{T}_h2048_e128k8_f768", T=T, H=2048, E=128, k=8, F=768,
        n_chan=64, n_chan_f=64, x_kind="outlier", n_outlier=10, outlier_scale=16.0,
        logit_kind="zipf",
        description=f"decode-shaped MoE layer: {T} tokens, hidden 2048, 128 experts "
                    "top-8, ffn 768, Zipf(1.1) router skew, 64 compensation channels")


PREFILL_T16384 = MoEConfig(
    "prefill_t16384_h4096_e128k8_f1536", T=16384, H=4096, E=128, k=8, F=1536,
    n_chan=128, n_chan_f=128, x_kind="student_t", logit_kind="zipf",
    description="large prefill MoE layer: 16384 tokens, hidden 4096, 128 experts "
                "top-8, ffn 1536, Student-t(3) channel scales, 128 compensation channels")

STACK8_T4096 = MoEConfig(
    "stack8_t4096_h2048_e64k4_f1024", T=4096, H=2048, E=64, k=4, F=1024,
    n_chan=64, n_chan_f=32, x_kind="outlier", n_outlier=10, outlier_scale=16.0,
    logit_kind="normal", layers=8,
    description="8-layer MoE stack: 4096 tokens, hidden 2048, 64 experts top-4, "
                "ffn 1024; the last 4 layers are recorded and replayed")

# The prefill layer's per-expert shape (1024 routed rows per expert on
# average, hidden 4096, ffn 1536, top-8, 128 + 128 channels) on 16 experts:
# small enough (a few GB on the device) for kernel profiles.
PREFILL_SLICE_T2048 = MoEConfig(
    "prefill_slice_t2048_h4096_e16k8_f1536", T=2048, H=4096, E=16, k=8, F=1536,
    n_chan=128, n_chan_f=128, x_kind="student_t", logit_kind="zipf",
    description="16-expert slice of the prefill layer: 2048 tokens, hidden 4096, 16 experts top-8, "
                "ffn 1536, Student-t(3) channel scales, 128 compensation channels (kernel profiles)")

CONFIGS = {c.name: c for c in [MOE_T2048, decode_config(64), decode_config(512),
                               decode_config(4096), PREFILL_T16384, STACK8_T4096, PREFILL_SLICE_T2048]}


def _gen(device, seed):
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def _randn_bf16(shape, std, gen, device, chunk=1 << 26):
    """N(0, std^2) rounded to BF16, drawn in float32 chunks to bound memory."""
    out = torch.empty(shape, dtype=torch.bfloat16, device=device)
    flat = out.view(-1)
    n = flat.numel()
    for s in range(0, n, chunk):
        m = min(chunk, n - s)
        flat[s:s + m] = (torch.randn(m, generator=gen, device=device) * std).to(torch.bfloat16)
    return out


def activations(T, H, kind, n_outlier, outlier_scale, gen, device):
    """BF16 [T, H] activations (see the module docstring)."""
    x = torch.randn(T, H, generator=gen, device=device)
    if kind == "outlier":
        if n_outlier:
            ch = torch.randperm(H, generator=gen, device=device)[:n_outlier]
            x[:, ch] *= outlier_scale
    elif kind == "student_t":
        z = torch.randn(H, generator=gen, device=device)
        chi2 = (torch.randn(3, H, generator=gen, device=device) ** 2).sum(0)
        sigma = (z / torch.sqrt(chi2 / 3.0)).abs()
        x *= sigma[None, :]
    else:
        raise ValueError(kind)
    return x.to(torch.bfloat16)


def router_logits(T, E, kind, gen, device):
    """FP32 [T, E] router logits."""
    l = torch.randn(T, E, generator=gen, device=device)
    if kind == "zipf":
        ranks = torch.arange(1, E + 1, device=device, dtype=torch.float64)
        p = ranks ** -1.1
        p = p / p.sum()
        perm = torch.randperm(E, generator=gen, device=device)
        logp = torch.empty(E, device=device, dtype=torch.float64)
        logp[perm] = torch.log(p)
        l = l + logp.to(torch.float32)[None, :]
    elif kind != "normal":
        raise ValueError(kind)
    return l.contiguous()


def moe_layer_inputs(cfg: MoEConfig, seed=0, device="cpu", layer=0, with_logits=True, with_weights=True):
    """Inputs of one MoE layer: x [T,H] bf16, logits [T,E] f32, w_gu [E,2F,H]
    bf16, w_d [E,H,F] bf16.  Layer l of a stack uses seed + 1000 * l for its
    weights (the stack's activations flow from layer to layer).  x and the
    logits are drawn first, so with_weights=False gives the same x and logits
    without the weights."""
    gen = _gen(device, seed * 7919 + layer * 1000 + 1)
    out = {}
    out["x"] = activations(cfg.T, cfg.H, cfg.x_kind, cfg.n_outlier, cfg.outlier_scale, gen, device)
    if with_logits:
        out["logits"] = router_logits(cfg.T, cfg.E, cfg.logit_kind, gen, device)
    if with_weights:
        out["w_gu"] = _randn_bf16((cfg.E, 2 * cfg.F, cfg.H), 0.02, gen, device)
        out["w_d"] = _randn_bf16((cfg.E, cfg.H, cfg.F), 0.02, gen, device)
    return out


def expert_weight_slice(cfg: MoEConfig, F_s, seed=0, device="cpu"):
    """Expert weights of the first F_s ffn columns only, with the layer's
    distribution (BF16 ~ N(0, 0.02)) from their own seeded generator (not the
    values moe_layer_inputs draws): w_gu [E, 2 F_s, H] (gate rows, then up
    rows), w_d [E, H, F_s].  Used where the whole layer's weights are too
    large to draw on the host."""
    gen = _gen(device, seed * 7919 + 271828)
    return {"w_gu": _randn_bf16((cfg.E, 2 * F_s, cfg.H), 0.02, gen, device),
            "w_d": _randn_bf16((cfg.E, cfg.H, F_s), 0.02, gen, device)}


def stack_router_weights(cfg: MoEConfig, seed=0, device="cpu"):
    """Router matrices W_r [layers, H, E] ~ N(0, 1/H) for the layer stack."""
    gen = _gen(device, seed * 7919 + 424242)
    return (torch.randn(cfg.layers, cfg.H, cfg.E, generator=gen, device=device)
            / math.sqrt(cfg.H)).contiguous()


def engine_drift(x, std, seed, device="cpu"):
    """x + N(0, std^2) rounded to BF16: the trainer's copy of an activation that
    drifted from the rollout's ([QUADS-fr §2.1] calls this engine drift)."""
    gen = _gen(device, seed * 7919 + 31337)
    n = torch.randn(x.shape, generator=gen, device=device)
    return (x.float() + std * n).to(torch.bfloat16)


def linear_inputs(cfg: LinearConfig = LINEAR_64x256x512, seed=0, device="cpu"):
    """x [M, K] bf16 with outlier channels, w [N, K] bf16 (row n = output n)."""
    gen = _gen(device, seed * 7919 + 5)
    x = activations(cfg.M, cfg.K, "outlier", cfg.n_outlier, cfg.outlier_scale, gen, device)
    w = _randn_bf16((cfg.N, cfg.K), 0.02, gen, device)
    return {"x": x, "w": w}


def random_bf16(shape, seed, std=1.0, device="cpu"):
    """Plain N(0, std^2) BF16 tensor (quantizer sweeps and unit tests)."""
    return _randn_bf16(tuple(shape), std, _gen(device, seed * 7919 + 99), device)
