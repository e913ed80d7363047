"""A stack of NVFP4 MoE layers on both sides of train/rollout alignment.

The pages' method acts per MoE layer; the model around the layers is not
described.  The stack joins layers in the plainest way the rest supports:
x_{l+1} = x_l + MoE_l(x_l), with router logits_l = x_l . W_r[l].

Rollout side: every layer runs the NVFP4 path (MoELayer) and the last
`recorded` layers export their TRACE record (codes, scales, per-tensor
scales, residuals, top-k indices) [TRACE "L'idée centrale"].

Trainer side ([QUADS-fr §2.2.A]): BF16 activations with the fake-quantized
weights W_fq.  In the recorded layers the trainer replays the record
[TRACE "L'idée centrale", "Fonctionnement"]:
  - its down projection reads the replayed h, bit-exact to what the
    rollout's compensated down GEMM multiplied;
  - its routing is the recorded top-k;
  - the mismatches of its own rounding of the layer input against the
    record are counted.
The other layers route and compute on the trainer's own activations.  The
trainer's expert FFNs are BF16 x W_fq products ([QUADS-fr §2.2.A]): by
default the W4A16 grouped GEMM, which reads the weights as their NVFP4 codes
and dequantizes them on chip (gate/up with the SwiGLU epilogue, then down,
then the combine kernel); trainer_gemm="library" runs per-expert BF16 library
matmuls on the stored W_fq instead.  The per-token gap between the two sides'
stack outputs is reported, not pinned.

The symmetric W4A4 trainer ([QUADS-fr §2.2, ablation studies; §2.1]: QAT
that fake-quantizes both weights and activations) is the ablation the pages
report as drifting further than the asymmetric scheme: every
layer fake-quantizes its input x (one per-tensor scale) and each expert's h
(one scale per expert) on the NVFP4 grid, without compensation and without
replay; its backward through those fake-quants is the same straight-through
identity as for the weights.  It runs on the same kernels as the W4A16
trainer: the fake-quant of x, the BF16 gather into expert order, the W4A16
gate/up + SwiGLU, the per-expert quantize and dequantize of h, the W4A16
down GEMM and the combine.
"""
import torch

from . import binding as B
from . import layer as L
from . import workloads as W


class LayerStack:
    def __init__(self, cfg: W.MoEConfig, seed=0, device="cuda", recorded=4, trainer_gemm="w4a16"):
        self.cfg = cfg
        self.dev = torch.device(device)
        self.recorded = min(recorded, cfg.layers)
        if trainer_gemm not in ("w4a16", "library"):
            raise ValueError(f"unknown trainer GEMM {trainer_gemm!r}")
        self.trainer_gemm = trainer_gemm
        self.w_r = W.stack_router_weights(cfg, seed, device)               # [L, H, E] fp32
        T, H, E = cfg.T, cfg.H, cfg.E
        inp0 = W.moe_layer_inputs(cfg, seed, device, layer=0, with_logits=False)
        self.x0 = inp0["x"]
        # build layer by layer: each layer's channel sets are calibrated on the
        # activations that actually reach it
        self.layers = []
        x = self.x0.clone()
        logits = torch.empty(T, E, dtype=torch.float32, device=self.dev)
        for l in range(cfg.layers):
            inp = inp0 if l == 0 else W.moe_layer_inputs(cfg, seed, device, layer=l, with_logits=False)
            B.router_logits(x, self.w_r[l], out=logits)
            layer = L.build_layer(cfg, {"x": x, "logits": logits, "w_gu": inp["w_gu"], "w_d": inp["w_d"]}, device)
            layer.weight_sync()
            out = layer.rollout_forward(x, logits)
            x = B.residual_add(x, out)
            self.layers.append(layer)
        self.logits = logits
        # the trainer's own routing and expert-ordered operands (W4A16 path)
        cap = B.moe_rows_capacity(T, cfg.k, E)
        i32, bf = torch.int32, torch.bfloat16
        self.t_off = torch.empty(E + 1, dtype=i32, device=self.dev)
        self.t_row_of = torch.empty(T * cfg.k, dtype=i32, device=self.dev)
        self.t_src_of = torch.full((cap,), -1, dtype=i32, device=self.dev)
        self.t_ws = torch.empty(B.moe_permute_workspace_bytes(T, cfg.k, E), dtype=torch.uint8, device=self.dev)
        self.t_x = torch.zeros(cap, H, dtype=bf, device=self.dev)
        self.t_h = torch.empty(cap, cfg.F, dtype=bf, device=self.dev)
        self.t_hq = torch.empty(cap, cfg.F, dtype=bf, device=self.dev)     # W4A4: fake-quantized h
        self.t_amax = torch.empty(E, dtype=torch.float32, device=self.dev)
        self.t_y = torch.empty(cap, H, dtype=bf, device=self.dev)
        self.x_roll = torch.empty(cfg.layers + 1, T, H, dtype=torch.bfloat16, device=self.dev)
        self.x_train = torch.empty_like(self.x_roll)

    def is_recorded(self, l):
        return l >= self.cfg.layers - self.recorded

    def rollout(self, x0):
        """The rollout side through every layer; layer inputs in x_roll[l],
        the stack output in x_roll[L]."""
        self.x_roll[0].copy_(x0)
        for l, layer in enumerate(self.layers):
            B.router_logits(self.x_roll[l], self.w_r[l], out=self.logits)
            layer.weight_sync()
            out = layer.rollout_forward(self.x_roll[l], self.logits)
            if self.is_recorded(l):
                layer.export(l)
            B.residual_add(self.x_roll[l], out, out=self.x_roll[l + 1])
        return self.x_roll[self.cfg.layers]

    def _trainer_ffn(self, layer, x, idx, w, w4a4=False):
        """BF16 MoE FFN of one layer with the fake-quantized weights:
        y_t = sum_s w[t,s] W_d,fq[e] (silu(W_g,fq[e] x) * W_u,fq[e] x), e = idx[t,s].
        w4a4: x (per tensor) and each expert's h (per expert) fake-quantized
        too, by the device fake-quant kernel."""
        cfg = self.cfg
        y = torch.zeros(cfg.T, cfg.H, dtype=torch.float32, device=self.dev)
        if w4a4:
            x = B.fakequant_weight_ste(x.unsqueeze(0), want_codes=False)[0][0]
        flat = idx.reshape(-1).long()
        for e in torch.unique(flat).tolist():
            pos = (flat == e).nonzero().squeeze(1)
            t = pos // cfg.k
            gu = x[t] @ layer.w_gu_fq[e].t()
            h = (torch.nn.functional.silu(gu[:, :cfg.F].float()) * gu[:, cfg.F:].float()).to(torch.bfloat16)
            if w4a4:
                h = B.fakequant_weight_ste(h.unsqueeze(0).contiguous(), want_codes=False)[0][0]
            yd = (h @ layer.w_d_fq[e].t()).float()
            y.index_add_(0, t, yd * w.reshape(-1)[pos, None])
        return y.to(torch.bfloat16)

    def _trainer_ffn_w4a16(self, layer, x, idx, w, w4a4=False):
        """The same FFN on the W4A16 kernels: the trainer's routing permutes
        its BF16 rows into expert order (the gather kernel; pad rows zero),
        gate/up + SwiGLU and down read the NVFP4 weight codes, the combine
        kernel sums the slots.  w4a4: x fake-quantized first (one per-tensor
        scale) and h quantized per expert segment and dequantized before the
        down GEMM (one scale per expert)."""
        cfg = self.cfg
        E, H, F = cfg.E, cfg.H, cfg.F
        cap = self.t_x.shape[0]
        if w4a4:
            x = B.fakequant_weight_ste(x.unsqueeze(0), want_codes=False)[0][0]
        B.moe_permute(idx, E, self.t_off, self.t_row_of, self.t_src_of, self.t_ws)
        B.moe_gather_bf16(self.t_src_of, self.t_off, E, cap, x, out=self.t_x)
        B.moe_grouped_gemm_w4a16(self.t_x, layer.w_gu_codes, layer.w_gu_scales, layer.g_w_gu, self.t_off, E, cap,
                                 2 * F, H, y=self.t_h, swiglu=True, amax=self.t_amax)
        h = self.t_h
        if w4a4:
            # the per-expert max |h| comes from the SwiGLU epilogue
            codes, scales, g_h, _ = B.quantize_nvfp4(self.t_h, group_off=self.t_off, n_groups=E,
                                                     amax_in=self.t_amax, scale_layout=B.SCALES_TILED)
            h = B.dequant(codes, scales, B.SCALES_TILED, g_h, cap, F, group_off=self.t_off, n_groups=E,
                          out=self.t_hq)
        B.moe_grouped_gemm_w4a16(h, layer.w_d_codes, layer.w_d_scales, layer.g_w_d, self.t_off, E, cap, H,
                                 F, y=self.t_y)
        return B.moe_unpermute_combine(self.t_y, self.t_row_of, w, cfg.T, cfg.k, H)

    def _trainer_down_replayed(self, layer):
        """Down projection of a recorded layer from the replayed h (the
        rollout's effective down-GEMM input, expert-ordered), combined with the
        recorded routing."""
        cfg = self.cfg
        if self.trainer_gemm == "w4a16":
            B.moe_grouped_gemm_w4a16(layer.h_hat, layer.w_d_codes, layer.w_d_scales, layer.g_w_d, layer.expert_off,
                                     cfg.E, layer.cap, cfg.H, cfg.F, y=self.t_y)
            return B.moe_unpermute_combine(self.t_y, layer.row_of, layer.topk_w, cfg.T, cfg.k, cfg.H)
        off = layer.expert_off.tolist()
        Y = torch.zeros(layer.cap, cfg.H, dtype=torch.bfloat16, device=self.dev)
        for e in range(cfg.E):
            if off[e + 1] > off[e]:
                Y[off[e]:off[e + 1]] = layer.h_hat[off[e]:off[e + 1]] @ layer.w_d_fq[e].t()
        return B.moe_unpermute_combine(Y, layer.row_of, layer.topk_w, cfg.T, cfg.k, cfg.H)

    def trainer(self, x0_train, w4a4=False):
        """The trainer side through every layer; layer inputs in x_train[l].
        Recorded layers replay the record; returns (stack output, code
        mismatches, scale mismatches) over the recorded layers.  w4a4: the
        symmetric W4A4 QAT trainer instead (no replay; mismatches 0)."""
        cfg = self.cfg
        self.x_train[0].copy_(x0_train)
        code_mis = scale_mis = 0
        for l, layer in enumerate(self.layers):
            xl = self.x_train[l]
            if self.is_recorded(l) and not w4a4:
                layer.reset_counts()
                layer.trainer_replay(xl, layer_id=l)
                assert int(layer.status.item()) == 0 and int(layer.status_h.item()) == 0, "bad TRACE record"
                cnt = layer.counts.tolist()
                code_mis += cnt[0]
                scale_mis += cnt[1]
                y = self._trainer_down_replayed(layer)
            else:
                B.router_logits(xl, self.w_r[l], out=self.logits)
                idx, w = B.moe_router_topk(self.logits, cfg.k, True)
                if self.trainer_gemm == "w4a16" and layer.fuse_swiglu:
                    y = self._trainer_ffn_w4a16(layer, xl, idx, w, w4a4)
                else:
                    y = self._trainer_ffn(layer, xl, idx, w, w4a4)
            B.residual_add(xl, y, out=self.x_train[l + 1])
        return self.x_train[cfg.layers], code_mis, scale_mis

    def alignment_pass(self, drift=1e-3, seed=0, w4a4=False):
        """One train/rollout alignment pass: rollout, then the trainer on the
        rollout's input plus N(0, drift) engine drift.  Returns the per-token
        relative gap between the two stack outputs (a reported diagnostic)
        and the mismatch counts of the replayed layers."""
        y_r = self.rollout(self.x0)
        x0_t = W.engine_drift(self.x0, drift, seed=seed, device=self.dev)
        y_t, cm, sm = self.trainer(x0_t, w4a4=w4a4)
        a, b = y_r.float(), y_t.float()
        gap = torch.linalg.vector_norm(a - b, dim=1) / torch.linalg.vector_norm(b, dim=1).clamp_min(1e-30)
        return gap, cm, sm
