"""One NVFP4 MoE expert layer on both sides of RL alignment, driven through
the C ABI (every step runs in libquads kernels; torch only allocates).

Rollout side ([QUADS-fr §1], [QUADS-fr §2.2.B]): NVFP4 quantization of the
layer input with the residual of the calibrated high-residual channels,
top-k routing and expert permutation, the NVFP4 grouped gate/up GEMM with
compensation, SwiGLU, per-expert NVFP4 re-quantization of h with its own
compensation channels, the grouped down GEMM with compensation, and the
weighted combine.

Trainer side ([QUADS-fr §2.2.A], [TRACE]): weight fake-quant onto the
rollout's grid (one pass also produces the rollout's NVFP4 weights and the
compensation weight columns), the straight-through backward accumulated
into the master gradient, the export of the rollout's quantization record
and its replay against the trainer's activation.
"""
import contextlib
import math

import torch

from . import binding as B
from .workloads import MoEConfig


class StageTimer:
    """Optional CUDA-event marks between stages, one chain per stream: mark()
    records on the current stream, and a stage's duration is the time between
    its mark and the previous mark of the same stream.  external=True records
    them as external event nodes, which is how timing events are captured into
    a CUDA graph and re-recorded at every replay.  Marks named "start", or
    starting with "wait" or "join", end no kernel stage."""

    def __init__(self, enabled=False, external=False, only=None):
        self.enabled = enabled
        self.external = external
        self.only = None if only is None else set(only)       # record only these marks
        self.chains = {}

    def mark(self, name):
        if self.enabled and (self.only is None or name in self.only):
            s = torch.cuda.current_stream()
            ev = torch.cuda.Event(enable_timing=True, external=self.external)
            ev.record(s)
            self.chains.setdefault(s.cuda_stream, []).append((name, ev))

    @property
    def marks(self):
        """The chain of the first stream marked (the step's own stream)."""
        return next(iter(self.chains.values())) if self.chains else []

    def durations_ms(self):
        out = {}
        for chain in self.chains.values():
            for (_, e0), (name, e1) in zip(chain, chain[1:]):
                if not is_stage(name):
                    continue
                out[name] = out.get(name, 0.0) + e0.elapsed_time(e1)
        return out


def is_stage(name):
    return name != "start" and not name.startswith("wait") and not name.startswith("join")


class MoELayer:
    """Weights, calibrated channel sets and every buffer of one layer at a
    fixed token count; step() runs the whole path without allocating."""

    def __init__(self, cfg: MoEConfig, w_gu, w_d, chan_x, chan_h, device="cuda", fuse_swiglu=None, overlap=True,
                 fuse_requant=False, amax_h_init=None, comp="bf16", materialize_wfq=True, side_sms=None):
        self.cfg = cfg
        T, H, E, k, F = cfg.T, cfg.H, cfg.E, cfg.k, cfg.F
        dev = torch.device(device)
        self.dev = dev
        # trainer master weights, both matrices in one allocation so that one
        # amax pass covers both: down [E, H, F] first, then gate/up [E, 2F, H].
        # The amax pass reads gate/up last, so much of it is still in L2 when
        # the gate/up fake-quant reads it again right after.
        n_gu, n_d = E * 2 * F * H, E * H * F
        self.n_gu, self.n_d = n_gu, n_d
        self.w_all = torch.empty(n_d + n_gu, dtype=torch.bfloat16, device=dev)
        self.w_all[:n_d].copy_(w_d.reshape(-1))
        self.w_all[n_d:].copy_(w_gu.reshape(-1))
        self.w_d = self.w_all[:n_d].view(E, H, F)
        self.w_gu = self.w_all[n_d:].view(E, 2 * F, H)
        # rows of a common width for the joint amax: each expert matrix is a group
        kw = math.gcd(H, F)
        self.amax_k = kw if kw % 16 == 0 else 0
        if self.amax_k:
            offs = [e * H * F // kw for e in range(E)] + [(n_d + e * 2 * F * H) // kw for e in range(E + 1)]
            self.w_groups = torch.tensor(offs, dtype=torch.int32, device=dev)
        # SwiGLU in the gate/up GEMM's epilogue (rollout gate/up weights kept
        # in the 64-row interleaved gate/up order), else a separate pass
        self.fuse_swiglu = (F % 64 == 0) if fuse_swiglu is None else bool(fuse_swiglu)
        # NVFP4 quantization of h in the same epilogue too (delayed scaling:
        # each expert's scale comes from the previous step's max |h|, or from
        # amax_h_init on the first step), else a separate pass with this
        # step's exact amax
        self.fuse_requant = bool(fuse_requant)
        if self.fuse_requant and not self.fuse_swiglu:
            raise ValueError("fuse_requant needs the fused SwiGLU epilogue (F % 64 == 0)")
        # the compensation on the high-residual channels: "bf16" (R . Wc in
        # BF16 on the tensor cores) or "fp4" (the literal second quantization
        # pass: R and Wc NVFP4-quantized, multiplied in the main FP4 product;
        # channel lists padded with -1 to multiples of 64)
        if comp not in ("bf16", "fp4"):
            raise ValueError(f"unknown compensation {comp!r}")
        self.comp = comp
        if comp == "fp4":
            if not self.fuse_swiglu or self.fuse_requant:
                raise ValueError("the FP4 compensation runs with the fused SwiGLU epilogue, without fuse_requant")
            chan_x, chan_h = _pad_chan(chan_x, 64), _pad_chan(chan_h, 64)
        # the trainer's fake-quantized weights W_fq in HBM (False: a trainer
        # whose GEMMs are the W4A16 kernels reads the NVFP4 codes instead, so
        # the weight sync writes codes, scales and Wc only)
        self.materialize_wfq = bool(materialize_wfq)
        # the weight side of a step on its own stream (False: one stream)
        self.overlap = bool(overlap)
        # SMs of the overlapped step's STE backward; the rollout's GEMMs run on
        # the others meanwhile (0: every kernel sized to the whole device)
        n_sm = torch.cuda.get_device_properties(dev).multi_processor_count
        self.side_sms = SIDE_SMS_DEFAULT if side_sms is None else int(side_sms)
        if not 0 <= self.side_sms < n_sm:
            raise ValueError(f"side_sms must be in [0, {n_sm})")
        self.gemm_sms = n_sm - self.side_sms if self.side_sms else 0
        self.nc_x = int(chan_x.numel())
        self.nc_h = int(chan_h.numel())
        cap = B.moe_rows_capacity(T, k, E)
        self.cap = cap
        e = lambda shape, dt: torch.empty(shape, dtype=dt, device=dev)
        bf, u8, f32, i32 = torch.bfloat16, torch.uint8, torch.float32, torch.int32
        # TRACE record: the rollout's kernels write the recorded tensors (codes,
        # scales, per-tensor scales, residuals, expert offsets, top-k indices)
        # straight into their sections, so the export writes only the header
        slot_x = B.qtensor_shape(T, H, B.SCALES_LINEAR, 1, self.nc_x)
        slot_h = B.qtensor_shape(cap, F, B.SCALES_TILED, E, self.nc_h)
        self.record_bytes, hdr = B.trace_qrecord_layout(0, T, k, [slot_x, slot_h])
        self.record = torch.zeros(self.record_bytes, dtype=u8, device=dev)
        vx, vh = B.record_views(self.record, hdr, 0), B.record_views(self.record, hdr, 1)
        none_i32 = torch.empty(0, dtype=i32, device=dev)
        self.chan_x = vx["chan"] if self.nc_x else none_i32
        self.chan_h = vh["chan"] if self.nc_h else none_i32
        self.chan_x.copy_(chan_x.to(dev, torch.int32))
        self.chan_h.copy_(chan_h.to(dev, torch.int32))
        # weight sync outputs
        self.w_gu_fq, self.w_d_fq = e((E, 2 * F, H), bf), e((E, H, F), bf)
        self.w_gu_codes, self.w_d_codes = e((E, 2 * F, H // 2), u8), e((E, H, F // 2), u8)
        self.w_gu_scales = e((B.scales_bytes(E * 2 * F, H, B.SCALES_TILED),), u8)
        self.w_d_scales = e((B.scales_bytes(E * H, F, B.SCALES_TILED),), u8)
        self.g_w_gu, self.g_w_d = e((E,), f32), e((E,), f32)
        self.amax_w_all, self.amax_x = e((2 * E,), f32), e((1,), f32)   # down experts, then gate/up
        self.amax_w_d, self.amax_w_gu = self.amax_w_all[:E], self.amax_w_all[E:]
        self.wc_gu, self.wc_d = e((E, 2 * F, self.nc_x), bf), e((E, H, self.nc_h), bf)
        self.ws_w = e((B.quantize_workspace_bytes(E),), u8)
        # STE gradients (master gradient accumulated in place)
        self.grad_all = torch.zeros(n_gu + n_d, dtype=torch.bfloat16, device=dev)   # gate/up, then down
        self.grad_gu, self.grad_d = self.grad_all[:n_gu].view(E, 2 * F, H), self.grad_all[n_gu:].view(E, H, F)
        # rollout activations
        self.x_codes, self.x_scales = vx["codes"].view(T, H // 2), vx["scales"]
        self.g_x = vx["g"]
        self.x_resid = vx["resid"].view(T, self.nc_x) if self.nc_x else None
        self.ws_x = e((B.quantize_workspace_bytes(1),), u8)
        self.topk_idx = self.record[hdr.topk_idx_off:hdr.topk_idx_off + 4 * T * k].view(i32).view(T, k)
        self.topk_w = e((T, k), f32)
        # one expert: the record keeps no group offsets, so they live outside it
        goff = vh["group_off"] if vh["group_off"] is not None else e((E + 1,), i32)
        self.expert_off, self.row_of, self.src_of = goff, e((T * k,), i32), e((cap,), i32)
        self.ws_perm = e((B.moe_permute_workspace_bytes(T, k, E),), u8)
        self.pa_codes, self.pa_scales = e((cap, H // 2), u8), e((B.scales_bytes(cap, H, B.SCALES_TILED),), u8)
        self.pa_resid = e((cap, self.nc_x), bf)
        self.y_gu = None if self.fuse_swiglu else e((cap, 2 * F), bf)
        self.h, self.amax_h = e((cap, F), bf), e((E,), f32)
        self.amax_h_prev = torch.zeros(E, dtype=f32, device=dev)
        if amax_h_init is not None:
            self.amax_h_prev.copy_(amax_h_init)
        self.h_codes, self.h_scales = vh["codes"].view(cap, F // 2), vh["scales"]
        self.g_h = vh["g"]
        self.h_resid = vh["resid"].view(cap, self.nc_h) if self.nc_h else None
        self.y_d = e((cap, H), bf)
        self.out = e((T, H), bf)
        # TRACE record and replay outputs
        self._tsrc = [
            B.qtensor_src(self.x_codes, self.x_scales, self.g_x, T, H, B.SCALES_LINEAR, chan=self.chan_x,
                          resid=self.x_resid),
            B.qtensor_src(self.h_codes, self.h_scales, self.g_h, cap, F, B.SCALES_TILED, group_off=self.expert_off,
                          chan=self.chan_h, resid=self.h_resid),
        ]
        if comp == "fp4":
            z = lambda shape, dt: torch.zeros(shape, dtype=dt, device=dev)
            ts = lambda rows, k: e((B.scales_bytes(rows, k, B.SCALES_TILED),), u8)
            self.wcq_gu_codes, self.wcq_gu_scales = e((E * 2 * F, self.nc_x // 2), u8), ts(E * 2 * F, self.nc_x)
            self.wcq_d_codes, self.wcq_d_scales = e((E * H, self.nc_h // 2), u8), ts(E * H, self.nc_h)
            self.g_wc_gu, self.g_wc_d = e((E,), f32), e((E,), f32)
            self.ws_wc = e((B.quantize_workspace_bytes(E),), u8)
            self.amax_r_gu, self.amax_r_d = e((E,), f32), e((E,), f32)
            self.rq_codes, self.rq_scales = z((cap, self.nc_x // 2), u8), z((B.scales_bytes(cap, self.nc_x,
                                                                                          B.SCALES_TILED),), u8)
            self.rhq_codes, self.rhq_scales = z((cap, self.nc_h // 2), u8), z((B.scales_bytes(cap, self.nc_h,
                                                                                            B.SCALES_TILED),), u8)
            self.g_rq, self.g_rhq = e((E,), f32), e((E,), f32)
        self.x_hat, self.h_hat = e((T, H), bf), e((cap, F), bf)
        self.counts, self.status = torch.zeros(2, dtype=torch.int64, device=dev), e((1,), i32)
        self.status_h = e((1,), i32)
        # the weight side of a step runs on its own stream (see step())
        self.side = torch.cuda.Stream(device=dev)
        self.ev_w_gu, self.ev_w_d = torch.cuda.Event(), torch.cuda.Event()
        # and the trainer's replays on a third, as soon as their operand is recorded
        self.trn = torch.cuda.Stream(device=dev)
        self.ev_x, self.ev_h = torch.cuda.Event(), torch.cuda.Event()

    # ---------------------------------------------------------------- stages

    def weight_sync(self, timer=None):
        """Trainer fake-quant + the rollout's NVFP4 weights: one amax pass over
        both weight tensors, then one quantize pass per weight tensor."""
        t = timer or StageTimer(False)
        self._amax_w(t)
        self._fakequant_gate_up(t)
        self._fakequant_down(t)

    def _amax_w(self, t):
        E, F, H = self.cfg.E, self.cfg.F, self.cfg.H
        if self.amax_k:
            B.amax_bf16(self.w_all.view(-1, self.amax_k), self.w_groups, 2 * E, out=self.amax_w_all)
        else:
            B.amax_bf16(self.w_gu.view(E * 2 * F, H), n_groups=E, out=self.amax_w_gu)
            B.amax_bf16(self.w_d.view(E * H, F), n_groups=E, out=self.amax_w_d)
        t.mark("amax_w")

    def _amax_w_gate_up(self, t):
        E, F, H = self.cfg.E, self.cfg.F, self.cfg.H
        B.amax_bf16(self.w_gu.view(E * 2 * F, H), n_groups=E, out=self.amax_w_gu)
        t.mark("amax_w_gate_up")

    def _amax_w_down(self, t):
        E, F, H = self.cfg.E, self.cfg.F, self.cfg.H
        B.amax_bf16(self.w_d.view(E * H, F), n_groups=E, out=self.amax_w_d)
        t.mark("amax_w_down")

    def _fakequant_gate_up(self, t):
        B.fakequant_weight_ste(self.w_gu, True, self.chan_x, False, True, self.w_gu_fq, self.w_gu_codes,
                               self.w_gu_scales, self.g_w_gu, self.wc_gu, None, self.amax_w_gu,
                               gate_up=self.fuse_swiglu, want_wfq=self.materialize_wfq)
        t.mark("fakequant_w_gate_up")
        if self.comp == "fp4":
            E, F = self.cfg.E, self.cfg.F
            B.quantize_nvfp4(self.wc_gu.view(E * 2 * F, self.nc_x), n_groups=E, scale_layout=B.SCALES_TILED,
                             codes=self.wcq_gu_codes, scales=self.wcq_gu_scales, g_out=self.g_wc_gu, ws=self.ws_wc)
            t.mark("quantize_wc_gate_up")

    def _fakequant_down(self, t):
        B.fakequant_weight_ste(self.w_d, True, self.chan_h, False, True, self.w_d_fq, self.w_d_codes,
                               self.w_d_scales, self.g_w_d, self.wc_d, None, self.amax_w_d,
                               want_wfq=self.materialize_wfq)
        t.mark("fakequant_w_down")
        if self.comp == "fp4":
            E, H = self.cfg.E, self.cfg.H
            B.quantize_nvfp4(self.wc_d.view(E * H, self.nc_h), n_groups=E, scale_layout=B.SCALES_TILED,
                             codes=self.wcq_d_codes, scales=self.wcq_d_scales, g_out=self.g_wc_d, ws=self.ws_wc)
            t.mark("quantize_wc_down")

    def ste_backward(self, grad_gu_fq, grad_d_fq, timer=None):
        """Straight-through backward of both weight tensors, accumulated into
        the master gradient; one pass when the two incoming gradients are
        adjacent in one allocation (as grad_fq_buffers() makes them)."""
        t = timer or StageTimer(False)
        flat = _adjacent(grad_gu_fq, grad_d_fq)
        if flat is not None:
            B.fakequant_weight_ste_backward(flat, self.grad_all, accumulate=True)
        else:
            B.fakequant_weight_ste_backward(grad_gu_fq, self.grad_gu, accumulate=True)
            B.fakequant_weight_ste_backward(grad_d_fq, self.grad_d, accumulate=True)
        t.mark("ste_backward")

    def grad_fq_buffers(self):
        """(flat, gate/up view, down view): one allocation for the gradients
        with respect to both fake-quantized weights."""
        flat = torch.empty_like(self.grad_all)
        E, F, H = self.cfg.E, self.cfg.F, self.cfg.H
        return flat, flat[:self.n_gu].view(E, 2 * F, H), flat[self.n_gu:].view(E, H, F)

    def rollout_forward(self, x, logits, timer=None):
        """The rollout side of the layer on the current stream (the weights
        must be synced)."""
        t = timer or StageTimer(False)
        self._rollout_front(x, logits, t)
        self._rollout_gate_up(t)
        return self._rollout_down(t)

    def _rollout_front(self, x, logits, t):
        cfg = self.cfg
        T, H, E, k = cfg.T, cfg.H, cfg.E, cfg.k
        B.amax_bf16(x, out=self.amax_x)
        t.mark("amax_x")
        B.quantize_nvfp4(x, amax_in=self.amax_x, scale_layout=B.SCALES_LINEAR, chan=self.chan_x,
                         codes=self.x_codes, scales=self.x_scales, g_out=self.g_x, resid_out=self.x_resid)
        t.mark("quantize_x")
        B.moe_router_topk(logits, k, True, idx=self.topk_idx, w=self.topk_w)
        t.mark("router_topk")
        B.moe_permute(self.topk_idx, E, self.expert_off, self.row_of, self.src_of, self.ws_perm)
        t.mark("permute")
        B.moe_gather(self.src_of, self.expert_off, E, self.cap, self.x_codes, self.x_scales, H, self.x_resid,
                     self.pa_codes, self.pa_scales, self.pa_resid)
        t.mark("gather")

    def _rollout_gate_up(self, t):
        cfg = self.cfg
        H, E, F = cfg.H, cfg.E, cfg.F
        if self.comp == "fp4":
            B.moe_fp4_comp_amax(self.g_x, self.g_w_gu, self.g_wc_gu, E, out=self.amax_r_gu)
            B.quantize_nvfp4(self.pa_resid, group_off=self.expert_off, n_groups=E, amax_in=self.amax_r_gu,
                             scale_layout=B.SCALES_TILED, codes=self.rq_codes, scales=self.rq_scales,
                             g_out=self.g_rq)
            t.mark("quantize_r")
            B.moe_grouped_gemm_nvfp4_fp4comp(self.pa_codes, self.pa_scales, self.g_x, self.w_gu_codes,
                                             self.w_gu_scales, self.g_w_gu, self.expert_off, E, self.cap, 2 * F, H,
                                             self.rq_codes, self.rq_scales, self.wcq_gu_codes, self.wcq_gu_scales,
                                             self.nc_x, y=self.h, swiglu=True, amax=self.amax_h)
            t.mark("gemm_gate_up_swiglu_fp4comp")
        elif self.fuse_requant:
            B.moe_grouped_gemm_nvfp4_swiglu_quant(
                self.pa_codes, self.pa_scales, self.g_x, self.w_gu_codes, self.w_gu_scales, self.g_w_gu,
                self.expert_off, E, self.cap, F, H, self.amax_h_prev, chan_h=self.chan_h if self.nc_h else None,
                a_resid=self.pa_resid, w_resid=self.wc_gu, h_codes=self.h_codes, h_scales=self.h_scales,
                h_resid=self.h_resid, g_h=self.g_h, amax_h_out=self.amax_h)
            t.mark("gemm_gate_up_swiglu_quant")
            B.copy_f32(self.amax_h, self.amax_h_prev)   # the next step's scale
        elif self.fuse_swiglu:
            B.moe_grouped_gemm_nvfp4_swiglu(self.pa_codes, self.pa_scales, self.g_x, self.w_gu_codes,
                                            self.w_gu_scales, self.g_w_gu, self.expert_off, E, self.cap, F, H,
                                            self.pa_resid, self.wc_gu, h=self.h, amax=self.amax_h)
            t.mark("gemm_gate_up_swiglu")
        else:
            B.moe_grouped_gemm_nvfp4(self.pa_codes, self.pa_scales, self.g_x, self.w_gu_codes, self.w_gu_scales,
                                     self.g_w_gu, self.expert_off, E, self.cap, 2 * F, H, self.pa_resid, self.wc_gu,
                                     y=self.y_gu)
            t.mark("gemm_gate_up")
            B.swiglu(self.y_gu, F, self.expert_off, E, h=self.h, amax=self.amax_h)
            t.mark("swiglu")

    def _rollout_down(self, t, on_h=None):
        """quantize h (unless the gate/up GEMM did), the down GEMM and the
        combine; on_h() runs once h's record section is written."""
        cfg = self.cfg
        T, H, E, k, F = cfg.T, cfg.H, cfg.E, cfg.k, cfg.F
        if not self.fuse_requant:
            B.quantize_nvfp4(self.h, group_off=self.expert_off, n_groups=E, amax_in=self.amax_h,
                             scale_layout=B.SCALES_TILED, chan=self.chan_h, codes=self.h_codes,
                             scales=self.h_scales, g_out=self.g_h, resid_out=self.h_resid)
            t.mark("quantize_h")
        if on_h is not None:
            on_h()
        if self.comp == "fp4":
            B.moe_fp4_comp_amax(self.g_h, self.g_w_d, self.g_wc_d, E, out=self.amax_r_d)
            B.quantize_nvfp4(self.h_resid, group_off=self.expert_off, n_groups=E, amax_in=self.amax_r_d,
                             scale_layout=B.SCALES_TILED, codes=self.rhq_codes, scales=self.rhq_scales,
                             g_out=self.g_rhq)
            t.mark("quantize_rh")
            B.moe_grouped_gemm_nvfp4_fp4comp(self.h_codes, self.h_scales, self.g_h, self.w_d_codes, self.w_d_scales,
                                             self.g_w_d, self.expert_off, E, self.cap, H, F, self.rhq_codes,
                                             self.rhq_scales, self.wcq_d_codes, self.wcq_d_scales, self.nc_h,
                                             y=self.y_d)
            t.mark("gemm_down_fp4comp")
        else:
            B.moe_grouped_gemm_nvfp4(self.h_codes, self.h_scales, self.g_h, self.w_d_codes, self.w_d_scales,
                                     self.g_w_d, self.expert_off, E, self.cap, H, F, self.h_resid, self.wc_d,
                                     y=self.y_d)
            t.mark("gemm_down")
        B.moe_unpermute_combine(self.y_d, self.row_of, self.topk_w, T, k, H, out=self.out)
        t.mark("combine")
        return self.out

    def export(self, layer_id=0):
        B.trace_export_qrecord(layer_id, self.cfg.T, self.cfg.k, self.topk_idx, self._tsrc, record=self.record)

    def trainer_replay(self, x_train, layer_id=0, timer=None):
        t = timer or StageTimer(False)
        self._replay_x(x_train, layer_id, t)
        self._replay_h(layer_id, t)

    def _replay_x(self, x_train, layer_id, t):
        cfg = self.cfg
        B.trace_replay_qrecord(self.record, layer_id, 0, cfg.T, cfg.H, x_train=x_train, x_hat=self.x_hat,
                               counts=self.counts, status=self.status)
        t.mark("replay_x")

    def _replay_h(self, layer_id, t):
        B.trace_replay_qrecord(self.record, layer_id, 1, self.cap, self.cfg.F, x_hat=self.h_hat, status=self.status_h)
        t.mark("replay_h")

    def step(self, x, logits, x_train, grad_gu_fq, grad_d_fq, timer=None, layer_id=0):
        """One pass of the whole path over one batch, on three streams: the
        weight side (amax, fake-quant of gate/up then down, STE backward) on
        a side stream; the rollout forward on the calling stream, each GEMM
        waiting only for its own weights; the TRACE export (the record's
        header: its sections are written in place by the rollout's kernels)
        and the trainer's replays on a third stream, each replay as soon as
        its operand is recorded.  While the rollout's GEMMs run, the STE
        backward keeps to side_sms SMs and the GEMMs to the rest (the
        library's SM budget), so that the HBM-bound and the tensor-core work
        share the GPU instead of taking turns.  The call returns with the
        calling stream joined to both.  The replay's mismatch counters
        accumulate across steps (zero them with reset_counts())."""
        cfg = self.cfg
        T, H, E, k, F = cfg.T, cfg.H, cfg.E, cfg.k, cfg.F
        t = timer or StageTimer(False)
        main = torch.cuda.current_stream()
        t.mark("start")
        if not self.overlap:
            self._amax_w(t)
            self._fakequant_gate_up(t)
            self._fakequant_down(t)
            self._rollout_front(x, logits, t)
            self._rollout_gate_up(t)
            out = self._rollout_down(t)
            self.export(layer_id)
            t.mark("export")
            self.trainer_replay(x_train, layer_id, t)
            self.ste_backward(grad_gu_fq, grad_d_fq, t)
            return out
        self.side.wait_stream(main)
        with torch.cuda.stream(self.side):
            t.mark("start")
            if self.side_sms:
                # SMs split between the GEMMs and the STE: the whole weight
                # sync first (on every SM), then the STE on its own SMs
                # beside the GEMMs
                self._amax_w(t)
                self._fakequant_gate_up(t)
                self.ev_w_gu.record(self.side)
                self._fakequant_down(t)
                self.ev_w_d.record(self.side)
                with _sm_budget(self.side_sms):
                    self.ste_backward(grad_gu_fq, grad_d_fq, t)
            else:
                # gate/up first, so that the gate/up GEMM can start as early as
                # possible (its amax pass leaves the weights in L2 for the
                # fake-quant)
                self._amax_w_gate_up(t)
                self._fakequant_gate_up(t)
                self.ev_w_gu.record(self.side)
                self._amax_w_down(t)
                self._fakequant_down(t)
                self.ev_w_d.record(self.side)
                self.ste_backward(grad_gu_fq, grad_d_fq, t)
        self._rollout_front(x, logits, t)
        self.ev_x.record(main)
        self.trn.wait_event(self.ev_x)
        with torch.cuda.stream(self.trn):
            t.mark("start")
            self.export(layer_id)
            t.mark("export")
            self._replay_x(x_train, layer_id, t)
        # with the SMs split, the gate/up GEMM starts once both weights are
        # synced, so that it does not share the SMs with the fake-quant
        main.wait_event(self.ev_w_d if self.side_sms else self.ev_w_gu)
        t.mark("wait_w_gate_up")
        with _sm_budget(self.gemm_sms):
            self._rollout_gate_up(t)
        main.wait_event(self.ev_w_d)
        t.mark("wait_w_down")

        def replay_h_when_recorded():
            self.ev_h.record(main)
            self.trn.wait_event(self.ev_h)
            with torch.cuda.stream(self.trn):
                self._replay_h(layer_id, t)

        with _sm_budget(self.gemm_sms):
            out = self._rollout_down(t, replay_h_when_recorded)
        main.wait_stream(self.trn)
        main.wait_stream(self.side)
        t.mark("join")
        return out

    def reset_counts(self):
        self.counts.zero_()


# SMs given to the STE backward while the rollout's GEMMs run beside it in
# the overlapped step (the STE's bulk-copy kernel moves about 110 GB/s per
# SM; the GEMMs keep the other 108 SMs)
SIDE_SMS_DEFAULT = 40


@contextlib.contextmanager
def _sm_budget(n):
    """The library's SM budget set to n (0: none) for the launches inside."""
    if not n:
        yield
        return
    prev = B.set_sm_budget(n)
    try:
        yield
    finally:
        B.set_sm_budget(prev)


def _pad_chan(chan, multiple):
    """A channel list padded with -1 entries to a multiple of `multiple`."""
    chan = torch.as_tensor(chan).to(torch.int32)
    n = -(-chan.numel() // multiple) * multiple
    out = torch.full((n,), -1, dtype=torch.int32, device=chan.device)
    out[:chan.numel()] = chan
    return out


def _adjacent(a, b):
    """A flat view over a then b when b directly follows a in one storage."""
    if a.dtype != b.dtype or a.device != b.device or not (a.is_contiguous() and b.is_contiguous()):
        return None
    if a.untyped_storage().data_ptr() != b.untyped_storage().data_ptr():
        return None
    if b.storage_offset() != a.storage_offset() + a.numel():
        return None
    return torch.as_strided(a, (a.numel() + b.numel(),), (1,), a.storage_offset())


def calibrate_channels(x, n_sel):
    """Calibrated high-residual channel set (device kernels), padded with -1
    to a multiple of 16."""
    K = x.shape[1]
    scores = B.channel_scores(x)
    sel = B.select_channels(scores, n_sel)
    n_pad = -(-n_sel // 16) * 16
    out = torch.full((n_pad,), -1, dtype=torch.int32, device=x.device)
    out[:n_sel] = sel
    return out


def build_layer(cfg: MoEConfig, inputs, device="cuda", overlap=True, fuse_requant=False, comp="bf16",
                materialize_wfq=True, side_sms=None):
    """Layer from generated inputs: channel sets calibrated on the layer's own
    batch (X for the gate/up input, the uncompensated h for the down input);
    with fuse_requant, h's first-step per-expert amax is calibrated on the
    same batch."""
    x, logits = inputs["x"], inputs["logits"]
    chan_x = calibrate_channels(x, cfg.n_chan)
    empty = torch.full((16,), -1, dtype=torch.int32, device=device)
    probe = MoELayer(cfg, inputs["w_gu"], inputs["w_d"], chan_x, empty, device)
    probe.weight_sync()
    probe.rollout_forward(x, logits)
    torch.cuda.synchronize()
    n_rows = int(probe.expert_off[-1].item())
    chan_h = calibrate_channels(probe.h[:n_rows].contiguous(), cfg.n_chan_f)
    amax_h = probe.amax_h.clone()
    del probe
    return MoELayer(cfg, inputs["w_gu"], inputs["w_d"], chan_x, chan_h, device, overlap=overlap,
                    fuse_requant=fuse_requant, amax_h_init=amax_h if fuse_requant else None, comp=comp,
                    materialize_wfq=materialize_wfq, side_sms=side_sms)
