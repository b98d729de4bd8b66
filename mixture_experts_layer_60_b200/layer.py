"""The DeepSeekMoE layer step built from the C-ABI calls.

MoELayer owns the layer's device state (centroids, bias, expert weights,
FP8 copies of them) and the per-step buffers, and runs one step as
    moe_route -> [moe_quantize_1x128] -> moe_permute
    -> gate/up and down of the routed experts (bf16: with the shared experts
       as extra groups of the same two launches; FP8 / f32: the shared
       experts' moe_expert_ffn after them) -> moe_combine [-> moe_bias_update]
on one CUDA stream.  For training (bf16 or FP8), forward_train keeps the
activations the backward needs and backward(dh) returns du and fills
self.grad with the gradients of E and of every expert weight.  Every step of the layer runs in libmoe's kernels; this
module only allocates buffers and sequences calls.
"""
from __future__ import annotations

import torch

from . import (MOE_BF16, MOE_E4M3, MOE_F32, moe_bias_update, moe_combine, moe_combine_backward,
               moe_expert_down, moe_expert_down_shared, moe_expert_ffn, moe_expert_ffn_backward,
               moe_expert_ffn_backward_workspace_size, moe_expert_ffn_workspace_size,
               moe_expert_gate_up, moe_expert_gate_up_save, moe_expert_gate_up_shared, moe_permute,
               moe_permute_workspace_size, moe_quantize_128x128, moe_quantize_1x128, moe_route,
               moe_route_grouped, moe_route_workspace_size, moe_router_weight_grad,
               moe_unpermute_backward)
from .configs import LayerConfig

GAMMA = 0.001


def _ws(nbytes, device):
    return torch.empty(max(int(nbytes), 256), dtype=torch.uint8, device=device)


class MoELayer:
    def __init__(self, cfg: LayerConfig, weights: dict, T_max: int | None = None, device="cuda"):
        self.cfg = cfg
        self.device = torch.device(device)
        self.T_max = cfg.T if T_max is None else T_max
        self.E = weights["E"]
        self.b = weights["b"].clone()
        self.fp8 = cfg.dtype == "e4m3"
        if self.fp8:
            self.W = {k: self._quantise(weights[k]) for k in
                      ("W_gate_up", "W_down", "Ws_gate_up", "Ws_down")}
        else:
            self.W = {k: (weights[k], None) for k in ("W_gate_up", "W_down", "Ws_gate_up", "Ws_down")}
        self._alloc(self.T_max)

    # -- setup ---------------------------------------------------------------
    def _quantise(self, w):
        G, R, C = w.shape
        q = torch.empty(G, R, C, dtype=torch.uint8, device=self.device)
        s = torch.empty(G, R // 128, C // 128, dtype=torch.float32, device=self.device)
        moe_quantize_128x128(w, q, s)
        return q, s

    def _alloc(self, T):
        c, dev = self.cfg, self.device
        d, K, N_r, N_s = c.d, c.K, c.N_r, c.N_s
        R = T * K
        act = torch.float32 if c.dtype == "f32" else torch.bfloat16
        xdt = torch.uint8 if self.fp8 else act
        ffn_dt = {"f32": MOE_F32, "bf16": MOE_BF16, "e4m3": MOE_E4M3}[c.dtype]
        self.topk_idx = torch.empty(T, K, dtype=torch.int32, device=dev)
        self.topk_gate = torch.empty(T, K, dtype=torch.float32, device=dev)
        self.counts = torch.zeros(N_r, dtype=torch.int32, device=dev)
        self.route_ws = _ws(moe_route_workspace_size(T, N_r), dev)
        self.perm_ws = _ws(moe_permute_workspace_size(T, N_r), dev)
        self.x_perm = torch.empty(R, d, dtype=xdt, device=dev)
        self.offsets = torch.zeros(N_r + 1, dtype=torch.int32, device=dev)
        self.perm_src = torch.empty(R, dtype=torch.int32, device=dev)
        self.inv_row = torch.empty(T, K, dtype=torch.int32, device=dev)
        # bf16: the shared experts run as extra groups of the routed launches,
        # their rows after the routed ones in the same h and y buffers
        self.merged_shared = (c.dtype == "bf16" and N_s > 0 and d % 256 == 0
                              and c.I % 128 == 0)
        self.y_all = torch.empty(R + N_s * T, d, dtype=act, device=dev)
        self.y_perm = self.y_all[:R]
        self.y_shared = self.y_all[R:].view(N_s, T, d)
        self.ffn_ws = _ws(moe_expert_ffn_workspace_size(ffn_dt, T, c.I), dev)
        hdt = torch.uint8 if self.fp8 else act
        self.h_all = torch.empty(R + (N_s * T if self.merged_shared else 0), c.I, dtype=hdt,
                                 device=dev)
        self.h_mid = self.h_all[:R]
        self.h_scale = torch.empty(R, c.I // 128, dtype=torch.float32, device=dev) if self.fp8 \
            else None
        self.h_out = torch.empty(T, d, dtype=act, device=dev)
        self.shared_offsets = torch.tensor([0, T], dtype=torch.int32, device=dev)
        if self.fp8:
            self.u_q = torch.empty(T, d, dtype=torch.uint8, device=dev)
            self.u_s = torch.empty(T, d // 128, dtype=torch.float32, device=dev)
            self.x_scale = torch.empty(R, d // 128, dtype=torch.float32, device=dev)
        self.T_alloc = T

    # -- one step ------------------------------------------------------------
    def forward(self, u: torch.Tensor, stream=None, gate_up_events=None,
                out: torch.Tensor | None = None, phase_events=None) -> torch.Tensor:
        """h' for the T tokens of u, written to `out` (default: the layer's own
        h_out buffer, overwritten by the next call).  gate_up_events=(start,
        end) records CUDA events around the routed gate/up GEMM launch on the
        same stream; phase_events, a dict name -> (start, end) for any of
        "route", "permute", "gate_up", "down", "shared", "combine", records
        events around those phases."""
        c = self.cfg
        T = u.shape[0]
        if T != self.T_alloc:
            self._alloc(T)
        st = torch.cuda.current_stream() if stream is None else stream
        pe = phase_events or {}
        if gate_up_events:
            pe = dict(pe, gate_up=gate_up_events)

        def mark(name, i):
            if name in pe:
                pe[name][i].record(st)
        mark("route", 0)
        if c.n_groups > 1:
            moe_route_grouped(u, self.E, self.b, c.K, c.n_groups, c.topk_groups, self.topk_idx,
                              self.topk_gate, self.counts, self.route_ws, stream)
        else:
            moe_route(u, self.E, self.b, c.K, self.topk_idx, self.topk_gate, self.counts,
                      self.route_ws, stream)
        mark("route", 1)
        mark("permute", 0)
        if self.fp8:
            moe_quantize_1x128(u, self.u_q, self.u_s, stream)
            moe_permute(self.u_q, self.topk_idx, c.N_r, self.x_perm, self.offsets, self.perm_src,
                        self.inv_row, self.perm_ws, u_scale=self.u_s, x_scale=self.x_scale,
                        stream=stream)
            x_sh, xs_sh = self.u_q, self.u_s
        else:
            moe_permute(u, self.topk_idx, c.N_r, self.x_perm, self.offsets, self.perm_src,
                        self.inv_row, self.perm_ws, stream=stream)
            x_sh, xs_sh = u, None
        mark("permute", 1)
        (wgu, sgu), (wdn, sdn) = self.W["W_gate_up"], self.W["W_down"]
        (wsgu, ssgu), (wsdn, ssdn) = self.W["Ws_gate_up"], self.W["Ws_down"]
        if self.merged_shared:
            # routed + shared experts: one gate/up launch, one down launch
            mark("gate_up", 0)
            moe_expert_gate_up_shared(self.x_perm, self.offsets, wgu, u, wsgu, self.h_all,
                                      stream=stream)
            mark("gate_up", 1)
            mark("down", 0)
            moe_expert_down_shared(self.h_all, self.offsets, wdn, wsdn, T * c.K, T, self.y_all,
                                   stream=stream)
            mark("down", 1)
        else:
            mark("gate_up", 0)
            moe_expert_gate_up(self.x_perm, self.offsets, wgu, self.h_mid,
                               x_scale=self.x_scale if self.fp8 else None, w_scale_gate_up=sgu,
                               h_scale=self.h_scale, stream=stream)
            mark("gate_up", 1)
            mark("down", 0)
            moe_expert_down(self.h_mid, self.offsets, wdn, self.y_perm, h_scale=self.h_scale,
                            w_scale_down=sdn, stream=stream)
            mark("down", 1)
            mark("shared", 0)
            for j in range(c.N_s):
                moe_expert_ffn(x_sh, self.shared_offsets, wsgu[j:j + 1], wsdn[j:j + 1],
                               self.y_shared[j], self.ffn_ws, x_scale=xs_sh,
                               w_scale_gate_up=None if ssgu is None else ssgu[j:j + 1],
                               w_scale_down=None if ssdn is None else ssdn[j:j + 1],
                               stream=stream)
            mark("shared", 1)
        u_res = u
        h = self.h_out if out is None else out
        mark("combine", 0)
        moe_combine(u_res, self.y_shared if c.N_s else None, self.y_perm, self.inv_row,
                    self.topk_gate, h, stream)
        mark("combine", 1)
        return h

    # -- training (bf16 / FP8): forward that keeps activations, then the backward
    def _alloc_train(self, T):
        c, dev = self.cfg, self.device
        R, bf = T * c.K, torch.bfloat16
        self.a_gu = torch.empty(R, 2 * c.I, dtype=bf, device=dev)
        hdt = torch.uint8 if self.fp8 else bf
        self.h_s = torch.empty(c.N_s, T, c.I, dtype=hdt, device=dev)
        self.h_s_scale = torch.empty(c.N_s, T, c.I // 128, dtype=torch.float32, device=dev) \
            if self.fp8 else None
        self.a_s = torch.empty(c.N_s, T, 2 * c.I, dtype=bf, device=dev)
        self.dy_perm = torch.empty(R, c.d, dtype=bf, device=dev)
        self.d_gate = torch.empty(T, c.K, dtype=torch.float32, device=dev)
        self.d_logit = torch.empty(T, c.K, dtype=torch.float32, device=dev)
        self.d_logit_perm = torch.empty(R, dtype=torch.float32, device=dev)
        self.dx_perm = torch.empty(R, c.d, dtype=bf, device=dev)
        self.dx_s = torch.empty(c.N_s, T, c.d, dtype=bf, device=dev)
        self.du = torch.empty(T, c.d, dtype=bf, device=dev)
        dt = MOE_E4M3 if self.fp8 else MOE_BF16
        self.bwd_ws = _ws(max(moe_expert_ffn_backward_workspace_size(dt, R, c.d, c.I, c.N_r),
                              moe_expert_ffn_backward_workspace_size(dt, T, c.d, c.I, 1)), dev)
        if not hasattr(self, "grad"):
            self.grad = {k: torch.empty(self.W[k][0].shape, dtype=bf, device=dev) for k in
                         ("W_gate_up", "W_down", "Ws_gate_up", "Ws_down")}
            self.grad["E"] = torch.empty(c.N_r, c.d, dtype=torch.float32, device=dev)
        self.T_train = T

    def forward_train(self, u: torch.Tensor, stream=None) -> torch.Tensor:
        """forward() that also keeps the gate/up pre-activations and h of the
        routed and shared experts for backward().  bf16 and FP8 layers."""
        c = self.cfg
        if c.dtype not in ("bf16", "e4m3"):
            raise ValueError("the backward is implemented for bf16 and FP8 layers")
        T = u.shape[0]
        if T != self.T_alloc:
            self._alloc(T)
        if getattr(self, "T_train", None) != T:
            self._alloc_train(T)
        if c.n_groups > 1:
            moe_route_grouped(u, self.E, self.b, c.K, c.n_groups, c.topk_groups, self.topk_idx,
                              self.topk_gate, self.counts, self.route_ws, stream)
        else:
            moe_route(u, self.E, self.b, c.K, self.topk_idx, self.topk_gate, self.counts,
                      self.route_ws, stream)
        (wgu, sgu), (wdn, sdn) = self.W["W_gate_up"], self.W["W_down"]
        (wsgu, ssgu), (wsdn, ssdn) = self.W["Ws_gate_up"], self.W["Ws_down"]
        sl = lambda t, j: None if t is None else t[j:j + 1]
        if self.fp8:
            moe_quantize_1x128(u, self.u_q, self.u_s, stream)
            moe_permute(self.u_q, self.topk_idx, c.N_r, self.x_perm, self.offsets, self.perm_src,
                        self.inv_row, self.perm_ws, u_scale=self.u_s, x_scale=self.x_scale,
                        stream=stream)
            x_sh, xs_sh = self.u_q, self.u_s
        else:
            moe_permute(u, self.topk_idx, c.N_r, self.x_perm, self.offsets, self.perm_src,
                        self.inv_row, self.perm_ws, stream=stream)
            x_sh, xs_sh = u, None
        moe_expert_gate_up_save(self.x_perm, self.offsets, wgu, self.h_mid, self.a_gu,
                                x_scale=self.x_scale if self.fp8 else None, w_scale_gate_up=sgu,
                                h_scale=self.h_scale, stream=stream)
        moe_expert_down(self.h_mid, self.offsets, wdn, self.y_perm, h_scale=self.h_scale,
                        w_scale_down=sdn, stream=stream)
        for j in range(c.N_s):
            hs_scale = None if self.h_s_scale is None else self.h_s_scale[j]
            moe_expert_gate_up_save(x_sh, self.shared_offsets, wsgu[j:j + 1], self.h_s[j],
                                    self.a_s[j], x_scale=xs_sh, w_scale_gate_up=sl(ssgu, j),
                                    h_scale=hs_scale, stream=stream)
            moe_expert_down(self.h_s[j], self.shared_offsets, wsdn[j:j + 1], self.y_shared[j],
                            h_scale=hs_scale, w_scale_down=sl(ssdn, j), stream=stream)
        moe_combine(u, self.y_shared if c.N_s else None, self.y_perm, self.inv_row,
                    self.topk_gate, self.h_out, stream)
        self._u = u
        return self.h_out

    def backward(self, dh: torch.Tensor, stream=None, ffn_events=None) -> torch.Tensor:
        """Gradients for upstream dh = dL/dh' of the last forward_train:
        returns du (overwritten by the next call) and fills self.grad
        (E: float32; W_gate_up, W_down, Ws_gate_up, Ws_down: bf16).
        ffn_events=(start, end) records CUDA events around the routed expert
        FFN backward on the same stream."""
        c, g = self.cfg, self.grad
        u = self._u
        st = torch.cuda.current_stream() if stream is None else stream
        moe_combine_backward(dh, u, self.E, self.y_perm, self.inv_row, self.topk_idx,
                             self.topk_gate, self.dy_perm, self.d_gate, self.d_logit,
                             self.d_logit_perm, stream)
        if ffn_events:
            ffn_events[0].record(st)
        (wgu, sgu), (wdn, sdn) = self.W["W_gate_up"], self.W["W_down"]
        (wsgu, ssgu), (wsdn, ssdn) = self.W["Ws_gate_up"], self.W["Ws_down"]
        sl = lambda t, j: None if t is None else t[j:j + 1]
        if self.fp8:
            # the FP8 Wgrad re-quantises the layer input: rows of u through perm_src
            x_r, x_rows, h_r = u, self.perm_src, None
        else:
            x_r, x_rows, h_r = self.x_perm, None, self.h_mid
        moe_expert_ffn_backward(x_r, self.offsets, wgu, wdn, self.a_gu, h_r, self.dy_perm,
                                self.dx_perm, g["W_gate_up"], g["W_down"], self.bwd_ws,
                                x_rows=x_rows, w_scale_gate_up=sgu, w_scale_down=sdn,
                                stream=stream)
        if ffn_events:
            ffn_events[1].record(st)
        for j in range(c.N_s):
            moe_expert_ffn_backward(u, self.shared_offsets, wsgu[j:j + 1], wsdn[j:j + 1],
                                    self.a_s[j], None if self.fp8 else self.h_s[j], dh,
                                    self.dx_s[j], g["Ws_gate_up"][j:j + 1],
                                    g["Ws_down"][j:j + 1], self.bwd_ws,
                                    w_scale_gate_up=sl(ssgu, j), w_scale_down=sl(ssdn, j),
                                    stream=stream)
        moe_unpermute_backward(dh, self.dx_s if c.N_s else None, self.dx_perm, self.inv_row,
                               self.topk_idx, self.d_logit, self.E, self.du, stream)
        if self.fp8:
            moe_router_weight_grad(u, self.d_logit_perm, self.offsets, g["E"],
                                   x_rows=self.perm_src, stream=stream)
        else:
            moe_router_weight_grad(self.x_perm, self.d_logit_perm, self.offsets, g["E"],
                                   stream=stream)
        return self.du

    def bias_update(self, counts=None, T_total=None, stream=None):
        """b <- b -/+ gamma from the load of the last step (or from the given
        global counts / token total of data-parallel replicas)."""
        counts = self.counts if counts is None else counts
        T_total = self.T_alloc if T_total is None else T_total
        moe_bias_update(self.b, counts, T_total, self.cfg.K, GAMMA, stream)

    def step(self, u, stream=None, process_group=None):
        """One training-style step: forward, global load, bias update."""
        h = self.forward(u, stream)
        if process_group is not None:
            from .parallel_load import allreduce_load
            counts, T_total = allreduce_load(self.counts, u.shape[0], process_group)
            self.bias_update(counts, T_total, stream)
        else:
            self.bias_update(stream=stream)
        return h
