"""Expert parallelism over W ranks built from the C-ABI calls.

Each rank keeps E_loc = N_r / W of the routed experts (expert e on rank
e // E_loc), a copy of the router and of every shared expert, and routes its
own tokens.  One step on rank s:

    moe_route -> moe_permute_index (offsets, inv_row) -> all-gather of the loads
    -> moe_ep_plan -> moe_ep_dispatch (rows straight into each expert's rank)
    -> [all rows arrived] -> moe_expert_ffn on the received rows (E_loc groups)
    -> moe_ep_return (outputs straight back to their source rank and grouped
       position) -> [all outputs arrived] -> shared experts -> moe_combine

The arithmetic of every token is the single-device layer's, so the result is
bit-identical to MoELayer.forward on the same tokens.

EPGroupEmulated runs W ranks in one process on one GPU (each rank's buffers
are separate tensors; "arrived" is stream order): it drives exactly the
indexing of the multi-GPU path.  EPRankDistributed is one rank per process:
loads are all-gathered with torch.distributed and the receive / return
buffers are symmetric memory, so the copy kernels store straight into the
peers' buffers over NVLink.
"""
from __future__ import annotations

import torch

from . import (moe_combine, moe_ep_dispatch, moe_ep_plan, moe_ep_return, moe_expert_ffn,
               moe_expert_ffn_workspace_size, moe_permute_index, moe_permute_workspace_size,
               moe_route, moe_route_workspace_size, MOE_BF16, MOE_F32)
from .configs import LayerConfig


def _ws(nbytes, device):
    return torch.empty(max(int(nbytes), 256), dtype=torch.uint8, device=device)


def gather_counts(counts: torch.Tensor, group=None) -> torch.Tensor:
    """counts_all [W, N_r]: every rank's per-expert load, in rank order
    (NCCL on GPUs, gloo on CPU)."""
    import torch.distributed as dist
    W = dist.get_world_size(group)
    parts = [torch.empty_like(counts) for _ in range(W)]
    dist.all_gather(parts, counts.contiguous(), group=group)
    return torch.stack(parts)


class _EPRank:
    """State and phases of one expert-parallel rank (T_max tokens, W ranks)."""

    def __init__(self, cfg: LayerConfig, weights: dict, W: int, rank: int, T_max: int,
                 device, recv_rows=None, recv_tags=None, ret_rows=None):
        if cfg.dtype not in ("f32", "bf16"):
            raise ValueError("expert parallelism is implemented for f32 and bf16 layers")
        if cfg.N_r % W:
            raise ValueError("N_r must be a multiple of the number of ranks")
        c, dev = cfg, torch.device(device)
        self.cfg, self.W, self.rank, self.dev = cfg, W, rank, dev
        self.E_loc = c.N_r // W
        lo, hi = rank * self.E_loc, (rank + 1) * self.E_loc
        self.E, self.b = weights["E"], weights["b"]
        self.Wgu = weights["W_gate_up"][lo:hi]
        self.Wdn = weights["W_down"][lo:hi]
        self.Wsgu, self.Wsdn = weights["Ws_gate_up"], weights["Ws_down"]
        act = torch.float32 if c.dtype == "f32" else torch.bfloat16
        R = T_max * c.K
        cap = W * R                                   # every token of every rank at most once
        self.cap = cap
        self.topk_idx = torch.empty(T_max, c.K, dtype=torch.int32, device=dev)
        self.topk_gate = torch.empty(T_max, c.K, dtype=torch.float32, device=dev)
        self.counts = torch.zeros(c.N_r, dtype=torch.int32, device=dev)
        self.route_ws = _ws(moe_route_workspace_size(T_max, c.N_r), dev)
        self.perm_ws = _ws(moe_permute_workspace_size(T_max, c.N_r), dev)
        self.offsets = torch.zeros(c.N_r + 1, dtype=torch.int32, device=dev)
        self.perm_src = torch.empty(R, dtype=torch.int32, device=dev)
        self.inv_row = torch.empty(T_max, c.K, dtype=torch.int32, device=dev)
        self.recv_offsets = torch.zeros(self.E_loc + 1, dtype=torch.int32, device=dev)
        self.send_base = torch.zeros(c.N_r, dtype=torch.int32, device=dev)
        self.recv_rows = recv_rows if recv_rows is not None else \
            torch.empty(cap, c.d, dtype=act, device=dev)
        self.recv_tags = recv_tags if recv_tags is not None else \
            torch.empty(cap, 2, dtype=torch.int32, device=dev)
        self.ret_rows = ret_rows if ret_rows is not None else \
            torch.empty(R, c.d, dtype=act, device=dev)
        self.y_recv = torch.empty(cap, c.d, dtype=act, device=dev)
        self.y_shared_buf = torch.empty(max(c.N_s, 1) * T_max * c.d, dtype=act, device=dev)
        ffn_dt = MOE_F32 if c.dtype == "f32" else MOE_BF16
        self.ffn_ws = _ws(moe_expert_ffn_workspace_size(ffn_dt, cap, c.I), dev)
        self.h_out = torch.empty(T_max, c.d, dtype=act, device=dev)
        self.shared_offsets = torch.tensor([0, T_max], dtype=torch.int32, device=dev)

    # phases -------------------------------------------------------------------
    def route_permute(self, u, stream=None):
        c = self.cfg
        T = u.shape[0]
        self.T = T
        self.shared_offsets.fill_(T)
        self.shared_offsets[0] = 0
        self.u = u
        moe_route(u, self.E, self.b, c.K, self.topk_idx[:T], self.topk_gate[:T], self.counts,
                  self.route_ws, stream)
        # the grouping only: moe_ep_dispatch copies the rows from u itself
        moe_permute_index(self.topk_idx[:T], c.N_r, self.offsets, self.perm_src[:T * c.K],
                          self.inv_row[:T], self.perm_ws, stream=stream)

    def plan(self, counts_all, stream=None):
        if stream is not None:
            stream.wait_stream(torch.cuda.current_stream())   # counts_all gathered there
        moe_ep_plan(counts_all, self.rank, self.recv_offsets, self.send_base, stream)

    def dispatch(self, recv_rows, recv_tags, stream=None):
        T = self.T
        moe_ep_dispatch(self.u, self.topk_idx[:T], self.inv_row[:T], self.offsets, self.send_base,
                        self.rank, recv_rows, recv_tags, stream)

    def experts(self, stream=None):
        moe_expert_ffn(self.recv_rows, self.recv_offsets, self.Wgu, self.Wdn, self.y_recv,
                       self.ffn_ws, stream=stream)

    def give_back(self, ret_rows, stream=None):
        moe_ep_return(self.y_recv, self.recv_tags, self.recv_offsets[self.E_loc:], ret_rows,
                      stream)

    def combine(self, stream=None):
        c, T = self.cfg, self.T
        ys = self.y_shared_buf[:c.N_s * T * c.d].view(c.N_s, T, c.d)
        for j in range(c.N_s):
            moe_expert_ffn(self.u, self.shared_offsets, self.Wsgu[j:j + 1], self.Wsdn[j:j + 1],
                           ys[j], self.ffn_ws, stream=stream)
        moe_combine(self.u, ys if c.N_s else None, self.ret_rows[:T * c.K],
                    self.inv_row[:T], self.topk_gate[:T], self.h_out[:T], stream)
        return self.h_out[:T]


class EPGroupEmulated:
    """W expert-parallel ranks in one process on one GPU, run phase by phase
    (stream order stands in for the cross-rank waits)."""

    def __init__(self, cfg: LayerConfig, weights: dict, W: int, T_max: int, device="cuda"):
        self.ranks = [_EPRank(cfg, weights, W, r, T_max, device) for r in range(W)]

    def forward(self, u_list, stream=None):
        R = self.ranks
        for r, u in zip(R, u_list):
            r.route_permute(u, stream)
        if stream is not None:
            torch.cuda.current_stream().wait_stream(stream)   # the stack reads the loads
        counts_all = torch.stack([r.counts for r in R])
        for r in R:
            r.plan(counts_all, stream)
        recv_rows = [r.recv_rows for r in R]
        recv_tags = [r.recv_tags for r in R]
        for r in R:
            r.dispatch(recv_rows, recv_tags, stream)
        for r in R:
            r.experts(stream)
        ret_rows = [r.ret_rows for r in R]
        for r in R:
            r.give_back(ret_rows, stream)
        return [r.combine(stream) for r in R]


class EPRankDistributed:
    """One rank per process (torch.distributed initialised, one GPU each).
    Receive and return buffers live in symmetric memory so that dispatch and
    return store straight into the peers' buffers; loads are all-gathered.
    Not exercised on more than one GPU in this repository's tests."""

    def __init__(self, cfg: LayerConfig, weights: dict, T_max: int, group=None):
        import torch.distributed as dist
        import torch.distributed._symmetric_memory as symm
        W, rank = dist.get_world_size(group), dist.get_rank(group)
        dev = torch.device("cuda", torch.cuda.current_device())
        act = torch.float32 if cfg.dtype == "f32" else torch.bfloat16
        cap, R = W * T_max * cfg.K, T_max * cfg.K
        self.group = group
        self._bufs = []

        def shared(shape, dtype):
            t = symm.empty(*shape, dtype=dtype, device=dev)
            h = symm.rendezvous(t, group if group is not None else dist.group.WORLD)
            self._bufs.append((t, h))
            return t, [h.get_buffer(p, shape, dtype) for p in range(W)], h

        recv, self.peer_recv, self.h = shared((cap, cfg.d), act)
        tags, self.peer_tags, _ = shared((cap, 2), torch.int32)
        ret, self.peer_ret, _ = shared((R, cfg.d), act)
        self.r = _EPRank(cfg, weights, W, rank, T_max, dev, recv, tags, ret)

    def _arrived(self, stream):
        """Cross-rank wait between two phases, in stream order: this rank's
        work queued so far on `stream` is ordered before a barrier collective
        (NCCL: an all-reduce queued on the current stream, which completes
        only after every rank's copy of it ran, i.e. after every rank's
        earlier work), and the work queued next on `stream` after it."""
        import torch.distributed as dist
        cur = torch.cuda.current_stream()
        other = stream is not None and stream != cur
        if other:
            cur.wait_stream(stream)
        dist.barrier(group=self.group)
        if other:
            stream.wait_stream(cur)

    def forward(self, u, stream=None):
        r = self.r
        r.route_permute(u, stream)
        counts = r.counts
        if stream is not None:
            torch.cuda.current_stream().wait_stream(stream)   # the gather reads the load
        r.plan(gather_counts(counts, self.group), stream)
        r.dispatch(self.peer_recv, self.peer_tags, stream)
        self._arrived(stream)                    # every rank's rows have arrived
        r.experts(stream)
        r.give_back(self.peer_ret, stream)
        self._arrived(stream)                    # every rank's outputs have arrived
        return r.combine(stream)
