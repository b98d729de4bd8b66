"""Layer steps on tokens that live in pinned host memory.

HostStepper overlaps each step's upload of u (host -> device) and download of
h' (device -> host) with the neighbouring steps' compute: uploads run on one
copy stream, downloads on another (both directions of the link at once), the
layer on the caller's current stream, with double-buffered device copies of
u and h' ordered by CUDA events.  Every step still moves its own bytes; only
the waiting is hidden.
"""
from __future__ import annotations

import torch


class HostStepper:
    def __init__(self, T: int, d: int, dtype: torch.dtype, device):
        self.device = torch.device(device)
        self.u_dev = [torch.empty(T, d, dtype=dtype, device=self.device) for _ in range(2)]
        self.h_dev = [torch.empty(T, d, dtype=dtype, device=self.device) for _ in range(2)]
        self.up = torch.cuda.Stream(self.device)
        self.down = torch.cuda.Stream(self.device)
        self.uploaded = [torch.cuda.Event() for _ in range(2)]
        self.computed = [torch.cuda.Event() for _ in range(2)]
        self.downloaded = [torch.cuda.Event() for _ in range(2)]

    def run(self, u_hosts, h_hosts, step_fn):
        """For i in range(len(u_hosts)): h_hosts[i] <- step_fn(u_dev, out) on
        u_hosts[i].  step_fn(u, out) must enqueue the step on the current
        stream and write h' into `out`.  Returns when everything is enqueued;
        the current stream waits for the last download."""
        n = len(u_hosts)
        comp = torch.cuda.current_stream(self.device)
        self.up.wait_stream(comp)
        self.down.wait_stream(comp)
        with torch.cuda.stream(self.up):
            self.u_dev[0].copy_(u_hosts[0], non_blocking=True)
            self.uploaded[0].record(self.up)
        for i in range(n):
            b = i % 2
            if i + 1 < n:
                nb = (i + 1) % 2
                with torch.cuda.stream(self.up):
                    if i >= 1:
                        self.up.wait_event(self.computed[nb])     # step i-1 is done with u_dev[nb]
                    self.u_dev[nb].copy_(u_hosts[i + 1], non_blocking=True)
                    self.uploaded[nb].record(self.up)
            comp.wait_event(self.uploaded[b])
            if i >= 2:
                comp.wait_event(self.downloaded[b])               # h_dev[b] of step i-2 is on the host
            step_fn(self.u_dev[b], self.h_dev[b])
            self.computed[b].record(comp)
            with torch.cuda.stream(self.down):
                self.down.wait_event(self.computed[b])
                h_hosts[i].copy_(self.h_dev[b], non_blocking=True)
                self.downloaded[b].record(self.down)
        comp.wait_stream(self.down)
        comp.wait_stream(self.up)
