"""A decode step captured once into a CUDA graph and replayed.

Plumbing around the C ABI: the step's host->device copies of the new query, key and value
(from pinned host buffers), one qs_decode call and the device->host copy of the output are
recorded into a torch.cuda.CUDAGraph on a side stream; each replay is one graph launch, so
the per-step host cost is independent of the number of kernels in the step. The caller
fills the pinned input buffers (`q_host`, `k_host`, `v_host`) before `step()` and reads
`out_host` after it. Every kernel still runs in libqs.
"""
from __future__ import annotations

import torch

from . import binding as B


class CapturedDecode:
    def __init__(self, cfg, cache, P, batch, out, sel, nsel, ws, q_dev, k_dev, v_dev,
                 before=None, warmup: int = 2):
        """`before`: an optional callable recorded ahead of the copies (e.g. a device-side
        reset the caller wants replayed every step)."""
        self.q_host = torch.empty(q_dev.shape, dtype=q_dev.dtype).pin_memory()
        self.k_host = torch.empty(k_dev.shape, dtype=k_dev.dtype).pin_memory()
        self.v_host = torch.empty(v_dev.shape, dtype=v_dev.dtype).pin_memory()
        self.out_host = torch.empty(out.shape, dtype=out.dtype).pin_memory()
        self.h2d_bytes = sum(t.numel() * t.element_size()
                             for t in (self.q_host, self.k_host, self.v_host))
        self.d2h_bytes = self.out_host.numel() * self.out_host.element_size()
        self.stream = torch.cuda.Stream()
        args = (cfg, cache, q_dev, k_dev, v_dev, P, batch, out, sel, nsel, ws)

        def body():
            if before is not None:
                before()
            q_dev.copy_(self.q_host, non_blocking=True)
            k_dev.copy_(self.k_host, non_blocking=True)
            v_dev.copy_(self.v_host, non_blocking=True)
            B.qs_decode(*args, stream=self.stream)
            self.out_host.copy_(out, non_blocking=True)

        self.stream.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(self.stream):
            for _ in range(warmup):           # one-time kernel attributes are set here
                body()
        self.stream.synchronize()
        self.graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(self.graph, stream=self.stream):
            body()
        torch.cuda.current_stream().wait_stream(self.stream)

    def step(self):
        """Replay the step and wait for its output to reach `out_host`."""
        self.graph.replay()
        torch.cuda.current_stream().synchronize()
