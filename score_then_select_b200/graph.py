"""A decode step captured once into a CUDA graph and replayed.

Plumbing around the C ABI: the step's new query, key and value live in one pinned host
buffer and one device buffer (each input a 256-byte aligned slice), so the step uploads
them with a single host->device copy; then one qs_decode call and the device->host copy
of the output. All of it is recorded into a torch.cuda.CUDAGraph on a side stream; each
replay is one graph launch, so the per-step host cost is independent of the number of
kernels in the step. The caller fills the pinned input views (`q_host`, `k_host`,
`v_host`) before `step()` and reads `out_host` after it. Every kernel runs in libqs.
"""
from __future__ import annotations

import torch

from . import binding as B

_ALIGN = 256


class CapturedDecode:
    def __init__(self, cfg, cache, P, batch, out, sel, nsel, ws, q_like, k_like, v_like,
                 before=None, warmup: int = 2, call=None):
        """`q_like`, `k_like`, `v_like`: tensors giving the shapes and dtypes of the step's
        inputs. `before`: an optional callable recorded ahead of the copy (e.g. a
        device-side reset the caller wants replayed every step). `call`: an optional
        callable (q, k_new, v_new, stream) that issues the step instead of qs_decode, e.g.
        qs_decode_top_p with its extra arguments bound."""
        offs, total = [], 0
        for t in (q_like, k_like, v_like):
            offs.append(total)
            total += -(-t.numel() * t.element_size() // _ALIGN) * _ALIGN
        self.host_buf = torch.empty(total, dtype=torch.uint8).pin_memory()
        self.dev_buf = torch.empty(total, dtype=torch.uint8, device=out.device)

        def view(buf, off, like):
            n = like.numel() * like.element_size()
            return buf[off:off + n].view(like.dtype).view(like.shape)

        self.q_host, self.k_host, self.v_host = (view(self.host_buf, o, t)
                                                 for o, t in zip(offs, (q_like, k_like, v_like)))
        q_dev, k_dev, v_dev = (view(self.dev_buf, o, t)
                               for o, t in zip(offs, (q_like, k_like, v_like)))
        self.out_host = torch.empty(out.shape, dtype=out.dtype).pin_memory()
        self.h2d_bytes = total
        self.d2h_bytes = self.out_host.numel() * self.out_host.element_size()
        self.stream = torch.cuda.Stream()
        args = (cfg, cache, q_dev, k_dev, v_dev, P, batch, out, sel, nsel, ws)

        def body():
            if before is not None:
                before()
            self.dev_buf.copy_(self.host_buf, non_blocking=True)
            if call is None:
                B.qs_decode(*args, stream=self.stream)
            else:
                call(q_dev, k_dev, v_dev, self.stream)
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
