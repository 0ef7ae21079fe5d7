"""A paged layer filled from a synthetic workload, ready for one decode step.

Set-up only: the caches are written through the library's own writer (qs_append_kv), and
the decode step is one qs_decode call. `inp` is a synthetic input set (synth.Inputs):
shapes, lengths, page table and the seeded key/value/query bits.
"""
from __future__ import annotations

import numpy as np
import torch

from . import binding as B
from .layer import Layer


def cfg_kwargs(w, attn_path: int = 0) -> dict:
    """qs_config fields of a workload description (synth.Workload)."""
    return dict(n_q_heads=w.n_q_heads, n_kv_heads=w.n_kv_heads, head_dim=w.head_dim,
                block_size=w.block_size, budget=w.budget, proxy_rank=w.proxy_rank,
                proxy_dtype=w.proxy_dtype, v_dtype=w.v_dtype, v_agg_dtype=w.v_agg_dtype,
                out_dtype=w.out_dtype, force_sink=w.force_sink, force_last=w.force_last,
                n_keep_hp=w.n_keep_hp, softmax_scale=w.softmax_scale, attn_path=attn_path,
                key_storage=getattr(w, "key_storage", "bf16"))


def u16(a: np.ndarray, dt=torch.bfloat16) -> torch.Tensor:
    """16-bit float bits held in a uint16 array, as a torch tensor of that float type."""
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(dt)


class Filled:
    """A layer holding L_b - 1 tokens per sequence, ready for one decode step."""

    def __init__(self, inp, dense=None, device="cuda", attn_path: int = 0):
        w = inp.w
        self.inp, self.w = inp, w
        lens = inp.lens
        K, V, Q = dense if dense is not None else inp.dense()
        self.K, self.V, self.Q = K, V, Q
        Lmax = int(lens.max())
        vdt = torch.float16 if w.v_dtype == "f16" else torch.bfloat16
        self.layer = Layer.allocate(cfg_kwargs(w, attn_path), w.batch, inp.num_pages,
                                    inp.page_table.shape[1], Lmax, device)
        lay = self.layer
        lay.page_table.copy_(torch.from_numpy(inp.page_table))
        if w.proxy_dtype in ("nvfp4", "rabitq"):
            lay.key_center.copy_(torch.from_numpy(inp.mu))
        if w.proxy_dtype == "nvfp4":
            lay.key_gscale.fill_(float(inp.g_k))
        self.P = torch.from_numpy(np.array(inp.P)).to(device) if inp.P is not None else None
        self.q = u16(Q).to(device)
        self.cfg = lay.cfg
        self.cache = lay.cache()
        # bulk append of the first L_b - 1 tokens of every sequence
        mx = max(Lmax - 1, 1)
        k_new = u16(K[:, :, :mx]).to(device)
        v_new = u16(V[:, :, :mx], vdt).to(device)
        n_new = torch.from_numpy((lens - 1).astype(np.int32)).to(device)
        B.qs_append_kv(self.cfg, self.cache, k_new, v_new, n_new, mx, self.P, w.batch, lay.ws)
        b_idx = np.arange(w.batch)
        self.k_last = u16(K[b_idx, :, lens - 1]).to(device)          # [b][Hkv][d]
        self.v_last = u16(V[b_idx, :, lens - 1], vdt).to(device)
        torch.cuda.synchronize()

    def decode(self):
        """One qs_decode step: (out [b][Hq][d], sel [b][Hkv][budget], n_sel [b][Hkv])."""
        w, lay = self.w, self.layer
        out_dt = torch.float32 if w.out_dtype == "f32" else torch.bfloat16
        out = torch.zeros((w.batch, w.n_q_heads, w.head_dim), dtype=out_dt, device="cuda")
        sel = torch.full((w.batch, w.n_kv_heads, w.budget), -7, dtype=torch.int32, device="cuda")
        nsel = torch.zeros((w.batch, w.n_kv_heads), dtype=torch.int32, device="cuda")
        B.qs_decode(self.cfg, self.cache, self.q, self.k_last, self.v_last, self.P, w.batch,
                    out, sel, nsel, lay.ws)
        return out, sel, nsel

    def status(self):
        return B.qs_device_status(self.layer.ws)
