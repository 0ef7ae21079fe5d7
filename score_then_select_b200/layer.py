"""Device buffers of one attention layer's paged caches, allocated with torch.

Plumbing only: torch provides device memory and streams; every step of the decode path
runs in libqs. Layouts are the ones documented in include/qs.h.
"""
from __future__ import annotations

from dataclasses import dataclass

import torch

from . import binding as B

_TORCH_DT = {"bf16": torch.bfloat16, "f16": torch.float16, "f32": torch.float32}


@dataclass
class Layer:
    cfg: B.qs_config
    batch: int
    max_context: int
    k: torch.Tensor
    v: torch.Tensor
    proxy: torch.Tensor
    page_table: torch.Tensor
    seq_lens: torch.Tensor
    ws: torch.Tensor
    proxy_scale: torch.Tensor | None = None
    block_err: torch.Tensor | None = None
    key_center: torch.Tensor | None = None
    key_gscale: torch.Tensor | None = None

    @staticmethod
    def allocate(cfg_kwargs: dict, batch: int, num_pages: int, max_pages_per_seq: int,
                 max_context: int, device="cuda") -> "Layer":
        cfg = B.make_config(**cfg_kwargs)
        Hkv, d, r = cfg.n_kv_heads, cfg.head_dim, cfg.proxy_rank
        ps = cfg.page_size
        vdt = _TORCH_DT["f16" if cfg.v_dtype == B.QS_F16 else "bf16"]
        k = torch.zeros((num_pages, Hkv, ps, d), dtype=torch.bfloat16, device=device)
        v = torch.zeros((num_pages, Hkv, ps, d), dtype=vdt, device=device)
        extra = {}
        if cfg.proxy_dtype == B.QS_SEMANTIC:
            # the semantic-block index lives outside the cache (qs_semantic_index)
            proxy = torch.zeros((16,), dtype=torch.uint8, device=device)
        elif cfg.proxy_dtype == B.QS_RABITQ:
            # per (page, KV head): page_size x d/8 bytes of code bits, then page_size FP32
            # factors; the row centres c
            proxy = torch.zeros((num_pages, Hkv, ps * (d // 8) + ps * 4), dtype=torch.uint8,
                                device=device)
            extra = dict(key_center=torch.zeros((batch, Hkv, d), dtype=torch.float32,
                                                device=device))
        elif cfg.proxy_dtype == B.QS_CENTROID:
            # per-block FP32 key sums: [num_pages][Hkv][page_size / S][d]
            proxy = torch.zeros((num_pages, Hkv, ps // cfg.block_size, d), dtype=torch.float32,
                                device=device)
        elif r > 0:
            pdt = {B.QS_F32: torch.float32, B.QS_E4M3: torch.uint8}.get(cfg.proxy_dtype,
                                                                        torch.bfloat16)
            proxy = torch.zeros((num_pages, Hkv, ps, r), dtype=pdt, device=device)
        else:
            proxy = torch.zeros((num_pages, Hkv, ps, d // 2), dtype=torch.uint8, device=device)
            nbs = -(-max_context // ps) * (ps // cfg.block_size)
            extra = dict(
                proxy_scale=torch.zeros((num_pages, Hkv, ps, d // 16), dtype=torch.uint8,
                                        device=device),
                block_err=torch.full((batch, Hkv, nbs), -1.0, dtype=torch.float32, device=device),
                key_center=torch.zeros((batch, Hkv, d), dtype=torch.float32, device=device),
                key_gscale=torch.zeros((1,), dtype=torch.float32, device=device))
        pt = torch.full((batch, max_pages_per_seq), -1, dtype=torch.int32, device=device)
        sl = torch.zeros((batch,), dtype=torch.int32, device=device)
        nbytes = B.qs_workspace_size(cfg, batch, max_context)
        ws = torch.zeros((nbytes,), dtype=torch.uint8, device=device)
        lay = Layer(cfg, batch, max_context, k, v, proxy, pt, sl, ws, **extra)
        B.qs_workspace_init(ws, nbytes)
        return lay

    def cache(self) -> B.qs_cache:
        return B.make_cache(k=self.k, v=self.v, proxy=self.proxy, page_table=self.page_table,
                            seq_lens=self.seq_lens, max_context=self.max_context,
                            proxy_scale=self.proxy_scale, block_err=self.block_err,
                            key_center=self.key_center, key_gscale=self.key_gscale)

    @property
    def nb_stride(self) -> int:
        ps = self.cfg.page_size
        return -(-self.max_context // ps) * (ps // self.cfg.block_size)


def workspace(nbytes: int, device="cuda") -> torch.Tensor:
    """A zeroed workspace of `nbytes` bytes, initialised for the library's calls."""
    ws = torch.zeros((nbytes,), dtype=torch.uint8, device=device)
    B.qs_workspace_init(ws, nbytes)
    return ws


@dataclass
class GatheredKV:
    """The compact buffers of gather-then-attend (filled by qs_gather_kv) and the cache view
    over them that qs_dense_attn reads: ceil(budget * block_size / 128) pages per sequence,
    page i of sequence b at b * pages_per_seq + i."""
    k: torch.Tensor
    v: torch.Tensor
    page_table: torch.Tensor
    seq_lens: torch.Tensor
    row_lens: torch.Tensor
    pages_per_seq: int

    @staticmethod
    def allocate(layer: Layer, fill: float | None = None) -> "GatheredKV":
        cfg = layer.cfg
        ps = cfg.page_size
        P = -(-cfg.budget * cfg.block_size // ps)
        dev = layer.k.device
        shape = (layer.batch * P, cfg.n_kv_heads, ps, cfg.head_dim)
        k = torch.empty(shape, dtype=layer.k.dtype, device=dev)
        v = torch.empty(shape, dtype=layer.v.dtype, device=dev)
        if fill is not None:
            k.fill_(fill)
            v.fill_(fill)
        pt = torch.arange(layer.batch * P, dtype=torch.int32, device=dev).reshape(layer.batch, P)
        sl = torch.zeros((layer.batch,), dtype=torch.int32, device=dev)
        rl = torch.zeros((layer.batch * cfg.n_kv_heads,), dtype=torch.int32, device=dev)
        return GatheredKV(k, v, pt, sl, rl, P)

    @property
    def max_context(self) -> int:
        return self.pages_per_seq * 128

    def cache(self) -> B.qs_cache:
        return B.make_cache(k=self.k, v=self.v, proxy=None, page_table=self.page_table,
                            seq_lens=self.seq_lens, max_context=self.max_context)
