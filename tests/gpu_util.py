"""GPU-side helpers for the parity tests: fill a paged layer from synthetic inputs through
the C ABI and read results back. Only the seeded generator and the library are used."""
import numpy as np
import torch

import synth
import score_then_select_b200 as qs
from score_then_select_b200.layer import Layer


def cfg_kwargs(w: synth.Workload, attn_path: int = 0) -> dict:
    return dict(n_q_heads=w.n_q_heads, n_kv_heads=w.n_kv_heads, head_dim=w.head_dim,
                block_size=w.block_size, budget=w.budget, proxy_rank=w.proxy_rank,
                proxy_dtype=w.proxy_dtype, v_dtype=w.v_dtype, v_agg_dtype=w.v_agg_dtype,
                out_dtype=w.out_dtype, force_sink=w.force_sink, force_last=w.force_last,
                n_keep_hp=w.n_keep_hp, softmax_scale=w.softmax_scale, attn_path=attn_path)


def u16(a: np.ndarray, dt=torch.bfloat16) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(dt)


class Filled:
    """A layer holding L_b - 1 tokens per sequence, ready for one decode step."""

    def __init__(self, inp: synth.Inputs, dense=None, device="cuda", attn_path: int = 0):
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
        qs.qs_append_kv(self.cfg, self.cache, k_new, v_new, n_new, mx, self.P, w.batch, lay.ws)
        b_idx = np.arange(w.batch)
        self.k_last = u16(K[b_idx, :, lens - 1]).to(device)          # [b][Hkv][d]
        self.v_last = u16(V[b_idx, :, lens - 1], vdt).to(device)
        torch.cuda.synchronize()

    def decode(self):
        w, lay = self.w, self.layer
        out_dt = torch.float32 if w.out_dtype == "f32" else torch.bfloat16
        out = torch.zeros((w.batch, w.n_q_heads, w.head_dim), dtype=out_dt, device="cuda")
        sel = torch.full((w.batch, w.n_kv_heads, w.budget), -7, dtype=torch.int32, device="cuda")
        nsel = torch.zeros((w.batch, w.n_kv_heads), dtype=torch.int32, device="cuda")
        qs.qs_decode(self.cfg, self.cache, self.q, self.k_last, self.v_last, self.P, w.batch,
                     out, sel, nsel, lay.ws)
        return out, sel, nsel

    def status(self):
        return qs.qs_device_status(self.layer.ws)

    def row_proxy(self, b: int, g: int) -> np.ndarray:
        """The row's scoring cache read back in token order ([L][r] or codes/scales)."""
        L = int(self.inp.lens[b])
        npg = -(-L // 128)
        pages = torch.from_numpy(self.inp.page_table[b, :npg].astype(np.int64)).cuda()
        if self.w.proxy_dtype == "nvfp4":
            # page codes: [4 chunks][128 tokens][16 bytes], chunk c = bytes 16c..16c+15 of
            # the token's 64-byte row; page scales: token m, group j at
            # (j // 4) * 512 + 16 * (m % 32) + 4 * (m // 32) + j % 4 (layouts of include/qs.h)
            raw = self.layer.proxy[pages, g].reshape(npg, 4, 128, 16).cpu().numpy()
            c = raw.transpose(0, 2, 1, 3).reshape(npg * 128, 64)[:L]
            rs = self.layer.proxy_scale[pages, g].reshape(npg, 1024).cpu().numpy()
            m = np.arange(128)[:, None]
            j = np.arange(8)[None, :]
            idx = (j // 4) * 512 + 16 * (m % 32) + 4 * (m // 32) + j % 4
            s = rs[:, idx].reshape(npg * 128, 8)[:L]
            codes = np.empty((L, 128), dtype=np.uint8)
            codes[:, 0::2] = c & 15
            codes[:, 1::2] = c >> 4
            return codes, s
        if self.w.proxy_dtype == "centroid":
            nb = -(-L // self.w.block_size)
            return self.layer.proxy[pages, g].reshape(-1, self.w.head_dim)[:nb].cpu().numpy()
        p = self.layer.proxy[pages, g].reshape(npg * 128, -1)[:L]
        if self.w.proxy_dtype in ("f32", "e4m3"):
            return p.cpu().numpy()
        return p.view(torch.int16).cpu().numpy().view(np.uint16)


def out_to_f64(out: torch.Tensor) -> np.ndarray:
    return out.float().cpu().numpy().astype(np.float64)
