"""GPU-side helpers for the parity tests: a paged layer filled from synthetic inputs through
the C ABI (score_then_select_b200.filled), and reading its caches back."""
import numpy as np
import torch

from score_then_select_b200.filled import Filled as _Filled, cfg_kwargs, u16  # noqa: F401


class Filled(_Filled):
    """The library's filled layer, plus reading a row's scoring cache back."""

    def host_caches(self):
        """Host copies of the scoring cache (and NVFP4 scales), for reading many rows."""
        lay = self.layer
        ps = lay.proxy_scale.cpu() if lay.proxy_scale is not None else None
        return lay.proxy.cpu(), ps

    def row_proxy(self, b: int, g: int, host=None) -> np.ndarray:
        """The row's scoring cache read back in token order ([L][r] or codes/scales), from
        the device or from host_caches()."""
        L = int(self.inp.lens[b])
        npg = -(-L // 128)
        pages = torch.from_numpy(self.inp.page_table[b, :npg].astype(np.int64))
        proxy, proxy_scale = host if host is not None else (self.layer.proxy,
                                                             self.layer.proxy_scale)
        if host is None:
            pages = pages.cuda()
        if self.w.proxy_dtype == "nvfp4":
            # page codes: [4 chunks][128 tokens][16 bytes], chunk c = bytes 16c..16c+15 of
            # the token's 64-byte row; page scales: token m, group j at
            # (j // 4) * 512 + 16 * (m % 32) + 4 * (m // 32) + j % 4 (layouts of include/qs.h)
            raw = proxy[pages, g].reshape(npg, 4, 128, 16).cpu().numpy()
            c = raw.transpose(0, 2, 1, 3).reshape(npg * 128, 64)[:L]
            rs = proxy_scale[pages, g].reshape(npg, 1024).cpu().numpy()
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
            return proxy[pages, g].reshape(-1, self.w.head_dim)[:nb].cpu().numpy()
        p = proxy[pages, g].reshape(npg * 128, -1)[:L]
        if self.w.proxy_dtype in ("f32", "e4m3"):
            return p.cpu().numpy()
        return p.view(torch.int16).cpu().numpy().view(np.uint16)


def out_to_f64(out: torch.Tensor) -> np.ndarray:
    return out.float().cpu().numpy().astype(np.float64)
