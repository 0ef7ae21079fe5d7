"""The NVFP4 scoring cache layout that include/qs.h documents is the one the library uses.

"Jet-QSparse: Accelerating Agentic LLM Inference with 4-Bit Sparse Attention" (Full text)
keeps the scoring keys in NVFP4 (E2M1 codes, one UE4M3 scale per 16 elements) and scans
them on FP4 tensor cores. The header gives the byte of every code and scale in a page:
  code of element e of token slot m:  (e / 32) * 2048 + m * 16 + (e % 32) / 2,
                                      low nibble for even e, high nibble for odd e;
  scale of elements 16j..16j+15:      (j / 4) * 512 + 16 * (m % 32) + 4 * (m / 32) + j % 4.
Through the C ABI: (1) pages written from the oracle's codes and scales with only those
formulas equal, byte for byte, the pages the library's writer (qs_append_kv) produces;
(2) qs_score over a cache filled with only those formulas (no library writer) gives the
oracle's block scores.
"""
import numpy as np
import pytest
import torch

import synth
from oracle import method as M
from tests.util import query_scale_all

pytestmark = pytest.mark.gpu


def _header_pages(codes, scales):
    """One row's codes [L][128] and scales [L][8] laid into pages with the header's
    formulas: (page codes [npg][8192], page scales [npg][1024])."""
    L = codes.shape[0]
    npg = -(-L // 128)
    pc = np.zeros((npg, 8192), dtype=np.uint8)
    ps = np.zeros((npg, 1024), dtype=np.uint8)
    for t in range(L):
        pg, m = divmod(t, 128)
        for e in range(128):
            byte = (e // 32) * 2048 + m * 16 + (e % 32) // 2
            pc[pg, byte] |= np.uint8(codes[t, e] << (4 * (e % 2)))
        for j in range(8):
            ps[pg, (j // 4) * 512 + 16 * (m % 32) + 4 * (m // 32) + j % 4] = scales[t, j]
    return pc, ps


def _rows(inp):
    w = inp.w
    out = {}
    for b in range(w.batch):
        L = int(inp.lens[b])
        for g in range(w.n_kv_heads):
            k, _, _ = inp.row(b, g)
            codes, scales = M.nvfp4_pack(M.centre(k[:L], inp.mu[b, g]), inp.g_k)
            out[b, g] = (codes, scales)
    return out


def test_writer_pages_follow_the_header():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from tests.gpu_util import Filled
    w = synth.small(synth.NVFP4_128K)
    inp = synth.Inputs(w)
    f = Filled(inp)
    f.decode()                                           # every row now holds L tokens
    proxy = f.layer.proxy.cpu().numpy().reshape(inp.num_pages, w.n_kv_heads, 8192)
    pscale = f.layer.proxy_scale.cpu().numpy().reshape(inp.num_pages, w.n_kv_heads, 1024)
    for (b, g), (codes, scales) in _rows(inp).items():
        L = int(inp.lens[b])
        pc, ps = _header_pages(codes, scales)
        pages = inp.page_table[b, :pc.shape[0]]
        tail = L % 128
        full = L // 128
        assert np.array_equal(proxy[pages[:full], g], pc[:full]), (b, g)
        assert np.array_equal(pscale[pages[:full], g], ps[:full]), (b, g)
        if tail:                                         # the written slots of the last page
            got_c = proxy[pages[full], g].reshape(4, 128, 16)[:, :tail]
            got_s = pscale[pages[full], g].reshape(2, 32, 4, 4)
            want_c = pc[full].reshape(4, 128, 16)[:, :tail]
            assert np.array_equal(got_c, want_c), (b, g)
            m = np.arange(tail)
            want_s = ps[full].reshape(2, 32, 4, 4)
            assert np.array_equal(got_s[:, m % 32, m // 32], want_s[:, m % 32, m // 32]), (b, g)


def test_scan_of_a_header_written_cache_matches_the_oracle():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import score_then_select_b200 as qs
    from score_then_select_b200.filled import cfg_kwargs, u16
    from score_then_select_b200.layer import Layer
    w = synth.small(synth.NVFP4_128K)
    inp = synth.Inputs(w)
    K, V, Q = inp.dense()
    lay = Layer.allocate(cfg_kwargs(w), w.batch, inp.num_pages, inp.page_table.shape[1],
                         int(inp.lens.max()))
    lay.page_table.copy_(torch.from_numpy(inp.page_table))
    lay.seq_lens.copy_(torch.from_numpy(inp.lens.astype(np.int32)))
    lay.key_center.copy_(torch.from_numpy(inp.mu))
    lay.key_gscale.fill_(float(inp.g_k))
    proxy = np.zeros((inp.num_pages, w.n_kv_heads, 8192), dtype=np.uint8)
    pscale = np.zeros((inp.num_pages, w.n_kv_heads, 1024), dtype=np.uint8)
    rows = _rows(inp)
    for (b, g), (codes, scales) in rows.items():
        pc, ps = _header_pages(codes, scales)
        pages = inp.page_table[b, :pc.shape[0]]
        proxy[pages, g] = pc
        pscale[pages, g] = ps
    lay.proxy.copy_(torch.from_numpy(proxy).view(lay.proxy.shape))
    lay.proxy_scale.copy_(torch.from_numpy(pscale).view(lay.proxy_scale.shape))
    q = u16(Q).cuda()
    scores = torch.full((w.batch, w.n_kv_heads, lay.nb_stride), np.nan, dtype=torch.float32,
                        device="cuda")
    qs.qs_score(lay.cfg, lay.cache(), q, None, w.batch, scores, lay.ws)
    st = qs.qs_device_status(lay.ws)
    assert st[0] == 0, f"device status {st}"
    scores = scores.cpu().numpy()
    gq = query_scale_all(inp, Q=Q)
    G = w.group
    for (b, g), (codes, scales) in rows.items():
        L = int(inp.lens[b])
        qx = (Q[b, g * G:(g + 1) * G].astype(np.uint32) << 16).view(np.float32)
        q_codes, q_scales = M.nvfp4_pack(qx, gq)
        hs = M.nvfp4_head_scores(q_codes, q_scales, gq, codes, scales, inp.g_k)
        beta = M.nvfp4_block_scores(hs, w.block_size)
        nb = -(-L // w.block_size)
        tol = 1e-4 * np.abs(beta).max()
        assert np.all(np.abs(scores[b, g, :nb] - beta) <= tol), (b, g)
