"""ctypes binding of libqs (include/qs.h): the same entry points, argument marshalling only.

Every function takes device buffers as torch tensors (or raw integer addresses) and a CUDA
stream (a torch.cuda.Stream, a raw handle, or None for torch's current stream), calls the
C entry point of the same name, and raises QsError when it returns a status other than
QS_OK. No computation happens here.
"""
from __future__ import annotations

import ctypes
import os

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libqs.so")

QS_OK, QS_ERR_INVALID_ARG, QS_ERR_UNSUPPORTED, QS_ERR_CUDA, QS_ERR_DEVICE_BOUNDS, \
    QS_ERR_DEVICE_TIMEOUT = range(6)
QS_F32, QS_BF16, QS_F16, QS_NVFP4, QS_E4M3, QS_CENTROID, QS_RABITQ, QS_SEMANTIC = range(8)
DTYPE_CODES = {"f32": QS_F32, "bf16": QS_BF16, "f16": QS_F16, "nvfp4": QS_NVFP4,
               "e4m3": QS_E4M3, "centroid": QS_CENTROID, "rabitq": QS_RABITQ,
               "semantic": QS_SEMANTIC}


class QsError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)} ({status})")


class qs_config(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in (
        "n_q_heads", "n_kv_heads", "head_dim", "page_size", "block_size", "budget",
        "proxy_rank", "proxy_dtype", "v_dtype", "v_agg_dtype", "out_dtype", "force_sink",
        "force_last", "n_keep_hp")] + [("softmax_scale", ctypes.c_float),
                                         ("attn_path", ctypes.c_int32),
                                         ("key_storage", ctypes.c_int32)]


class qs_cache(ctypes.Structure):
    _fields_ = [("k", ctypes.c_void_p), ("v", ctypes.c_void_p), ("proxy", ctypes.c_void_p),
                ("proxy_scale", ctypes.c_void_p), ("block_err", ctypes.c_void_p),
                ("key_center", ctypes.c_void_p), ("key_gscale", ctypes.c_void_p),
                ("page_table", ctypes.c_void_p), ("seq_lens", ctypes.c_void_p),
                ("max_pages_per_seq", ctypes.c_int32), ("num_pages", ctypes.c_int32),
                ("max_context", ctypes.c_int32)]


_lib = None


def lib() -> ctypes.CDLL:
    """Load libqs.so from the package directory; fail loudly if it was not built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: build it with "
                              "`python -m score_then_select_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        vp, i32, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_size_t
        cfgp, cachep = ctypes.POINTER(qs_config), ctypes.POINTER(qs_cache)
        sig = {
            "qs_version": ([], i32),
            "qs_status_string": ([i32], ctypes.c_char_p),
            "qs_workspace_size": ([cfgp, i32, i32, ctypes.POINTER(sz)], i32),
            "qs_workspace_init": ([vp, sz, vp], i32),
            "qs_attention_launches": ([cfgp, i32, i32, ctypes.POINTER(i32)], i32),
            "qs_selftest_wait_timeout": ([vp, vp], i32),
            "qs_append_kv": ([cfgp, cachep, vp, vp, vp, i32, vp, i32, vp, vp], i32),
            "qs_score": ([cfgp, cachep, vp, vp, i32, vp, vp, vp], i32),
            "qs_select_topk": ([cfgp, cachep, vp, i32, vp, vp, vp, vp], i32),
            "qs_sparse_attn": ([cfgp, cachep, vp, vp, vp, i32, vp, vp, vp], i32),
            "qs_decode": ([cfgp, cachep, vp, vp, vp, vp, i32, vp, vp, vp, vp, vp], i32),
            "qs_device_status": ([vp, vp, ctypes.POINTER(ctypes.c_uint32)], i32),
            "qs_sparse_attn_noalloc": ([cfgp, cachep, vp, vp, vp, i32, vp, vp], i32),
            "qs_dense_workspace_size": ([cfgp, i32, i32, ctypes.POINTER(sz)], i32),
            "qs_dense_attn": ([cfgp, cachep, vp, vp, i32, vp, vp, vp], i32),
            "qs_gather_kv": ([cfgp, cachep, vp, vp, i32, vp, vp, vp, vp, vp], i32),
            "qs_calib_workspace_size": ([cfgp, ctypes.POINTER(sz)], i32),
            "qs_calibrate_basis": ([cfgp, vp, vp, i32, vp, vp, vp, vp], i32),
            "qs_rabitq_score": ([cfgp, cachep, vp, vp, vp, i32, vp, vp, vp], i32),
            "qs_select_top_p": ([cfgp, cachep, vp, ctypes.c_float, i32, vp, vp, vp, vp], i32),
            "qs_decode_top_p": ([cfgp, cachep, vp, vp, vp, vp, vp, ctypes.c_float, i32, vp, vp,
                                 vp, vp, vp], i32),
            "qs_gather_kv_nvfp4k": ([cfgp, cachep, vp, vp, i32, vp, vp, vp, vp, vp], i32),
            "qs_select_topk_radix": ([cfgp, cachep, vp, i32, vp, vp, vp, vp], i32),
            "qs_semantic_index_workspace_size": ([cfgp, i32, i32, ctypes.POINTER(sz)], i32),
            "qs_semantic_index": ([cfgp, cachep, vp, i32, vp, vp, vp, i32, vp, vp], i32),
            "qs_semantic_select": ([cfgp, cachep, vp, vp, vp, vp, vp, i32, vp, vp, i32, vp, vp],
                                   i32),
        }
        for name, (args, res) in sig.items():
            f = getattr(L, name)
            f.argtypes = args
            f.restype = res
        _lib = L
    return _lib


EXPORTS = ("qs_version", "qs_status_string", "qs_workspace_size", "qs_workspace_init",
           "qs_append_kv", "qs_score", "qs_select_topk", "qs_sparse_attn", "qs_decode",
           "qs_device_status", "qs_sparse_attn_noalloc", "qs_attention_launches",
           "qs_selftest_wait_timeout", "qs_dense_workspace_size", "qs_dense_attn",
           "qs_gather_kv", "qs_calib_workspace_size", "qs_calibrate_basis", "qs_rabitq_score",
           "qs_select_top_p", "qs_decode_top_p", "qs_gather_kv_nvfp4k", "qs_select_topk_radix",
           "qs_semantic_index_workspace_size",
           "qs_semantic_index", "qs_semantic_select")


def status_string(s: int) -> str:
    return lib().qs_status_string(int(s)).decode()


def _ptr(x) -> int | None:
    if x is None:
        return None
    if isinstance(x, int):
        return x
    return x.data_ptr()


def _stream(s) -> int | None:
    if s is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(s, int):
        return s
    return s.cuda_stream


def _check(st: int, where: str):
    if st != QS_OK:
        raise QsError(st, where)


def make_config(*, n_q_heads, n_kv_heads, head_dim, block_size, budget, proxy_rank,
                proxy_dtype, v_dtype="bf16", v_agg_dtype="bf16", out_dtype="bf16",
                force_sink=False, force_last=False, n_keep_hp=0, softmax_scale=0.0,
                page_size=128, attn_path=0, key_storage="bf16") -> qs_config:
    c = qs_config()
    c.n_q_heads, c.n_kv_heads, c.head_dim = n_q_heads, n_kv_heads, head_dim
    c.page_size, c.block_size, c.budget = page_size, block_size, budget
    c.proxy_rank = proxy_rank
    c.proxy_dtype = DTYPE_CODES[proxy_dtype]
    c.v_dtype, c.v_agg_dtype = DTYPE_CODES[v_dtype], DTYPE_CODES[v_agg_dtype]
    c.out_dtype = DTYPE_CODES[out_dtype]
    c.force_sink, c.force_last, c.n_keep_hp = int(force_sink), int(force_last), n_keep_hp
    c.softmax_scale = softmax_scale
    c.attn_path = attn_path
    c.key_storage = 0 if key_storage == "bf16" else DTYPE_CODES[key_storage]
    return c


def make_cache(*, k, v, proxy, page_table, seq_lens, max_context, proxy_scale=None,
               block_err=None, key_center=None, key_gscale=None) -> qs_cache:
    c = qs_cache()
    c.k, c.v, c.proxy = _ptr(k), _ptr(v), _ptr(proxy)
    c.proxy_scale, c.block_err = _ptr(proxy_scale), _ptr(block_err)
    c.key_center, c.key_gscale = _ptr(key_center), _ptr(key_gscale)
    c.page_table, c.seq_lens = _ptr(page_table), _ptr(seq_lens)
    c.max_pages_per_seq = int(page_table.shape[1]) if hasattr(page_table, "shape") else 0
    c.num_pages = int(k.shape[0]) if hasattr(k, "shape") else 0
    c.max_context = int(max_context)
    return c


# ------------------------------------------------------------------ entry points

def qs_version() -> int:
    return lib().qs_version()


def qs_workspace_size(cfg: qs_config, batch: int, max_context: int) -> int:
    n = ctypes.c_size_t(0)
    _check(lib().qs_workspace_size(ctypes.byref(cfg), batch, max_context, ctypes.byref(n)),
           "qs_workspace_size")
    return n.value


def qs_attention_launches(cfg: qs_config, batch: int, max_context: int) -> int:
    n = ctypes.c_int32(0)
    _check(lib().qs_attention_launches(ctypes.byref(cfg), batch, max_context, ctypes.byref(n)),
           "qs_attention_launches")
    return n.value


def qs_selftest_wait_timeout(ws, stream=None):
    _check(lib().qs_selftest_wait_timeout(_ptr(ws), _stream(stream)), "qs_selftest_wait_timeout")


def qs_workspace_init(ws, nbytes: int, stream=None):
    _check(lib().qs_workspace_init(_ptr(ws), nbytes, _stream(stream)), "qs_workspace_init")


def qs_append_kv(cfg, cache, k_new, v_new, n_new, max_new, P, batch, ws, stream=None):
    _check(lib().qs_append_kv(ctypes.byref(cfg), ctypes.byref(cache), _ptr(k_new), _ptr(v_new),
                              _ptr(n_new), max_new, _ptr(P), batch, _ptr(ws), _stream(stream)),
           "qs_append_kv")


def qs_score(cfg, cache, q, P, batch, block_scores, ws, stream=None):
    _check(lib().qs_score(ctypes.byref(cfg), ctypes.byref(cache), _ptr(q), _ptr(P), batch,
                          _ptr(block_scores), _ptr(ws), _stream(stream)), "qs_score")


def qs_select_topk(cfg, cache, block_scores, batch, sel, n_sel, ws, stream=None):
    _check(lib().qs_select_topk(ctypes.byref(cfg), ctypes.byref(cache), _ptr(block_scores),
                                batch, _ptr(sel), _ptr(n_sel), _ptr(ws), _stream(stream)),
           "qs_select_topk")


def qs_select_topk_radix(cfg, cache, block_scores, batch, sel, n_sel, ws, stream=None):
    """qs_select_topk's selection by histogram passes instead of pairwise ranking."""
    _check(lib().qs_select_topk_radix(ctypes.byref(cfg), ctypes.byref(cache), _ptr(block_scores),
                                      batch, _ptr(sel), _ptr(n_sel), _ptr(ws), _stream(stream)),
           "qs_select_topk_radix")


def qs_sparse_attn(cfg, cache, q, sel, n_sel, batch, out, ws, stream=None):
    _check(lib().qs_sparse_attn(ctypes.byref(cfg), ctypes.byref(cache), _ptr(q), _ptr(sel),
                                _ptr(n_sel), batch, _ptr(out), _ptr(ws), _stream(stream)),
           "qs_sparse_attn")


def qs_decode(cfg, cache, q, k_new, v_new, P, batch, out, sel_out, n_sel_out, ws, stream=None):
    _check(lib().qs_decode(ctypes.byref(cfg), ctypes.byref(cache), _ptr(q), _ptr(k_new),
                           _ptr(v_new), _ptr(P), batch, _ptr(out), _ptr(sel_out),
                           _ptr(n_sel_out), _ptr(ws), _stream(stream)), "qs_decode")


def qs_sparse_attn_noalloc(cfg, cache, q, sel, n_sel, batch, out, stream=None):
    """qs_sparse_attn without a workspace: the library's static device scratch is used.

    For callers that cannot allocate device memory (a framework that owns all of it, or a
    loop where an allocation would synchronise the device). Calls that overlap on the GPU
    share that scratch and race.
    """
    _check(lib().qs_sparse_attn_noalloc(ctypes.byref(cfg), ctypes.byref(cache), _ptr(q),
                                        _ptr(sel), _ptr(n_sel), batch, _ptr(out),
                                        _stream(stream)), "qs_sparse_attn_noalloc")


def qs_dense_workspace_size(cfg: qs_config, batch: int, max_context: int) -> int:
    """Workspace bytes qs_dense_attn needs for caches of up to max_context tokens."""
    n = ctypes.c_size_t(0)
    _check(lib().qs_dense_workspace_size(ctypes.byref(cfg), batch, max_context, ctypes.byref(n)),
           "qs_dense_workspace_size")
    return n.value


def qs_dense_attn(cfg, cache, q, row_lens, batch, out, ws, stream=None):
    """Full-KV attention over every valid token of each row: q [batch][Hq][d] BF16, row_lens
    [batch * Hkv] int32 or None (then seq_lens[b]), out [batch][Hq][d]."""
    _check(lib().qs_dense_attn(ctypes.byref(cfg), ctypes.byref(cache), _ptr(q), _ptr(row_lens),
                               batch, _ptr(out), _ptr(ws), _stream(stream)), "qs_dense_attn")


def qs_gather_kv(cfg, cache, sel, n_sel, batch, k_dst, v_dst, row_lens, ws, stream=None):
    """Copy each row's selected blocks into compact pages k_dst / v_dst [batch * P][Hkv][128][d]
    (P = ceil(budget * block_size / 128)) and write the valid lengths to row_lens
    [batch * Hkv] (the first half of gather-then-attend)."""
    _check(lib().qs_gather_kv(ctypes.byref(cfg), ctypes.byref(cache), _ptr(sel), _ptr(n_sel),
                              batch, _ptr(k_dst), _ptr(v_dst), _ptr(row_lens), _ptr(ws),
                              _stream(stream)), "qs_gather_kv")


def qs_gather_kv_nvfp4k(cfg, cache, sel, n_sel, batch, k_dst, v_dst, row_lens, ws, stream=None):
    """qs_gather_kv for the NVFP4 storage variant: kept blocks' keys from BF16, every
    other selected key dequantised from NVFP4, un-centred and rounded to BF16."""
    _check(lib().qs_gather_kv_nvfp4k(ctypes.byref(cfg), ctypes.byref(cache), _ptr(sel),
                                     _ptr(n_sel), batch, _ptr(k_dst), _ptr(v_dst),
                                     _ptr(row_lens), _ptr(ws), _stream(stream)),
           "qs_gather_kv_nvfp4k")


def qs_calib_workspace_size(cfg: qs_config) -> int:
    """Workspace bytes qs_calibrate_basis needs (2 * Hkv * d * d FP64 moments + 256)."""
    n = ctypes.c_size_t(0)
    _check(lib().qs_calib_workspace_size(ctypes.byref(cfg), ctypes.byref(n)),
           "qs_calib_workspace_size")
    return n.value


def qs_calibrate_basis(cfg, q, k, n, P, eigvals, ws, stream=None):
    """The scoring basis P [Hkv][d][r] FP32 from n calibration positions: q [n][Hq][d] and
    k [n][Hkv][d] BF16; eigvals [Hkv][r] FP32 or None. r = cfg.proxy_rank."""
    _check(lib().qs_calibrate_basis(ctypes.byref(cfg), _ptr(q), _ptr(k), n, _ptr(P),
                                    _ptr(eigvals), _ptr(ws), _stream(stream)),
           "qs_calibrate_basis")


def qs_rabitq_score(cfg, cache, q, R, u, batch, block_scores, ws, stream=None):
    """Binary-proxy block scores: q [batch][Hq][d] BF16, R [Hkv][d][d] FP32 rotations,
    u [batch][Hkv][d] FP32 rounding draws in [0, 1); block_scores [batch][Hkv][nb_stride]
    receive the natural log of each block's estimated attention mass."""
    _check(lib().qs_rabitq_score(ctypes.byref(cfg), ctypes.byref(cache), _ptr(q), _ptr(R),
                                 _ptr(u), batch, _ptr(block_scores), _ptr(ws),
                                 _stream(stream)), "qs_rabitq_score")


def qs_select_top_p(cfg, cache, block_scores, p, batch, sel, n_sel, ws, stream=None):
    """Forced blocks, then the highest-mass blocks until their mass reaches p of the row's
    (block_scores are log masses), at most cfg.budget; sel ascending, padded with -1."""
    _check(lib().qs_select_top_p(ctypes.byref(cfg), ctypes.byref(cache), _ptr(block_scores),
                                 float(p), batch, _ptr(sel), _ptr(n_sel), _ptr(ws),
                                 _stream(stream)), "qs_select_top_p")


def qs_decode_top_p(cfg, cache, q, k_new, v_new, R, u, p, batch, out, sel_out, n_sel_out, ws,
                    stream=None):
    """One decode step with the binary proxy: append, qs_rabitq_score, qs_select_top_p and
    qs_sparse_attn in stream order (sel_out / n_sel_out may both be None)."""
    _check(lib().qs_decode_top_p(ctypes.byref(cfg), ctypes.byref(cache), _ptr(q), _ptr(k_new),
                                 _ptr(v_new), _ptr(R), _ptr(u), float(p), batch, _ptr(out),
                                 _ptr(sel_out), _ptr(n_sel_out), _ptr(ws), _stream(stream)),
           "qs_decode_top_p")


def qs_semantic_index_workspace_size(cfg: qs_config, batch: int, max_context: int) -> int:
    """Workspace bytes qs_semantic_index needs."""
    n = ctypes.c_size_t(0)
    _check(lib().qs_semantic_index_workspace_size(ctypes.byref(cfg), batch, max_context,
                                                  ctypes.byref(n)),
           "qs_semantic_index_workspace_size")
    return n.value


def qs_semantic_index(cfg, cache, prompt_lens, iters, centroids, offsets, members, batch, ws,
                      stream=None):
    """Build the semantic-block index over each sequence's first prompt_lens[b] keys:
    centroids [rows][C_max][d] FP32, offsets [rows][C_max + 1], members [rows][max_context]."""
    _check(lib().qs_semantic_index(ctypes.byref(cfg), ctypes.byref(cache), _ptr(prompt_lens),
                                   iters, _ptr(centroids), _ptr(offsets), _ptr(members), batch,
                                   _ptr(ws), _stream(stream)), "qs_semantic_index")


def qs_semantic_select(cfg, cache, q, prompt_lens, centroids, offsets, members, batch, tokens,
                       n_tokens, max_tokens, ws, stream=None):
    """Score the clusters, select cfg.budget of them and expand them (plus the tokens after
    the prompt) into tokens [rows][max_tokens] / n_tokens [rows] for the token-level
    attention."""
    _check(lib().qs_semantic_select(ctypes.byref(cfg), ctypes.byref(cache), _ptr(q),
                                    _ptr(prompt_lens), _ptr(centroids), _ptr(offsets),
                                    _ptr(members), batch, _ptr(tokens), _ptr(n_tokens),
                                    max_tokens, _ptr(ws), _stream(stream)), "qs_semantic_select")


def qs_device_status(ws, stream=None) -> tuple[int, int, int]:
    """(status, kernel id, index) of the first device-side error since the last read."""
    detail = (ctypes.c_uint32 * 2)()
    st = lib().qs_device_status(_ptr(ws), _stream(stream), detail)
    return st, detail[0], detail[1]
