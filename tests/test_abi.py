"""The C-ABI library loads and exports every entry point declared in include/qs.h; host
validation and workspace sizing work without a GPU (no compute call is made)."""
import os
import re

import pytest

import score_then_select_b200 as qs
from score_then_select_b200 import binding as B

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    names = []
    for fn in sorted(os.listdir(os.path.join(ROOT, "include"))):
        if fn.endswith(".h"):
            txt = open(os.path.join(ROOT, "include", fn)).read()
            txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
            names += re.findall(r"\b(qs_[a-z0-9_]+)\s*\(", txt)
    return sorted(set(names))


def test_library_exports_every_declared_symbol():
    L = qs.lib()
    declared = _declared()
    assert "qs_decode" in declared and "qs_sparse_attn" in declared
    for name in declared:
        assert hasattr(L, name), name


def test_version_and_status_strings():
    assert qs.qs_version() >= 10000
    assert qs.status_string(B.QS_ERR_DEVICE_TIMEOUT).startswith("device-side")


def _cfg(**kw):
    base = dict(n_q_heads=40, n_kv_heads=8, head_dim=128, block_size=128, budget=64,
                proxy_rank=32, proxy_dtype="bf16", force_sink=True, force_last=True)
    base.update(kw)
    return qs.make_config(**base)


def test_workspace_size_is_positive_and_monotone():
    a = qs.qs_workspace_size(_cfg(), 16, 131072)
    b = qs.qs_workspace_size(_cfg(), 16, 262144)
    assert 0 < a < b


@pytest.mark.parametrize("kw,status", [
    (dict(head_dim=96), B.QS_ERR_UNSUPPORTED),
    (dict(n_q_heads=41), B.QS_ERR_INVALID_ARG),
    (dict(n_q_heads=80), B.QS_ERR_UNSUPPORTED),          # group of 10 > 8
    (dict(block_size=48), B.QS_ERR_INVALID_ARG),
    (dict(budget=0), B.QS_ERR_INVALID_ARG),
    (dict(proxy_rank=48), B.QS_ERR_UNSUPPORTED),
    (dict(proxy_rank=0), B.QS_ERR_INVALID_ARG),          # rank 0 needs the NVFP4 proxy
    (dict(v_dtype="f16", v_agg_dtype="bf16"), B.QS_ERR_UNSUPPORTED),
    (dict(block_size=1, budget=2048), None),
    (dict(proxy_dtype="e4m3"), None),                     # FP8 projected keys, r = 32
    (dict(proxy_dtype="e4m3", proxy_rank=64), None),
    (dict(proxy_dtype="e4m3", proxy_rank=16), B.QS_ERR_UNSUPPORTED),
])
def test_host_validation(kw, status):
    if status is None:
        assert qs.qs_workspace_size(_cfg(**kw), 16, 32768) > 0
        return
    with pytest.raises(qs.QsError) as e:
        qs.qs_workspace_size(_cfg(**kw), 16, 131072)
    assert e.value.status == status


def test_token_level_context_limit():
    # token-level selection runs up to 131,072 candidates per row (a cluster of 4 CTAs)
    assert qs.qs_workspace_size(_cfg(block_size=1, budget=2048), 16, 131072) > 0
    with pytest.raises(qs.QsError) as e:
        qs.qs_workspace_size(_cfg(block_size=1, budget=2048), 16, 131073)
    assert e.value.status == B.QS_ERR_UNSUPPORTED


def test_null_pointers_rejected_without_launch():
    cfg = _cfg()
    cache = B.qs_cache()
    with pytest.raises(qs.QsError) as e:
        qs.qs_decode(cfg, cache, 0, 0, 0, 0, 16, 0, None, None, 0, stream=0)
    assert e.value.status == B.QS_ERR_INVALID_ARG


def test_dense_workspace_covers_every_page_and_limits_context():
    # full-KV attention plans every 128-token page of the row: more partials than the sparse
    # plan of the same cache, and contexts past 128K tokens are refused on the host
    sparse = qs.qs_workspace_size(_cfg(), 16, 131072)
    dense = qs.qs_dense_workspace_size(_cfg(), 16, 131072)
    assert dense > sparse
    assert qs.qs_dense_workspace_size(_cfg(), 16, 2048) < dense
    with pytest.raises(qs.QsError) as e:
        qs.qs_dense_workspace_size(_cfg(), 16, 131073)
    assert e.value.status == B.QS_ERR_UNSUPPORTED
    with pytest.raises(qs.QsError) as e:                      # an invalid configuration
        qs.qs_dense_workspace_size(_cfg(n_q_heads=41), 16, 4096)
    assert e.value.status == B.QS_ERR_INVALID_ARG


def test_comparison_calls_reject_null_pointers_without_launch():
    cfg = _cfg()
    cache = B.qs_cache()
    with pytest.raises(qs.QsError) as e:
        qs.qs_dense_attn(cfg, cache, 0, None, 16, 0, 0, stream=0)
    assert e.value.status == B.QS_ERR_INVALID_ARG
    with pytest.raises(qs.QsError) as e:
        qs.qs_gather_kv(cfg, cache, 0, 0, 16, 0, 0, 0, 0, stream=0)
    assert e.value.status == B.QS_ERR_INVALID_ARG


def test_centroid_and_fp8_configurations():
    # centroid scoring: rank 0 with the centroid proxy; kept blocks are NVFP4-only
    assert qs.qs_workspace_size(_cfg(proxy_rank=0, proxy_dtype="centroid"), 16, 131072) > 0
    with pytest.raises(qs.QsError) as e:
        qs.qs_workspace_size(_cfg(proxy_rank=0, proxy_dtype="centroid", n_keep_hp=2), 16, 4096)
    assert e.value.status == B.QS_ERR_INVALID_ARG
    # a rank-r proxy cannot be a centroid cache
    with pytest.raises(qs.QsError) as e:
        qs.qs_workspace_size(_cfg(proxy_dtype="centroid"), 16, 4096)
    assert e.value.status == B.QS_ERR_UNSUPPORTED


def test_calibration_entry_points_validate_on_the_host():
    cfg = _cfg(n_q_heads=32, n_kv_heads=8, proxy_rank=32)
    assert qs.qs_calib_workspace_size(cfg) == 256 + 2 * 8 * 128 * 128 * 8
    with pytest.raises(qs.QsError) as e:                      # no rank, no basis
        qs.qs_calib_workspace_size(_cfg(proxy_rank=0, proxy_dtype="nvfp4", block_size=128))
    assert e.value.status == B.QS_ERR_UNSUPPORTED
    with pytest.raises(qs.QsError) as e:                      # null pointers, no launch
        qs.qs_calibrate_basis(cfg, 0, 0, 16, 0, None, 0, stream=0)
    assert e.value.status == B.QS_ERR_INVALID_ARG
    with pytest.raises(qs.QsError) as e:                      # no positions
        qs.qs_calibrate_basis(cfg, 16, 16, 0, 16, None, 256, stream=0)
    assert e.value.status == B.QS_ERR_INVALID_ARG


def test_kept_blocks_limited_to_one_cta_rows():
    # NVFP4 kept blocks with more than 32,768 blocks per row are refused on the host
    cfg = _cfg(proxy_rank=0, proxy_dtype="nvfp4", block_size=128, n_keep_hp=2)
    assert qs.qs_workspace_size(cfg, 1, 128 * 32768) > 0
    with pytest.raises(qs.QsError) as e:
        qs.qs_workspace_size(cfg, 1, 128 * 32768 + 1)
    assert e.value.status == B.QS_ERR_UNSUPPORTED


def _prototypes():
    """{name: number of parameters} of every entry point declared in include/qs.h."""
    out = {}
    for fn in sorted(os.listdir(os.path.join(ROOT, "include"))):
        if not fn.endswith(".h"):
            continue
        txt = open(os.path.join(ROOT, "include", fn)).read()
        txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
        for m in re.finditer(r"\b(qs_[a-z0-9_]+)\s*\(([^;{]*?)\)\s*;", txt):
            params = m.group(2).strip()
            out[m.group(1)] = 0 if params in ("", "void") else params.count(",") + 1
    return out


def test_binding_argument_counts_match_the_header():
    L = qs.lib()
    protos = _prototypes()
    assert set(protos) == set(_declared())
    for name, n in protos.items():
        f = getattr(L, name)
        assert f.argtypes is not None, f"{name}: no argtypes in the binding"
        assert len(f.argtypes) == n, f"{name}: header has {n} parameters, binding {len(f.argtypes)}"


def _fake_cache(with_center=True):
    """A cache whose pointers are aligned placeholders: valid for the host checks, never
    dereferenced (every call below returns before any launch)."""
    c = B.qs_cache()
    c.k = c.v = c.proxy = c.page_table = c.seq_lens = 1 << 20
    c.key_center = (1 << 20) if with_center else None
    c.max_pages_per_seq, c.num_pages, c.max_context = 8, 64, 1024
    return c


def test_binary_proxy_configuration_and_calls_validate_on_the_host():
    rq = dict(proxy_rank=0, proxy_dtype="rabitq", block_size=1, budget=256)
    assert qs.qs_workspace_size(_cfg(**rq), 16, 131072) > 0
    assert qs.qs_workspace_size(_cfg(head_dim=64, **rq), 2, 1000) > 0
    with pytest.raises(qs.QsError) as e:                      # kept blocks are NVFP4-only
        qs.qs_workspace_size(_cfg(n_keep_hp=1, **rq), 16, 4096)
    assert e.value.status == B.QS_ERR_INVALID_ARG
    with pytest.raises(qs.QsError) as e:
        qs.qs_workspace_size(_cfg(head_dim=96, **rq), 16, 4096)
    assert e.value.status == B.QS_ERR_UNSUPPORTED
    cfg, cache, a = _cfg(**rq), _fake_cache(), 1 << 20
    # its stages are separate calls: the fused step and the draw-less score refuse it
    with pytest.raises(qs.QsError) as e:
        qs.qs_score(cfg, cache, a, a, 4, a, a, stream=0)
    assert e.value.status == B.QS_ERR_UNSUPPORTED
    with pytest.raises(qs.QsError) as e:
        qs.qs_decode(cfg, cache, a, a, a, a, 4, a, None, None, a, stream=0)
    assert e.value.status == B.QS_ERR_UNSUPPORTED
    # the binary scan needs the binary proxy, its centres and its rotation
    with pytest.raises(qs.QsError) as e:
        qs.qs_rabitq_score(_cfg(), cache, a, a, a, 4, a, a, stream=0)
    assert e.value.status == B.QS_ERR_UNSUPPORTED
    with pytest.raises(qs.QsError) as e:
        qs.qs_rabitq_score(cfg, _fake_cache(with_center=False), a, a, a, 4, a, a, stream=0)
    assert e.value.status == B.QS_ERR_INVALID_ARG
    with pytest.raises(qs.QsError) as e:
        qs.qs_rabitq_score(cfg, cache, a, None, a, 4, a, a, stream=0)
    assert e.value.status == B.QS_ERR_INVALID_ARG
    with pytest.raises(qs.QsError) as e:                      # the writer needs R
        qs.qs_append_kv(cfg, cache, a, a, a, 1, None, 4, a, stream=0)
    assert e.value.status == B.QS_ERR_INVALID_ARG
    # top-p: 0 < p <= 1, and room for the forced blocks
    for p in (0.0, -0.5, 1.5, float("nan")):
        with pytest.raises(qs.QsError) as e:
            qs.qs_select_top_p(cfg, cache, a, p, 4, a, a, a, stream=0)
        assert e.value.status == B.QS_ERR_INVALID_ARG, p
    with pytest.raises(qs.QsError) as e:
        qs.qs_select_top_p(_cfg(budget=1, **{k: v for k, v in rq.items() if k != "budget"}),
                           cache, a, 0.5, 4, a, a, a, stream=0)
    assert e.value.status == B.QS_ERR_INVALID_ARG
    # the binary step: its own proxy only, its rotation and draws, 0 < p <= 1
    with pytest.raises(qs.QsError) as e:
        qs.qs_decode_top_p(_cfg(), cache, a, a, a, a, a, 0.9, 4, a, None, None, a, stream=0)
    assert e.value.status == B.QS_ERR_UNSUPPORTED
    for R, u, p in ((None, a, 0.9), (a, None, 0.9), (a, a, 0.0), (a, a, 1.01)):
        with pytest.raises(qs.QsError) as e:
            qs.qs_decode_top_p(cfg, cache, a, a, a, R, u, p, 4, a, None, None, a, stream=0)
        assert e.value.status == B.QS_ERR_INVALID_ARG, (R, u, p)
    with pytest.raises(qs.QsError) as e:                      # sel_out without n_sel_out
        qs.qs_decode_top_p(cfg, cache, a, a, a, a, a, 0.9, 4, a, a, None, a, stream=0)
    assert e.value.status == B.QS_ERR_INVALID_ARG


def test_semantic_configuration_and_calls_validate_on_the_host():
    sem = dict(proxy_rank=0, proxy_dtype="semantic", block_size=64, budget=16,
               force_sink=False, force_last=False)
    cfg = _cfg(**sem)
    assert qs.qs_workspace_size(cfg, 4, 8192) > 0
    rows, c_max = 4 * 8, 8192 // 64
    assert qs.qs_semantic_index_workspace_size(cfg, 4, 8192) == 256 + 4 * rows * (8192 + c_max)
    with pytest.raises(qs.QsError) as e:                      # only the semantic kind
        qs.qs_semantic_index_workspace_size(_cfg(), 4, 8192)
    assert e.value.status == B.QS_ERR_UNSUPPORTED
    with pytest.raises(qs.QsError) as e:                      # kept blocks are NVFP4-only
        qs.qs_workspace_size(_cfg(n_keep_hp=1, **sem), 4, 8192)
    assert e.value.status == B.QS_ERR_INVALID_ARG
    cache, a = _fake_cache(with_center=False), 1 << 20
    cache.proxy = None                                        # the index is outside the cache
    for call in (lambda: qs.qs_score(cfg, cache, a, a, 4, a, a, stream=0),
                 lambda: qs.qs_decode(cfg, cache, a, a, a, a, 4, a, None, None, a, stream=0),
                 lambda: qs.qs_semantic_index(_cfg(), cache, a, 2, a, a, a, 4, a, stream=0),
                 lambda: qs.qs_semantic_select(_cfg(), cache, a, a, a, a, a, 4, a, a, 64, a,
                                               stream=0)):
        with pytest.raises(qs.QsError) as e:
            call()
        assert e.value.status == B.QS_ERR_UNSUPPORTED
    for call in (lambda: qs.qs_semantic_index(cfg, cache, a, 0, a, a, a, 4, a, stream=0),
                 lambda: qs.qs_semantic_index(cfg, cache, None, 2, a, a, a, 4, a, stream=0),
                 lambda: qs.qs_semantic_select(cfg, cache, a, a, a, a, a, 4, a, a, 0, a,
                                               stream=0),
                 lambda: qs.qs_semantic_select(cfg, cache, a, a, None, a, a, 4, a, a, 64, a,
                                               stream=0)):
        with pytest.raises(qs.QsError) as e:
            call()
        assert e.value.status == B.QS_ERR_INVALID_ARG


def test_nvfp4_storage_gather_validates_on_the_host():
    cache, a = _fake_cache(), 1 << 20
    with pytest.raises(qs.QsError) as e:                      # only the NVFP4 configuration
        qs.qs_gather_kv_nvfp4k(_cfg(), cache, a, a, 4, a, a, a, a, stream=0)
    assert e.value.status == B.QS_ERR_UNSUPPORTED
    nv = _cfg(proxy_rank=0, proxy_dtype="nvfp4", block_size=128, n_keep_hp=2)
    with pytest.raises(qs.QsError) as e:                      # no scales / tensor scale
        qs.qs_gather_kv_nvfp4k(nv, cache, a, a, 4, a, a, a, a, stream=0)
    assert e.value.status == B.QS_ERR_INVALID_ARG
    cache.proxy_scale = a
    cache.key_gscale = a
    with pytest.raises(qs.QsError) as e:                      # kept blocks need block_err
        qs.qs_gather_kv_nvfp4k(nv, cache, a, a, 4, a, a, a, a, stream=0)
    assert e.value.status == B.QS_ERR_INVALID_ARG
    cache.block_err = a
    with pytest.raises(qs.QsError) as e:                      # no destination
        qs.qs_gather_kv_nvfp4k(nv, cache, a, a, 4, None, a, a, a, stream=0)
    assert e.value.status == B.QS_ERR_INVALID_ARG


def test_radix_select_validates_on_the_host():
    cache, a = B.qs_cache(), 1 << 20
    with pytest.raises(qs.QsError) as e:                      # no seq_lens
        qs.qs_select_topk_radix(_cfg(), cache, a, 4, a, a, a, stream=0)
    assert e.value.status == B.QS_ERR_INVALID_ARG
    cache.seq_lens = a
    with pytest.raises(qs.QsError) as e:                      # kept blocks need block_err
        qs.qs_select_topk_radix(_cfg(proxy_rank=0, proxy_dtype="nvfp4", block_size=128,
                                     n_keep_hp=2), cache, a, 4, a, a, a, stream=0)
    assert e.value.status == B.QS_ERR_INVALID_ARG


def test_nvfp4_key_storage_validates_on_the_host():
    """Attention over the NVFP4 keys: only on the NVFP4 configuration and the tile pipeline;
    every attending call needs the NVFP4 pointers (16-byte aligned codes, scales, centres)
    and the block errors for kept blocks; full-KV attention plans the BF16 keys regardless;
    the no-allocation entry point refuses it. All rejected before any launch."""
    nv = dict(proxy_rank=0, proxy_dtype="nvfp4", block_size=128, n_keep_hp=2, budget=128,
              v_dtype="f16", v_agg_dtype="f16")
    st = _cfg(key_storage="nvfp4", **nv)
    assert qs.qs_workspace_size(st, 16, 131072) > qs.qs_workspace_size(_cfg(**nv), 16, 131072)
    assert qs.qs_attention_launches(st, 16, 131072) == 3
    assert qs.qs_attention_launches(_cfg(**nv), 16, 131072) == 2
    assert qs.qs_dense_workspace_size(st, 16, 131072) == qs.qs_dense_workspace_size(
        _cfg(**nv), 16, 131072)
    with pytest.raises(qs.QsError) as e:                      # rank-r scoring copy
        qs.qs_workspace_size(_cfg(key_storage="nvfp4"), 16, 131072)
    assert e.value.status == B.QS_ERR_INVALID_ARG
    with pytest.raises(qs.QsError) as e:                      # the gather kernel cannot decode
        qs.qs_workspace_size(_cfg(key_storage="nvfp4", attn_path=2, **nv), 16, 131072)
    assert e.value.status == B.QS_ERR_UNSUPPORTED
    a = 1 << 20
    cache = _fake_cache()
    with pytest.raises(qs.QsError) as e:                      # no scales / tensor scale
        qs.qs_sparse_attn(st, cache, a, a, a, 4, a, a, stream=0)
    assert e.value.status == B.QS_ERR_INVALID_ARG
    cache.proxy_scale = a
    cache.key_gscale = a
    with pytest.raises(qs.QsError) as e:                      # kept blocks need block_err
        qs.qs_sparse_attn(st, cache, a, a, a, 4, a, a, stream=0)
    assert e.value.status == B.QS_ERR_INVALID_ARG
    cache.block_err = a
    cache.key_center = a + 8                                  # centres copied in 16-byte units
    with pytest.raises(qs.QsError) as e:
        qs.qs_sparse_attn(st, cache, a, a, a, 4, a, a, stream=0)
    assert e.value.status == B.QS_ERR_INVALID_ARG
    cache.key_center = a
    with pytest.raises(qs.QsError) as e:
        qs.qs_sparse_attn_noalloc(st, cache, a, a, a, 4, a, stream=0)
    assert e.value.status == B.QS_ERR_UNSUPPORTED
