"""The bench's byte accounting (the numerators of its roofline fractions), checked against
hand counts for each kind of proxy, on CPU."""
import numpy as np

import bench
import synth


def _full_selection(w, lens):
    """Every row selects its first `budget` blocks (all full when lens are multiples)."""
    sel = np.tile(np.arange(w.budget, dtype=np.int32), (w.batch, w.n_kv_heads, 1))
    nsel = np.full((w.batch, w.n_kv_heads), w.budget, dtype=np.int32)
    return sel, nsel


def test_rank_r_bf16_bytes_at_128k():
    w = synth.BLOCK128K
    lens = np.full(w.batch, 131072, dtype=np.int64)
    sel, nsel = _full_selection(w, lens)
    by = bench.step_bytes(w, lens, sel, nsel)
    assert by["proxy"] == 16 * 8 * 131072 * 32 * 2 == 1 << 30          # 1 GiB of r = 32 BF16
    assert by["kv"] == 16 * 8 * 64 * 128 * 128 * 2 * 2                  # K and V of 64 blocks
    assert by["q"] == 16 * 40 * 128 * 2 and by["out"] == 16 * 40 * 128 * 2
    assert by["total"] == by["proxy"] + by["kv"] + by["q"] + by["out"]
    assert by["selected_tokens"] == 16 * 8 * 64 * 128


def test_fp8_nvfp4_centroid_and_binary_proxy_bytes():
    lens = np.full(16, 131072, dtype=np.int64)
    fp8 = synth.FP8_128K
    sel, nsel = _full_selection(fp8, lens)
    assert bench.step_bytes(fp8, lens, sel, nsel)["proxy"] == 16 * 8 * 131072 * 32      # 1 B
    nv = synth.NVFP4_128K
    sel, nsel = _full_selection(nv, lens)
    # 64 code bytes + 8 scale bytes per token
    assert bench.step_bytes(nv, lens, sel, nsel)["proxy"] == 16 * 8 * 131072 * (64 + 8)
    ce = synth.CENTROID_128K
    sel, nsel = _full_selection(ce, lens)
    # one FP32 key sum of d = 128 per 128-token block
    assert bench.step_bytes(ce, lens, sel, nsel)["proxy"] == 16 * 8 * 1024 * 128 * 4
    rq = synth.RABITQ_TOKEN128K
    sel, nsel = _full_selection(rq, lens)
    # 128 code bits (16 bytes) + one FP32 factor per token
    assert bench.step_bytes(rq, lens, sel, nsel)["proxy"] == 16 * 8 * 131072 * (16 + 4)


def test_ragged_lengths_count_valid_tokens_only():
    # a selected last block cut by the length counts only its valid tokens
    w = synth.RAGGED.replace(batch=2)
    lens = np.array([1000, 64 * 40 + 7], dtype=np.int64)
    nb = (lens + 63) // 64
    sel = np.full((2, w.n_kv_heads, w.budget), -1, dtype=np.int32)
    nsel = np.zeros((2, w.n_kv_heads), dtype=np.int32)
    for b in range(2):
        take = np.arange(min(w.budget, nb[b]))
        if nb[b] > w.budget:
            take = np.concatenate([np.arange(w.budget - 1), [nb[b] - 1]])   # includes the last
        sel[b, :, :len(take)] = take
        nsel[b, :] = len(take)
    by = bench.step_bytes(w, lens, sel, nsel)
    want_tokens = 0
    for b in range(2):
        for j in sel[b, 0, :nsel[b, 0]]:
            want_tokens += min(64, int(lens[b]) - int(j) * 64)
    assert by["selected_tokens"] == want_tokens * w.n_kv_heads
    assert by["kv"] == want_tokens * w.n_kv_heads * 128 * 2 * 2
    assert by["proxy"] == int(lens.sum()) * w.n_kv_heads * 64 * 2           # r = 64 BF16


def test_steps_per_s_aggregates_over_ranks():
    assert bench.aggregate_steps_per_s(0.5, 1) == 2000.0
    assert bench.aggregate_steps_per_s(0.5, 4) == 8000.0


def test_nvfp4_key_storage_bytes():
    """The NVFP4 storage variant reads 72 bytes of key per selected token (64 of codes, 8 of
    scales), 256 for the two kept blocks' BF16 keys, and the FP16 values in full."""
    w = synth.NVFP4_STORE_128K
    lens = np.full(16, 131072, dtype=np.int64)
    sel, nsel = _full_selection(w, lens)
    by = bench.step_bytes(w, lens, sel, nsel)
    rows, tok_row = 16 * 8, 128 * 128
    v = rows * tok_row * 256
    k = rows * ((tok_row - 2 * 128) * 72 + 2 * 128 * 256)
    assert by["kv"] == v + k
    assert by["proxy"] == rows * 131072 * 72
