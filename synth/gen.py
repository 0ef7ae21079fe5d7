"""Seeded synthetic input generator shared by the oracle tests, the GPU tests and the bench.

Holds none of the method's arithmetic: it draws keys, values, queries, projection
matrices, lengths and page tables, rounds them to their storage formats, and (for the
NVFP4 workload) computes the calibration inputs that the method takes as given (the
per-row centring mean and the per-tensor key scale).

Every array is drawn from its own stream, ``SeedSequence([seed, tag, *ids])``, so one row
(sequence b, KV head g) can be regenerated alone, and a prefix of a row equals the same
prefix drawn on its own.

Recipe (Gaussians are written N(mean, variance)):
  * draws are float32; stored tensors are rounded to nearest-even BF16 (or FP16 for the
    NVFP4 workload's V);
  * 'outliers' keys: N(0,1) with a few per-KV-head channels scaled (x8 or x10);
  * 'offset' keys: N(0,1) plus a per-row channel offset drawn N(0,2);
  * 'mixture' keys: per token, with probability 0.3 one of 16 row centres c ~ N(0,4I)
    plus N(0, 0.3^2 I) noise, else N(0, I);
  * V ~ N(0,1); q ~ N(0,1) unless planted:
      - 'needle': every head's query is 3 * m / |m|, m the mean stored key of the needle
        block (optionally that block's keys are first pushed by +boost * w, w a drawn
        unit vector);
      - 'planted': n distinct blocks per row drawn from [1, nb-2];
        q_h = z_h + 3 * sum_j unit(mean key of block j - mean key of the row), z_h ~ N(0, I);
  * P: QR of a Gaussian d x r matrix, columns sign-fixed so diag(R) > 0; one P per layer,
    repeated for every KV head;
  * binary proxy: one rotation per KV head (QR of a Gaussian d x d matrix, sign-fixed),
    the row centres as the NVFP4 centring mean below, and rounding draws uniform in
    [0, 1) per (sequence, KV head, dimension);
  * ragged lengths: integers uniform in [min, max], redrawn while a multiple of the block
    size, then fixed overrides for the last few sequences;
  * paging: 128-token pages; each sequence's physical pages are a slice of one seeded
    permutation of all pages.
"""
from __future__ import annotations

import concurrent.futures as cf
import math
import os

import numpy as np

from .workloads import Workload

TAG_K, TAG_V, TAG_Q, TAG_P, TAG_LENS, TAG_PAGES, TAG_OUTL, TAG_PLANT, TAG_ROWPAR, TAG_MIX = (
    1, 2, 3, 4, 5, 6, 7, 8, 9, 10)
TAG_ROT, TAG_U = 11, 12


def _rng(w: Workload, tag: int, *ids: int) -> np.random.Generator:
    return np.random.default_rng(np.random.SeedSequence([w.seed, tag, *[int(i) for i in ids]]))


# ---- storage rounding (input preparation only) ------------------------------------------

def to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """float32 -> BF16 bit patterns, round to nearest even (finite inputs)."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    t = np.right_shift(u, np.uint32(16))
    np.bitwise_and(t, np.uint32(1), out=t)
    t += np.uint32(0x7FFF)
    t += u
    np.right_shift(t, np.uint32(16), out=t)
    return t.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (b.astype(np.uint32) << np.uint32(16)).view(np.float32)


def to_f16_bits(x: np.ndarray) -> np.ndarray:
    return np.ascontiguousarray(x, dtype=np.float32).astype(np.float16).view(np.uint16)


# ---- small per-workload arrays ------------------------------------------------------------

def lengths(w: Workload) -> np.ndarray:
    """Context length per sequence (tokens, including the one appended this step)."""
    if not w.ragged:
        return np.full(w.batch, w.context, dtype=np.int32)
    rng = _rng(w, TAG_LENS)
    out = np.empty(w.batch, dtype=np.int32)
    for b in range(w.batch):
        while True:
            v = int(rng.integers(w.ragged_min, w.ragged_max, endpoint=True))
            if v % w.block_size != 0:
                break
        out[b] = v
    for b, L in w.ragged_overrides:
        if b < w.batch:
            out[b] = L
    return out


def proj_matrix(w: Workload) -> np.ndarray:
    """P as float32 [Hkv][d][r]: one random orthonormal basis per layer, repeated per head."""
    assert w.proxy_rank > 0
    rng = _rng(w, TAG_P)
    a = rng.standard_normal((w.head_dim, w.proxy_rank))
    q, r = np.linalg.qr(a)
    q = q * np.sign(np.diag(r))[None, :]
    p = q.astype(np.float32)
    return np.ascontiguousarray(np.broadcast_to(p, (w.n_kv_heads,) + p.shape))


def rotations(w: Workload) -> np.ndarray:
    """R as float32 [Hkv][d][d]: one uniformly random rotation per KV head (QR of a Gaussian
    matrix, columns sign-fixed so diag(R) > 0), the binary proxy's random rotation."""
    out = np.empty((w.n_kv_heads, w.head_dim, w.head_dim), dtype=np.float32)
    for g in range(w.n_kv_heads):
        a = _rng(w, TAG_ROT, g).standard_normal((w.head_dim, w.head_dim))
        q, r = np.linalg.qr(a)
        out[g] = (q * np.sign(np.diag(r))[None, :]).astype(np.float32)
    return out


def rounding_draws(w: Workload) -> np.ndarray:
    """u as float32 [batch][Hkv][d], uniform in [0, 1): the binary proxy's random rounding
    of the rotated query to its 4-bit grid (one draw per dimension per step)."""
    return _rng(w, TAG_U).random((w.batch, w.n_kv_heads, w.head_dim), dtype=np.float32)


def outlier_channels(w: Workload, g: int) -> np.ndarray:
    return _rng(w, TAG_OUTL, g).choice(w.head_dim, size=w.n_outlier_ch, replace=False)


def page_table(w: Workload, lens: np.ndarray, extra_tokens: int = 0):
    """(page_table int32 [batch][max_pages], num_pages). Unused entries are -1."""
    ps = w.page_size
    need = [(int(L) + extra_tokens + ps - 1) // ps for L in lens]
    total = int(sum(need))
    max_pages = max(need)
    perm = _rng(w, TAG_PAGES).permutation(total).astype(np.int32)
    pt = np.full((w.batch, max_pages), -1, dtype=np.int32)
    off = 0
    for b, n in enumerate(need):
        pt[b, :n] = perm[off:off + n]
        off += n
    return pt, total


# ---- per-row key / value / query draws ------------------------------------------------------

def row_keys_f32(w: Workload, b: int, g: int, L: int) -> np.ndarray:
    """Unrounded keys of row (b, g): float32 [L][d]."""
    d = w.head_dim
    rng = _rng(w, TAG_K, b, g)
    if w.key_recipe == "outliers":
        k = rng.standard_normal((L, d), dtype=np.float32)
        ch = outlier_channels(w, g)
        k[:, ch] *= np.float32(w.outlier_scale)
        if w.needle_boost > 0:
            wdir = _rng(w, TAG_PLANT, b, g).standard_normal(d)
            wdir = (wdir / np.linalg.norm(wdir)).astype(np.float32)
            s = w.needle_block * w.block_size
            e = min(s + w.block_size, L)
            k[s:e] += np.float32(w.needle_boost) * wdir
        return k
    if w.key_recipe == "offset":
        off = (_rng(w, TAG_ROWPAR, b, g).standard_normal(d) * math.sqrt(2.0)).astype(np.float32)
        k = rng.standard_normal((L, d), dtype=np.float32)
        k += off
        return k
    if w.key_recipe == "mixture":
        pr = _rng(w, TAG_ROWPAR, b, g)
        centres = (pr.standard_normal((16, d)) * 2.0).astype(np.float32)
        k = rng.standard_normal((L, d), dtype=np.float32)
        mix = _rng(w, TAG_MIX, b, g)
        u = mix.random(L)
        which = mix.integers(0, 16, size=L)
        sel = u < 0.3
        k[sel] = centres[which[sel]] + np.float32(0.3) * k[sel]
        return k
    raise ValueError(w.key_recipe)


def row_kv(w: Workload, b: int, g: int, L: int):
    """Stored (K, V) of row (b, g) as 16-bit patterns [L][d]: K BF16, V BF16 or FP16."""
    k = to_bf16_bits(row_keys_f32(w, b, g, L))
    v32 = _rng(w, TAG_V, b, g).standard_normal((L, w.head_dim), dtype=np.float32)
    v = to_f16_bits(v32) if w.v_dtype == "f16" else to_bf16_bits(v32)
    return k, v


def row_queries(w: Workload, b: int, g: int, k_bits: np.ndarray, L: int) -> np.ndarray:
    """Queries of the G heads of row (b, g) as BF16 bits [G][d]."""
    G, d = w.group, w.head_dim
    if w.query_recipe == "normal":
        q = _rng(w, TAG_Q, b, g).standard_normal((G, d), dtype=np.float32)
        return to_bf16_bits(q)
    kf = bf16_bits_to_f32(k_bits[:L]).astype(np.float64)
    S = w.block_size
    if w.query_recipe == "needle":
        s = w.needle_block * S
        m = kf[s:s + S].mean(axis=0)
        q = np.broadcast_to(3.0 * m / np.linalg.norm(m), (G, d))
        return to_bf16_bits(q.astype(np.float32))
    if w.query_recipe == "planted":
        nb = (L + S - 1) // S
        rng = _rng(w, TAG_PLANT, b, g)
        blocks = rng.choice(np.arange(1, nb - 1), size=w.n_planted, replace=False)
        mu = kf.mean(axis=0)
        direction = np.zeros(d)
        for j in blocks:
            m = kf[j * S:(j + 1) * S].mean(axis=0) - mu
            direction += m / np.linalg.norm(m)
        z = _rng(w, TAG_Q, b, g).standard_normal((G, d))
        return to_bf16_bits((z + 3.0 * direction).astype(np.float32))
    raise ValueError(w.query_recipe)


def planted_blocks(w: Workload, b: int, g: int, L: int) -> np.ndarray:
    nb = (L + w.block_size - 1) // w.block_size
    return _rng(w, TAG_PLANT, b, g).choice(np.arange(1, nb - 1), size=w.n_planted, replace=False)


# ---- NVFP4 calibration inputs ---------------------------------------------------------------

def calibration(w: Workload, lens: np.ndarray, threads: int | None = None):
    """Centring mean mu [batch][Hkv][d] (float32) and key tensor scale g_k (float32).

    mu[b, g] is the float64 mean of the row's first ``calib_tokens`` stored keys, rounded
    to float32. g_k = fp32(A / 2688), A the largest |fp32(k) - mu| (float32 subtraction)
    over those tokens of every row; 2688 = 6 * 448 is the product of the largest E2M1 and
    UE4M3 magnitudes. Calibration happens before decoding and is an input of the step.
    """
    mu = np.zeros((w.batch, w.n_kv_heads, w.head_dim), dtype=np.float32)
    amax = np.zeros((w.batch, w.n_kv_heads), dtype=np.float32)

    def one(bg):
        b, g = bg
        n = min(int(lens[b]), w.calib_tokens)
        k = bf16_bits_to_f32(to_bf16_bits(row_keys_f32(w, b, g, n)))
        m = k.astype(np.float64).mean(axis=0).astype(np.float32)
        mu[b, g] = m
        amax[b, g] = np.max(np.abs(k - m))

    rows = [(b, g) for b in range(w.batch) for g in range(w.n_kv_heads)]
    with cf.ThreadPoolExecutor(threads or os.cpu_count()) as ex:
        list(ex.map(one, rows))
    gk = np.float32(np.float32(amax.max()) / np.float32(2688.0))
    return mu, gk


# ---- whole-workload assembly -----------------------------------------------------------------

class Inputs:
    """All host-side inputs of one workload (possibly only a subset of rows filled)."""

    def __init__(self, w: Workload, threads: int | None = None, rows=None, extra_tokens: int = 0):
        self.w = w
        self.lens = lengths(w)
        self.page_table, self.num_pages = page_table(w, self.lens, extra_tokens)
        self.P = proj_matrix(w) if w.proxy_rank > 0 else None
        self.threads = threads or os.cpu_count()
        self.u = None
        if w.proxy_dtype == "nvfp4":
            self.mu, self.g_k = calibration(w, self.lens, self.threads)
        elif w.proxy_dtype == "rabitq":
            # the rotation R takes P's place; the row centres are the calibration means
            self.P = rotations(w)
            self.mu, _ = calibration(w, self.lens, self.threads)
            self.g_k = None
            self.u = rounding_draws(w)
        else:
            self.mu, self.g_k = None, None

    def row(self, b: int, g: int):
        """(K bits [L][d], V bits [L][d], q bits [G][d]) of row (b, g)."""
        L = int(self.lens[b])
        k, v = row_kv(self.w, b, g, L)
        q = row_queries(self.w, b, g, k, L)
        return k, v, q

    def dense(self, max_len: int | None = None):
        """Row-major host arrays for the whole workload.

        Returns (K [b][Hkv][Lmax][d] u16, V same, q [b][Hq][d] u16); entries past a
        sequence's length are zero.
        """
        w = self.w
        Lmax = int(self.lens.max()) if max_len is None else max_len
        K = np.zeros((w.batch, w.n_kv_heads, Lmax, w.head_dim), dtype=np.uint16)
        V = np.zeros_like(K)
        Q = np.zeros((w.batch, w.n_q_heads, w.head_dim), dtype=np.uint16)
        G = w.group

        def one(bg):
            b, g = bg
            k, v, q = self.row(b, g)
            L = min(int(self.lens[b]), Lmax)
            K[b, g, :L] = k[:L]
            V[b, g, :L] = v[:L]
            Q[b, g * G:(g + 1) * G] = q

        rows = [(b, g) for b in range(w.batch) for g in range(w.n_kv_heads)]
        with cf.ThreadPoolExecutor(self.threads) as ex:
            list(ex.map(one, rows))
        return K, V, Q
