#!/usr/bin/env python
"""Decode-step benchmark of score-then-select sparse attention on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

A step is one qs_decode call over one batch: append the new token of every sequence,
score the whole key history through the proxy cache, select the top-k blocks per
(sequence, KV head), and attend over the selected keys and values. For the binary proxy
(--workload rabitq128k) it is one qs_decode_top_p call, which selects a top-p set. The default workload
is the 128K-context, batch-16 block-level step (40 query / 8 KV heads, d = 128, rank-32
BF16 proxy, 128-token blocks, budget 64 with the sink and last blocks forced); its
seeded synthetic caches (about 9 GiB) exceed the L2, so no flush is needed.

One JSON line is printed by rank 0. With N > 1 (torchrun), every rank runs its own batch
of the same shape on its own GPU (weak scaling: the rows are independent, no collective
is on the data path); the process group only provides the barrier and the max-over-ranks
time.

--impl reference times the CPU oracle (tests-only float64 implementation) on a bounded
sample of the same workload, on the host cores, and prints the same line with
"impl": "reference".
"""
from __future__ import annotations

import argparse
import concurrent.futures as cf
import datetime
import hashlib
import json
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

import synth  # noqa: E402

METRIC = "sparse decode attn steps/s at 128K ctx, batch 16; achieved HBM GB/s vs peak"
WORKLOADS = {"block128k": synth.BLOCK128K, "token32k": synth.TOKEN32K, "ragged": synth.RAGGED,
             "nvfp4": synth.NVFP4_128K, "nvfp4store": synth.NVFP4_STORE_128K,
             "tiny": synth.TINY, "fp8": synth.FP8_128K,
             "fp8token": synth.FP8_TOKEN32K, "centroid": synth.CENTROID_128K,
             "centroid32": synth.CENTROID_S32, "token128k": synth.TOKEN128K,
             "rabitq128k": synth.RABITQ_TOKEN128K, "semantic128k": synth.SEMANTIC_128K}
FALLBACK_HBM_GBS = 6650.0


def parse(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--workload", default="block128k", choices=sorted(WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--cpu-rows", type=int, default=16, help="rows timed for the CPU baseline")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--batch", type=int, default=0,
                    help="override the workload's batch (small cases for profiling only)")
    ap.add_argument("--context", type=int, default=0,
                    help="override the workload's context (small cases for profiling only)")
    ap.add_argument("--no-compare", action="store_true",
                    help="skip the full-KV and gather-then-attend comparison")
    ap.add_argument("--attn-path", type=int, default=0, choices=[0, 1, 2],
                    help="attention kernel: 0 chosen per shape, 1 tile pipeline, 2 gather "
                         "(for profiling small cases)")
    return ap.parse_args(argv)


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "MEASURED_PEAKS.json hbm_gbs (measured copy bandwidth)"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback 6650 GB/s (an earlier copy-bandwidth measurement on B200)"


# ------------------------------------------------------------------ clocks (NVML sampling)

_REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
            0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
            0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
            0x100: "display_clock_setting"}


class Clocks:
    """Samples SM clock and clock-event reasons of one GPU from a thread (read-only)."""

    def __init__(self, index: int, period_s: float = 0.005):
        self.ok = False
        self.samples, self.reasons = [], set()
        self.period = period_s
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            self.max_mhz = None

    def _read(self):
        nv = self.nv
        self.samples.append(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
        try:
            r = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
        except Exception:
            r = nv.nvmlDeviceGetCurrentClocksThrottleReasons(self.h)
        for bit, name in _REASONS.items():
            if r & bit and bit != 0x1:
                self.reasons.add(name)

    def _loop(self):
        while not self._stop.is_set():
            try:
                self._read()
            except Exception:
                pass
            time.sleep(self.period)

    def start(self):
        if not self.ok:
            return
        self._stop = threading.Event()
        self._t = threading.Thread(target=self._loop, daemon=True)
        self._t.start()

    def stop(self):
        if not self.ok:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvml unavailable"]}
        self._stop.set()
        self._t.join()
        try:
            self._read()
        except Exception:
            pass
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
                "samples": len(self.samples)}


# ------------------------------------------------------------------ byte accounting

def step_bytes(w, lens, sel, nsel):
    """Algorithmic bytes of one decode step: proxy-cache bytes streamed + selected K/V bytes
    (valid tokens only) + q + out."""
    d, S = w.head_dim, w.block_size
    if w.proxy_dtype == "centroid":                 # one FP32 key sum per block
        nbs = (lens.astype(np.int64) + S - 1) // S
        proxy = int(nbs.sum()) * w.n_kv_heads * d * 4
    else:
        if w.proxy_dtype == "nvfp4":
            per_tok = d // 2 + d // 16
        elif w.proxy_dtype == "rabitq":                # d code bits + one FP32 factor
            per_tok = d // 8 + 4
        else:
            per_tok = w.proxy_rank * {"f32": 4, "bf16": 2, "e4m3": 1}[w.proxy_dtype]
        proxy = int(np.sum(lens.astype(np.int64))) * w.n_kv_heads * per_tok
    tokens = 0
    kept_tokens = 0                      # NVFP4 key storage: tokens of the kept BF16 blocks
    for b in range(w.batch):
        L = int(lens[b])
        for g in range(w.n_kv_heads):
            blk = sel[b, g, :int(nsel[b, g])].astype(np.int64)
            tokens += int(np.minimum(S, L - blk * S).sum())
            kept_tokens += min(w.n_keep_hp, L // S) * S     # complete, always selected
    if getattr(w, "key_storage", "bf16") == "nvfp4":
        # K: 72 bytes per token (d/2 of codes, d/16 of scales) except the kept blocks' BF16
        kv = tokens * d * 2 + (tokens - kept_tokens) * (d // 2 + d // 16) + kept_tokens * d * 2
    else:
        kv = tokens * d * 2 * 2
    q = w.batch * w.n_q_heads * d * 2
    out = w.batch * w.n_q_heads * d * (4 if w.out_dtype == "f32" else 2)
    return {"proxy": proxy, "kv": kv, "q": q, "out": out, "total": proxy + kv + q + out,
            "selected_tokens": tokens}


def src_hash(*names):
    h = hashlib.sha1()
    for n in names:
        with open(os.path.join(ROOT, "score_then_select_b200", "csrc", n), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:12]


def profiled_traffic(kernel_file: str, workload: str):
    """DRAM bytes per launch recorded by a committed ncu summary, if its source hash still
    matches the kernel's current source; else None."""
    p = os.path.join(ROOT, "profiles", f"{kernel_file}.json")
    try:
        with open(p) as f:
            d = json.load(f)
        if d.get("workload") != workload:
            return None
        if d.get("src_hash") != src_hash(*d["sources"]):
            return None
        return d.get("dram_bytes_per_launch")
    except Exception:
        return None


# ------------------------------------------------------------------ CPU oracle timing

def oracle_prepare(w, inp, rows, threads):
    """The rows' stored inputs and scoring caches, built by the oracle (untimed)."""
    from threadpoolctl import threadpool_limits
    from oracle import method as M
    from oracle import step as OS

    p = OS.top_p_params_of(w) if w.proxy_dtype == "rabitq" else OS.row_params_of(w)

    def prep(bg):
        b, g = bg
        k, v, q = inp.row(b, g)
        L = int(inp.lens[b])
        P = inp.P[g] if inp.P is not None else None
        mu = inp.mu[b, g] if inp.mu is not None else None
        if w.proxy_dtype == "rabitq":                 # the binary codes (P holds R)
            cache = M.rabitq_encode(k[:L], P, mu)
        else:
            cache = OS.row_scoring_cache(p, k[:L], P, mu, inp.g_k)
        return (b, g, k, v, q, L, P, cache)

    with threadpool_limits(limits=1):
        with cf.ThreadPoolExecutor(threads) as ex:
            prepared = list(ex.map(prep, rows))
    g_q = None
    if w.proxy_dtype == "nvfp4":
        g_q = M.query_scale(np.stack([x[4] for x in prepared]))
    return p, prepared, g_q


def oracle_time(w, inp, prep, threads):
    """Seconds for the oracle's decode step (score + select + attend) over prepared rows,
    one row per thread, BLAS pinned to one thread."""
    from threadpoolctl import threadpool_limits
    from oracle import formats as F
    from oracle import method as M
    from oracle import step as OS

    p, prepared, g_q = prep

    def one(x):
        b, g, k, v, q, L, P, cache = x
        if w.proxy_dtype == "rabitq":
            bits, gk = cache
            n, delta, vl, qbar = M.rabitq_query(q, P, inp.u[b, g])
            s = M.rabitq_scores(bits, gk, n, delta, vl, inp.mu[b, g], qbar)
            mass = M.block_mass(M.estimated_weights(s, p.scale), p.S)
            forced = M.forced_blocks(mass.shape[0], p.force_sink, p.force_last)
            sel = M.select_top_p(mass, p.p, p.budget, forced)
        else:
            beta = OS.row_block_scores(p, cache, q, L, P=P, g_q=g_q, g_k=inp.g_k)
            forced, _ = OS.row_forced(p, beta.shape[0], cache, L, inp.g_k)
            sel = M.select_blocks(beta, p.budget, forced)
        tok = M.block_tokens(sel, p.S, L)
        return M.sparse_attention(F.bf16_to_f64(q), F.bf16_to_f64(k[tok]),
                                  OS.decode_v(v[tok], p.v_dtype), np.arange(len(tok)), p.scale)

    with threadpool_limits(limits=1):
        with cf.ThreadPoolExecutor(threads) as ex:
            t0 = time.perf_counter()
            list(ex.map(one, prepared))
            return time.perf_counter() - t0


def host_cores():
    try:
        return len(os.sched_getaffinity(0))
    except Exception:
        return os.cpu_count() or 1


def cpu_baseline(w, inp, nrows, cpu_work_s=10.0, max_wall_s=20.0):
    """The oracle on a bounded sample: `nrows` rows of one step, one row per host thread,
    repeated until about `cpu_work_s` seconds of CPU work (wall time x threads) are done."""
    rows = [(b, g) for b in range(w.batch) for g in range(w.n_kv_heads)][:nrows]
    threads = min(host_cores(), len(rows))
    prep = oracle_prepare(w, inp, rows, threads)
    total, passes = 0.0, 0
    while passes < 1 or (total * threads < cpu_work_s and total < max_wall_s):
        total += oracle_time(w, inp, prep, threads)
        passes += 1
    t = total / passes
    total_rows = w.batch * w.n_kv_heads
    return {"value": (len(rows) / total_rows) / t, "unit": "steps/s", "cores": threads,
            "kind": "oracle",
            "sample": f"{len(rows)} of {total_rows} (sequence, KV head) rows of one step, "
                      f"{passes} passes ({total:.1f} s wall); score+select+attend from "
                      f"prepared scoring caches, float64 numpy, one row per thread"}


# ------------------------------------------------------------------ distributed plumbing

def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def rank_workload(w, rank: int):
    """Each rank decodes its own batch of the same shape (weak scaling): rank r > 0 draws
    its inputs from seed + 1000 r, so no two ranks process the same rows."""
    return w if rank == 0 else w.replace(seed=w.seed + 1000 * rank)


def max_over_ranks(x: float, world: int, device) -> float:
    """The slowest rank's value (all ranks call this in the same order)."""
    if world <= 1:
        return float(x)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate_steps_per_s(ms_per_step_max: float, world: int) -> float:
    """Whole-job throughput: every rank ran the same number of steps; the job took as long
    as its slowest rank."""
    return world * 1e3 / ms_per_step_max


def config_of(w, lens):
    return {"workload": w.name, "global_batch": w.batch, "context": int(lens.max()),
            "q_heads": w.n_q_heads, "kv_heads": w.n_kv_heads, "head_dim": w.head_dim,
            "block_size": w.block_size, "budget_blocks": w.budget, "proxy": w.proxy_dtype,
            "proxy_rank": w.proxy_rank, "parallelism": "independent rows per GPU",
            "l2": "no flush: per-step inputs (proxy cache + selected K/V) exceed the 126 MB L2"}


# ------------------------------------------------------------------ reference arm

def run_reference(args):
    world, rank, local = dist_setup()
    if rank != 0:
        return 0
    w = WORKLOADS[args.workload]
    if w.proxy_dtype == "semantic":
        print(json.dumps({"impl": "reference", "unavailable": (
            "the oracle's float32 k-means index over a 131,072-token prompt per row takes far "
            "longer than a bounded timing run")}), flush=True)
        return 0
    inp = synth.Inputs(w)
    rows_all = [(b, g) for b in range(w.batch) for g in range(w.n_kv_heads)]
    threads = min(host_cores(), len(rows_all))
    # untimed: the rows' stored inputs and scoring caches (the writer's output)
    prep = oracle_prepare(w, inp, rows_all, threads)
    times = []
    t_run = time.perf_counter()
    for i in range(args.warmup + args.steps):
        t = oracle_time(w, inp, prep, threads)            # one whole step: every row
        if i >= args.warmup:
            times.append(t)
    run_s = time.perf_counter() - t_run
    t_step = sum(times) / len(times)
    value = 1.0 / t_step
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "steps/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * t_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": config_of(w, inp.lens),
            "cpu_baseline": {"value": value, "unit": "steps/s", "cores": threads,
                             "kind": "oracle",
                             "sample": f"whole steps: all {len(rows_all)} (sequence, KV head) "
                                       f"rows, score+select+attend from prepared scoring "
                                       f"caches, float64 numpy, one row per host thread; "
                                       f"{args.warmup}+{args.steps} steps in {run_s:.1f} s"},
            "e2e": {"value": value, "unit": "steps/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------------ our arm

def run_compare(args, w, f, lens, sel, nsel, out, stream):
    """Attention-stage comparison: gather-free sparse attention, gather-then-attend and
    full-KV attention, each timed with CUDA events on `stream` (mean of n launches after 3
    untimed rounds), with the algorithmic HBM bytes of each."""
    import torch
    import score_then_select_b200 as qs
    from score_then_select_b200.layer import GatheredKV, workspace
    lay, cfg, cache, B = f.layer, f.cfg, f.cache, w.batch
    ws_d = workspace(qs.qs_dense_workspace_size(cfg, B, lay.max_context))
    gk = GatheredKV.allocate(lay)
    ws_g = workspace(qs.qs_dense_workspace_size(cfg, B, gk.max_context))
    gcache = gk.cache()
    out_c = torch.empty_like(out)
    n = min(args.steps, 20)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(n + 3)]
    for ev in evs:
        ev[0].record(stream)
        qs.qs_sparse_attn(cfg, cache, f.q, sel, nsel, B, out_c, lay.ws, stream)
        ev[1].record(stream)
        qs.qs_gather_kv(cfg, cache, sel, nsel, B, gk.k, gk.v, gk.row_lens, lay.ws, stream)
        ev[2].record(stream)
        qs.qs_dense_attn(cfg, gcache, f.q, gk.row_lens, B, out_c, ws_g, stream)
        ev[3].record(stream)
        qs.qs_dense_attn(cfg, cache, f.q, None, B, out_c, ws_d, stream)
        ev[4].record(stream)
    torch.cuda.synchronize()
    for ws in (lay.ws, ws_d, ws_g):
        st = qs.qs_device_status(ws)
        if st[0] != 0:
            raise RuntimeError(f"device status in the comparison {st}")
    acc = np.zeros(4)
    for ev in evs[3:]:
        acc += [ev[j].elapsed_time(ev[j + 1]) for j in range(4)]
    attend, gather, attend_g, full = (acc / n * 1e3).tolist()
    by = step_bytes(w, lens, sel.cpu().numpy(), nsel.cpu().numpy())
    qo = by["q"] + by["out"]
    full_bytes = int(np.sum(lens.astype(np.int64))) * w.n_kv_heads * w.head_dim * 2 * 2 + qo
    peak, _ = peaks()
    gta = gather + attend_g

    def hbm(nbytes, us):
        return {"bytes": int(nbytes), "GB/s": nbytes / (us * 1e-6) / 1e9,
                "frac": nbytes / (us * 1e-6) / 1e9 / peak}

    return {"attend_us": attend, "gather_us": gather, "attend_gathered_us": attend_g,
            "gather_then_attend_us": gta, "full_kv_us": full,
            "speedup_vs_full_kv": full / attend,
            "gather_then_attend_speedup_vs_full_kv": full / gta,
            "gather_free_speedup_vs_gather_then_attend": gta / attend,
            "hbm": {"attend": hbm(by["kv"] + qo, attend), "gather": hbm(2 * by["kv"], gather),
                    "attend_gathered": hbm(by["kv"] + qo, attend_g),
                    "full_kv": hbm(full_bytes, full)},
            "launches": {"attend": qs.qs_attention_launches(cfg, B, lay.max_context),
                         "gather_then_attend": 3, "full_kv": 2},
            "timed_launches": n}


def run_ours(args):
    import torch
    import torch.distributed as dist

    world, rank, local = dist_setup()
    if world != args.gpus:
        print(f"--gpus {args.gpus} but WORLD_SIZE {world}: launch N > 1 with torchrun",
              file=sys.stderr)
        return 2
    torch.cuda.set_device(local)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local))
    import score_then_select_b200 as qs
    from score_then_select_b200.filled import Filled

    w0 = WORKLOADS[args.workload]
    if args.batch:
        w0 = w0.replace(batch=args.batch)
    if args.context:
        w0 = w0.replace(context=args.context, calib_tokens=min(w0.calib_tokens, args.context))
    w = rank_workload(w0, rank)
    inp = synth.Inputs(w)
    f = Filled(inp, attn_path=args.attn_path)
    if w.proxy_dtype == "rabitq":
        return run_ours_top_p(args, w, inp, f, world, rank, local)
    if w.proxy_dtype == "semantic":
        return run_ours_semantic(args, w, inp, f, world, rank, local)
    lay, cfg, cache = f.layer, f.cfg, f.cache
    B = w.batch
    lens = inp.lens
    start_lens = torch.from_numpy((lens - 1).astype(np.int32)).cuda()
    out = torch.zeros((B, w.n_q_heads, w.head_dim),
                      dtype=torch.float32 if w.out_dtype == "f32" else torch.bfloat16, device="cuda")
    sel = torch.zeros((B, w.n_kv_heads, w.budget), dtype=torch.int32, device="cuda")
    nsel = torch.zeros((B, w.n_kv_heads), dtype=torch.int32, device="cuda")
    stream = torch.cuda.current_stream()

    def step():
        lay.seq_lens.copy_(start_lens, non_blocking=True)
        qs.qs_decode(cfg, cache, f.q, f.k_last, f.v_last, f.P, B, out, sel, nsel, lay.ws, stream)

    for _ in range(max(args.warmup, 3)):
        step()
    st = qs.qs_device_status(lay.ws)
    if st[0] != 0:
        raise RuntimeError(f"device status {st}")
    nsel_h = nsel.cpu().numpy()
    sel_h = sel.cpu().numpy()
    # append [+ block errors + query tiles] + score + select + attention (1 or 2 launches)
    launches_per_step = (5 if w.proxy_dtype == "nvfp4" else 3) + qs.qs_attention_launches(
        lay.cfg, w.batch, lay.max_context)

    def barrier():
        if world > 1:
            dist.barrier()

    # ---------------- timed region: K fused decode steps
    clocks = Clocks(local)
    barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks.start()
    e0.record(stream)
    for _ in range(args.steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize()
    clk = clocks.stop()
    barrier()
    t_ms = max_over_ranks(e0.elapsed_time(e1) / args.steps, world, "cuda")
    st = qs.qs_device_status(lay.ws)
    if st[0] != 0:
        raise RuntimeError(f"device status after timing {st}")

    # ---------------- per-stage breakdown through the standalone entry points
    n_stage = min(args.steps, 50)
    ones = torch.ones((B,), dtype=torch.int32, device="cuda")
    scores = torch.empty((B, w.n_kv_heads, lay.nb_stride), dtype=torch.float32, device="cuda")
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(n_stage + 3)]
    for i in range(n_stage + 3):          # no host sync inside: the host stays ahead
        ev = evs[i]
        lay.seq_lens.copy_(start_lens, non_blocking=True)
        ev[0].record(stream)
        qs.qs_append_kv(cfg, cache, f.k_last, f.v_last, ones, 1, f.P, B, lay.ws, stream)
        ev[1].record(stream)
        qs.qs_score(cfg, cache, f.q, f.P, B, scores, lay.ws, stream)
        ev[2].record(stream)
        qs.qs_select_topk(cfg, cache, scores, B, sel, nsel, lay.ws, stream)
        ev[3].record(stream)
        qs.qs_sparse_attn(cfg, cache, f.q, sel, nsel, B, out, lay.ws, stream)
        ev[4].record(stream)
    torch.cuda.synchronize()
    acc = np.zeros(4)
    for ev in evs[3:]:
        acc += [ev[j].elapsed_time(ev[j + 1]) for j in range(4)]
    stage_us = dict(zip(["append", "score", "select", "attend"], (acc / n_stage * 1e3).tolist()))

    # ---------------- comparison ("Joint Subspace Sparse Attention ...", Figure 2 (b) and
    # Figure 6 (a)): the sparse attention stage (gather-free, reading the selected blocks in
    # place) against full-KV attention over every cached token and against gather-then-attend
    # (qs_gather_kv into a compact buffer, then the same dense kernel over it), on the
    # selection of the steps above; CUDA events on the launching stream, caches > L2.
    compare = None
    if not args.no_compare:
        compare = run_compare(args, w, f, lens, sel, nsel, out, stream)

    # ---------------- end to end: host buffers, copies inside the timed region. Through the
    # public API twice: eager qs_decode calls, and the same step captured once into a CUDA
    # graph (score_then_select_b200.graph.CapturedDecode) and replayed; each step copies q,
    # k_new, v_new from pinned host memory (the graph: one packed copy), decodes, copies the
    # output back and syncs.
    from score_then_select_b200.graph import CapturedDecode
    q_h = f.q.cpu().pin_memory()
    k_h = f.k_last.cpu().pin_memory()
    v_h = f.v_last.cpu().pin_memory()
    out_h = torch.empty(out.shape, dtype=out.dtype).pin_memory()
    q_d, k_d, v_d = torch.empty_like(f.q), torch.empty_like(f.k_last), torch.empty_like(f.v_last)

    def e2e_step():
        q_d.copy_(q_h, non_blocking=True)
        k_d.copy_(k_h, non_blocking=True)
        v_d.copy_(v_h, non_blocking=True)
        lay.seq_lens.copy_(start_lens, non_blocking=True)
        qs.qs_decode(cfg, cache, q_d, k_d, v_d, f.P, B, out, sel, nsel, lay.ws, stream)
        out_h.copy_(out, non_blocking=True)
        stream.synchronize()

    for _ in range(3):
        e2e_step()
    n_e2e = max(args.steps, 10)
    barrier()
    t0 = time.perf_counter()
    for _ in range(n_e2e):
        e2e_step()
    eager_ms = max_over_ranks((time.perf_counter() - t0) * 1e3 / n_e2e, world, "cuda")

    cap = CapturedDecode(cfg, cache, f.P, B, out, sel, nsel, lay.ws, q_d, k_d, v_d,
                         before=lambda: lay.seq_lens.copy_(start_lens, non_blocking=True))
    cap.q_host.copy_(q_h)
    cap.k_host.copy_(k_h)
    cap.v_host.copy_(v_h)
    for _ in range(3):
        cap.step()
    barrier()
    t0 = time.perf_counter()
    for _ in range(n_e2e):
        cap.step()
    e2e_ms = max_over_ranks((time.perf_counter() - t0) * 1e3 / n_e2e, world, "cuda")
    st = qs.qs_device_status(lay.ws)
    if st[0] != 0:
        raise RuntimeError(f"device status after the end-to-end runs {st}")
    if not torch.equal(cap.out_host, out_h):
        raise RuntimeError("graph-replayed step differs from the eager step")
    h2d = cap.h2d_bytes
    d2h = cap.d2h_bytes

    # ---------------- roofline
    peak, peak_src = peaks()
    by = step_bytes(w, lens, sel_h, nsel_h)
    score_us = stage_us["score"]
    score_kernel_file = {"nvfp4": "score_nvfp4.cu", "centroid": "score_centroid.cu"}.get(
        w.proxy_dtype, "score.cu")
    traffic = profiled_traffic(score_kernel_file.replace(".cu", ""), w.name)
    roof = {"bound": "hbm", "kernel": "score (scoring prep + proxy scan, one qs_score call)",
            "achieved": by["proxy"] / (score_us * 1e-6) / 1e9, "peak": peak, "unit": "GB/s",
            "frac": by["proxy"] / (score_us * 1e-6) / 1e9 / peak, "peak_source": peak_src,
            "algorithmic_bytes_per_launch": by["proxy"], "launch_us": score_us,
            "traffic": traffic}
    step_gbs = by["total"] / (t_ms * 1e-3) / 1e9
    value = aggregate_steps_per_s(t_ms, world)
    line = {"metric": METRIC, "value": value, "unit": "steps/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": t_ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": {"bf16": "bf16", "f32": "f32+bf16", "centroid": "f32+bf16"}.get(
                w.proxy_dtype, f"{w.proxy_dtype}+bf16"),
            "data": "synthetic (seeded; shapes of the pages' 128K batch-16 decode)",
            "config": config_of(w, lens),
            "tokens_per_s": value * B, "us_per_layer_step": t_ms * 1e3,
            "step_hbm": {"achieved": step_gbs, "peak": peak, "unit": "GB/s",
                         "frac": step_gbs / peak, "bytes_per_step": by},
            "stage_us": stage_us, "roofline": roof, "clocks": clk,
            "e2e": {"value": aggregate_steps_per_s(e2e_ms, world), "unit": "steps/s",
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                    "ms_per_step": e2e_ms, "path": "CapturedDecode (CUDA graph of the step)",
                    "eager_ms_per_step": eager_ms},
            "gpu_launches": args.steps * launches_per_step}
    # the attention stage's own roofline: selected K/V bytes + q + out over its stage time
    att_b = by["kv"] + by["q"] + by["out"]
    line["attend_hbm"] = {"achieved": att_b / (stage_us["attend"] * 1e-6) / 1e9, "peak": peak,
                          "unit": "GB/s",
                          "frac": att_b / (stage_us["attend"] * 1e-6) / 1e9 / peak,
                          "bytes": att_b, "us": stage_us["attend"]}
    if getattr(w, "key_storage", "bf16") == "nvfp4":
        # capacity of the storage variant ("Jet-QSparse ...", Full text): bytes held per
        # cached token by the key and value pages the attention needs, against a BF16 K/V
        # cache (the two kept BF16 blocks of each row are spread over its tokens)
        d = w.head_dim
        kept = w.n_keep_hp * w.block_size * d * 2 / float(lens.mean())
        per_tok = (d // 2 + d // 16) + d * 2 + kept
        line["capacity"] = {"bytes_per_token": per_tok, "bf16_kv_bytes_per_token": 4 * d,
                            "tokens_vs_bf16_kv": 4 * d / per_tok,
                            "note": "NVFP4 keys (codes + scales), FP16 values, 2 BF16 blocks "
                                    "per (sequence, KV head)"}
    if compare is not None:
        line["comparison"] = compare
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(w, inp, args.cpu_rows)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def run_ours_top_p(args, w, inp, f, world, rank, local):
    """The binary proxy's step ("RaBitQCache", Abstract): qs_decode_top_p (append with the
    binary writer, query code + scan, top-p select, sparse attention) timed like the fused
    step of the other proxies; the stage breakdown issues the four stage calls with events
    between them; end to end, the step is captured once into a CUDA graph with its host
    copies (CapturedDecode) and replayed."""
    import torch
    import torch.distributed as dist
    import score_then_select_b200 as qs

    lay, cfg, cache = f.layer, f.cfg, f.cache
    B, lens, Hkv = w.batch, inp.lens, w.n_kv_heads
    start_lens = torch.from_numpy((lens - 1).astype(np.int32)).cuda()
    ones = torch.ones((B,), dtype=torch.int32, device="cuda")
    u = torch.from_numpy(inp.u).cuda()
    out = torch.zeros((B, w.n_q_heads, w.head_dim),
                      dtype=torch.float32 if w.out_dtype == "f32" else torch.bfloat16, device="cuda")
    sel = torch.zeros((B, Hkv, w.budget), dtype=torch.int32, device="cuda")
    nsel = torch.zeros((B, Hkv), dtype=torch.int32, device="cuda")
    scores = torch.empty((B, Hkv, lay.nb_stride), dtype=torch.float32, device="cuda")
    stream = torch.cuda.current_stream()
    p = float(w.top_p)

    def step(q, k, v):
        lay.seq_lens.copy_(start_lens, non_blocking=True)
        qs.qs_decode_top_p(cfg, cache, q, k, v, f.P, u, p, B, out, sel, nsel, lay.ws, stream)

    def stages(q, k, v, ev):
        lay.seq_lens.copy_(start_lens, non_blocking=True)
        ev[0].record(stream)
        qs.qs_append_kv(cfg, cache, k, v, ones, 1, f.P, B, lay.ws, stream)
        ev[1].record(stream)
        qs.qs_rabitq_score(cfg, cache, q, f.P, u, B, scores, lay.ws, stream)
        ev[2].record(stream)
        qs.qs_select_top_p(cfg, cache, scores, p, B, sel, nsel, lay.ws, stream)
        ev[3].record(stream)
        qs.qs_sparse_attn(cfg, cache, q, sel, nsel, B, out, lay.ws, stream)
        ev[4].record(stream)

    for _ in range(max(args.warmup, 3)):
        step(f.q, f.k_last, f.v_last)
    st = qs.qs_device_status(lay.ws)
    if st[0] != 0:
        raise RuntimeError(f"device status {st}")
    sel_h, nsel_h = sel.cpu().numpy(), nsel.cpu().numpy()
    # append + query code + scan + top-p select + attention (1 or 2 launches)
    launches_per_step = 4 + qs.qs_attention_launches(cfg, B, lay.max_context)

    def barrier():
        if world > 1:
            dist.barrier()

    # ---------------- timed region: K steps
    clocks = Clocks(local)
    barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks.start()
    e0.record(stream)
    for _ in range(args.steps):
        step(f.q, f.k_last, f.v_last)
    e1.record(stream)
    torch.cuda.synchronize()
    clk = clocks.stop()
    barrier()
    t_ms = max_over_ranks(e0.elapsed_time(e1) / args.steps, world, "cuda")
    st = qs.qs_device_status(lay.ws)
    if st[0] != 0:
        raise RuntimeError(f"device status after timing {st}")

    # ---------------- per-stage breakdown (events between the four calls)
    n_stage = min(args.steps, 50)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(n_stage + 3)]
    for ev in evs:
        stages(f.q, f.k_last, f.v_last, ev)
    torch.cuda.synchronize()
    acc = np.zeros(4)
    for ev in evs[3:]:
        acc += [ev[j].elapsed_time(ev[j + 1]) for j in range(4)]
    stage_us = dict(zip(["append", "score", "select", "attend"], (acc / n_stage * 1e3).tolist()))

    # ---------------- end to end: the step captured once with its host copies (q, k_new,
    # v_new from pinned host memory in one packed copy; the output back to pinned memory)
    # and replayed; each replay is followed by a sync
    from score_then_select_b200.graph import CapturedDecode
    cap = CapturedDecode(
        cfg, cache, f.P, B, out, sel, nsel, lay.ws, f.q, f.k_last, f.v_last,
        before=lambda: lay.seq_lens.copy_(start_lens, non_blocking=True),
        call=lambda q, k, v, s_: qs.qs_decode_top_p(cfg, cache, q, k, v, f.P, u, p, B, out,
                                                    sel, nsel, lay.ws, s_))
    cap.q_host.copy_(f.q.cpu())
    cap.k_host.copy_(f.k_last.cpu())
    cap.v_host.copy_(f.v_last.cpu())
    for _ in range(3):
        cap.step()
    n_e2e = max(args.steps, 10)
    barrier()
    t0 = time.perf_counter()
    for _ in range(n_e2e):
        cap.step()
    e2e_ms = max_over_ranks((time.perf_counter() - t0) * 1e3 / n_e2e, world, "cuda")
    st = qs.qs_device_status(lay.ws)
    if st[0] != 0:
        raise RuntimeError(f"device status after the end-to-end runs {st}")
    h2d, d2h = cap.h2d_bytes, cap.d2h_bytes

    # ---------------- roofline: the scan (query code + binary scan, one qs_rabitq_score)
    peak, peak_src = peaks()
    by = step_bytes(w, lens, sel_h, nsel_h)
    score_us = stage_us["score"]
    roof = {"bound": "hbm", "kernel": "score (query code + binary scan, one qs_rabitq_score call)",
            "achieved": by["proxy"] / (score_us * 1e-6) / 1e9, "peak": peak, "unit": "GB/s",
            "frac": by["proxy"] / (score_us * 1e-6) / 1e9 / peak, "peak_source": peak_src,
            "algorithmic_bytes_per_launch": by["proxy"], "launch_us": score_us,
            "traffic": profiled_traffic("rabitq", w.name)}
    step_gbs = by["total"] / (t_ms * 1e-3) / 1e9
    value = aggregate_steps_per_s(t_ms, world)
    cfg_line = config_of(w, lens)
    cfg_line["top_p"] = w.top_p
    cfg_line["mean_selected_blocks"] = float(nsel_h.mean())
    line = {"metric": METRIC, "value": value, "unit": "steps/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": t_ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "b1xi4+f32+bf16",
            "data": "synthetic (seeded; shapes of the pages' 128K batch-16 decode)",
            "config": cfg_line, "tokens_per_s": value * B, "us_per_layer_step": t_ms * 1e3,
            "step_hbm": {"achieved": step_gbs, "peak": peak, "unit": "GB/s",
                         "frac": step_gbs / peak, "bytes_per_step": by},
            "stage_us": stage_us, "roofline": roof, "clocks": clk,
            "e2e": {"value": aggregate_steps_per_s(e2e_ms, world), "unit": "steps/s",
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                    "ms_per_step": e2e_ms,
                    "path": "CapturedDecode (CUDA graph of qs_decode_top_p)"},
            "gpu_launches": args.steps * launches_per_step}
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(w, inp, args.cpu_rows)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def run_ours_semantic(args, w, inp, f, world, rank, local):
    """The semantic-block step ("Coarse Semantic Blocks ...", Abstract). Before timing, the
    k-means index over each sequence's prompt (all but the newest token) is built once.
    Each timed step appends the newest token (K/V only), runs qs_semantic_select (cluster
    scores, top clusters, expansion into a token list) and attends over that list with the
    token-level attention. No CPU baseline: the oracle's float32 k-means is far too slow at
    this size."""
    import torch
    import torch.distributed as dist
    import score_then_select_b200 as qs
    from score_then_select_b200.graph import CapturedDecode
    from score_then_select_b200.layer import workspace
    from score_then_select_b200.filled import cfg_kwargs

    lay, cfg, cache = f.layer, f.cfg, f.cache
    B, Hkv, d = w.batch, w.n_kv_heads, w.head_dim
    lens = inp.lens
    start_lens = torch.from_numpy((lens - 1).astype(np.int32)).cuda()
    prompt = start_lens.clone()
    Lmax = lay.max_context
    rows, c_max = B * Hkv, -(-Lmax // w.block_size)
    cent = torch.empty((rows, c_max, d), dtype=torch.float32, device="cuda")
    offsets = torch.empty((rows, c_max + 1), dtype=torch.int32, device="cuda")
    members = torch.empty((rows, Lmax), dtype=torch.int32, device="cuda")
    ws_idx = workspace(qs.qs_semantic_index_workspace_size(cfg, B, Lmax))
    lay.seq_lens.copy_(start_lens)
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    qs.qs_semantic_index(cfg, cache, prompt, 4, cent, offsets, members, B, ws_idx)
    torch.cuda.synchronize()
    index_ms = (time.perf_counter() - t0) * 1e3
    st = qs.qs_device_status(ws_idx)
    if st[0] != 0:
        raise RuntimeError(f"device status after the index build {st}")
    max_tokens = Lmax
    cfg_tok = qs.make_config(**dict(cfg_kwargs(w), block_size=1, budget=max_tokens))
    ws_tok = workspace(qs.qs_workspace_size(cfg_tok, B, Lmax))
    tokens = torch.empty((B, Hkv, max_tokens), dtype=torch.int32, device="cuda")
    ntok = torch.empty((B, Hkv), dtype=torch.int32, device="cuda")
    ones = torch.ones((B,), dtype=torch.int32, device="cuda")
    out = torch.zeros((B, w.n_q_heads, d), dtype=torch.bfloat16, device="cuda")
    stream = torch.cuda.current_stream()

    def calls(q, k, v, s_, ev=None):
        if ev:
            ev[0].record(s_)
        qs.qs_append_kv(cfg, cache, k, v, ones, 1, None, B, lay.ws, s_)
        if ev:
            ev[1].record(s_)
        qs.qs_semantic_select(cfg, cache, q, prompt, cent, offsets, members, B, tokens, ntok,
                              max_tokens, lay.ws, s_)
        if ev:
            ev[2].record(s_)
        qs.qs_sparse_attn(cfg_tok, cache, q, tokens, ntok, B, out, ws_tok, s_)
        if ev:
            ev[3].record(s_)

    def step(ev=None):
        lay.seq_lens.copy_(start_lens, non_blocking=True)
        calls(f.q, f.k_last, f.v_last, stream, ev)

    for _ in range(max(args.warmup, 3)):
        step()
    for ws in (lay.ws, ws_tok):
        st = qs.qs_device_status(ws)
        if st[0] != 0:
            raise RuntimeError(f"device status {st}")
    ntok_h = ntok.cpu().numpy()
    launches_per_step = 1 + 3 + qs.qs_attention_launches(cfg_tok, B, Lmax)

    def barrier():
        if world > 1:
            dist.barrier()

    clocks = Clocks(local)
    barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks.start()
    e0.record(stream)
    for _ in range(args.steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize()
    clk = clocks.stop()
    barrier()
    t_ms = max_over_ranks(e0.elapsed_time(e1) / args.steps, world, "cuda")

    n_stage = min(args.steps, 50)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(n_stage + 3)]
    for ev in evs:
        step(ev)
    torch.cuda.synchronize()
    acc = np.zeros(3)
    for ev in evs[3:]:
        acc += [ev[j].elapsed_time(ev[j + 1]) for j in range(3)]
    stage_us = dict(zip(["append", "score+select", "attend"], (acc / n_stage * 1e3).tolist()))

    cap = CapturedDecode(cfg, cache, None, B, out, None, None, lay.ws, f.q, f.k_last, f.v_last,
                         before=lambda: lay.seq_lens.copy_(start_lens, non_blocking=True),
                         call=lambda q, k, v, s_: calls(q, k, v, s_))
    cap.q_host.copy_(f.q.cpu())
    cap.k_host.copy_(f.k_last.cpu())
    cap.v_host.copy_(f.v_last.cpu())
    for _ in range(3):
        cap.step()
    n_e2e = max(args.steps, 10)
    barrier()
    t0 = time.perf_counter()
    for _ in range(n_e2e):
        cap.step()
    e2e_ms = max_over_ranks((time.perf_counter() - t0) * 1e3 / n_e2e, world, "cuda")
    for ws in (lay.ws, ws_tok):
        st = qs.qs_device_status(ws)
        if st[0] != 0:
            raise RuntimeError(f"device status after the end-to-end runs {st}")

    # bytes: centroids scanned, the attended tokens' K and V, q and out
    peak, peak_src = peaks()
    clusters = -(-(lens.astype(np.int64) - 1) // w.block_size)
    by_cent = int(clusters.sum()) * Hkv * d * 4
    by_kv = int(ntok_h.astype(np.int64).sum()) * d * 2 * 2
    by_qo = 2 * B * w.n_q_heads * d * 2
    by = {"centroids": by_cent, "kv": by_kv, "q+out": by_qo, "total": by_cent + by_kv + by_qo,
          "attended_tokens": int(ntok_h.sum())}
    att_us = stage_us["attend"]
    roof = {"bound": "hbm", "kernel": "attend (token-level attention over the expanded list)",
            "achieved": by_kv / (att_us * 1e-6) / 1e9, "peak": peak, "unit": "GB/s",
            "frac": by_kv / (att_us * 1e-6) / 1e9 / peak, "peak_source": peak_src,
            "algorithmic_bytes_per_launch": by_kv, "launch_us": att_us, "traffic": None}
    value = aggregate_steps_per_s(t_ms, world)
    cfg_line = config_of(w, lens)
    cfg_line.update({"index_build_ms": index_ms, "kmeans_iters": 4,
                     "mean_attended_tokens": float(ntok_h.mean())})
    step_gbs = by["total"] / (t_ms * 1e-3) / 1e9
    line = {"metric": METRIC, "value": value, "unit": "steps/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": t_ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "f32+bf16", "data": "synthetic (seeded; shapes of the pages' 128K batch-16 decode)",
            "config": cfg_line, "tokens_per_s": value * B, "us_per_layer_step": t_ms * 1e3,
            "step_hbm": {"achieved": step_gbs, "peak": peak, "unit": "GB/s",
                         "frac": step_gbs / peak, "bytes_per_step": by},
            "stage_us": stage_us, "roofline": roof, "clocks": clk,
            "e2e": {"value": aggregate_steps_per_s(e2e_ms, world), "unit": "steps/s",
                    "h2d_bytes_per_step": cap.h2d_bytes, "d2h_bytes_per_step": cap.d2h_bytes,
                    "ms_per_step": e2e_ms, "path": "CapturedDecode (CUDA graph of the three calls)"},
            "gpu_launches": args.steps * launches_per_step}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def main(argv=None):
    args = parse(argv)
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
