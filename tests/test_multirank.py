"""Host logic of multi-GPU runs, on CPU with two gloo ranks: each rank decodes its own
batch (distinct seeds, same shapes), and the job's time is the slowest rank's."""
import os
import socket

import pytest
import torch.multiprocessing as mp

import synth


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import torch.distributed as dist
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w = bench.rank_workload(synth.BLOCK128K, rank)
        t = bench.max_over_ranks(1.0 + rank * 0.5, world, "cpu")
        lens = synth.lengths(w)
        q.put((rank, w.seed, t, bench.aggregate_steps_per_s(t, world), tuple(lens.tolist())))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_weak_scaling():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=5) for _ in range(2))
    (r0, s0, t0, v0, l0), (r1, s1, t1, v1, l1) = res
    assert s0 != s1                              # different rows on different ranks
    assert l0 == l1                              # same shapes
    assert t0 == t1 == 1.5                       # the slowest rank's time on every rank
    assert v0 == v1 == pytest.approx(2 * 1e3 / 1.5)


def test_single_rank_is_identity():
    import bench
    assert bench.max_over_ranks(3.25, 1, "cpu") == 3.25
    assert bench.rank_workload(synth.TINY, 0) is synth.TINY
