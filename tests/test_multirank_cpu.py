"""The N > 1 host logic of bench.py on CPU: two gloo ranks.

Layers are independent problems, so the multi-GPU bench gives every rank its own
layer (weak scaling, no data-path collective); the only collective is the
max-over-ranks of the timings.
"""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
import synthetic as S


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        r, lr, w = bench.env_rank()
        wl = S.workloads()["layer-256x512"]
        layer = bench.rank_layer(wl.layers[0], r)
        x = S.make_x(layer.x, 0, 64)
        ms = 10.0 + 5.0 * r                       # rank 1 is the slower one
        slowest = bench.max_over_ranks(ms, w)
        value = bench.job_gparams_per_s(w, layer.w.out, layer.w.n, slowest)
        q.put((r, lr, w, layer.x.seed, int(x[:2, :4].sum()), slowest, value))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_slowest_time_and_distinct_layers():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    (r0, lr0, w0, seed0, x0, ms0, v0), (r1, lr1, w1, seed1, x1, ms1, v1) = res
    assert (r0, r1, w0, w1, lr0, lr1) == (0, 1, 2, 2, 0, 1)
    assert seed0 != seed1 and x0 != x1                 # independent problems per rank
    assert ms0 == ms1 == 15.0                          # max over ranks
    assert v0 == v1 == pytest.approx(2 * 256 * 512 / 15e-3 / 1e9)


def test_single_rank_is_the_identity():
    assert bench.max_over_ranks(3.5, 1) == 3.5
    assert bench.job_gparams_per_s(1, 1024, 4096, 2.0) == pytest.approx(1024 * 4096 / 2e-3 / 1e9)
