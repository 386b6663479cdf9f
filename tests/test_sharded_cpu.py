"""The host logic of one layer split over ranks (sharded.py), on two gloo ranks on CPU.

The library's kernels need a B200; here each rank's kernel results are stood in for
by the oracle on the same shard (partial H of the rank's tokens; the sweep of the
rank's rows with the shared U), so that what is tested is what sharded.py adds: the
partition of tokens and rows, the all-reduce that completes H, and the gather that
puts the row shards back together along the outputs.  The whole must equal the
oracle's unsplit layer: H to rounding, the quantized layer exactly (rows are
independent given U, "polydesk.ai/glossaire/gptq", "Etape 1").
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import synthetic as S
from oracle import gptq_oracle as O
from post_weight_quantization_15_b200 import sharded as SH

OUT, N_IN, TOKENS = 150, 256, 1000          # rows and tokens that two ranks split unevenly


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        W, x = S.small_case(OUT, N_IN, TOKENS, seed=12)
        # tokens: this rank's partial Hessian (the oracle stands in for the kernel), then the sum
        t0, t1 = SH.split_range(TOKENS, world, rank, align=8)
        H = torch.from_numpy(O.hessian(x[:, t0:t1]))
        hdiag = torch.from_numpy(O.hessian_diag(x[:, t0:t1]))
        SH.allreduce_hessian(H, hdiag)
        H = H.numpy()
        prep = O.prepare(H, 0.01, True, order_key=hdiag.numpy())
        # rows: this rank's rows given the shared U, then the gather along the outputs
        o0, o1 = SH.split_range(OUT, world, rank)
        sw, codes = O.quantize_layer(W[o0:o1], prep, 3, 64, False, 128)
        qweight = torch.from_numpy(O.pack(codes, 3))
        scales = torch.from_numpy(sw.scales.astype(np.float16))
        zeros = torch.from_numpy(sw.zeros.astype(np.float16))
        sizes = [SH.split_range(OUT, world, r)[1] - SH.split_range(OUT, world, r)[0] for r in range(world)]
        qw, sc, zr = SH.gather_rows([qweight, scales, zeros], sizes, 1)
        cd, none = SH.gather_rows([torch.from_numpy(codes), None], sizes, 0)
        q.put((rank, (t0, t1), (o0, o1), H, hdiag.numpy(), prep.perm, qw.numpy(), sc.numpy(), zr.numpy(),
               cd.numpy(), none))
    finally:
        dist.destroy_process_group()


def test_split_range_partitions():
    for total, world, align in [(1000, 2, 8), (65536, 8, 8), (150, 4, 1), (7, 8, 1), (0, 3, 1), (100, 3, 64)]:
        rs = [SH.split_range(total, world, r, align) for r in range(world)]
        assert rs[0][0] == 0 and rs[-1][1] == total
        for (a, b), (c, d) in zip(rs, rs[1:]):
            assert b == c and a <= b
        for a, b in rs[:-1]:
            assert b % align == 0 or b == total
    with pytest.raises(ValueError):
        SH.split_range(10, 2, 2)


def test_two_gloo_ranks_rebuild_the_unsplit_layer():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted((q.get(timeout=180) for _ in procs), key=lambda t: t[0])
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    W, x = S.small_case(OUT, N_IN, TOKENS, seed=12)
    H_ref = O.hessian(x)
    (_, tr0, or0, H0, d0, p0, qw0, sc0, zr0, cd0, n0), (_, tr1, or1, H1, d1, p1, qw1, sc1, zr1, cd1, n1) = res
    assert tr0 == (0, 496) and tr1 == (496, TOKENS)            # token shards, row-aligned to 8
    assert or0 == (0, 75) and or1 == (75, OUT)
    # the all-reduce leaves the same bits on both ranks: the unsplit H to rounding
    assert np.array_equal(H0, H1) and np.array_equal(d0, d1) and np.array_equal(p0, p1)
    assert np.allclose(H0, H_ref, rtol=1e-12, atol=1e-12 * np.abs(H_ref).max())
    assert np.allclose(d0, np.diag(H_ref), rtol=1e-13)
    # given that H, the gathered row shards are exactly the unsplit layer, on both ranks
    prep = O.prepare(H0, 0.01, True, order_key=d0)
    assert np.array_equal(p0, prep.perm)
    sw, codes = O.quantize_layer(W, prep, 3, 64, False, 128)
    for a, b in ((qw0, qw1), (sc0, sc1), (zr0, zr1), (cd0, cd1)):
        assert np.array_equal(a, b)
    assert n0 is None and n1 is None
    assert qw0.shape == (N_IN * 3 // 32, OUT) and cd0.shape == (OUT, N_IN)
    assert np.array_equal(cd0, codes)
    assert np.array_equal(qw0.view(np.uint32), O.pack(codes, 3).view(np.uint32))
    assert np.array_equal(sc0, sw.scales.astype(np.float16)) and np.array_equal(zr0, sw.zeros.astype(np.float16))
    # a planted mistake in the gather (shards concatenated in the wrong order) is seen
    wrong = np.concatenate([qw0[:, 75:], qw0[:, :75]], axis=1)
    assert not np.array_equal(wrong, O.pack(codes, 3))
