"""Host logic of the multi-GPU bench on CPU: two gloo ranks.

bench.py runs one independent layer-step per rank (no collective on the data
path) and reports the slowest rank's time; this checks that reduction with a
world of two processes.
"""
import os
import socket

import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    import sys
    sys.path.insert(0, ROOT)
    import bench

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        vals = bench.max_over_ranks([10.0 + rank, 5.0 - rank, 1.5], world, "cpu")
        out[rank] = vals
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    out = mgr.dict()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    assert out[0] == [11.0, 5.0, 1.5] and out[1] == [11.0, 5.0, 1.5]


def test_max_over_ranks_single_rank_is_identity():
    import sys
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks([3, 4.5], 1, "cpu") == [3.0, 4.5]


def _sharded_worker(rank, world, port, out):
    import sys
    sys.path.insert(0, ROOT)
    import numpy as np
    import torch

    import kv_cached_segment_b200 as nm
    import oracle

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        g = torch.Generator().manual_seed(0)
        q = torch.randn((9, 16, 128), generator=g, dtype=torch.float64)
        k = torch.randn((50, 16, 128), generator=g, dtype=torch.float64)
        v = torch.randn((50, 16, 128), generator=g, dtype=torch.float64)
        a, b = nm.shard_rows(50, rank, world, align=8)

        def attend(qq, spans, lse_out):  # the oracle stands in for the kernel on CPU
            o, l = oracle.attention(qq.numpy(), [(s[0].numpy(), s[1].numpy()) for s in spans])
            lse_out.copy_(torch.from_numpy(l).reshape(-1))
            return torch.from_numpy(o)

        def merge(op, lp, lse_out):
            o, _ = oracle.merge_partials(op.numpy(), lp.double().numpy())
            return torch.from_numpy(o)

        o = nm.sharded_segment_attention(q, [(k[a:b], v[a:b])], attend=attend, merge=merge)
        o_ref, _ = oracle.attention(q.numpy(), [(k.numpy(), v.numpy())])
        out[rank] = float(np.abs(o.numpy() - o_ref).max())
    finally:
        dist.destroy_process_group()


def test_sharded_attention_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    out = mgr.dict()
    port = _free_port()
    procs = [ctx.Process(target=_sharded_worker, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=180)
        assert p.exitcode == 0
    assert out[0] < 1e-6 and out[1] < 1e-6


def test_shard_rows_covers_everything_once():
    import kv_cached_segment_b200 as nm
    for n in (0, 1, 7, 920, 55200, 55201):
        for world in (1, 2, 3, 8):
            cuts = [nm.shard_rows(n, r, world, align=920) for r in range(world)]
            assert cuts[0][0] == 0 and cuts[-1][1] == n
            assert all(cuts[i][1] == cuts[i + 1][0] for i in range(world - 1))
