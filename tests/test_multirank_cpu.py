"""Host logic of the multi-GPU paths on CPU, with gloo ranks.

bench.py either runs one independent layer-step per rank (no collective on
the data path) or, with --key-shards equal to the number of GPUs, shares one
layer-step over the ranks by keys (partials all-gathered and merged); it
reports the slowest rank's time.  Checked here with two and three processes,
the oracle standing in for the kernels: the cross-rank reduction, the
binding's sharded attention, and the bench's split of the key sequence.
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


def _bench_shard_worker(rank, world, port, out):
    # The key-sharded bench step's orchestration, with the oracle standing in
    # for the kernels: this rank's share of [history | text | segment] keys
    # (bench.local_key_spans), partial attention, all-gather, merge.
    import sys
    sys.path.insert(0, ROOT)
    import numpy as np
    import torch

    import bench
    import kv_cached_segment_b200 as nm
    import oracle

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        g = torch.Generator().manual_seed(1)
        lens = [700, 37, 300]  # history, text, segment; shares on 128-key tiles
        q = torch.randn((23, 16, 128), generator=g, dtype=torch.float64)
        kv = [(torch.randn((n, 16, 128), generator=g, dtype=torch.float64),
               torch.randn((n, 16, 128), generator=g, dtype=torch.float64)) for n in lens]
        local = bench.local_key_spans(lens, rank, world)
        spans = [(kv[s][0][lo:hi], kv[s][1][lo:hi]) for s, lo, hi in local]

        def attend(qq, sp, lse_out):
            if not sp:
                lse_out.fill_(-float("inf"))
                return torch.zeros_like(qq)
            o, l = oracle.attention(qq.numpy(), [(a.numpy(), b.numpy()) for a, b in sp])
            lse_out.copy_(torch.from_numpy(l).reshape(-1))
            return torch.from_numpy(o)

        def merge(op, lp, lse_out):
            o, _ = oracle.merge_partials(op.numpy(), lp.double().numpy())
            return torch.from_numpy(o)

        lse = torch.empty(16 * 23, dtype=torch.float32)
        o = nm.sharded_segment_attention(q, spans, attend=attend, merge=merge, lse=lse)
        o_ref, _ = oracle.attention(q.numpy(), [(a.numpy(), b.numpy()) for a, b in kv])
        keys = sum(hi - lo for _, lo, hi in local)
        out[rank] = (float(np.abs(o.numpy() - o_ref).max()), keys)
    finally:
        dist.destroy_process_group()


def test_bench_key_shards_on_gloo_ranks():
    for world in (2, 3):
        ctx = mp.get_context("spawn")
        mgr = ctx.Manager()
        out = mgr.dict()
        port = _free_port()
        procs = [ctx.Process(target=_bench_shard_worker, args=(r, world, port, out))
                 for r in range(world)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(timeout=180)
            assert p.exitcode == 0
        assert all(out[r][0] < 1e-6 for r in range(world))
        assert sum(out[r][1] for r in range(world)) == 700 + 37 + 300  # every key once


def test_local_key_spans_partition_in_order():
    import sys
    sys.path.insert(0, ROOT)
    import bench
    lens = [55200, 512, 27600]
    for world in (1, 2, 3, 8):
        seen = []
        for r in range(world):
            for s, lo, hi in bench.local_key_spans(lens, r, world):
                base = sum(lens[:s])
                seen.extend(range(base + lo, base + hi))
        assert seen == list(range(sum(lens)))


def _head_sharded_worker(rank, world, port, out):
    # Head-sharded (Ulysses-style) attention: query and key rows spread over
    # the ranks, one all-to-all to heads, attention over 16/world heads, one
    # all-to-all back; the oracle stands in for the kernel.
    import sys
    sys.path.insert(0, ROOT)
    import numpy as np
    import torch

    import kv_cached_segment_b200 as nm
    import oracle

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        g = torch.Generator().manual_seed(2)
        lens = [70, 9, 40]
        q = torch.randn((23, 16, 128), generator=g, dtype=torch.float64)
        kv = [(torch.randn((n, 16, 128), generator=g, dtype=torch.float64),
               torch.randn((n, 16, 128), generator=g, dtype=torch.float64)) for n in lens]
        qa, qb = nm.shard_rows(23, rank, world, align=1)
        spans = []
        for k, v in kv:
            a, b = nm.shard_rows(k.shape[0], rank, world, align=1)
            if b > a:
                spans.append((k[a:b], v[a:b]))
        seen = {}

        def attend(qq, sp, lse_out):
            seen["heads"] = qq.shape[1]
            seen["rows"] = qq.shape[0]
            seen["keys"] = sum(a.shape[0] for a, _ in sp)
            o, l = oracle.attention(qq.numpy(), [(a.numpy(), b.numpy()) for a, b in sp])
            lse_out.copy_(torch.from_numpy(l).reshape(-1))
            return torch.from_numpy(o)

        lse = torch.empty(16 * (qb - qa), dtype=torch.float32)
        o = nm.head_sharded_segment_attention(q[qa:qb], spans, attend=attend, lse=lse)
        o_ref, l_ref = oracle.attention(q.numpy(), [(a.numpy(), b.numpy()) for a, b in kv])
        out[rank] = (float(np.abs(o.numpy() - o_ref[qa:qb]).max()),
                     float(np.abs(lse.view(16, -1).double().numpy() - l_ref[:, qa:qb]).max()),
                     seen["heads"], seen["rows"], seen["keys"])
    finally:
        dist.destroy_process_group()


def test_head_sharded_attention_on_gloo_ranks():
    for world in (2, 4):
        ctx = mp.get_context("spawn")
        mgr = ctx.Manager()
        out = mgr.dict()
        port = _free_port()
        procs = [ctx.Process(target=_head_sharded_worker, args=(r, world, port, out))
                 for r in range(world)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(timeout=180)
            assert p.exitcode == 0
        for r in range(world):
            err_o, err_l, heads, rows, keys = out[r]
            assert err_o < 1e-9 and err_l < 1e-5, (world, r, err_o, err_l)
            # every rank attends over all rows and all keys for 16/world heads
            assert heads == 16 // world and rows == 23 and keys == 70 + 9 + 40
