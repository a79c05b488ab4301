"""Host logic of bench.py that needs no GPU: how keys are split into shards."""
import pytest
import torch

import bench
import kv_cached_segment_b200 as nm


class _Step(bench.LayerStep):
    def __init__(self, shards):  # no device buffers: only the span split is used
        self.nm, self.torch, self.shards = nm, torch, shards


@pytest.mark.parametrize("shards", [1, 2, 3, 8, 40])
def test_key_shards_cover_the_key_sequence_once_in_order(shards):
    lens = [1000, 37, 700]
    spans = []
    start = 0
    for n in lens:
        ids = torch.arange(start, start + n, dtype=torch.float32).view(n, 1, 1)
        spans.append((ids, -ids))
        start += n
    parts = _Step(shards)._shard_spans(spans)
    assert len(parts) == shards
    keys = torch.cat([k.flatten() for sub in parts for k, _ in sub])
    vals = torch.cat([v.flatten() for sub in parts for _, v in sub])
    assert torch.equal(keys, torch.arange(sum(lens), dtype=torch.float32))
    assert torch.equal(vals, -keys)
    for sub in parts:
        assert 1 <= len(sub) <= 4  # the attention call takes at most 4 spans
    # shard boundaries sit on 128-key tiles
    firsts = [int(sub[0][0].flatten()[0]) for sub in parts if sub[0][0].numel()]
    assert all(f % 128 == 0 for f in firsts)
    if shards > (sum(lens) + 127) // 128:
        assert any(sub[0][0].numel() == 0 for sub in parts)


def test_auto_kv_splits_fills_the_gpu_only_when_it_pays():
    from seeded_inputs import WORKLOADS

    def splits(name):
        w = WORKLOADS[name]
        hist = w.n_window if w.select_frames else w.n_cache
        return nm.auto_kv_splits(w.n_q, [hist, w.n_text, w.n_seg])

    # 11.9 waves of query blocks already: no split; 3.35 waves: split in two
    assert splits("720p") == 1 and splits("bounded") == 1 and splits("bounded90") == 1
    assert splits("short") == 2
    # too few tiles to split
    assert splits("tiny") == 1
    # 2 query blocks x 16 heads over 652 key tiles: as many splits as fit one wave
    s = nm.auto_kv_splits(512, [55200, 512, 27600])
    assert 32 * s <= 148 and 32 * (s + 1) > 148
    assert nm.auto_kv_splits(0, [100]) == 1 and nm.auto_kv_splits(100, []) == 1


def test_sparse_tile_lists_keep_spans_whole_and_sample_candidates():
    from seeded_inputs import sparse_tile_lists

    lens = [1000, 37, 700]                 # 8 + 1 + 6 tiles, global ids 0-7, 8, 9-14
    lists, counts = sparse_tile_lists(600, lens, keep_spans=[1], candidate_spans=[0, 2],
                                      fraction=0.25, seed=3)
    assert lists.shape == (3, 16, 1 + 4) and counts.shape == (3, 16)   # round(0.25 * 14) = 4
    assert (counts == 5).all()
    seen = set()
    for b in range(3):
        for h in range(16):
            row = lists[b, h, :counts[b, h]].tolist()
            assert row == sorted(set(row))                 # sorted, no repeats
            assert 8 in row                                # the kept span's only tile
            assert all(0 <= g < 15 for g in row)
            picked = [g for g in row if g != 8]              # the sampled candidates
            assert len(picked) == 4 and all(g in range(0, 8) or g in range(9, 15) for g in picked)
            seen.add(tuple(row))
    assert len(seen) > 1                                   # blocks and heads differ
    again, _ = sparse_tile_lists(600, lens, [1], [0, 2], 0.25, seed=3)
    assert (again == lists).all()                          # seeded: reproducible
    other, _ = sparse_tile_lists(600, lens, [1], [0, 2], 0.25, seed=4)
    assert not (other == lists).all()


def test_sparse_tile_lists_pad_with_minus_one():
    from seeded_inputs import sparse_tile_lists

    lists, counts = sparse_tile_lists(100, [300], keep_spans=[], candidate_spans=[0],
                                      fraction=0.0, seed=1)
    assert (counts == 0).all() and (lists == -1).all() and lists.shape[-1] == 1


def test_owner_rows_partition_the_queries_on_16_row_steps():
    for n_q, world in ((28112, 8), (700, 3), (130, 4), (15, 2), (0, 3)):
        rows = nm.owner_rows(n_q, world)
        assert len(rows) == world + 1 and rows[0] == 0 and rows[-1] == n_q
        assert all(a <= b for a, b in zip(rows, rows[1:]))
        assert all(r % 16 == 0 for r in rows[:-1])
        # the same shares as the merge of owned rows uses
        for r in range(world):
            assert (rows[r], rows[r + 1]) == nm.shard_rows(n_q, r, world, align=16)


def test_auto_kv_splits_counts_the_heads_of_the_launch():
    # head-sharded launches: fewer heads, fewer CTAs, more splits pay off
    lens = [55200, 512, 27600]
    s16 = nm.auto_kv_splits(28112, lens, heads=16)
    s2 = nm.auto_kv_splits(28112, lens, heads=2)
    s1 = nm.auto_kv_splits(28112, lens, heads=1)
    assert s16 == 1 and s2 >= 2 and s1 >= s2
    # 110 query blocks x 1 head: the splits fill at least one wave of 148 SMs
    assert 110 * s1 >= 148


def test_head_sharded_attention_single_process_reshapes_back():
    # world 1 (no process group): the two all-to-alls are identities and the
    # head slicing round-trips; a reference attend checks what it is given
    import torch

    g = torch.Generator().manual_seed(3)
    q = torch.randn((13, 16, 128), generator=g, dtype=torch.float64)
    k = torch.randn((20, 16, 128), generator=g, dtype=torch.float64)
    v = torch.randn((20, 16, 128), generator=g, dtype=torch.float64)
    seen = {}

    def attend(qq, spans, lse_out):
        seen["shape"] = tuple(qq.shape)
        seen["keys"] = sum(a.shape[0] for a, _ in spans)
        lse_out.copy_(torch.arange(lse_out.numel(), dtype=torch.float32))
        return qq * 2.0  # per (row, head) and dims: any mix-up of rows or heads shows

    lse = torch.empty(16 * 13, dtype=torch.float32)
    o = nm.head_sharded_segment_attention(q, [(k[:7], v[:7]), (k[7:], v[7:])], attend=attend,
                                          lse=lse)
    assert seen == {"shape": (13, 16, 128), "keys": 20}
    assert torch.equal(o, q * 2.0)
    assert torch.equal(lse, torch.arange(16 * 13, dtype=torch.float32))
