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
