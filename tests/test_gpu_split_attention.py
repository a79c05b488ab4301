"""Key-split attention (partial results per key range, merged) against the oracle."""
import numpy as np
import pytest
import torch

import kv_cached_segment_b200 as nm
import oracle
from seeded_inputs import randn_bf16
from tests._util import assert_close, bits, f64

pytestmark = pytest.mark.gpu


def _inputs(n_q, lens, seed):
    q = randn_bf16((n_q, 16, 128), seed)
    spans = [(randn_bf16((n, 16, 128), seed * 10 + i), randn_bf16((n, 16, 128), seed * 10 + 5 + i))
             for i, n in enumerate(lens)]
    return q, spans


def _run(q, spans, splits, want_lse=True):
    qd = q.cuda()
    sd = [(k.cuda(), v.cuda()) for k, v in spans]
    lse = torch.empty(16 * q.shape[0], dtype=torch.float32, device="cuda") if want_lse else None
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    o = nm.segment_attention(qd, sd, lse=lse, dev_err=err, kv_splits=splits)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    return o, lse


@pytest.mark.parametrize("n_q,lens,splits", [
    (300, [1000], 2),
    (129, [128, 1, 255], 3),          # ragged spans: 1 + 1 + 2 tiles
    (513, [37, 300, 5, 128], 7),      # four spans
    (40, [200], 8),                   # more splits than tiles: six ranges are empty
    (256, [5000, 64, 900], nm.MAX_MERGE_PARTS),
])
def test_split_matches_oracle(n_q, lens, splits):
    q, spans = _inputs(n_q, lens, n_q + splits)
    o, lse = _run(q, spans, splits)
    o_ref, l_ref = oracle.attention(f64(q), [(f64(k), f64(v)) for k, v in spans])
    assert_close(f64(o), o_ref, what=f"split {splits} O")
    assert_close(lse.view(16, -1).cpu().numpy().astype(np.float64), l_ref, what=f"split {splits} LSE")


def test_split_without_lse_and_deterministic():
    q, spans = _inputs(200, [3000], 5)
    o1, _ = _run(q, spans, 5, want_lse=False)
    o2, _ = _run(q, spans, 5, want_lse=False)
    assert np.array_equal(bits(o1), bits(o2))
    o_ref, _ = oracle.attention(f64(q), [(f64(k), f64(v)) for k, v in spans])
    assert_close(f64(o1), o_ref, what="split 5 O without LSE")


def test_auto_split_on_a_small_query_set():
    # 2 query blocks over 40 key tiles: the heuristic splits the keys
    q, spans = _inputs(300, [4000, 64, 1000], 6)
    assert nm.auto_kv_splits(300, [4000, 64, 1000]) > 1
    o, lse = _run(q, spans, "auto")
    o_ref, l_ref = oracle.attention(f64(q), [(f64(k), f64(v)) for k, v in spans])
    assert_close(f64(o), o_ref, what="auto split O")
    assert_close(lse.view(16, -1).cpu().numpy().astype(np.float64), l_ref, what="auto split LSE")


def test_split_with_no_keys():
    q = randn_bf16((50, 16, 128), 7)
    empty = torch.empty((0, 16, 128), dtype=torch.bfloat16)
    o, lse = _run(q, [(empty, empty)], 4)
    assert torch.all(o == 0) and torch.all(torch.isneginf(lse))


@pytest.mark.slow
def test_short_layer_step_with_automatic_splits_sampled_rows():
    # The bench's short configuration (3.35 waves of query blocks, so the
    # automatic choice splits the keys), sampled rows against the oracle.
    from seeded_inputs import WORKLOADS, layer_inputs

    w = WORKLOADS["short"]
    inp = layer_inputs(w, seed=6)
    ns = w.n_seg
    lay = nm.SegLayout(w.frames, w.grid_h, w.grid_w, w.t0, w.n_text)
    cache = nm.KVCache.empty(w.n_cache + ns, w.tokens_per_frame)
    cache.k[:w.n_cache] = inp["cache_k"].cuda()
    cache.v[:w.n_cache] = inp["cache_v"].cuda()
    cache.len = w.n_cache
    q, k, v = inp["q"].cuda(), inp["k"].cuda(), inp["v"].cuda()
    q_rot = torch.empty_like(q)
    nm.kvcache_append(cache, k[:ns], v[:ns], q_in=q, q_out=q_rot, layout=lay, cfg=nm.RopeConfig())
    spans = [cache.span(0, w.n_cache), (k[ns:], v[ns:]), cache.span(w.n_cache, w.n_cache + ns)]
    assert nm.auto_kv_splits(w.n_q, [w.n_cache, w.n_text, ns]) > 1
    lse = torch.empty(16 * w.n_q, dtype=torch.float32, device="cuda")
    o = nm.segment_attention(q_rot, spans, lse=lse, kv_splits="auto")
    torch.cuda.synchronize()
    t, h, ww = oracle.video_positions(w.frames, w.grid_h, w.grid_w, w.t0)
    qf = oracle.rope3d(f64(inp["q"]), ns, t, h, ww)
    kf = oracle.rope3d(f64(inp["k"][:ns]), ns, t, h, ww)
    rows = np.unique(np.concatenate([np.random.default_rng(2).integers(0, w.n_q, 40),
                                     [0, ns - 1, ns, w.n_q - 1]]))
    o_ref, l_ref = oracle.attention_rows(
        qf, rows, [(f64(inp["cache_k"]), f64(inp["cache_v"])),
                   (f64(inp["k"][ns:]), f64(inp["v"][ns:])), (kf, f64(inp["v"][:ns]))])
    assert_close(f64(o[torch.as_tensor(rows)]), o_ref, what="short, split keys, O")
    got_l = lse.view(16, -1)[:, torch.as_tensor(rows).cuda()].cpu().numpy().astype(np.float64)
    assert_close(got_l, l_ref, what="short, split keys, LSE")
