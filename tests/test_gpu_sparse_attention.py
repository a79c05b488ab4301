"""Block-sparse segment attention against the oracle."""
import numpy as np
import pytest
import torch

import kv_cached_segment_b200 as nm
import oracle
from seeded_inputs import randn_bf16, sparse_tile_lists
from tests._util import assert_close, f64

pytestmark = pytest.mark.gpu


def _run(q, spans, lists, counts):
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    lse = torch.empty(16 * q.shape[0], dtype=torch.float32, device="cuda")
    o = nm.segment_attention_sparse(q.cuda(), [(k.cuda(), v.cuda()) for k, v in spans],
                                    torch.from_numpy(lists).cuda(), torch.from_numpy(counts).cuda(),
                                    lse=lse, dev_err=err)
    torch.cuda.synchronize()
    return o, lse, int(err.item())


def _oracle(q, spans, lists, counts):
    tl = [[lists[b, h, :counts[b, h]].tolist() for h in range(16)] for b in range(lists.shape[0])]
    return oracle.block_sparse_attention(f64(q), [(f64(k), f64(v)) for k, v in spans], tl)


def _spans(lens, seed):
    return [(randn_bf16((n, 16, 128), seed + i), randn_bf16((n, 16, 128), seed + 50 + i))
            for i, n in enumerate(lens)]


@pytest.mark.parametrize("n_q,lens,frac", [(300, [700, 64, 300], 0.25), (513, [1000, 33], 0.5),
                                           (100, [129, 128, 1], 0.34)])
def test_sparse_matches_oracle(n_q, lens, frac):
    q = randn_bf16((n_q, 16, 128), n_q)
    spans = _spans(lens, 7)
    # keep the text-like and segment-like spans whole, sample the history
    lists, counts = sparse_tile_lists(n_q, lens, keep_spans=range(1, len(lens)),
                                      candidate_spans=[0], fraction=frac, seed=n_q)
    o, lse, err = _run(q, spans, lists, counts)
    assert err == 0
    o_ref, l_ref = _oracle(q, spans, lists, counts)
    assert_close(f64(o), o_ref, what="sparse O")
    assert_close(lse.view(16, -1).cpu().numpy().astype(np.float64), l_ref, what="sparse LSE")


def test_every_tile_listed_equals_dense_bit_for_bit():
    q = randn_bf16((600, 16, 128), 3)
    lens = [500, 77, 300]
    spans = _spans(lens, 11)
    lists, counts = sparse_tile_lists(600, lens, keep_spans=[0, 1, 2], candidate_spans=[],
                                      fraction=0.0, seed=0)
    o, lse, err = _run(q, spans, lists, counts)
    dense_lse = torch.empty_like(lse)
    dense = nm.segment_attention(q.cuda(), [(k.cuda(), v.cuda()) for k, v in spans], lse=dense_lse)
    torch.cuda.synchronize()
    assert err == 0
    assert torch.equal(o.view(torch.int16), dense.view(torch.int16))
    assert torch.equal(lse, dense_lse)


def test_invalid_ids_skipped_empty_blocks_and_duplicates():
    q = randn_bf16((700, 16, 128), 4)
    lens = [400, 100]
    spans = _spans(lens, 21)  # tiles: span 0 -> 0..3, span 1 -> 4
    lists = np.full((3, 16, 6), -1, dtype=np.int32)
    counts = np.zeros((3, 16), dtype=np.int32)
    lists[0, :, :4] = [0, -7, 4, 99]        # two invalid ids
    counts[0] = 4
    lists[1, :, :3] = [2, 2, 4]             # a duplicate tile counts twice
    counts[1] = 3
    counts[2, :8] = 0                        # empty for half the heads of block 2
    lists[2, 8:, :1] = 1
    counts[2, 8:] = 1
    o, lse, err = _run(q, spans, lists, counts)
    assert err == nm.DEVERR_BAD_TILE_INDEX
    o_ref, l_ref = _oracle(q, spans, lists, counts)
    got_l = lse.view(16, -1).cpu().numpy().astype(np.float64)
    fin = np.isfinite(l_ref)
    assert np.array_equal(np.isfinite(got_l), fin)
    assert_close(f64(o), o_ref, what="sparse O (edge cases)")
    assert np.allclose(got_l[fin], l_ref[fin], atol=2e-2)
    assert torch.all(o[512:, :8] == 0)


def test_sparse_deterministic():
    q = randn_bf16((512, 16, 128), 5)
    lens = [1200, 256]
    spans = _spans(lens, 31)
    lists, counts = sparse_tile_lists(512, lens, [1], [0], 0.25, seed=9)
    o1, l1, _ = _run(q, spans, lists, counts)
    o2, l2, _ = _run(q, spans, lists, counts)
    assert torch.equal(o1.view(torch.int16), o2.view(torch.int16)) and torch.equal(l1, l2)


@pytest.mark.slow
def test_sparse_720p_layer_step_sampled_blocks():
    # The bench's block-sparse configuration at full size: the 720p
    # layer-step (RoPE + append on the GPU), every text tile and a seeded 25%
    # of the history and segment tiles per 256-query block and head.  Three
    # query blocks are checked against the oracle, each as its own one-block
    # problem (its 256 rows with its own tile lists).
    from seeded_inputs import WORKLOADS, layer_inputs

    w = WORKLOADS["720p"]
    inp = layer_inputs(w, seed=5)
    ns = w.n_seg
    lay = nm.SegLayout(w.frames, w.grid_h, w.grid_w, w.t0, w.n_text)
    cache = nm.KVCache.empty(w.n_cache + ns, w.tokens_per_frame)
    cache.k[:w.n_cache] = inp["cache_k"].cuda()
    cache.v[:w.n_cache] = inp["cache_v"].cuda()
    cache.len = w.n_cache
    q, k, v = inp["q"].cuda(), inp["k"].cuda(), inp["v"].cuda()
    q_rot = torch.empty_like(q)
    nm.kvcache_append(cache, k[:ns], v[:ns], q_in=q, q_out=q_rot, layout=lay, cfg=nm.RopeConfig())
    lens = [w.n_cache, w.n_text, ns]
    lists, counts = sparse_tile_lists(w.n_q, lens, keep_spans=[1], candidate_spans=[0, 2],
                                      fraction=0.25, seed=5)
    spans = [cache.span(0, w.n_cache), (k[ns:], v[ns:]), cache.span(w.n_cache, w.n_cache + ns)]
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    lse = torch.empty(16 * w.n_q, dtype=torch.float32, device="cuda")
    o = nm.segment_attention_sparse(q_rot, spans, torch.from_numpy(lists).cuda(),
                                    torch.from_numpy(counts).cuda(), lse=lse, dev_err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0

    t, h, ww = oracle.video_positions(w.frames, w.grid_h, w.grid_w, w.t0)
    qf = oracle.rope3d(f64(inp["q"]), ns, t, h, ww)
    kf = oracle.rope3d(f64(inp["k"][:ns]), ns, t, h, ww)
    spans_f = [(f64(inp["cache_k"]), f64(inp["cache_v"])),
               (f64(inp["k"][ns:]), f64(inp["v"][ns:])), (kf, f64(inp["v"][:ns]))]
    lse_g = lse.view(16, -1).cpu().numpy().astype(np.float64)
    last = lists.shape[0] - 1
    for b in (0, 57, last):      # first, middle (video rows) and last (text rows) blocks
        rows = np.arange(b * 256, min(w.n_q, (b + 1) * 256))
        tl = [[lists[b, hh, :counts[b, hh]].tolist() for hh in range(16)]]
        o_ref, l_ref = oracle.block_sparse_attention(qf[rows], spans_f, tl)
        assert_close(f64(o[torch.as_tensor(rows)]), o_ref, what=f"720p sparse block {b} O")
        assert_close(lse_g[:, rows], l_ref, what=f"720p sparse block {b} LSE")
