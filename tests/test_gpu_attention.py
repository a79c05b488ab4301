"""Parity of the tcgen05 segment attention kernel with the fp64 oracle."""
import math

import numpy as np
import pytest
import torch

import kv_cached_segment_b200 as nm
import oracle
from seeded_inputs import WORKLOADS, bounded_frame_list, layer_inputs, randn_bf16
from tests._util import assert_close, f64

pytestmark = pytest.mark.gpu


# Every test runs under each kernel schedule (same results expected).
@pytest.fixture(autouse=True, params=[nm.PIPELINE_TWO_TILE, nm.PIPELINE_ONE_TILE, nm.PIPELINE_PAIR],
                ids=["two_tile", "one_tile", "pair"])
def pipeline(request):
    nm.set_attention_pipeline(request.param)
    yield request.param
    nm.set_attention_pipeline(0)


def _attn(q, spans, scale=0.0, want_lse=True):
    qd = q.cuda()
    sd = [(k.cuda(), v.cuda()) for k, v in spans]
    lse = torch.empty(q.shape[1] * q.shape[0], dtype=torch.float32, device="cuda") if want_lse else None
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    o = nm.segment_attention(qd, sd, lse=lse, softmax_scale=scale, dev_err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    return o, lse


def _check(q, spans, scale=None, rows=None, what=""):
    o, lse = _attn(q, spans, 0.0 if scale is None else scale)
    fs = [(f64(k), f64(v)) for k, v in spans]
    if rows is None:
        o_ref, l_ref = oracle.attention(f64(q), fs, scale)
        got_o, got_l = f64(o), lse.view(16, -1).cpu().numpy().astype(np.float64)
    else:
        o_ref, l_ref = oracle.attention_rows(f64(q), rows, fs, scale)
        got_o = f64(o[torch.as_tensor(rows)])
        got_l = lse.view(16, -1)[:, torch.as_tensor(rows).cuda()].cpu().numpy().astype(np.float64)
    assert_close(got_o, o_ref, what=f"{what} O")
    assert_close(got_l, l_ref, what=f"{what} LSE")
    return o


@pytest.mark.parametrize("n_q,lens", [
    (112, [48, 64, 48]),          # tiny shapes
    (1, [1]),                     # one query, one key
    (127, [129]),                 # one-row tails on both sides
    (129, [128, 1, 255]),
    (256, [37, 300, 5, 128]),     # four spans with ragged tails
    (300, [1000]),
    (513, [0, 200, 0, 77]),       # empty spans are skipped
])
def test_attention_ragged_shapes(n_q, lens):
    q = randn_bf16((n_q, 16, 128), n_q)
    spans = [(randn_bf16((n, 16, 128), 1000 + i), randn_bf16((n, 16, 128), 2000 + i))
             for i, n in enumerate(lens)]
    _check(q, spans, what=f"n_q={n_q} lens={lens}")


def test_attention_custom_scale():
    q = randn_bf16((200, 16, 128), 1)
    spans = [(randn_bf16((333, 16, 128), 2), randn_bf16((333, 16, 128), 3))]
    _check(q, spans, scale=0.2, what="scale 0.2")


def test_attention_growing_scores_force_rescale():
    # Later spans have much larger logits, so the running max must be raised
    # (and O rescaled) several times along the key sequence.
    q = randn_bf16((256, 16, 128), 4)
    spans = []
    for i, mag in enumerate((0.25, 1.0, 3.0, 6.0)):
        k = (randn_bf16((200, 16, 128), 10 + i).float() * mag).to(torch.bfloat16)
        spans.append((k, randn_bf16((200, 16, 128), 20 + i)))
    _check(q, spans, what="growing logits")


def test_attention_shrinking_scores():
    q = randn_bf16((130, 16, 128), 5)
    spans = []
    for i, mag in enumerate((6.0, 1.0, 0.1)):
        k = (randn_bf16((150, 16, 128), 30 + i).float() * mag).to(torch.bfloat16)
        spans.append((k, randn_bf16((150, 16, 128), 40 + i)))
    _check(q, spans, what="shrinking logits")


def test_attention_zero_query_gives_mean_of_v():
    q = torch.zeros((130, 16, 128), dtype=torch.bfloat16)
    k = randn_bf16((333, 16, 128), 6)
    v = randn_bf16((333, 16, 128), 7)
    o, lse = _attn(q, [(k, v)])
    mean_v = f64(v).mean(axis=0)
    assert_close(f64(o), np.broadcast_to(mean_v, (130, 16, 128)), what="q=0")
    assert np.allclose(lse.cpu().numpy(), math.log(333), atol=1e-4)


def test_attention_no_keys():
    q = randn_bf16((40, 16, 128), 8)
    empty = torch.empty((0, 16, 128), dtype=torch.bfloat16)
    o, lse = _attn(q, [(empty, empty)])
    assert torch.all(o == 0) and torch.all(torch.isneginf(lse))


def test_attention_deterministic():
    q = randn_bf16((600, 16, 128), 9)
    spans = [(randn_bf16((900, 16, 128), 11), randn_bf16((900, 16, 128), 12))]
    o1, l1 = _attn(q, spans)
    o2, l2 = _attn(q, spans)
    assert torch.equal(o1.view(torch.int16), o2.view(torch.int16))
    assert torch.equal(l1, l2)


def _layer_step(w, seed, select=False):
    """Append (fused RoPE) + attention through the C ABI, as one layer-step."""
    inp = layer_inputs(w, seed)
    ns, nt = w.n_seg, w.n_text
    lay = nm.SegLayout(w.frames, w.grid_h, w.grid_w, w.t0, nt)
    cfg = nm.RopeConfig()
    cache = nm.KVCache.empty(w.n_cache + ns, w.tokens_per_frame)
    cache.k[:w.n_cache] = inp["cache_k"].cuda()
    cache.v[:w.n_cache] = inp["cache_v"].cuda()
    cache.len = w.n_cache
    q = inp["q"].cuda()
    k = inp["k"].cuda()
    v = inp["v"].cuda()
    q_rot = torch.empty_like(q)
    nm.kvcache_append(cache, k[:ns], v[:ns], q_in=q, q_out=q_rot, layout=lay, cfg=cfg)
    if select:
        idx = bounded_frame_list(w, seed)
        window = nm.KVCache.empty(idx.size * w.tokens_per_frame, 0)
        nm.kvcache_select(cache, idx.tolist(), window)
        hist = window.span()
    else:
        idx = None
        hist = cache.span(0, w.n_cache)
    spans = [hist, (k[ns:], v[ns:]), cache.span(w.n_cache, w.n_cache + ns)]
    lse = torch.empty(16 * w.n_q, dtype=torch.float32, device="cuda")
    o = nm.segment_attention(q_rot, spans, lse=lse)
    torch.cuda.synchronize()
    return inp, idx, o, lse


def _oracle_step(w, inp, idx, rows=None):
    ns = w.n_seg
    t, h, ww = oracle.video_positions(w.frames, w.grid_h, w.grid_w, w.t0)
    qf = oracle.rope3d(f64(inp["q"]), ns, t, h, ww)
    kf = oracle.rope3d(f64(inp["k"][:ns]), ns, t, h, ww)
    ck, cv = f64(inp["cache_k"]), f64(inp["cache_v"])
    if idx is not None:
        ck = oracle.kvcache_select(ck, idx, w.tokens_per_frame)
        cv = oracle.kvcache_select(cv, idx, w.tokens_per_frame)
    spans = [(ck, cv), (f64(inp["k"][ns:]), f64(inp["v"][ns:])), (kf, f64(inp["v"][:ns]))]
    if rows is None:
        return oracle.attention(qf, spans)
    return oracle.attention_rows(qf, rows, spans)


@pytest.mark.parametrize("name", ["tiny", "mid"])
def test_layer_step_matches_oracle(name):
    w = WORKLOADS[name]
    inp, idx, o, lse = _layer_step(w, seed=1)
    o_ref, l_ref = _oracle_step(w, inp, idx)
    assert_close(f64(o), o_ref, what=f"{name} O")
    assert_close(lse.view(16, -1).cpu().numpy().astype(np.float64), l_ref, what=f"{name} LSE")


def _sample_rows(w, n=48, seed=0):
    r = np.random.default_rng(seed).integers(0, w.n_q, n)
    return np.unique(np.concatenate([r, [0, w.n_seg - 1, w.n_seg, w.n_q - 1]]))


@pytest.mark.slow
def test_layer_step_720p_sampled_rows():
    w = WORKLOADS["720p"]
    inp, idx, o, lse = _layer_step(w, seed=2)
    rows = _sample_rows(w)
    o_ref, l_ref = _oracle_step(w, inp, idx, rows)
    assert_close(f64(o[torch.as_tensor(rows)]), o_ref, what="720p O")
    got_l = lse.view(16, -1)[:, torch.as_tensor(rows).cuda()].cpu().numpy().astype(np.float64)
    assert_close(got_l, l_ref, what="720p LSE")
    # rows are independent: the full output must be finite everywhere
    assert torch.isfinite(o.float()).all()


@pytest.mark.slow
@pytest.mark.parametrize("name", ["bounded", "bounded90"])
def test_layer_step_bounded_sampled_rows(name):
    w = WORKLOADS[name]
    inp, idx, o, lse = _layer_step(w, seed=3, select=True)
    rows = _sample_rows(w, seed=1)
    o_ref, l_ref = _oracle_step(w, inp, idx, rows)
    assert_close(f64(o[torch.as_tensor(rows)]), o_ref, what=f"{name} O")
    got_l = lse.view(16, -1)[:, torch.as_tensor(rows).cuda()].cpu().numpy().astype(np.float64)
    assert_close(got_l, l_ref, what=f"{name} LSE")


def test_wait_timeout_is_reported_and_context_survives():
    # The producer leaves out one K/V load, so a consumer wait can never
    # complete: the kernel must give up after its (short) limit, report
    # NOMAS_DEVERR_WAIT_TIMEOUT and leave the context usable.
    q = randn_bf16((112, 16, 128), 1)
    spans = [(randn_bf16((48, 16, 128), 2), randn_bf16((48, 16, 128), 3)),
             (randn_bf16((64, 16, 128), 4), randn_bf16((64, 16, 128), 5)),
             (randn_bf16((48, 16, 128), 6), randn_bf16((48, 16, 128), 7))]
    sd = [(k.cuda(), v.cuda()) for k, v in spans]
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    o = torch.full((112, 16, 128), 7.0, dtype=torch.bfloat16, device="cuda")
    lse = torch.full((16 * 112,), 7.0, dtype=torch.float32, device="cuda")
    nm.segment_attention(q.cuda(), sd, o=o, lse=lse, dev_err=err, wait_limit_ns=50_000_000,
                         testing_skip_kv_load=3)
    torch.cuda.synchronize()
    assert int(err.item()) == nm.DEVERR_WAIT_TIMEOUT
    # every block leaves out its fourth load and aborts: its rows are NaN, so
    # nothing earlier in the buffers can pass for a result
    assert torch.all(torch.isnan(o)) and torch.all(torch.isnan(lse))
    # the same context still computes correct results
    _check(q, spans, what="after timeout")


@pytest.mark.parametrize("col", [2, 5, 17, 64, 66])
@pytest.mark.parametrize("spike", [100.0, 300.0])
def test_attention_logit_spike_in_later_tile(col, spike):
    # One key, in the second 128-key tile, scores `spike` (natural-log units)
    # above the others, so the softmax is that key's V row.  Its column lands
    # on exponentials computed on either pipe and in either half of the tile:
    # a running max that is not raised in time would overflow there.
    n_k = 400
    q = torch.ones((64, 16, 128), dtype=torch.bfloat16)
    k = randn_bf16((n_k, 16, 128), 50)
    k[128 + col] = spike / math.sqrt(128.0)
    v = randn_bf16((n_k, 16, 128), 51)
    o = _check(q, [(k, v)], what=f"spike {spike} at column {col}")
    assert_close(f64(o), np.broadcast_to(f64(v[128 + col]), (64, 16, 128)), what="spike row")


@pytest.mark.parametrize("heads", [1, 2, 4, 8])
def test_attention_fewer_heads_matches_oracle_and_full_run(heads):
    # Rows of 1, 2, 4 or 8 heads: the local heads of head-sharded attention.
    # Each head is computed alone, so the result equals the 16-head run's
    # heads bit for bit, and the oracle within the bar.
    n_q, lens = 300, [200, 37, 129]
    q = randn_bf16((n_q, 16, 128), 70 + heads)
    spans = [(randn_bf16((n, 16, 128), 80 + i), randn_bf16((n, 16, 128), 90 + i))
             for i, n in enumerate(lens)]
    o16, l16 = _attn(q, spans)
    h0 = 16 - heads  # the last heads of the row
    qs = q[:, h0:].contiguous()
    ss = [(k[:, h0:].contiguous(), v[:, h0:].contiguous()) for k, v in spans]
    o, lse = _attn(qs, ss)
    assert torch.equal(o, o16[:, h0:].contiguous())
    assert torch.equal(lse.view(heads, n_q), l16.view(16, n_q)[h0:])
    o_ref, l_ref = oracle.attention(f64(qs), [(f64(k), f64(v)) for k, v in ss])
    assert_close(f64(o), o_ref, what=f"{heads} heads O")
    assert_close(lse.view(heads, -1).cpu().numpy().astype(np.float64), l_ref, what=f"{heads} heads LSE")
    # key splits and their merge at the same head count: the 16-head split's heads
    qd, sd = q.cuda(), [(k.cuda(), v.cuda()) for k, v in spans]
    l16s = torch.empty(16 * n_q, dtype=torch.float32, device="cuda")
    o16s = nm.segment_attention(qd, sd, lse=l16s, kv_splits=3)
    ls = torch.empty(heads * n_q, dtype=torch.float32, device="cuda")
    os_ = nm.segment_attention(qs.cuda(), [(k.cuda(), v.cuda()) for k, v in ss], lse=ls, kv_splits=3)
    torch.cuda.synchronize()
    assert torch.equal(os_, o16s[:, h0:].contiguous())
    assert torch.equal(ls.view(heads, n_q), l16s.view(16, n_q)[h0:])
    assert_close(f64(os_), o_ref, what=f"{heads} heads, 3 key splits O")


def test_head_sharded_single_rank_is_plain_attention():
    q = randn_bf16((257, 16, 128), 5).cuda()
    k, v = randn_bf16((300, 16, 128), 6).cuda(), randn_bf16((300, 16, 128), 7).cuda()
    lse = torch.empty(16 * 257, dtype=torch.float32, device="cuda")
    o = nm.head_sharded_segment_attention(q, [(k[:100], v[:100]), (k[100:], v[100:])], lse=lse)
    o_ref, l_ref = _attn(q.cpu(), [(k.cpu(), v.cpu())])
    torch.cuda.synchronize()
    assert torch.equal(o, o_ref) and torch.equal(lse, l_ref)
