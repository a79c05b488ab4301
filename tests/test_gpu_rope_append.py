"""Parity of the fused RoPE-3D + cache append kernel with the fp64 oracle."""
import numpy as np
import pytest
import torch

import kv_cached_segment_b200 as nm
import oracle
from seeded_inputs import WORKLOADS, randn_bf16
from tests._util import assert_bf16_rounding, assert_close, bits, f64

pytestmark = pytest.mark.gpu
CANARY = 0x7E57


def _positions(lay: nm.SegLayout):
    return oracle.video_positions(lay.frames, lay.grid_h, lay.grid_w, lay.t0)


def _run_append(frames, gh, gw, t0, n_text, cache_len, spare, cfg, seed):
    lay = nm.SegLayout(frames, gh, gw, t0, n_text)
    ns, nq = lay.n_video, lay.n_video + n_text
    q = randn_bf16((nq, 16, 128), seed)
    k = randn_bf16((ns, 16, 128), seed + 1)
    v = randn_bf16((ns, 16, 128), seed + 2)
    cap = cache_len + ns + spare
    ck = torch.full((cap, 16, 128), 0, dtype=torch.int16).fill_(CANARY).view(torch.bfloat16)
    cv = ck.clone()
    ck[:cache_len] = randn_bf16((cache_len, 16, 128), seed + 3)
    cv[:cache_len] = randn_bf16((cache_len, 16, 128), seed + 4)
    cache = nm.KVCache(ck.cuda(), cv.cuda(), cache_len, gh * gw)
    qd = q.cuda()
    q_out = torch.empty_like(qd)
    nm.kvcache_append(cache, k.cuda(), v.cuda(), q_in=qd, q_out=q_out, layout=lay, cfg=cfg)
    torch.cuda.synchronize()
    return lay, q, k, v, ck, cv, cache, q_out


@pytest.mark.parametrize("shape", [
    (2, 4, 6, 2, 64, 48, 7),       # tiny workload
    (8, 12, 20, 24, 256, 5760, 0),  # mid workload
    (3, 5, 7, 11, 37, 13, 129),     # ragged: odd grid, tail rows, spare capacity
    (1, 1, 1, 0, 0, 0, 0),          # a single token, empty cache, no text
])
def test_append_matches_oracle(shape):
    frames, gh, gw, t0, n_text, cache_len, spare = shape
    cfg = nm.RopeConfig()
    lay, q, k, v, ck, cv, cache, q_out = _run_append(frames, gh, gw, t0, n_text, cache_len,
                                                     spare, cfg, seed=100 + frames)
    ns = lay.n_video
    assert cache.len == cache_len + ns
    t, h, w = _positions(lay)
    split = (cfg.d_t, cfg.d_h, cfg.d_w)
    k_ref = oracle.rope3d(f64(k), ns, t, h, w, split, cfg.theta)
    q_ref = oracle.rope3d(f64(q), ns, t, h, w, split, cfg.theta)
    got_k = f64(cache.k[cache_len:cache_len + ns])
    assert_bf16_rounding(got_k, k_ref, "K'")
    assert_close(got_k, k_ref, what="K'")
    assert_bf16_rounding(f64(q_out[:ns]), q_ref[:ns], "Q' video rows")
    # text rows of Q are copied bit for bit; V rows are copied bit for bit
    assert np.array_equal(bits(q_out[ns:]), bits(q[ns:]))
    assert np.array_equal(bits(cache.v[cache_len:cache_len + ns]), bits(v))
    # rows outside [len, len + ns) are untouched (earlier cache and canaries)
    for dev, host in ((cache.k, ck), (cache.v, cv)):
        assert np.array_equal(bits(dev[:cache_len]), bits(host[:cache_len]))
        assert np.array_equal(bits(dev[cache_len + ns:]), bits(host[cache_len + ns:]))


def test_append_page_rope_variant():
    # The page's own split and base: 16/56/56, theta 256.
    cfg = nm.RopeConfig(16, 56, 56, 256.0)
    lay, q, k, v, ck, cv, cache, q_out = _run_append(4, 22, 40, 60, 16, 880, 0, cfg, seed=7)
    ns = lay.n_video
    t, h, w = _positions(lay)
    k_ref = oracle.rope3d(f64(k), ns, t, h, w, (16, 56, 56), 256.0)
    assert_bf16_rounding(f64(cache.k[880:880 + ns]), k_ref, "K' (16/56/56)")
    q_ref = oracle.rope3d(f64(q), ns, t, h, w, (16, 56, 56), 256.0)
    assert_bf16_rounding(f64(q_out), q_ref, "Q' (16/56/56)")


def test_append_plain_copy_without_rope():
    lay = nm.SegLayout(2, 3, 4, 0, 5)
    ns = lay.n_video
    k = randn_bf16((ns, 16, 128), 1).cuda()
    v = randn_bf16((ns, 16, 128), 2).cuda()
    cache = nm.KVCache.empty(ns + 3, 12)
    nm.kvcache_append(cache, k, v)  # no cfg: bit copy
    torch.cuda.synchronize()
    assert np.array_equal(bits(cache.k[:ns]), bits(k)) and np.array_equal(bits(cache.v[:ns]), bits(v))
    assert cache.len == ns


def test_append_capacity_error_leaves_cache_untouched():
    lay = nm.SegLayout(2, 2, 2, 0, 0)
    k = randn_bf16((8, 16, 128), 1).cuda()
    cache = nm.KVCache.empty(10, 4)
    cache.len = 4
    before = bits(cache.k)
    with pytest.raises(nm.NomasError) as e:
        nm.kvcache_append(cache, k, k.clone(), layout=lay, cfg=nm.RopeConfig())
    assert e.value.status == nm.NOMAS_ERR_CAPACITY
    torch.cuda.synchronize()
    assert cache.len == 4 and np.array_equal(bits(cache.k), before)


@pytest.mark.parametrize("inplace", [False, True])
def test_rope3d_qk_matches_oracle(inplace):
    lay = nm.SegLayout(5, 9, 11, 17, 33)
    n = lay.n_video + lay.n_text
    q = randn_bf16((n, 16, 128), 21)
    k = randn_bf16((n, 16, 128), 22)
    qd, kd = q.cuda(), k.cuda()
    if inplace:
        qo, ko = qd, kd
    else:
        qo, ko = torch.empty_like(qd), torch.empty_like(kd)
    cfg = nm.RopeConfig()
    nm.rope3d_qk(qd, kd, qo, ko, lay, cfg)
    torch.cuda.synchronize()
    t, h, w = _positions(lay)
    for got, src in ((qo, q), (ko, k)):
        ref = oracle.rope3d(f64(src), lay.n_video, t, h, w)
        assert_bf16_rounding(f64(got), ref, "rope3d_qk")
        assert np.array_equal(bits(got[lay.n_video:]), bits(src[lay.n_video:]))


def test_rope_deterministic():
    lay = nm.SegLayout(3, 8, 8, 4, 10)
    n = lay.n_video + lay.n_text
    q = randn_bf16((n, 16, 128), 3).cuda()
    outs = []
    for _ in range(2):
        o = torch.empty_like(q)
        nm.rope3d_qk(q, None, o, None, lay, nm.RopeConfig())
        outs.append(bits(o))
    assert np.array_equal(outs[0], outs[1])


@pytest.mark.slow
def test_append_720p_full_size():
    w = WORKLOADS["720p"]
    cfg = nm.RopeConfig()
    lay, q, k, v, ck, cv, cache, q_out = _run_append(w.frames, w.grid_h, w.grid_w, w.t0, w.n_text,
                                                     w.n_cache, 0, cfg, seed=3)
    ns = lay.n_video
    t, h, w_ = _positions(lay)
    rows = np.unique(np.concatenate([[0, ns - 1], np.random.default_rng(0).integers(0, ns, 2000)]))
    k_ref = oracle.rope3d(f64(k[rows]), rows.size, t[rows], h[rows], w_[rows])
    assert_bf16_rounding(f64(cache.k[w.n_cache + rows]), k_ref, "720p K'")
    assert np.array_equal(bits(cache.v[w.n_cache:]), bits(v))
    assert torch.equal(cache.k[:w.n_cache].cpu().view(torch.int16), ck[:w.n_cache].view(torch.int16))
