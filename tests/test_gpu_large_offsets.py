"""Maximum-size edge cases: every kernel addresses rows beyond 4 GiB.

A row of Q, K, V or the cache is 4 KiB, so past 1,048,576 rows a byte offset
no longer fits 32 bits (past 2,097,152 rows for INT8 codes).  Each test puts
the data that decides the result beyond that point and takes the expected
values from the inputs themselves or from the oracle on a few rows.  About
9-10 GB of device memory per test.
"""
import math

import numpy as np
import pytest
import torch

import kv_cached_segment_b200 as nm
import oracle
from seeded_inputs import randn_bf16
from tests._util import assert_bf16_rounding, bits, f64

pytestmark = pytest.mark.gpu

FAR_ROWS = 1_100_000          # 4.5 GB per bf16 tensor of rows
FAR_ROWS_I8 = 2_200_000       # 4.5 GB per INT8 code tensor


def _seeded_rows(n, seed):
    """n seeded N(0,1) bf16 rows, made on the host and copied to the device."""
    return randn_bf16((n, 16, 128), seed).cuda()


def test_attention_one_hot_key_beyond_4gib():
    # q = 1 everywhere and one key of 8s: its logit is 128 * 8 / sqrt(128) =
    # 90.5 above the zero logits of every other key, so each output row is
    # that key's V row (weight 1 - 1.1e6 * e^-90.5) and LSE is its logit.
    n_q, far = 300, FAR_ROWS - 5
    q = torch.ones((n_q, 16, 128), dtype=torch.bfloat16, device="cuda")
    k = torch.zeros((FAR_ROWS, 16, 128), dtype=torch.bfloat16, device="cuda")
    v = torch.zeros_like(k)
    k[far] = 8.0
    v[far] = _seeded_rows(1, 71)[0]
    tail_k = torch.zeros((77, 16, 128), dtype=torch.bfloat16, device="cuda")
    tail_v = _seeded_rows(77, 72)
    lse = torch.empty(16 * n_q, dtype=torch.float32, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    o = nm.segment_attention(q, [(k, v), (tail_k, tail_v)], lse=lse, dev_err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    want = bits(v[far : far + 1])
    assert np.array_equal(bits(o), np.broadcast_to(want, (n_q, 16, 128)))
    logit = 128 * 8.0 / math.sqrt(128.0)
    assert np.allclose(lse.cpu().numpy(), logit, atol=1e-4)


def test_append_beyond_4gib():
    # 100 segment tokens rotated and appended at row FAR_ROWS - 100 of the
    # cache; the row before them (a canary) stays as it was.
    lay = nm.SegLayout(2, 5, 10, 1195, 0)
    ns = lay.n_video
    cache = nm.KVCache.empty(FAR_ROWS, 920)
    start = FAR_ROWS - ns
    cache.k[start - 1] = 3.0
    cache.v[start - 1] = -3.0
    cache.len = start
    k = randn_bf16((ns, 16, 128), 73)
    v = randn_bf16((ns, 16, 128), 74)
    nm.kvcache_append(cache, k.cuda(), v.cuda(), layout=lay, cfg=nm.RopeConfig())
    torch.cuda.synchronize()
    assert cache.len == FAR_ROWS
    t, h, w = oracle.video_positions(lay.frames, lay.grid_h, lay.grid_w, lay.t0)
    assert_bf16_rounding(f64(cache.k[start:]), oracle.rope3d(f64(k), ns, t, h, w), what="K'")
    assert np.array_equal(bits(cache.v[start:]), bits(v))
    assert torch.all(cache.k[start - 1] == 3.0) and torch.all(cache.v[start - 1] == -3.0)


def test_select_frames_beyond_4gib():
    # Frames at the far end of a 1,195-frame cache (P = 920) are gathered bit
    # for bit, in list order, with a near frame between them.
    tpf = 920
    n_frames = FAR_ROWS // tpf
    cache = nm.KVCache.empty(n_frames * tpf, tpf)
    cache.len = n_frames * tpf
    picks = [n_frames - 1, 3, n_frames - 5]
    for i, f in enumerate(picks):
        cache.k[f * tpf : (f + 1) * tpf] = _seeded_rows(tpf, 80 + i)
        cache.v[f * tpf : (f + 1) * tpf] = _seeded_rows(tpf, 90 + i)
    window = nm.KVCache.empty(len(picks) * tpf, 0)
    nm.kvcache_select(cache, picks, window)
    torch.cuda.synchronize()
    assert window.len == len(picks) * tpf
    for i, f in enumerate(picks):
        rows = slice(i * tpf, (i + 1) * tpf)
        assert np.array_equal(bits(window.k[rows]), bits(cache.k[f * tpf : (f + 1) * tpf]))
        assert np.array_equal(bits(window.v[rows]), bits(cache.v[f * tpf : (f + 1) * tpf]))


def test_int8_append_and_select_beyond_4gib():
    # INT8 codes are 2 KiB per row: 2.2 M rows put the appended rows beyond
    # 4 GiB.  Codes and scales equal the oracle's; the gather dequantises
    # them bit for bit.
    n = 64
    cache = nm.KVCacheI8.empty(FAR_ROWS_I8, 32)
    start = FAR_ROWS_I8 - n
    cache.len = start
    k = randn_bf16((n, 16, 128), 75) * 2
    v = randn_bf16((n, 16, 128), 76)
    k = k.to(torch.bfloat16)
    nm.kvcache_append_i8(cache, k.cuda(), v.cuda())
    torch.cuda.synchronize()
    for codes, scales, src in ((cache.k, cache.k_scale, k), (cache.v, cache.v_scale, v)):
        want_c, want_s = oracle.quantize_int8(bits(src))
        assert np.array_equal(codes[start:].cpu().numpy(), want_c)
        assert np.array_equal(scales[start:].cpu().numpy().view(np.uint32), want_s.view(np.uint32))
    last = FAR_ROWS_I8 // 32 - 1            # the frame holding the appended rows
    window = nm.KVCache.empty(2 * 32, 0)
    nm.kvcache_select(cache, [last, last], window)
    torch.cuda.synchronize()
    kc = cache.k[last * 32 :].cpu().numpy()
    ks = cache.k_scale[last * 32 :].cpu().numpy()
    want = oracle.dequantize_int8(kc, ks)
    assert np.array_equal(bits(window.k[:32]), want)
    assert np.array_equal(bits(window.k[32:]), want)
