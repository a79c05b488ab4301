"""INT8 KV cache: quantising append and dequantising gather against the oracle."""
import numpy as np
import pytest
import torch

import kv_cached_segment_b200 as nm
import oracle
from seeded_inputs import WORKLOADS, random_frame_list, randn_bf16
from tests._util import assert_close, bits, f64

pytestmark = pytest.mark.gpu


def _codes(t):
    return t.detach().cpu().numpy()


def test_append_plain_quantisation_is_bit_exact():
    # No rotation: K and V are quantised straight from the seeded bf16 input,
    # so codes and scales must equal the oracle's bit for bit.
    n = 300
    k = randn_bf16((n, 16, 128), 1) * 3
    v = randn_bf16((n, 16, 128), 2)
    k[5, 3] = 0  # an all-zero head
    cache = nm.KVCacheI8.empty(n + 10, 20)
    cache.len = 7
    nm.kvcache_append_i8(cache, k.to(torch.bfloat16).cuda(), v.cuda())
    torch.cuda.synchronize()
    assert cache.len == 7 + n
    near_ties = 0
    for codes, scales, src in ((cache.k, cache.k_scale, k), (cache.v, cache.v_scale, v)):
        want_c, want_s = oracle.quantize_int8(bits(src.to(torch.bfloat16)))
        assert np.array_equal(_codes(codes[7:7 + n]), want_c)
        assert np.array_equal(scales[7:7 + n].cpu().numpy().view(np.uint32), want_s.view(np.uint32))
        near_ties += _fp32_reciprocal_route_misses(src, want_c)
    # the sample holds quotients near half-integers, where x * fl(127 / a)
    # in float32 alone would give the wrong code
    print(f"codes the float32 reciprocal route would miss: {near_ties}")
    assert near_ties > 0


def _fp32_reciprocal_route_misses(src, want_codes):
    x = f64(src.to(torch.bfloat16)).astype(np.float32)
    a = np.max(np.abs(x), axis=2)
    inv = (np.float32(127.0) / np.where(a == 0, np.float32(1), a)).astype(np.float32)
    route = np.rint((x * inv[:, :, None]).astype(np.float32))
    return int(np.count_nonzero(route != want_codes))


def test_append_hand_ties():
    # a = 127 per head: codes are x rounded half to even; a = 2: a / 2 -> 64.
    x = torch.zeros((3, 16, 128))
    x[0, :, :8] = torch.tensor([127.0, 0.5, 1.5, 2.5, -2.5, 126.5, 3.25, -127.0])
    x[1, :, :3] = torch.tensor([1.0, -2.0, -1.0])
    x[2, :, 0] = 2.0 ** -130  # absmax so small that 127 / a overflows float32
    xb = x.to(torch.bfloat16)
    cache = nm.KVCacheI8.empty(3, 1)
    nm.kvcache_append_i8(cache, xb.cuda(), xb.cuda())
    torch.cuda.synchronize()
    got = _codes(cache.k)
    assert got[0, :, :8].tolist() == [[127, 0, 2, 2, -2, 126, 3, -127]] * 16
    assert got[1, :, :3].tolist() == [[64, -127, -64]] * 16
    assert np.all(got[2, :, 0] == 127) and np.all(got[2, :, 1:] == 0)
    want_c, want_s = oracle.quantize_int8(bits(xb))
    assert np.array_equal(got, want_c) and np.array_equal(_codes(cache.v), want_c)
    assert np.array_equal(cache.k_scale.cpu().numpy().view(np.uint32), want_s.view(np.uint32))


def test_append_rotated_keys_within_quantisation_error():
    lay = nm.SegLayout(4, 9, 11, 20, 40)
    ns = lay.n_video
    q = randn_bf16((ns + 40, 16, 128), 3)
    k = randn_bf16((ns, 16, 128), 4)
    v = randn_bf16((ns, 16, 128), 5)
    cache = nm.KVCacheI8.empty(ns, 99)
    q_out = torch.empty_like(q.cuda())
    nm.kvcache_append_i8(cache, k.cuda(), v.cuda(), q_in=q.cuda(), q_out=q_out, layout=lay,
                         cfg=nm.RopeConfig())
    torch.cuda.synchronize()
    t, h, w = oracle.video_positions(lay.frames, lay.grid_h, lay.grid_w, lay.t0)
    k_ref = oracle.rope3d(f64(k), ns, t, h, w)
    scales = cache.k_scale.cpu().numpy().astype(np.float64)
    k_hat = _codes(cache.k).astype(np.float64) * scales[:, :, None]
    # half a quantisation step, plus the bf16 rounding of the rotated key
    bound = 0.5 * scales[:, :, None] * (1 + 1e-6) + np.abs(k_ref) * 2.0 ** -7 + 1e-6
    assert np.all(np.abs(k_hat - k_ref) <= bound)
    want_c, want_s = oracle.quantize_int8(bits(v))
    assert np.array_equal(_codes(cache.v), want_c)
    assert np.array_equal(cache.v_scale.cpu().numpy().view(np.uint32), want_s.view(np.uint32))
    assert_close(f64(q_out[:ns]), oracle.rope3d(f64(q), ns, t, h, w)[:ns], what="Q'")
    # text rows of Q are not rotated: copied bit for bit
    assert np.array_equal(bits(q_out[ns:]), bits(q[ns:]))


def _i8_source(n_frames, tpf, seed):
    g = torch.Generator().manual_seed(seed)
    rows = n_frames * tpf
    kc = torch.randint(-127, 128, (rows, 16, 128), generator=g, dtype=torch.int8)
    vc = torch.randint(-127, 128, (rows, 16, 128), generator=g, dtype=torch.int8)
    ks = torch.rand((rows, 16), generator=g) * 0.05
    vs = torch.rand((rows, 16), generator=g) * 0.05
    ks[0, 0] = 0.0
    src = nm.KVCacheI8(kc.cuda(), vc.cuda(), ks.cuda(), vs.cuda(), rows, tpf)
    return (kc.numpy(), ks.numpy()), (vc.numpy(), vs.numpy()), src


@pytest.mark.parametrize("n_src,tpf,n_sel", [(10, 24, 7), (37, 5, 60), (3, 920, 2)])
def test_select_dequantises_bit_exactly(n_src, tpf, n_sel):
    kk, vv, src = _i8_source(n_src, tpf, n_src)
    idx = random_frame_list(n_src, n_sel, seed=tpf)
    win = nm.KVCache.empty(n_sel * tpf, 0)
    nm.kvcache_select(src, idx.tolist(), win)
    torch.cuda.synchronize()
    assert win.len == n_sel * tpf and win.tokens_per_frame == tpf
    for dev, (codes, scales) in ((win.k, kk), (win.v, vv)):
        want = oracle.dequantize_int8(oracle.kvcache_select(codes, idx, tpf),
                                      oracle.kvcache_select(scales, idx, tpf))
        assert np.array_equal(bits(dev), want)


def test_select_dequantises_with_one_rounding():
    # Random float32 scales make some float32 products land on a bf16 tie that
    # the exact product is not on; rounding twice (float32, then bf16) would
    # pick the wrong neighbour there.  The gather must equal the one-step
    # rounding of the oracle everywhere, those cases included.
    kk, vv, src = _i8_source(16, 920, 7)
    idx = np.arange(16)[::-1].copy()
    win = nm.KVCache.empty(16 * 920, 0)
    nm.kvcache_select(src, idx.tolist(), win)
    torch.cuda.synchronize()
    twice = 0
    for dev, (codes, scales) in ((win.k, kk), (win.v, vv)):
        c = oracle.kvcache_select(codes, idx, 920)
        s = oracle.kvcache_select(scales, idx, 920)
        want = oracle.dequantize_int8(c, s)
        assert np.array_equal(bits(dev), want)
        prod32 = (c.astype(np.float32) * s[:, :, None]).astype(np.float32)
        twice += int(np.count_nonzero(oracle.f32_to_bf16_bits(prod32) != want))
    print(f"elements where rounding twice would differ: {twice}")
    assert twice > 0


def test_select_int8_device_list_bad_index():
    kk, vv, src = _i8_source(6, 8, 1)
    idx = torch.tensor([1, 6, 2], dtype=torch.int32, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    win = nm.KVCache.empty(24, 0)
    win.k.view(torch.int16).fill_(0x7E57)
    nm.kvcache_select(src, idx, win, dev_err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == nm.DEVERR_BAD_FRAME_INDEX
    got = bits(win.k)
    assert np.all(got[8:16] == 0x7E57)
    want = oracle.dequantize_int8(oracle.kvcache_select(kk[0], [1, 2], 8),
                                  oracle.kvcache_select(kk[1], [1, 2], 8))
    assert np.array_equal(got[:8], want[:8]) and np.array_equal(got[16:], want[8:])


def test_int8_bounded_history_layer_step():
    # History appended to an INT8 cache (quantised on the GPU), a frame list
    # gathered back to bf16, then attention; the oracle runs the same steps.
    w = WORKLOADS["mid"]
    tpf = w.tokens_per_frame
    hist_k = randn_bf16((w.n_cache, 16, 128), 11)
    hist_v = randn_bf16((w.n_cache, 16, 128), 12)
    cache = nm.KVCacheI8.empty(w.n_cache, tpf)
    nm.kvcache_append_i8(cache, hist_k.cuda(), hist_v.cuda())
    idx = random_frame_list(w.cache_frames, 10, seed=3)
    win = nm.KVCache.empty(10 * tpf, 0)
    nm.kvcache_select(cache, idx.tolist(), win)
    q = randn_bf16((w.n_q, 16, 128), 13)
    ks = randn_bf16((w.n_seg, 16, 128), 14)
    vs = randn_bf16((w.n_seg, 16, 128), 15)
    o = nm.segment_attention(q.cuda(), [win.span(), (ks.cuda(), vs.cuda())])
    torch.cuda.synchronize()
    kc, ksc = oracle.quantize_int8(bits(hist_k))
    vc, vsc = oracle.quantize_int8(bits(hist_v))
    wk = oracle.dequantize_int8(oracle.kvcache_select(kc, idx, tpf), oracle.kvcache_select(ksc, idx, tpf))
    wv = oracle.dequantize_int8(oracle.kvcache_select(vc, idx, tpf), oracle.kvcache_select(vsc, idx, tpf))
    assert np.array_equal(bits(win.k), wk) and np.array_equal(bits(win.v), wv)
    o_ref, _ = oracle.attention(f64(q), [(oracle.bf16_bits_to_f64(wk), oracle.bf16_bits_to_f64(wv)),
                                         (f64(ks), f64(vs))])
    assert_close(f64(o), o_ref, what="int8 bounded O")
