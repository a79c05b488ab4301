"""Bit-exact parity of the frame-list gather with the oracle."""
import numpy as np
import pytest
import torch

import kv_cached_segment_b200 as nm
import oracle
from seeded_inputs import WORKLOADS, bounded_frame_list, random_frame_list, randn_bf16
from tests._util import bits

pytestmark = pytest.mark.gpu
CANARY = 0x7E57


def _src(n_frames, tpf, seed):
    k = randn_bf16((n_frames * tpf, 16, 128), seed)
    v = randn_bf16((n_frames * tpf, 16, 128), seed + 1)
    return k, v, nm.KVCache(k.cuda(), v.cuda(), n_frames * tpf, tpf)


def _window(rows):
    k = torch.empty((rows, 16, 128), dtype=torch.int16, device="cuda").fill_(CANARY)
    return nm.KVCache(k.view(torch.bfloat16), k.clone().view(torch.bfloat16), 0, 0)


@pytest.mark.parametrize("n_src,tpf,n_sel,spare", [(10, 24, 4, 0), (37, 7, 50, 3), (5, 1, 1, 2),
                                                    (24, 240, 9, 0)])
def test_select_host_list(n_src, tpf, n_sel, spare):
    k, v, src = _src(n_src, tpf, 5 + n_src)
    idx = random_frame_list(n_src, n_sel, seed=n_src)
    win = _window((n_sel + spare) * tpf)
    nm.kvcache_select(src, idx.tolist(), win)
    torch.cuda.synchronize()
    assert win.len == n_sel * tpf and win.tokens_per_frame == tpf
    for dev, host in ((win.k, k), (win.v, v)):
        want = oracle.kvcache_select(bits(host), idx, tpf)
        assert np.array_equal(bits(dev[:n_sel * tpf]), want)
        assert np.all(bits(dev[n_sel * tpf:]) == CANARY)


def test_select_device_list_and_bad_index():
    k, v, src = _src(12, 16, 9)
    idx = np.array([3, 11, 12, 0, -5, 3], dtype=np.int32)  # entries 2 and 4 are out of range
    idx_d = torch.from_numpy(idx).cuda()
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    win = _window(6 * 16)
    nm.kvcache_select(src, idx_d, win, dev_err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == nm.DEVERR_BAD_FRAME_INDEX
    for dev, host in ((win.k, k), (win.v, v)):
        got = bits(dev)
        for j, f in enumerate(idx):
            rows = got[j * 16:(j + 1) * 16]
            if 0 <= f < 12:
                assert np.array_equal(rows, oracle.kvcache_select(bits(host), [f], 16))
            else:
                assert np.all(rows == CANARY)


def test_select_device_list_good():
    k, v, src = _src(30, 8, 2)
    idx = random_frame_list(30, 100, seed=4)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    win = _window(100 * 8)
    nm.kvcache_select(src, torch.from_numpy(idx).cuda(), win, dev_err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    assert np.array_equal(bits(win.k), oracle.kvcache_select(bits(k), idx, 8))
    assert np.array_equal(bits(win.v), oracle.kvcache_select(bits(v), idx, 8))


def test_select_empty_list():
    k, v, src = _src(3, 4, 1)
    win = _window(8)
    nm.kvcache_select(src, [], win)
    torch.cuda.synchronize()
    assert win.len == 0 and np.all(bits(win.k) == CANARY)


def test_select_many_frames_spans_several_launches():
    # More host entries than one launch carries.
    k, v, src = _src(50, 1, 3)
    idx = random_frame_list(50, 5000, seed=8)
    win = _window(5000)
    nm.kvcache_select(src, idx.tolist(), win)
    torch.cuda.synchronize()
    assert np.array_equal(bits(win.k), oracle.kvcache_select(bits(k), idx, 1))


@pytest.mark.slow
def test_select_bounded_full_size():
    w = WORKLOADS["bounded"]
    tpf = w.tokens_per_frame
    k, v, src = _src(w.cache_frames, tpf, 11)
    idx = bounded_frame_list(w, seed=4)
    assert idx.size == w.select_frames and idx.size * tpf == 57960
    win = _window(idx.size * tpf)
    nm.kvcache_select(src, idx.tolist(), win)
    torch.cuda.synchronize()
    for dev, host in ((win.k, k), (win.v, v)):
        assert np.array_equal(bits(dev), oracle.kvcache_select(bits(host), idx, tpf))
