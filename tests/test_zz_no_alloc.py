"""The key-split attention entry point that allocates nothing.

Some callers cannot allocate device memory: a serving process whose whole
device budget is claimed up front and handed out from its own pools, a host
framework that owns the device allocator, or a latency-critical loop where
cudaMalloc and cudaFree, which can synchronise the device, are not allowed.
For them nomas_segment_attention_split_noalloc runs the key-split attention
on a scratch array built into the library instead of caller memory.

Through the C ABI, two calls in a row (with different shapes, so the second
reads nothing the first left behind) must give, bit for bit, the result of
the existing key-split entry point with caller scratch (the same kernel, the
same split, the same stream), plain attention's result within the parity
bar, and the fp64 oracle's within the same bar; a request larger than the
array must be refused before anything runs.  This file is collected last on purpose, and passes alone in
a fresh process as well as after every other test.
"""
import ctypes

import numpy as np
import pytest
import torch

import kv_cached_segment_b200 as nm
import oracle
from seeded_inputs import randn_bf16
from tests._util import assert_close, bits, f64

pytestmark = pytest.mark.gpu


def _entry(lib):
    f = lib.nomas_segment_attention_split_noalloc
    P, I32, I64, F32 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_float
    f.restype = ctypes.c_int
    f.argtypes = [P, I64, ctypes.POINTER(nm._KVSpan), I32, P, P, F32, I32, I32, I32, P, P]
    return f


def _span_array(spans):
    return (nm._KVSpan * len(spans))(*[nm._KVSpan(k.data_ptr(), v.data_ptr(), k.shape[0])
                                       for k, v in spans])


def _inputs(n_q, lens, seed):
    q = randn_bf16((n_q, 16, 128), seed).cuda()
    spans = [(randn_bf16((n, 16, 128), seed * 10 + i).cuda(),
              randn_bf16((n, 16, 128), seed * 10 + 5 + i).cuda()) for i, n in enumerate(lens)]
    return q, spans


def test_noalloc_split_matches_the_existing_entry_points_on_two_calls_in_a_row():
    lib = nm.load_library()
    f = _entry(lib)
    for seed, (n_q, lens, splits) in ((31, (600, [3000, 64, 1200], 3)),
                                      (32, (300, [5000, 17], 5))):
        q, spans = _inputs(n_q, lens, seed)
        # the existing entry points: the same split with caller scratch, and
        # plain attention
        lse_ref = torch.empty(16 * n_q, dtype=torch.float32, device="cuda")
        o_ref = nm.segment_attention(q, spans, lse=lse_ref, kv_splits=splits)
        o_plain = nm.segment_attention(q, spans)
        o = torch.full_like(q, 7.0)
        lse = torch.full_like(lse_ref, 7.0)
        err = torch.zeros(1, dtype=torch.int32, device="cuda")
        st = f(q.data_ptr(), n_q, _span_array(spans), len(spans), o.data_ptr(), lse.data_ptr(),
               0.0, 16, 128, splits, err.data_ptr(), None)
        torch.cuda.synchronize()
        assert st == nm.NOMAS_OK, lib.nomas_last_error().decode()
        assert int(err.item()) == 0
        # same kernel, same split, same stream: identical bits
        assert np.array_equal(bits(o), bits(o_ref)), f"no-alloc vs caller scratch, call {seed}"
        assert np.array_equal(lse.cpu().numpy().view(np.uint32),
                              lse_ref.cpu().numpy().view(np.uint32))
        assert_close(f64(o), f64(o_plain), what=f"no-alloc vs plain attention, call {seed}")
        o_or, l_or = oracle.attention(f64(q), [(f64(k), f64(v)) for k, v in spans])
        assert_close(f64(o), o_or, what=f"no-alloc vs oracle, call {seed}")
        assert_close(lse.view(16, n_q).cpu().double().numpy(), l_or,
                     what=f"no-alloc LSE vs oracle, call {seed}")


def test_noalloc_refuses_more_than_its_array():
    lib = nm.load_library()
    f = _entry(lib)
    n_q, splits = 600, nm.MAX_MERGE_PARTS        # 32 x 600 x 4,160 B = 80 MB > 64 MiB
    q, spans = _inputs(n_q, [1000], 33)
    o = torch.full_like(q, 7.0)
    st = f(q.data_ptr(), n_q, _span_array(spans), 1, o.data_ptr(), None, 0.0, 16, 128, splits,
           None, None)
    torch.cuda.synchronize()
    assert st == nm.NOMAS_ERR_CAPACITY
    msg = lib.nomas_last_error().decode()
    assert str(64 << 20) in msg and str(splits * n_q * 4160) in msg
    assert torch.all(o == 7.0)  # refused before anything ran
