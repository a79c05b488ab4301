"""Attention over a history held in INT8, dequantised inside the kernel.

The single-GPU preset keeps its resident history frames on the GPU in INT8
and computes in bf16 ("Hy-Nomas: an 8.6B world model whose memory is a KV
cache", section "The 4090 preset"; "Hy-Nomas en una RTX 4090", section
"El preset de una GPU").  The oracle is plain fp64 attention over the exact
dequantised history (code * scale) followed by the bf16 spans; the kernel
rounds each dequantised value to bf16 once more on its way to the tensor
cores, which the parity bar covers.
"""
import numpy as np
import pytest
import torch

import kv_cached_segment_b200 as nm
import oracle
from seeded_inputs import WORKLOADS, bounded_frame_list, randn_bf16
from tests._util import assert_close, bits, f64

pytestmark = pytest.mark.gpu


def _i8_history(n, seed):
    """Codes and scales shaped like a quantised N(0, 1) history: codes about
    N(0, 40^2) clipped to +-127, scales near 1/40, so values are about
    N(0, 1) like the bf16 spans; one (token, head) has scale 0."""
    g = torch.Generator().manual_seed(seed)
    kc = (torch.randn((n, 16, 128), generator=g) * 40).round().clamp(-127, 127).to(torch.int8)
    vc = (torch.randn((n, 16, 128), generator=g) * 40).round().clamp(-127, 127).to(torch.int8)
    ks = (1.0 + 0.5 * torch.rand((n, 16), generator=g)) / 48.0
    vs = (1.0 + 0.5 * torch.rand((n, 16), generator=g)) / 48.0
    if n > 3:
        ks[3, 5] = 0.0  # an all-zero (token, head)
        vs[3, 5] = 0.0
    return kc, vc, ks, vs


def _run(n_q, n_hist, text_lens, seed, **kw):
    kc, vc, ks, vs = _i8_history(n_hist, seed)
    hist = nm.I8Span(kc.cuda(), vc.cuda(), ks.cuda(), vs.cuda())
    q = randn_bf16((n_q, 16, 128), seed + 1)
    rest = [(randn_bf16((n, 16, 128), seed + 10 + i), randn_bf16((n, 16, 128), seed + 20 + i))
            for i, n in enumerate(text_lens)]
    lse = torch.empty(16 * n_q, dtype=torch.float32, device="cuda")
    o = nm.segment_attention(q.cuda(), [hist] + [(k.cuda(), v.cuda()) for k, v in rest], lse=lse,
                             **kw)
    torch.cuda.synchronize()
    spans = [(oracle.dequantize_int8_f64(kc.numpy(), ks.numpy()),
              oracle.dequantize_int8_f64(vc.numpy(), vs.numpy()))]
    spans += [(f64(k), f64(v)) for k, v in rest]
    return o, lse, q, spans


@pytest.mark.parametrize("n_q,n_hist,text_lens", [
    (300, 1000, [64, 200]),     # ragged history tail, two bf16 spans
    (112, 48, [64, 48]),        # history shorter than one tile
    (513, 128 * 5, []),         # whole tiles, history only
    (256, 777, [1, 129]),       # a one-key span
])
def test_int8_history_attention_matches_oracle(n_q, n_hist, text_lens):
    o, lse, q, spans = _run(n_q, n_hist, text_lens, seed=n_hist)
    o_ref, l_ref = oracle.attention(f64(q), spans)
    assert_close(f64(o), o_ref, what="INT8-history O")
    assert_close(lse.view(16, n_q).cpu().double().numpy(), l_ref, what="INT8-history LSE")


def test_int8_history_of_length_zero_is_plain_attention():
    q = randn_bf16((200, 16, 128), 5).cuda()
    k = randn_bf16((300, 16, 128), 6).cuda()
    v = randn_bf16((300, 16, 128), 7).cuda()
    empty = nm.KVCacheI8.empty(16, 1).span(0, 0)
    o1 = nm.segment_attention(q, [empty, (k, v)])
    o2 = nm.segment_attention(q, [(k, v)])
    torch.cuda.synchronize()
    assert np.array_equal(bits(o1), bits(o2))


def test_int8_history_equals_bf16_window_of_the_same_values():
    # When every code * scale is a bf16 value (scales that are powers of
    # two), the kernel's conversion is exact, and attention over the INT8
    # history must equal attention over the same values as a bf16 span.
    n = 700
    kc, vc, _, _ = _i8_history(n, 9)
    g = torch.Generator().manual_seed(10)
    ks = torch.exp2(torch.randint(-9, -3, (n, 16), generator=g).float())
    vs = torch.exp2(torch.randint(-9, -3, (n, 16), generator=g).float())
    kb = (kc.float() * ks[:, :, None]).to(torch.bfloat16)
    vb = (vc.float() * vs[:, :, None]).to(torch.bfloat16)
    assert torch.equal(kb.float(), kc.float() * ks[:, :, None])  # exact in bf16
    q = randn_bf16((400, 16, 128), 11).cuda()
    seg = (randn_bf16((90, 16, 128), 12).cuda(), randn_bf16((90, 16, 128), 13).cuda())
    hist = nm.I8Span(kc.cuda(), vc.cuda(), ks.cuda(), vs.cuda())
    l1 = torch.empty(16 * 400, dtype=torch.float32, device="cuda")
    l2 = torch.empty_like(l1)
    o1 = nm.segment_attention(q, [hist, seg], lse=l1)
    o2 = nm.segment_attention(q, [(kb.cuda(), vb.cuda()), seg], lse=l2)
    torch.cuda.synchronize()
    assert np.array_equal(bits(o1), bits(o2))
    assert torch.equal(l1, l2)


def test_int8_window_gather_copies_codes_and_scales():
    tpf, n_src = 40, 12
    kc, vc, ks, vs = _i8_history(tpf * n_src, 21)
    src = nm.KVCacheI8(kc.cuda(), vc.cuda(), ks.cuda(), vs.cuda(), tpf * n_src, tpf)
    idx = [11, 0, 5, 5, 3]
    win = nm.KVCacheI8.empty(tpf * 6, 0)
    nm.kvcache_select(src, idx, win)
    torch.cuda.synchronize()
    assert win.len == len(idx) * tpf and win.tokens_per_frame == tpf
    n = len(idx) * tpf
    for got, want in ((win.k, kc), (win.v, vc), (win.k_scale, ks), (win.v_scale, vs)):
        ref = oracle.kvcache_select(want.numpy(), idx, tpf)
        assert np.array_equal(got[:n].cpu().numpy(), ref)
    # device list with a bad entry: its rows are left alone, the rest copied
    win2 = nm.KVCacheI8.empty(tpf * 3, 0)
    win2.k.fill_(9)
    win2.k_scale.fill_(9.0)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    nm.kvcache_select(src, torch.tensor([2, 99, 4], dtype=torch.int32, device="cuda"), win2,
                      dev_err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == nm.DEVERR_BAD_FRAME_INDEX
    assert torch.all(win2.k[tpf:2 * tpf] == 9) and torch.all(win2.k_scale[tpf:2 * tpf] == 9.0)
    assert np.array_equal(win2.k[:tpf].cpu().numpy(), kc[2 * tpf:3 * tpf].numpy())
    assert np.array_equal(win2.v_scale[2 * tpf:].cpu().numpy(), vs[4 * tpf:5 * tpf].numpy())


def test_int8_history_wait_timeout_marks_rows_and_context_survives():
    # The producer leaves out the first INT8 code tile, so the converters'
    # wait can never complete: every block must give up, report the timeout
    # and mark its rows NaN; the context then still computes correctly.
    kc, vc, ks, vs = _i8_history(300, 31)
    hist = nm.I8Span(kc.cuda(), vc.cuda(), ks.cuda(), vs.cuda())
    q = randn_bf16((300, 16, 128), 32).cuda()
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    o = torch.full_like(q, 7.0)
    nm.segment_attention(q, [hist], o=o, dev_err=err, wait_limit_ns=50_000_000,
                         testing_skip_kv_load=0)
    torch.cuda.synchronize()
    assert int(err.item()) == nm.DEVERR_WAIT_TIMEOUT
    assert torch.all(torch.isnan(o))
    o2, lse, q2, spans = _run(300, 500, [64], seed=33)
    assert_close(f64(o2), oracle.attention(f64(q2), spans)[0], what="after timeout")


def test_int8_bounded_layer_step_full_size():
    # The bounded workload with its history in INT8 end to end: the history
    # quantised into an INT8 cache on the GPU, the frame list gathered as
    # codes and scales, attention over window + text + segment.  Sampled
    # rows (segment and text) against the oracle over the same codes.
    w = WORKLOADS["bounded"]
    tpf, ns = w.tokens_per_frame, w.n_seg
    cache = nm.KVCacheI8.empty(w.n_cache, tpf)
    chunk = tpf * 30
    for r0 in range(0, w.n_cache, chunk):
        r1 = min(w.n_cache, r0 + chunk)
        nm.kvcache_append_i8(cache, randn_bf16((r1 - r0, 16, 128), 40 + r0, "cuda"),
                             randn_bf16((r1 - r0, 16, 128), 41 + r0, "cuda"))
    frames = bounded_frame_list(w, 1)
    win = nm.KVCacheI8.empty(w.n_window, 0)
    nm.kvcache_select(cache, frames.tolist(), win)
    q = randn_bf16((w.n_q, 16, 128), 42, "cuda")
    k = randn_bf16((w.n_q, 16, 128), 43, "cuda")
    v = randn_bf16((w.n_q, 16, 128), 44, "cuda")
    lse = torch.empty(16 * w.n_q, dtype=torch.float32, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    o = nm.segment_attention(q, [win.span(), (k[ns:], v[ns:]), (k[:ns], v[:ns])], lse=lse,
                             dev_err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    codes = [x.cpu().numpy() for x in (win.k, win.v, win.k_scale, win.v_scale)]
    spans = [(oracle.dequantize_int8_f64(codes[0], codes[2]),
              oracle.dequantize_int8_f64(codes[1], codes[3])),
             (f64(k[ns:]), f64(v[ns:])), (f64(k[:ns]), f64(v[:ns]))]
    rows = np.unique(np.concatenate([np.random.default_rng(2).integers(0, w.n_q, 40),
                                     [0, ns - 1, ns, w.n_q - 1]]))
    o_ref, l_ref = oracle.attention_rows(f64(q), rows, spans)
    assert_close(f64(o[torch.as_tensor(rows).cuda()]), o_ref, what="bounded INT8 O")
    got_l = lse.view(16, -1)[:, torch.as_tensor(rows).cuda()].cpu().double().numpy()
    assert_close(got_l, l_ref, what="bounded INT8 LSE")
    # the window is the oracle's gather of the oracle's quantisation
    kc, ksc = oracle.quantize_int8(bits(randn_bf16((chunk, 16, 128), 40, "cuda")))
    first = np.nonzero(frames < 30)[0]
    if first.size:
        j = int(first[0])
        f = int(frames[j])
        assert np.array_equal(codes[0][j * tpf:(j + 1) * tpf], kc[f * tpf:(f + 1) * tpf])
