"""Merging attention partials over key shards, and the sharded path on one GPU."""
import numpy as np
import pytest
import torch

import kv_cached_segment_b200 as nm
import oracle
from seeded_inputs import randn_bf16
from tests._util import assert_bf16_rounding, assert_close, f64

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("r,n_q", [(5, 300), (1, 17), (7, 1000), (nm.MAX_MERGE_PARTS, 129)])
def test_merge_kernel_matches_oracle_formula(r, n_q):
    g = torch.Generator().manual_seed(3)
    o_parts = randn_bf16((r, n_q, 16, 128), 7)
    lse_parts = torch.randn((r, 16, n_q), generator=g) * 4
    lse_parts[r // 2] = -float("inf")       # an empty shard (the only one when r = 1)
    lse_parts[:, 3, :10] = -float("inf")    # rows where every shard is empty
    lse = torch.empty(16 * n_q, dtype=torch.float32, device="cuda")
    o = nm.attention_merge(o_parts.cuda(), lse_parts.cuda(), lse=lse)
    torch.cuda.synchronize()
    want_o, want_l = oracle.merge_partials(f64(o_parts), lse_parts.double().numpy())
    # fp32 weights and sums, one rounding to bf16 at the end: every element
    # is the exact merge rounded to bf16, to within one unit in the last place
    # (partials of unit variance reach |O| ~ 4, where that unit is 2^-5).
    assert_bf16_rounding(f64(o), want_o, what="merged O")
    got_l = lse.view(16, n_q).cpu().double().numpy()
    fin = np.isfinite(want_l)
    assert np.array_equal(np.isfinite(got_l), fin)
    assert np.allclose(got_l[fin], want_l[fin], atol=1e-5)


def test_merge_nan_partial_poisons_only_its_rows():
    # A NaN LSE marks a partial whose attention block aborted: those (row,
    # head) pairs come out NaN, never as a merge of the remaining parts; every
    # other row is the plain merge.
    r, n_q = 4, 300
    o_parts = randn_bf16((r, n_q, 16, 128), 8)
    lse_parts = torch.randn((r, 16, n_q), generator=torch.Generator().manual_seed(4)) * 3
    lse_parts[2, 5, 100:120] = float("nan")
    lse = torch.empty(16 * n_q, dtype=torch.float32, device="cuda")
    o = nm.attention_merge(o_parts.cuda(), lse_parts.cuda(), lse=lse)
    torch.cuda.synchronize()
    got_o, got_l = f64(o), lse.view(16, n_q).cpu().double().numpy()
    bad = np.zeros((n_q, 16), dtype=bool)
    bad[100:120, 5] = True
    assert np.all(np.isnan(got_o[bad])) and np.all(np.isnan(got_l.T[bad]))
    clean = lse_parts.clone()
    clean[2, 5, 100:120] = 0.0
    want_o, want_l = oracle.merge_partials(f64(o_parts), clean.double().numpy())
    assert not np.any(np.isnan(got_o[~bad]))
    assert_bf16_rounding(np.where(bad[:, :, None], 0.0, got_o),
                         np.where(bad[:, :, None], 0.0, want_o), what="merged O, clean rows")
    assert np.allclose(got_l.T[~bad], want_l.T[~bad], atol=1e-5)


@pytest.mark.parametrize("cuts", [[0, 1000, 2500, 4000], [0, 0, 4000], [0, 1, 3999, 4000]])
def test_sharded_keys_merge_to_full_attention(cuts):
    q = randn_bf16((700, 16, 128), 1)
    k = randn_bf16((4000, 16, 128), 2)
    v = randn_bf16((4000, 16, 128), 3)
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    parts_o, parts_l = [], []
    for a, b in zip(cuts[:-1], cuts[1:]):
        l_r = torch.empty(16 * 700, dtype=torch.float32, device="cuda")
        parts_o.append(nm.segment_attention(qd, [(kd[a:b], vd[a:b])], lse=l_r))
        parts_l.append(l_r.view(16, 700))
    lse = torch.empty(16 * 700, dtype=torch.float32, device="cuda")
    o = nm.attention_merge(torch.stack(parts_o), torch.stack(parts_l), lse=lse)
    torch.cuda.synchronize()
    o_ref, l_ref = oracle.attention(f64(q), [(f64(k), f64(v))])
    assert_close(f64(o), o_ref, what="sharded O")
    assert_close(lse.view(16, -1).cpu().double().numpy(), l_ref, what="sharded LSE")


def test_sharded_attention_single_rank_is_plain_attention():
    q = randn_bf16((300, 16, 128), 4).cuda()
    spans = [(randn_bf16((500, 16, 128), 5).cuda(), randn_bf16((500, 16, 128), 6).cuda())]
    o1 = nm.sharded_segment_attention(q, spans)
    o2 = nm.segment_attention(q, spans)
    torch.cuda.synchronize()
    assert (o1.float() - o2.float()).abs().max().item() <= 2 ** -7


@pytest.mark.parametrize("world,n_q,n_k", [(3, 700, 4000), (2, 130, 300), (4, 1000, 2000)])
def test_peer_merge_emulating_ranks_on_one_gpu(world, n_q, n_k):
    # Each "GPU" is a set of buffers on this one: phase 1 runs for every rank,
    # then phase 2 for every rank, in stream order (nothing waits on anything
    # else).  Every rank's output must be the whole attention.
    q, k, v = (randn_bf16((n, 16, 128), s) for n, s in ((n_q, 41), (n_k, 42), (n_k, 43)))
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    part_o = [torch.empty((n_q, 16, 128), dtype=torch.bfloat16, device="cuda")
              for _ in range(world)]
    part_lse = [torch.empty((16, n_q), dtype=torch.float32, device="cuda") for _ in range(world)]
    o_out = [torch.full((n_q, 16, 128), 7.0, dtype=torch.bfloat16, device="cuda")
             for _ in range(world)]
    lse_out = [torch.full((16, n_q), 7.0, dtype=torch.float32, device="cuda")
               for _ in range(world)]
    for r in range(world):
        a, b = nm.shard_rows(n_k, r, world, align=128)
        nm.peer_partial_attention(qd, [(kd[a:b], vd[a:b])], part_o[r], part_lse[r])
    for r in range(world):
        nm.peer_merge_owned_rows(part_o, part_lse, o_out, lse_out, r, world)
    stacked = nm.attention_merge(torch.stack(part_o), torch.stack(part_lse))
    torch.cuda.synchronize()
    o_ref, l_ref = oracle.attention(f64(q), [(f64(k), f64(v))])
    for r in range(world):
        assert torch.equal(o_out[r].view(torch.int16), o_out[0].view(torch.int16))
        assert torch.equal(lse_out[r], lse_out[0])
    assert torch.equal(o_out[0].view(torch.int16), stacked.view(torch.int16))
    assert_close(f64(o_out[0]), o_ref, what=f"peer merge over {world} ranks O")
    assert_close(lse_out[0].cpu().double().numpy(), l_ref, what=f"peer merge over {world} ranks LSE")


def test_peer_merge_writes_only_its_rows():
    n_q = 300
    parts = [randn_bf16((n_q, 16, 128), 50 + r).cuda() for r in range(2)]
    lses = [torch.zeros((16, n_q), dtype=torch.float32, device="cuda") for _ in range(2)]
    outs = [torch.full((n_q, 16, 128), 7.0, dtype=torch.bfloat16, device="cuda")]
    nm.attention_merge_peers(parts, lses, outs, None, row0=100, n_rows=37)
    torch.cuda.synchronize()
    assert torch.all(outs[0][:100] == 7.0) and torch.all(outs[0][137:] == 7.0)
    # equal LSEs: the merged rows are the average of the two parts, rounded once
    want = (f64(parts[0][100:137]) + f64(parts[1][100:137])) / 2   # on the host, in fp64
    assert_bf16_rounding(f64(outs[0][100:137]), want, what="average of two parts")


@pytest.mark.parametrize("world,n_q,n_k", [(3, 700, 4000), (4, 130, 300), (2, 1000, 2000)])
def test_attention_routed_to_owners_emulating_ranks_on_one_gpu(world, n_q, n_k):
    # Phase 1 on every "GPU": its partial rows go straight into part `rank`
    # of each row owner's inbox; phase 2 on every "GPU": the owner merges its
    # rows from its inbox into every output.  With n_k = 300 over 4 ranks,
    # rank 0 has no keys and stores O = 0, LSE = -inf.
    q, k, v = (randn_bf16((n, 16, 128), s) for n, s in ((n_q, 61), (n_k, 62), (n_k, 63)))
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    inbox_o = [torch.full((world, n_q, 16, 128), 7.0, dtype=torch.bfloat16, device="cuda")
               for _ in range(world)]
    inbox_l = [torch.full((world, 16, n_q), 7.0, dtype=torch.float32, device="cuda")
               for _ in range(world)]
    o_out = [torch.full((n_q, 16, 128), 7.0, dtype=torch.bfloat16, device="cuda")
             for _ in range(world)]
    lse_out = [torch.full((16, n_q), 7.0, dtype=torch.float32, device="cuda")
               for _ in range(world)]
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    for r in range(world):
        a, b = nm.shard_rows(n_k, r, world, align=128)
        nm.peer_attention_to_owners(qd, [(kd[a:b], vd[a:b])], inbox_o, inbox_l, slot=r,
                                    dev_err=err)
    for r in range(world):
        nm.peer_merge_inbox(inbox_o[r], inbox_l[r], o_out, lse_out, r)
    # the same partials computed the plain way, merged by the stacked kernel
    parts_o, parts_l = [], []
    for r in range(world):
        a, b = nm.shard_rows(n_k, r, world, align=128)
        l_r = torch.empty(16 * n_q, dtype=torch.float32, device="cuda")
        parts_o.append(nm.segment_attention(qd, [(kd[a:b], vd[a:b])], lse=l_r))
        parts_l.append(l_r.view(16, n_q))
    stacked = nm.attention_merge(torch.stack(parts_o), torch.stack(parts_l))
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    for r in range(world):
        assert torch.equal(o_out[r].view(torch.int16), stacked.view(torch.int16))
        assert torch.equal(lse_out[r], lse_out[0])
    o_ref, l_ref = oracle.attention(f64(q), [(f64(k), f64(v))])
    assert_close(f64(o_out[0]), o_ref, what=f"routed attention over {world} ranks O")
    assert_close(lse_out[0].cpu().double().numpy(), l_ref, what=f"routed over {world} ranks LSE")


def test_routed_sharded_attention_on_one_rank_is_plain_attention():
    q = randn_bf16((300, 16, 128), 71).cuda()
    k, v = randn_bf16((900, 16, 128), 72).cuda(), randn_bf16((900, 16, 128), 73).cuda()
    inbox_o = [torch.empty((1, 300, 16, 128), dtype=torch.bfloat16, device="cuda")]
    inbox_l = [torch.empty((1, 16, 300), dtype=torch.float32, device="cuda")]
    o_out = [torch.empty((300, 16, 128), dtype=torch.bfloat16, device="cuda")]
    l_out = [torch.empty((16, 300), dtype=torch.float32, device="cuda")]
    o = nm.sharded_segment_attention_routed(q, [(k, v)], inbox_o, inbox_l, o_out, l_out, rank=0)
    lse = torch.empty(16 * 300, dtype=torch.float32, device="cuda")
    plain = nm.segment_attention(q, [(k, v)], lse=lse)
    torch.cuda.synchronize()
    # one part with weight 1: the merge only re-rounds values already in bf16
    assert torch.equal(o.view(torch.int16), plain.view(torch.int16))
    assert torch.allclose(l_out[0].view(-1), lse, atol=1e-5)
