#!/usr/bin/env python
"""Segment-over-cache attention layer-step benchmark on B200.

One step = one pass of the whole hot path over one layer's inputs, resident
in HBM: fused RoPE-3D + cache append of the segment (rotated Q out, rotated K
and V into the cache), for the bounded-history workload the frame-list gather
of the history window, then segment attention of the segment + text queries
over history + text + segment keys.  Prints ONE JSON line on rank 0.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload 720p]
  python bench.py --impl reference ...   # the fp64 CPU oracle, same metric

Multi-GPU (torchrun): every rank runs its own independent layer-step (weak
scaling, no collective on the data path); with --key-shards N on N GPUs the
ranks instead share one layer-step, each attending over 1/N of the keys, the
partials all-gathered over NCCL and merged (strong scaling).  Timing is the
max over ranks.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time
import types

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "segment-over-cache attention TFLOP/s and % of B200 BF16 peak; ms per layer-step"
UNIT = "TFLOP/s"
DATASHEET_BF16_TFLOPS = 2250.0
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def parse_args():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=40)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--impl", choices=["nomas", "reference"], default="nomas")
    p.add_argument("--workload", choices=["720p", "bounded", "bounded90", "short", "mid", "tiny",
                                          "sweep"],
                   default="720p")
    p.add_argument("--int8", action="store_true",
                   help="the history in INT8 (quantising append; for a workload with a frame "
                        "window, a gather of codes and scales; attention dequantising the "
                        "history tiles in the kernel)")
    p.add_argument("--int8-window", choices=["int8", "bf16"], default="int8",
                   help="with --int8 and a frame window: keep the gathered window in INT8 and "
                        "dequantise inside attention (int8), or dequantise once in the gather "
                        "into a transient bf16 window read by the bf16 kernel (bf16)")
    p.add_argument("--sparse", type=float, default=0.0,
                   help="block-sparse attention keeping this fraction of the video key tiles "
                        "(text tiles always kept); 0 = dense")
    p.add_argument("--key-shards", type=int, default=0,
                   help="split the key sequence into this many contiguous shards, attend over "
                        "each into a partial (O, LSE) and merge them.  Equal to the number of "
                        "GPUs: each rank holds one shard and the partials are all-gathered over "
                        "NCCL; on one GPU with more shards: every shard on that GPU (the per-GPU "
                        "work of key-sharded attention); 0 = one launch over all keys")
    p.add_argument("--head-shards", type=int, default=0,
                   help="on one GPU: attention in this many launches of 16/N heads each, with "
                        "head-sliced copies of the rows (the per-GPU work of N-way head-sharded "
                        "attention, all N shares on this GPU); 0 = one launch of 16 heads")
    p.add_argument("--kv-splits", default="1",
                   help="key splits of the attention launch (an integer, or 'auto': chosen from "
                        "the grid's wave count); 1 = one CTA per query block and head")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-e2e", action="store_true")
    return p.parse_args()


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return FALLBACK_PEAKS, "fallback"


def kernel_source_hash() -> str:
    """Hash of the attention kernel's code: its sources with // comments and
    blank lines removed, so that editing a comment keeps a capture valid."""
    h = hashlib.sha256()
    for name in ("attention.cu", "attn_device.cuh", "f32x2.cuh", "tmem_ops.cuh", "nomas_internal.h"):
        with open(os.path.join(ROOT, "kv_cached_segment_b200", "csrc", name)) as f:
            for line in f:
                code = line.split("//", 1)[0].rstrip()
                if code:
                    h.update(code.encode() + b"\n")
    return h.hexdigest()[:16]


def recorded_traffic(workload: str):
    """DRAM bytes per attention launch from a committed ncu summary, if the
    kernel source has not changed since it was captured."""
    path = os.path.join(ROOT, "profiles", f"attention_{workload}_dram.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        d = json.load(f)
    if d.get("source_hash") != kernel_source_hash():
        return None
    return d.get("dram_bytes_per_launch")


# ------------------------------------------------------------------ clocks --
class ClockSampler:
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, uuid: str | None):
        self.proc = None
        try:
            cmd = ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                   "-lms", "200"]
            if uuid:
                cmd += ["-i", uuid]
            self.proc = subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.DEVNULL,
                                         text=True)
        except (OSError, ValueError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sm, smax, power, reasons = [], [], [], set()
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        for line in out.strip().splitlines():
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 7:
                continue
            try:
                sm.append(float(parts[0]))
                smax.append(float(parts[1]))
                power.append(float(parts[2]))
            except ValueError:
                continue
            for n, flag in zip(names, parts[3:7]):
                if flag.lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None,
                "power_w_max": max(power) if power else None,
                "samples": len(sm), "reasons": sorted(reasons)}


# ---------------------------------------------------------------- workload --
def _mark(ev, name: str, which: int) -> None:
    """Records the start (0) or end (1) event of `name` if the step is timed."""
    if ev is not None and name in ev:
        ev[name][which].record()


class LayerStep:
    """Device-resident buffers of one layer-step and the launches of a step."""

    def __init__(self, wname: str, seed: int):
        import torch

        import kv_cached_segment_b200 as nm
        from seeded_inputs import WORKLOADS, bounded_frame_list, randn_bf16

        self.nm, self.torch = nm, torch
        w = self.w = WORKLOADS[wname]
        dev = "cuda"
        ns, nt = w.n_seg, w.n_text
        self.layout = nm.SegLayout(w.frames, w.grid_h, w.grid_w, w.t0, nt)
        self.cfg = nm.RopeConfig(*w.rope_split, w.rope_theta)
        self.cache = nm.KVCache.empty(w.n_cache + ns, w.tokens_per_frame)
        self.cache.k[:w.n_cache] = randn_bf16((w.n_cache, 16, 128), seed * 16 + 4, dev)
        self.cache.v[:w.n_cache] = randn_bf16((w.n_cache, 16, 128), seed * 16 + 5, dev)
        self.q = randn_bf16((w.n_q, 16, 128), seed * 16 + 1, dev)
        self.k = randn_bf16((w.n_q, 16, 128), seed * 16 + 2, dev)
        self.v = randn_bf16((w.n_q, 16, 128), seed * 16 + 3, dev)
        self.q_rot = torch.empty_like(self.q)
        self.o = torch.empty_like(self.q)
        self.lse = torch.empty(16 * w.n_q, dtype=torch.float32, device=dev)
        self.err = torch.zeros(1, dtype=torch.int32, device=dev)
        if w.select_frames:
            self.frames = bounded_frame_list(w, seed).tolist()
            self.window = nm.KVCache.empty(w.n_window, 0)
        else:
            self.frames = None
        self.launches_per_step = 3 if self.frames else 2
        self.append_kernels = "rope_append_kernel<bf16> (fused RoPE + append)"
        self.select_kernel = "select_kernel"
        self.sparse = None
        self.shards = 0
        self.head_shards = 0
        self.kv_splits = 1

    def use_key_shards(self, n_shards: int):
        """Attention over `n_shards` contiguous ranges of the key sequence
        (boundaries on 128-key tiles), each into its own partial (O, LSE),
        then one merge: what each GPU of key-sharded attention computes."""
        torch, w = self.torch, self.w
        self.shards = n_shards
        self.part_o = torch.empty((n_shards, w.n_q, 16, 128), dtype=torch.bfloat16,
                                  device="cuda")
        self.part_lse = torch.empty((n_shards, 16, w.n_q), dtype=torch.float32, device="cuda")
        self.launches_per_step += n_shards  # n_shards attention launches + 1 merge, was 1

    def use_head_shards(self, n_shards: int):
        """Attention in `n_shards` launches of 16 / n_shards heads each: what
        each GPU of head-sharded attention computes, all shares on this GPU.
        Each share's history rows are resident in a head-sliced layout (as a
        GPU of head-sharded attention holds its heads' cache); per step the
        rotated Q and the text and segment K/V are copied into head-sliced
        buffers and O back (the local data movement of the two all-to-alls),
        and each launch picks its key splits (kv_splits="auto")."""
        torch, w = self.torch, self.w
        if 16 % n_shards:
            raise SystemExit("--head-shards must divide 16")
        self.head_shards = n_shards
        hl = 16 // n_shards
        sl = [slice(g * hl, (g + 1) * hl) for g in range(n_shards)]
        self.head_slices = sl
        if self.frames is not None:
            raise SystemExit("--head-shards uses a workload without a frame window")
        self.hist_g = [(self.cache.k[:w.n_cache, s].contiguous(), self.cache.v[:w.n_cache, s].contiguous())
                       for s in sl]
        self.q_g = [torch.empty((w.n_q, hl, 128), dtype=torch.bfloat16, device="cuda") for _ in sl]
        self.o_g = [torch.empty_like(t) for t in self.q_g]
        self.lse_g = [torch.empty(hl * w.n_q, dtype=torch.float32, device="cuda") for _ in sl]
        self.ks_g = [torch.empty((w.n_text + w.n_seg, hl, 128), dtype=torch.bfloat16, device="cuda")
                     for _ in sl]
        self.vs_g = [torch.empty_like(t) for t in self.ks_g]
        sm = torch.cuda.get_device_properties(0).multi_processor_count
        splits = self.nm.auto_kv_splits(w.n_q, [w.n_cache, w.n_text + w.n_seg], sm, heads=hl)
        # n_shards attention launches (was 1), and a merge each when keys are split
        self.launches_per_step += n_shards - 1 + (n_shards if splits > 1 else 0)

    def _shard_spans(self, spans):
        lens = [int(k.shape[0]) for k, _ in spans]
        n_k = sum(lens)
        out = []
        for r in range(self.shards):
            a, b = self.nm.shard_rows(n_k, r, self.shards, align=128)
            sub, base = [], 0
            for (k, v), n in zip(spans, lens):
                lo, hi = max(a, base), min(b, base + n)
                if hi > lo:
                    sub.append((k[lo - base:hi - base], v[lo - base:hi - base]))
                base += n
            out.append(sub if sub else [(spans[0][0][:0], spans[0][1][:0])])
        return out

    def use_sparse(self, fraction: float, seed: int):
        """Seeded block-sparse selection: text tiles kept, `fraction` of the
        history and segment tiles per (query block, head)."""
        from seeded_inputs import sparse_tile_lists

        w, torch = self.w, self.torch
        hist = w.n_window if w.select_frames else w.n_cache
        lens = [hist, w.n_text, w.n_seg]
        lists, counts = sparse_tile_lists(w.n_q, lens, keep_spans=[1], candidate_spans=[0, 2],
                                          fraction=fraction, seed=seed)
        # keys actually attended: every listed tile is full except span ends
        tile_keys = []
        for n in lens:
            tile_keys += [min(128, n - a) for a in range(0, n, 128)]
        tile_keys = np.asarray(tile_keys)
        rows = np.minimum(256, w.n_q - 256 * np.arange(lists.shape[0]))
        keys = np.array([[tile_keys[lists[b, h, :counts[b, h]]].sum() for h in range(16)]
                         for b in range(lists.shape[0])])
        self.sparse_flops = float(4.0 * 128 * (rows[:, None] * keys).sum())
        self.sparse = (torch.from_numpy(lists).cuda(), torch.from_numpy(counts).cuda())

    def flops(self) -> float:
        return self.sparse_flops if self.sparse is not None else self.w.attention_flops()

    def run(self, ev=None, bufs=None):
        """One layer-step; `ev` (optional) maps "append", "select" and "attn" to
        (start, end) CUDA events recorded around those launches."""
        nm, w = self.nm, self.w
        ns = w.n_seg
        q, k, v, o = (self.q, self.k, self.v, self.o) if bufs is None else bufs
        self.cache.len = w.n_cache
        _mark(ev, "append", 0)
        nm.kvcache_append(self.cache, k[:ns], v[:ns], q_in=q, q_out=self.q_rot,
                          layout=self.layout, cfg=self.cfg)
        _mark(ev, "append", 1)
        if self.frames is not None:
            _mark(ev, "select", 0)
            nm.kvcache_select(self.cache, self.frames, self.window)
            _mark(ev, "select", 1)
            hist = self.window.span()
        else:
            hist = self.cache.span(0, w.n_cache)
        spans = [hist, (k[ns:], v[ns:]), self.cache.span(w.n_cache, w.n_cache + ns)]
        _mark(ev, "attn", 0)
        if self.sparse is not None:
            nm.segment_attention_sparse(self.q_rot, spans, *self.sparse, o=o, lse=self.lse,
                                        dev_err=self.err)
        elif self.head_shards:
            nt = w.n_text
            for g, sl in enumerate(self.head_slices):
                self.q_g[g].copy_(self.q_rot[:, sl])
                self.ks_g[g][:nt].copy_(k[ns:, sl])
                self.vs_g[g][:nt].copy_(v[ns:, sl])
                self.ks_g[g][nt:].copy_(self.cache.k[w.n_cache:w.n_cache + ns, sl])
                self.vs_g[g][nt:].copy_(self.cache.v[w.n_cache:w.n_cache + ns, sl])
                nm.segment_attention(self.q_g[g], [self.hist_g[g], (self.ks_g[g], self.vs_g[g])],
                                     o=self.o_g[g], lse=self.lse_g[g], dev_err=self.err,
                                     kv_splits="auto")
                o[:, sl].copy_(self.o_g[g])
                self.lse.view(16, w.n_q)[sl].copy_(self.lse_g[g].view(-1, w.n_q))
        elif self.shards:
            for r, sub in enumerate(self._shard_spans(spans)):
                nm.segment_attention(self.q_rot, sub, o=self.part_o[r],
                                     lse=self.part_lse[r].view(-1), dev_err=self.err)
            _mark(ev, "merge", 0)
            nm.attention_merge(self.part_o, self.part_lse, o=o, lse=self.lse)
            _mark(ev, "merge", 1)
        else:
            nm.segment_attention(self.q_rot, spans, o=o, lse=self.lse, dev_err=self.err,
                                 kv_splits=self.kv_splits)
        _mark(ev, "attn", 1)


class LayerStepI8:
    """Bounded-history layer-step with the history held in INT8 on the GPU.

    Per step: 3D RoPE of the segment's Q and K into bf16 buffers, the rotated
    K and V quantised into the INT8 cache, the frame list gathered as codes
    and scales into an INT8 window (4,224 B per token), then attention over
    window + text + segment, the window's tiles dequantised inside the
    attention kernel.
    """

    def __init__(self, wname: str, seed: int, window: str = "int8"):
        import torch

        import kv_cached_segment_b200 as nm
        from seeded_inputs import WORKLOADS, bounded_frame_list, randn_bf16

        self.nm, self.torch = nm, torch
        w = self.w = WORKLOADS[wname]
        dev = "cuda"
        ns, nt = w.n_seg, w.n_text
        self.layout = nm.SegLayout(w.frames, w.grid_h, w.grid_w, w.t0, nt)
        self.cfg = nm.RopeConfig(*w.rope_split, w.rope_theta)
        self.window_kind = window if w.select_frames else "int8"
        self.cache = nm.KVCacheI8.empty(w.n_cache + ns, w.tokens_per_frame)
        chunk = 4 * w.tokens_per_frame * 30  # quantise the history in pieces
        for r0 in range(0, w.n_cache, chunk):
            r1 = min(w.n_cache, r0 + chunk)
            hk = randn_bf16((r1 - r0, 16, 128), seed * 16 + 4 + r0, dev)
            hv = randn_bf16((r1 - r0, 16, 128), seed * 16 + 5 + r0, dev)
            nm.kvcache_append_i8(self.cache, hk, hv)
        self.q = randn_bf16((w.n_q, 16, 128), seed * 16 + 1, dev)
        self.k = randn_bf16((w.n_q, 16, 128), seed * 16 + 2, dev)
        self.v = randn_bf16((w.n_q, 16, 128), seed * 16 + 3, dev)
        self.q_rot = torch.empty_like(self.q)
        self.k_rot = torch.empty_like(self.k)
        self.o = torch.empty_like(self.q)
        self.lse = torch.empty(16 * w.n_q, dtype=torch.float32, device=dev)
        self.err = torch.zeros(1, dtype=torch.int32, device=dev)
        # with a frame window: the listed frames gathered as codes and scales;
        # without one, attention reads the INT8 cache's history directly
        self.frames = bounded_frame_list(w, seed).tolist() if w.select_frames else None
        self.window = None
        if w.select_frames:
            self.window = (nm.KVCache.empty(w.n_window, 0) if self.window_kind == "bf16"
                           else nm.KVCacheI8.empty(w.n_window, 0))
        # rope3d_qk, INT8 append, gather (codes and scales: 2 launches; or one
        # dequantising launch), attention
        self.launches_per_step = 3 + (0 if not w.select_frames
                                      else 1 if self.window_kind == "bf16" else 2)
        self.append_kernels = "rope_append_kernel<bf16> (RoPE of Q, K) + rope_append_kernel<int8>"
        self.select_kernel = ("select_i8_kernel (gather + dequantise into bf16)"
                              if self.window_kind == "bf16" else "select_kernel (codes, then scales)")

    def flops(self) -> float:
        return self.w.attention_flops()

    def run(self, ev=None, bufs=None):
        nm, w = self.nm, self.w
        ns = w.n_seg
        q, k, v, o = (self.q, self.k, self.v, self.o) if bufs is None else bufs
        self.cache.len = w.n_cache
        _mark(ev, "append", 0)
        nm.rope3d_qk(q, k, self.q_rot, self.k_rot, self.layout, self.cfg)
        nm.kvcache_append_i8(self.cache, self.k_rot[:ns], v[:ns])
        _mark(ev, "append", 1)
        if self.frames is not None:
            _mark(ev, "select", 0)
            nm.kvcache_select(self.cache, self.frames, self.window)
            _mark(ev, "select", 1)
            hist = self.window.span()
        else:
            hist = self.cache.span(0, w.n_cache)
        spans = [hist, (self.k_rot[ns:], v[ns:]), (self.k_rot[:ns], v[:ns])]
        _mark(ev, "attn", 0)
        nm.segment_attention(self.q_rot, spans, o=o, lse=self.lse, dev_err=self.err)
        _mark(ev, "attn", 1)


def local_key_spans(span_lens, rank: int, world: int, align: int = 128):
    """The rows of each key span that fall in this rank's contiguous share of
    the concatenated key sequence (shares on `align`-key boundaries): a list
    of (span index, first row, end row), in key order, empty spans left out."""
    import kv_cached_segment_b200 as nm

    a, b = nm.shard_rows(int(sum(span_lens)), rank, world, align=align)
    out, base = [], 0
    for s, n in enumerate(span_lens):
        lo, hi = max(a, base), min(b, base + n)
        if hi > lo:
            out.append((s, lo - base, hi - base))
        base += n
    return out


class ShardedLayerStep:
    """A layer-step with its keys spread over the ranks (key-sharded attention,
    as the pages' standard preset spreads the cache over eight GPUs).

    Every rank holds a contiguous 1/N of the key sequence (history, then
    text, then segment keys; shares on 128-key tiles) and all query rows.  Per
    step each rank runs the fused RoPE + append of the segment (the rotated Q
    and the segment's keys and values), attends with every query over its own
    keys into a partial (O, LSE), all-gathers the partials over NCCL and
    merges them (sharded_segment_attention).  The whole job computes one
    layer-step: total work is fixed as N grows.
    """

    def __init__(self, wname: str, seed: int, rank: int, world: int):
        import torch

        import kv_cached_segment_b200 as nm
        from seeded_inputs import WORKLOADS, randn_bf16

        self.nm, self.torch = nm, torch
        w = self.w = WORKLOADS[wname]
        if w.select_frames:
            raise SystemExit("key-sharded steps use a workload without a frame window")
        dev = "cuda"
        ns, nt = w.n_seg, w.n_text
        self.rank, self.world = rank, world
        self.layout = nm.SegLayout(w.frames, w.grid_h, w.grid_w, w.t0, nt)
        self.cfg = nm.RopeConfig(*w.rope_split, w.rope_theta)
        # the same seeded inputs on every rank; each keeps only its share of
        # the history
        self.local = local_key_spans([w.n_cache, nt, ns], rank, world)
        self.hist = None
        for s, lo, hi in self.local:
            if s == 0:
                hk = randn_bf16((w.n_cache, 16, 128), seed * 16 + 4, dev)[lo:hi].clone()
                hv = randn_bf16((w.n_cache, 16, 128), seed * 16 + 5, dev)[lo:hi].clone()
                self.hist = (hk, hv)
        torch.cuda.empty_cache()
        self.seg = nm.KVCache.empty(ns, w.tokens_per_frame)
        self.q = randn_bf16((w.n_q, 16, 128), seed * 16 + 1, dev)
        self.k = randn_bf16((w.n_q, 16, 128), seed * 16 + 2, dev)
        self.v = randn_bf16((w.n_q, 16, 128), seed * 16 + 3, dev)
        self.q_rot = torch.empty_like(self.q)
        self.o = torch.empty_like(self.q)
        self.lse = torch.empty(16 * w.n_q, dtype=torch.float32, device=dev)
        self.err = torch.zeros(1, dtype=torch.int32, device=dev)
        self.frames = None
        # append, attention over the local share, two all-gathers (NCCL), merge
        self.launches_per_step = 3
        self.append_kernels = "rope_append_kernel<bf16> (fused RoPE + append)"
        self.shards = world

    def flops(self) -> float:
        return self.w.attention_flops()  # of the whole job: every rank does 1/N

    def local_flops(self) -> float:
        keys = sum(hi - lo for _, lo, hi in self.local)
        return 4.0 * self.w.n_q * keys * 128 * 16

    def spans(self, k, v):
        w, ns = self.w, self.w.n_seg
        out = []
        for s, lo, hi in self.local:
            if s == 0:
                out.append(self.hist)
            elif s == 1:
                out.append((k[ns + lo:ns + hi], v[ns + lo:ns + hi]))
            else:
                out.append(self.seg.span(lo, hi))
        return out

    def run(self, ev=None, bufs=None):
        nm, w = self.nm, self.w
        ns = w.n_seg
        q, k, v, o = (self.q, self.k, self.v, self.o) if bufs is None else bufs
        self.seg.len = 0
        _mark(ev, "append", 0)
        nm.kvcache_append(self.seg, k[:ns], v[:ns], q_in=q, q_out=self.q_rot, layout=self.layout,
                          cfg=self.cfg)
        _mark(ev, "append", 1)
        _mark(ev, "attn", 0)
        nm.sharded_segment_attention(
            self.q_rot, self.spans(k, v), lse=self.lse,
            merge=lambda op, lp, lse: nm.attention_merge(op, lp, o=o, lse=lse))
        _mark(ev, "attn", 1)


class SweepStep:
    """One denoising step of a whole segment: 54 layers of the 720p layer-step.

    Every layer has its own resident cache of 55,200 tokens plus 512 text
    tokens; each step uses fresh seeded Q and segment K/V (one set per
    denoising step, 8 sets).  Per layer: 3D RoPE of Q and the segment K into
    bf16 buffers, then attention over cache + text + segment.
    """

    def __init__(self, seed: int, layers: int | None = None):
        import torch

        import kv_cached_segment_b200 as nm
        from seeded_inputs import SWEEP_LAYERS, SWEEP_STEPS, WORKLOADS, randn_bf16

        self.nm, self.torch = nm, torch
        w = self.w = WORKLOADS["720p"]
        dev = "cuda"
        ns, nt = w.n_seg, w.n_text
        self.seed = seed
        self.layers = SWEEP_LAYERS if layers is None else layers
        self.steps_per_segment = SWEEP_STEPS
        self.cfg = nm.RopeConfig(*w.rope_split, w.rope_theta)
        # text rows of Q are copied by the RoPE pass; text K/V live with each layer
        self.lay_q = nm.SegLayout(w.frames, w.grid_h, w.grid_w, w.t0, nt)
        self.lay_k = nm.SegLayout(w.frames, w.grid_h, w.grid_w, w.t0, 0)
        self.cache = []
        for l in range(self.layers):
            k = randn_bf16((w.n_cache + nt, 16, 128), self.cache_seed(l, 0), dev)
            v = randn_bf16((w.n_cache + nt, 16, 128), self.cache_seed(l, 1), dev)
            self.cache.append((k, v))
        self.inputs = [tuple(randn_bf16((w.n_q if i == 0 else ns, 16, 128),
                                        self.input_seed(s, i), dev) for i in range(3))
                       for s in range(self.steps_per_segment)]
        self.q_rot = torch.empty((w.n_q, 16, 128), dtype=torch.bfloat16, device=dev)
        self.k_rot = torch.empty((ns, 16, 128), dtype=torch.bfloat16, device=dev)
        self.o = torch.empty_like(self.q_rot)
        self.lse = torch.empty(16 * w.n_q, dtype=torch.float32, device=dev)
        self.err = torch.zeros(1, dtype=torch.int32, device=dev)
        self.i = 0
        self.launches_per_step = 3 * self.layers

    def cache_seed(self, layer: int, which: int) -> int:
        """Seed of layer `layer`'s resident K (which 0) or V (1), text rows last."""
        return self.seed * 1000 + 2 * layer + which

    def input_seed(self, step: int, which: int) -> int:
        """Seed of denoising step `step`'s Q (which 0), segment K (1), V (2)."""
        return self.seed * 100000 + 3 * step + which

    def flops(self) -> float:
        return self.w.attention_flops() * self.layers

    def spans(self, layer: int, v):
        """Key/value spans of one layer: its cached rows, the text rows stored
        with it, then the segment's rotated K (in k_rot) and its V."""
        w = self.w
        ck, cv = self.cache[layer]
        return [(ck[:w.n_cache], cv[:w.n_cache]), (ck[w.n_cache:], cv[w.n_cache:]),
                (self.k_rot, v)]

    def run_layer(self, layer: int, q, k, v, lse=None):
        nm = self.nm
        nm.rope3d_qk(q, None, self.q_rot, None, self.lay_q, self.cfg)
        nm.rope3d_qk(k, None, self.k_rot, None, self.lay_k, self.cfg)
        nm.segment_attention(self.q_rot, self.spans(layer, v), o=self.o, lse=lse,
                             dev_err=self.err)

    def run(self, ev=None):
        q, k, v = self.inputs[self.i % self.steps_per_segment]
        self.i += 1
        _mark(ev, "attn", 0)
        for layer in range(self.layers):
            self.run_layer(layer, q, k, v)
        _mark(ev, "attn", 1)


def max_over_ranks(values, world: int, device):
    """Element-wise max of per-rank floats over all ranks (identity at world 1)."""
    if world <= 1:
        return [float(x) for x in values]
    import torch
    import torch.distributed as dist

    t = torch.tensor([float(x) for x in values], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(x) for x in t.tolist()]


def rotated_query_rows(oracle, q_rows, rows, n_video: int, t, h, ww, split=(32, 48, 48),
                       theta: float = 10000.0):
    """The oracle's RoPE of sampled query rows (sorted, so video rows come
    first); text rows (index >= n_video) pass unrotated."""
    nv = int(np.count_nonzero(rows < n_video))
    vid = rows[:nv]
    return oracle.rope3d(q_rows, nv, t[vid], h[vid], ww[vid], split=split, theta=theta)


def parity_summary(err_o, err_l, rows: int) -> dict:
    parity = {"rows": rows, "max_abs_o": float(err_o.max()), "mean_abs_o": float(err_o.mean()),
              "max_abs_lse": float(err_l.max()), "bar_max_abs": 2e-2, "bar_mean_abs": 2e-3}
    parity["pass"] = bool(parity["max_abs_o"] <= 2e-2 and parity["mean_abs_o"] <= 2e-3
                          and parity["max_abs_lse"] <= 2e-2)
    return parity


def sweep_parity(step, layer: int, n_rows: int = 24) -> dict:
    """Runs one layer of the sweep (denoising step 0's inputs) and compares
    sampled query rows, the first and last text rows among them, with the
    fp64 oracle over that layer's spans built from the seeded inputs."""
    import numpy as np
    import torch

    import oracle

    def f64(x):
        b = x.detach().contiguous().cpu().view(torch.int16).numpy().view(np.uint16)
        return oracle.bf16_bits_to_f64(b)

    w = step.w
    ns = w.n_seg
    q, k, v = step.inputs[0]
    step.run_layer(layer, q, k, v, lse=step.lse)
    torch.cuda.synchronize()
    # the oracle starts from host copies of the seeded inputs (the layer's
    # resident cache with its text rows, the step's Q, K, V), never from a
    # kernel's output
    ck, cv = (f64(x) for x in step.cache[layer])
    qh, kh, vh = f64(q), f64(k), f64(v)
    t, h, ww = oracle.video_positions(w.frames, w.grid_h, w.grid_w, w.t0)
    spans = [(ck[:w.n_cache], cv[:w.n_cache]), (ck[w.n_cache:], cv[w.n_cache:]),
             (oracle.rope3d(kh, ns, t, h, ww), vh)]
    rows = np.random.default_rng(layer).integers(0, w.n_q, n_rows)
    rows = np.unique(np.concatenate([rows, [0, ns - 1, ns, w.n_q - 1]]))
    o_ref, l_ref = oracle.attention(rotated_query_rows(oracle, qh[rows], rows, ns, t, h, ww), spans)
    err_o = np.abs(f64(step.o[torch.as_tensor(rows)]) - o_ref)
    lse = step.lse.view(16, w.n_q).cpu().numpy().astype(np.float64)[:, rows]
    out = parity_summary(err_o, np.abs(lse - l_ref), int(rows.size))
    out["layer"] = layer
    return out


def cpu_oracle_rate(step, budget_s: float, rows_per_chunk: int, max_rows: int):
    """Times the fp64 oracle (RoPE of sampled query rows + their attention over
    every key of the workload) on host cores; returns (TFLOP/s, rows, s,
    threads, parity).

    The oracle works from the seeded inputs (host copies of the resident
    cache, the frame list and the segment), never from kernel outputs.  The
    sampled rows of the step's last output are then compared with the
    oracle's (`parity`: max and mean absolute error of O and LSE)."""
    import numpy as np
    import torch

    import oracle

    def f64(t):
        b = t.detach().contiguous().cpu().view(torch.int16).numpy().view(np.uint16)
        return oracle.bf16_bits_to_f64(b)

    w = step.w
    ns = w.n_seg
    hist_k, hist_v = f64(step.cache.k[:w.n_cache]), f64(step.cache.v[:w.n_cache])
    if w.select_frames:
        hist_k = oracle.kvcache_select(hist_k, step.frames, w.tokens_per_frame)
        hist_v = oracle.kvcache_select(hist_v, step.frames, w.tokens_per_frame)
    t, h, ww = oracle.video_positions(w.frames, w.grid_h, w.grid_w, w.t0)
    spans = [(hist_k, hist_v), (f64(step.k[ns:]), f64(step.v[ns:])),
             (oracle.rope3d(f64(step.k[:ns]), ns, t, h, ww), f64(step.v[:ns]))]
    q_all = step.q
    rng = np.random.default_rng(0)
    done, elapsed = 0, 0.0
    refs = []
    t0 = time.perf_counter()
    while elapsed < budget_s and done < max_rows:
        # every query row, text rows included (the last n_text rows)
        rows = np.sort(rng.integers(0, w.n_q, rows_per_chunk))
        if not refs:
            rows[0], rows[-1] = ns, w.n_q - 1  # first and last text rows
            rows = np.sort(rows)
        q_rows = rotated_query_rows(oracle, f64(q_all[torch.as_tensor(rows)]), rows, ns, t, h, ww)
        refs.append((rows, oracle.attention(q_rows, spans)))
        done += rows.size
        elapsed = time.perf_counter() - t0
    flops = 4.0 * done * w.n_k * 128 * 16
    # parity of the step's output on the sampled rows (outside the timing)
    err_o = np.concatenate([np.abs(f64(step.o[torch.as_tensor(r)]) - o).ravel()
                            for r, (o, _) in refs])
    lse_gpu = step.lse.view(16, w.n_q).cpu().numpy().astype(np.float64)
    err_l = np.concatenate([np.abs(lse_gpu[:, r] - lse).ravel() for r, (_, lse) in refs])
    parity = parity_summary(err_o, err_l, done)
    parity["text_rows"] = int(sum(np.count_nonzero(r >= ns) for r, _ in refs))
    return flops / elapsed / 1e12, done, elapsed, blas_threads(), parity


def cpu_model() -> str:
    """The host CPU's model name and logical core count."""
    name = "unknown CPU"
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    name = line.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    return f"{name}, {os.cpu_count()} logical cores"


def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        return max((i.get("num_threads", 1) for i in threadpool_info()), default=1)
    except Exception:  # noqa: BLE001
        return os.cpu_count() or 1


def make_step(args, rank, world=1):
    if args.key_shards > 0 and args.key_shards == world:
        if args.sparse > 0 or args.int8 or args.workload == "sweep" or args.kv_splits != "1":
            raise SystemExit("--key-shards across ranks runs the dense bf16 layer-step only")
        # one seed for all ranks: together they compute one layer-step
        return ShardedLayerStep(args.workload, seed=1, rank=rank, world=world)
    if args.key_shards > 0 and world > 1:
        raise SystemExit("--key-shards across ranks must equal the number of GPUs")
    if args.workload == "sweep":
        return SweepStep(seed=1 + rank)
    if args.int8:
        return LayerStepI8(args.workload, seed=1 + rank, window=args.int8_window)
    step = LayerStep(args.workload, seed=1 + rank)
    if args.sparse > 0:
        step.use_sparse(args.sparse, seed=1 + rank)
    if args.key_shards > 0:
        if args.sparse > 0:
            raise SystemExit("--key-shards and --sparse are exclusive")
        step.use_key_shards(args.key_shards)
    if args.head_shards > 0:
        if world > 1 or args.sparse > 0 or args.key_shards > 0 or args.kv_splits != "1":
            raise SystemExit("--head-shards runs on one GPU, dense, without key shards or "
                             "--kv-splits (each launch picks its own)")
        step.use_head_shards(args.head_shards)
    if args.kv_splits != "1":
        if not isinstance(step, LayerStep) or step.sparse is not None or step.shards:
            raise SystemExit("--kv-splits applies to the dense bf16 layer-step only")
        step.kv_splits = args.kv_splits if args.kv_splits == "auto" else int(args.kv_splits)
        if step.kv_splits == "auto":
            w = step.w
            hist = w.n_window if w.select_frames else w.n_cache
            step.kv_splits = step.nm.auto_kv_splits(
                w.n_q, [hist, w.n_text, w.n_seg],
                step.torch.cuda.get_device_properties(0).multi_processor_count)
        step.launches_per_step += 1 if step.kv_splits > 1 else 0  # the merge
    return step


def workload_text(args, step) -> str:
    w = step.w
    if args.workload == "sweep":
        return (f"sweep: {step.layers} layers x one denoising step of the 720p layer-step "
                f"({w.frames}x{w.grid_h}x{w.grid_w} segment + {w.n_text} text over "
                f"{w.n_cache} cached tokens per layer)")
    hist = w.n_window if w.select_frames else w.n_cache
    extra = ""
    if args.int8:
        extra = (" (history in INT8; gathered frames dequantised once into a bf16 window)"
                 if w.select_frames and getattr(args, "int8_window", "int8") == "bf16"
                 else " (history in INT8, dequantised in the attention kernel)")
    if getattr(step, "kv_splits", 1) > 1:
        extra += f" (keys split {step.kv_splits} ways per query block, partials merged)"
    if getattr(args, "key_shards", 0) > 0:
        extra += (f" (keys split into {args.key_shards} contiguous shards, partial results "
                  f"merged)")
    if getattr(args, "head_shards", 0) > 0:
        extra += (f" (heads split into {args.head_shards} launches of "
                  f"{16 // args.head_shards} heads, rows copied to head-sliced buffers and back)")
    if args.sparse > 0:
        extra += (f" (block-sparse: text kept, {100 * args.sparse:.0f}% of video key tiles "
                  f"per 256-query block and head)")
    return (f"{w.name}: {w.frames}x{w.grid_h}x{w.grid_w} segment tokens + {w.n_text} text "
            f"over {hist} history tokens{extra}")


def main():
    args = parse_args()
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        return run_reference(args, rank, world)

    import torch
    import torch.distributed as dist

    torch.cuda.set_device(local_rank)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=300),
                                device_id=torch.device("cuda", local_rank))

    def barrier():
        if world > 1:
            dist.barrier()

    peaks, peak_src = load_peaks()
    step = make_step(args, rank, world)
    sharded = isinstance(step, ShardedLayerStep)
    torch.cuda.synchronize()

    warmup = max(3, args.warmup)
    for _ in range(warmup):
        step.run()
    torch.cuda.synchronize()
    if int(step.err.item()) != 0:
        raise RuntimeError(f"device error word {int(step.err.item())}")

    uuid = None
    try:
        uuid = str(torch.cuda.get_device_properties(local_rank).uuid)
        uuid = uuid if uuid.startswith("GPU-") else "GPU-" + uuid
    except Exception:  # noqa: BLE001
        uuid = None
    sampler = ClockSampler(uuid) if rank == 0 else None
    time.sleep(0.3 if sampler else 0)

    def ev_pair():
        return (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))

    timed = step_kernels(step)
    evs = [{name: ev_pair() for name in timed} for _ in range(args.steps)]
    start, stop = ev_pair()
    barrier()
    torch.cuda.synchronize()
    start.record()
    for i in range(args.steps):
        step.run(evs[i])
    stop.record()
    torch.cuda.synchronize()
    barrier()
    clocks = sampler.stop() if sampler else None
    if int(step.err.item()) != 0:
        raise RuntimeError(f"device error word {int(step.err.item())}")

    def mean_ms(name):
        if name not in timed:
            return 0.0
        return statistics.mean(e[name][0].elapsed_time(e[name][1]) for e in evs)

    ms, attn_ms, merge_ms, append_ms, select_ms = max_over_ranks(
        [start.elapsed_time(stop), mean_ms("attn"), mean_ms("merge"), mean_ms("append"),
         mean_ms("select")], world, "cuda")
    attn_ms -= merge_ms  # attention launches only
    ms_per_step = ms / args.steps
    flops = step.flops()
    # replicas: every rank computes a layer-step; key shards: all ranks
    # together compute one
    jobs = 1 if sharded else world
    value = flops * args.steps * jobs / (ms / 1e3) / 1e12
    attn_tflops = flops / (attn_ms / 1e3) / 1e12
    hbm = peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"])

    # The memory-bound kernels against the copy bandwidth: the append (or
    # RoPE + INT8 append) timed inside the steps above; the frame gather
    # inside the steps when the workload has one, else a gather of every
    # cached frame timed here on its own.
    roof_append = roof_select = None
    if "append" in timed:
        a_bytes = append_bytes(step)
        roof_append = memory_roofline(step.append_kernels, a_bytes, append_ms, hbm, peak_src,
                                      "inside the timed steps")
    if "select" in timed:
        roof_select = memory_roofline(step.select_kernel, select_bytes(step, step.w.n_window),
                                      select_ms, hbm, peak_src, "inside the timed steps")
    elif isinstance(step, (LayerStep, ShardedLayerStep)) and not sharded:
        sel_ms, n_tok = time_full_gather(step, repeats=20)
        (sel_ms,) = max_over_ranks([sel_ms], world, "cuda")
        roof_select = memory_roofline("select_kernel", select_bytes(step, n_tok), sel_ms, hbm,
                                      peak_src, f"gather of all {n_tok // step.w.tokens_per_frame} "
                                      f"cached frames ({n_tok} tokens) in a seeded order, mean "
                                      f"of 20 launches timed alone")

    # ---- end to end through the public API with host buffers: every step
    # copies its inputs from pinned host memory and reads its output back;
    # two buffer sets and two copy streams overlap step i+1's upload and step
    # i-1's download with step i's kernels.
    e2e = None
    if not args.no_e2e and args.workload != "sweep" and not sharded:
        pipe = E2EPipeline(step)
        pipe.run(2)
        torch.cuda.synchronize()
        barrier()
        n_e2e = max(3, min(args.steps, 20))
        e_ms = pipe.run(n_e2e)
        (e_ms,) = max_over_ranks([e_ms], world, "cuda")
        e2e = {"value": flops * n_e2e * world / (e_ms / 1e3) / 1e12, "unit": UNIT,
               "h2d_bytes_per_step": pipe.h2d_bytes, "d2h_bytes_per_step": pipe.d2h_bytes,
               "ms_per_step": e_ms / n_e2e, "steps": n_e2e,
               "overlap": "double-buffered inputs/outputs, separate H2D and D2H streams"}

    cpu = None
    parity = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline and isinstance(step, LayerStep):
        rate, rows, secs, threads, parity = cpu_oracle_rate(step, budget_s=12.0,
                                                            rows_per_chunk=16, max_rows=512)
        cpu = {"value": rate, "unit": UNIT, "cores": threads, "kind": "oracle", "host": cpu_model(),
               "sample": f"fp64 oracle RoPE + attention of {rows} sampled query rows (segment "
                         f"and text) x 16 heads over all {step.w.n_k} keys ({secs:.1f} s)"}
        if step.sparse is not None:
            parity = None  # the oracle above is dense attention
    elif rank == 0 and world == 1 and not args.no_cpu_baseline and args.workload == "sweep":
        parity = [sweep_parity(step, 0), sweep_parity(step, step.layers - 1)]

    if world > 1:
        dist.destroy_process_group()
    if rank != 0:
        return

    # burst peak for a kernel timed over well under a second of steps; the
    # seconds-long sweep runs under the power cap: its sustained peak
    peak_kind = "sustained" if args.workload == "sweep" else "burst"
    peak = (peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"])
            if peak_kind == "sustained" else peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    w = step.w
    attn_per_step = getattr(step, "layers", 1)
    out = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
        "scaling": "strong" if sharded else "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": workload_config(args, step, world),
        # per GPU: value is the whole job's aggregate over `world` GPUs
        "pct_of_measured_bf16_peak": 100.0 * value / world / peak,
        "pct_of_datasheet_bf16_peak": 100.0 * value / world / DATASHEET_BF16_TFLOPS,
        "attention_ms": attn_ms / attn_per_step,
        "roofline": {"kernel": "attention_kernel", "bound": "tensor",
                     "achieved": attn_tflops, "peak": peak, "unit": "TFLOP/s",
                     "frac": attn_tflops / peak, "peak_source": f"{peak_src} bf16 {peak_kind}",
                     "traffic": recorded_traffic(args.workload)},
        "roofline_append": roof_append, "roofline_select": roof_select,
        "cpu_baseline": cpu, "e2e": e2e, "parity": parity,
        "gpu_launches": step.launches_per_step * args.steps * world,  # all ranks
        "clocks": clocks,
    }
    n_shards = getattr(step, "shards", 0)
    if sharded:
        # attention_ms holds this rank's partial attention, the two
        # all-gathers and the merge; the roofline counts this rank's keys
        loc = step.local_flops()
        out["roofline"].update({"achieved": loc / (attn_ms / 1e3) / 1e12,
                                "frac": loc / (attn_ms / 1e3) / 1e12 / peak,
                                "note": "per rank: partial attention over its key share + NCCL "
                                        "all-gather of the partials + merge"})
    elif n_shards:
        # merge: R partial O rows (+ LSE) read, one O row (+ LSE) written per query row
        mbytes = (n_shards + 1) * w.n_q * (16 * 128 * 2 + 16 * 4)
        out["merge"] = memory_roofline("merge_kernel", mbytes, merge_ms, hbm, peak_src,
                                       "inside the timed steps")
    if args.workload == "sweep":
        out["ms_per_segment"] = ms_per_step * step.steps_per_segment
        out["roofline"]["note"] = "per-step average over the 54 layers (rope3d_qk launches included)"
    print(json.dumps(out), flush=True)


def step_kernels(step) -> list:
    """Names of the launch groups a step records events around."""
    if isinstance(step, SweepStep):
        return ["attn"]
    if isinstance(step, ShardedLayerStep):
        return ["append", "attn"]
    names = ["append", "attn"]
    if getattr(step, "frames", None) is not None:
        names.append("select")
    if getattr(step, "shards", 0):
        names.append("merge")
    return names


def append_bytes(step) -> float:
    """Algorithmic HBM bytes of a step's append group.

    Fused RoPE + append: 24 KiB per video token (Q, K, V read; Q', K', V
    written) + 8 KiB per text row of Q (read and written).  INT8 path:
    RoPE of every Q and K row (16 KiB per row), then the quantising append of
    the video rows (K', V read: 8 KiB; codes + scales written: 4,224 B)."""
    w = step.w
    if isinstance(step, LayerStepI8):
        return float(w.n_q * 16384 + w.n_seg * (8192 + 4224))
    return float(w.n_seg * 24576 + w.n_text * 8192)


def select_bytes(step, n_tokens: int) -> float:
    """Frame gather: 16 KiB per token (K and V rows read and written); from
    an INT8 cache into an INT8 window, 4,224 B read and written per token
    (codes and scales of K and V); dequantising into a bf16 window, 4,224 B
    read and 8 KiB written."""
    if isinstance(step, LayerStepI8):
        if step.window_kind == "bf16":
            return float(n_tokens * (4224 + 8192))
        return float(n_tokens * 2 * 4224)
    return float(n_tokens * 16384)


def memory_roofline(kernel: str, nbytes: float, ms: float, hbm: float, peak_src: str,
                    how: str) -> dict:
    achieved = nbytes / (ms / 1e3) / 1e9
    return {"kernel": kernel, "bound": "hbm", "bytes": nbytes, "ms": ms, "achieved": achieved,
            "peak": hbm, "unit": "GB/s", "frac": achieved / hbm,
            "peak_source": f"{peak_src} copy bandwidth", "timed": how}


def time_full_gather(step, repeats: int):
    """Mean time of gathering every cached frame (seeded order) into a window."""
    import torch

    w = step.w
    frames = np.random.default_rng(11).permutation(w.cache_frames).astype(np.int32).tolist()
    window = step.nm.KVCache.empty(w.n_cache, 0)
    step.cache.len = w.n_cache
    for _ in range(3):
        step.nm.kvcache_select(step.cache, frames, window)
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(repeats)]
    torch.cuda.synchronize()
    for a, b in evs:
        a.record()
        step.nm.kvcache_select(step.cache, frames, window)
        b.record()
    torch.cuda.synchronize()
    ms = statistics.mean(a.elapsed_time(b) for a, b in evs)
    del window
    return ms, w.n_cache


def workload_config(args, step, world: int) -> dict:
    """The `config` object of the JSON line, the same for both arms."""
    w = step.w
    attn_per_step = getattr(step, "layers", 1)
    cfg = {
        "workload": workload_text(args, step),
        "n_q": w.n_q, "n_k": w.n_k, "heads": 16, "head_dim": 128,
        "attention_flops_per_step": w.attention_flops() * attn_per_step,
        "step": ("per layer: rope3d_qk x2 + segment attention" if args.workload == "sweep"
                 else "rope3d_qk + int8 append + " + (
                     ("dequantising select + segment attention over the bf16 window"
                      if getattr(args, "int8_window", "int8") == "bf16" else
                      "int8 select + segment attention over the int8 window")
                     if w.select_frames else "segment attention over the int8 history")
                 if args.int8
                 else "fused rope3d+append" + (" + select" if w.select_frames else "")
                 + " + segment attention"),
        "l2": "inputs larger than L2: each step reads "
              f"{attn_per_step * (w.n_q * 3 + w.n_k * 2) * 4096 / 1e9:.2f} GB > 126 MB",
        "parallelism": (f"keys sharded over {world} GPUs (partials all-gathered over NCCL and "
                        f"merged)" if isinstance(step, ShardedLayerStep)
                        else f"independent layer-step per GPU x{world}"),
    }
    if getattr(args, "key_shards", 0):
        cfg["key_shards"] = args.key_shards
    if getattr(args, "head_shards", 0):
        cfg["head_shards"] = args.head_shards
    return cfg


class E2EPipeline:
    """End-to-end steps through the public API from pinned host buffers."""

    def __init__(self, step):
        import torch

        self.torch, self.step = torch, step
        self.host_in = [{n: getattr(step, n).cpu().pin_memory() for n in ("q", "k", "v")}
                        for _ in range(2)]
        self.host_o = [torch.empty_like(step.o, device="cpu").pin_memory() for _ in range(2)]
        self.dev = [(step.q, step.k, step.v, step.o),
                    (torch.empty_like(step.q), torch.empty_like(step.k),
                     torch.empty_like(step.v), torch.empty_like(step.o))]
        self.h2d_bytes = sum(x.numel() * x.element_size() for x in self.host_in[0].values())
        self.d2h_bytes = step.o.numel() * step.o.element_size()
        self.s_h2d = torch.cuda.Stream()
        self.s_d2h = torch.cuda.Stream()

    def run(self, n: int) -> float:
        """Runs n steps; returns elapsed ms from the first upload to the last download."""
        torch = self.torch
        comp = torch.cuda.current_stream()
        ev = lambda: torch.cuda.Event(enable_timing=False)  # noqa: E731
        in_ready = [ev(), ev()]
        done = [ev(), ev()]
        out_read = [ev(), ev()]
        start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        start.record(comp)
        self.s_h2d.wait_event(start)
        self.s_d2h.wait_event(start)

        def upload(i):
            b = i % 2
            with torch.cuda.stream(self.s_h2d):
                if i >= 2:
                    self.s_h2d.wait_event(done[b])  # step i-2 no longer reads buffer b
                q, k, v, _ = self.dev[b]
                q.copy_(self.host_in[b]["q"], non_blocking=True)
                k.copy_(self.host_in[b]["k"], non_blocking=True)
                v.copy_(self.host_in[b]["v"], non_blocking=True)
                in_ready[b].record(self.s_h2d)

        upload(0)
        for i in range(n):
            b = i % 2
            if i + 1 < n:
                upload(i + 1)
            comp.wait_event(in_ready[b])
            if i >= 2:
                comp.wait_event(out_read[b])  # step i-2's output has been read back
            self.step.run(bufs=self.dev[b])
            done[b].record(comp)
            with torch.cuda.stream(self.s_d2h):
                self.s_d2h.wait_event(done[b])
                self.host_o[b].copy_(self.dev[b][3], non_blocking=True)
                out_read[b].record(self.s_d2h)
        stop.record(self.s_d2h)
        torch.cuda.synchronize()
        return start.elapsed_time(stop)


def run_reference(args, rank, world):
    """The fp64 CPU oracle as it stands, on the same workload, metric and unit."""
    if rank != 0:
        return
    import numpy as np
    import torch

    import oracle
    from seeded_inputs import WORKLOADS, layer_inputs

    w = WORKLOADS["720p" if args.workload == "sweep" else args.workload]
    inp = layer_inputs(w, seed=1)

    def f64(t):
        b = t.detach().contiguous().view(torch.int16).numpy().view(np.uint16)
        return oracle.bf16_bits_to_f64(b)

    ns = w.n_seg
    t, h, ww = oracle.video_positions(w.frames, w.grid_h, w.grid_w, w.t0)
    hist_k, hist_v = f64(inp["cache_k"]), f64(inp["cache_v"])
    if w.select_frames:
        from seeded_inputs import bounded_frame_list
        idx = bounded_frame_list(w, 1)
        hist_k = oracle.kvcache_select(hist_k, idx, w.tokens_per_frame)
        hist_v = oracle.kvcache_select(hist_v, idx, w.tokens_per_frame)
    k_seg = oracle.rope3d(f64(inp["k"][:ns]), ns, t, h, ww)
    spans = [(hist_k, hist_v), (f64(inp["k"][ns:]), f64(inp["v"][ns:])), (k_seg, f64(inp["v"][:ns]))]
    q_all = inp["q"]
    rows_per_step = 8
    rng = np.random.default_rng(0)

    def one_step():
        rows = np.sort(rng.integers(0, w.n_q, rows_per_step))  # segment and text rows
        q_rows = rotated_query_rows(oracle, f64(q_all[torch.as_tensor(rows)]), rows, ns, t, h, ww)
        oracle.attention(q_rows, spans)

    for _ in range(max(3, args.warmup)):
        one_step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        one_step()
    secs = time.perf_counter() - t0
    flops = 4.0 * rows_per_step * w.n_k * 128 * 16 * args.steps
    value = flops / secs / 1e12
    try:
        from threadpoolctl import threadpool_info
        threads = max((i.get("num_threads", 1) for i in threadpool_info()), default=1)
    except Exception:  # noqa: BLE001
        threads = os.cpu_count()
    out = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": max(3, args.warmup),
        "ms_per_step": secs * 1e3 / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        # the same workload and config as the CUDA arm's line; what this arm
        # ran (host cores, a row sample) is in cpu_baseline
        "config": workload_config(args, types.SimpleNamespace(w=w, kv_splits=1), world),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle",
                         "host": cpu_model(), "memory": "host memory, one process",
                         "sample": f"fp64 oracle RoPE + attention of {rows_per_step} sampled "
                                   f"query rows (segment and text) per step x 16 heads over all "
                                   f"{w.n_k} keys, {args.steps} steps"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(out), flush=True)


if __name__ == "__main__":
    main()
