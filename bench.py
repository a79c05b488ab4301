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
scaling, no collective on the data path); timing is the max over ranks.
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
                   help="bounded workload with an INT8 history cache (quantising append, "
                        "dequantising gather)")
    p.add_argument("--sparse", type=float, default=0.0,
                   help="block-sparse attention keeping this fraction of the video key tiles "
                        "(text tiles always kept); 0 = dense")
    p.add_argument("--key-shards", type=int, default=0,
                   help="split the key sequence into this many contiguous shards, attend over "
                        "each into a partial (O, LSE) and merge them (the per-GPU work of "
                        "key-sharded attention, on one GPU); 0 = one launch over all keys")
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
    for name in ("attention.cu", "f32x2.cuh", "tmem_ops.cuh", "nomas_internal.h"):
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
        self.sparse = None
        self.shards = 0
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
        self.merge_ev = []
        self.launches_per_step += n_shards  # n_shards attention launches + 1 merge, was 1

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
        nm, w = self.nm, self.w
        ns = w.n_seg
        q, k, v, o = (self.q, self.k, self.v, self.o) if bufs is None else bufs
        self.cache.len = w.n_cache
        nm.kvcache_append(self.cache, k[:ns], v[:ns], q_in=q, q_out=self.q_rot,
                          layout=self.layout, cfg=self.cfg)
        if self.frames is not None:
            nm.kvcache_select(self.cache, self.frames, self.window)
            hist = self.window.span()
        else:
            hist = self.cache.span(0, w.n_cache)
        spans = [hist, (k[ns:], v[ns:]), self.cache.span(w.n_cache, w.n_cache + ns)]
        if ev is not None:
            ev[0].record()
        if self.sparse is not None:
            nm.segment_attention_sparse(self.q_rot, spans, *self.sparse, o=o, lse=self.lse,
                                        dev_err=self.err)
        elif self.shards:
            for r, sub in enumerate(self._shard_spans(spans)):
                nm.segment_attention(self.q_rot, sub, o=self.part_o[r],
                                     lse=self.part_lse[r].view(-1), dev_err=self.err)
            if ev is not None:
                mev = (self.torch.cuda.Event(enable_timing=True),
                       self.torch.cuda.Event(enable_timing=True))
                mev[0].record()
            nm.attention_merge(self.part_o, self.part_lse, o=o, lse=self.lse)
            if ev is not None:
                mev[1].record()
                self.merge_ev.append(mev)
        else:
            nm.segment_attention(self.q_rot, spans, o=o, lse=self.lse, dev_err=self.err,
                                 kv_splits=self.kv_splits)
        if ev is not None:
            ev[1].record()


class LayerStepI8:
    """Bounded-history layer-step with an INT8 history cache.

    Per step: 3D RoPE of the segment's Q and K into bf16 buffers, the rotated
    K and V quantised into the INT8 cache, the frame list gathered back to a
    bf16 window, then attention over window + text + segment.
    """

    def __init__(self, wname: str, seed: int):
        import torch

        import kv_cached_segment_b200 as nm
        from seeded_inputs import WORKLOADS, bounded_frame_list, randn_bf16

        self.nm, self.torch = nm, torch
        w = self.w = WORKLOADS[wname]
        if not w.select_frames:
            raise SystemExit("--int8 needs the bounded workload")
        dev = "cuda"
        ns, nt = w.n_seg, w.n_text
        self.layout = nm.SegLayout(w.frames, w.grid_h, w.grid_w, w.t0, nt)
        self.cfg = nm.RopeConfig(*w.rope_split, w.rope_theta)
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
        self.frames = bounded_frame_list(w, seed).tolist()
        self.window = nm.KVCache.empty(w.n_window, 0)
        self.launches_per_step = 4

    def flops(self) -> float:
        return self.w.attention_flops()

    def run(self, ev=None, bufs=None):
        nm, w = self.nm, self.w
        ns = w.n_seg
        q, k, v, o = (self.q, self.k, self.v, self.o) if bufs is None else bufs
        self.cache.len = w.n_cache
        nm.rope3d_qk(q, k, self.q_rot, self.k_rot, self.layout, self.cfg)
        nm.kvcache_append_i8(self.cache, self.k_rot[:ns], v[:ns])
        nm.kvcache_select(self.cache, self.frames, self.window)
        spans = [self.window.span(), (self.k_rot[ns:], v[ns:]), (self.k_rot[:ns], v[:ns])]
        if ev is not None:
            ev[0].record()
        nm.segment_attention(self.q_rot, spans, o=o, lse=self.lse, dev_err=self.err)
        if ev is not None:
            ev[1].record()


class SweepStep:
    """One denoising step of a whole segment: 54 layers of the 720p layer-step.

    Every layer has its own resident cache of 55,200 tokens plus 512 text
    tokens; each step uses fresh seeded Q and segment K/V (one set per
    denoising step, 8 sets).  Per layer: 3D RoPE of Q and the segment K into
    bf16 buffers, then attention over cache + text + segment.
    """

    def __init__(self, seed: int):
        import torch

        import kv_cached_segment_b200 as nm
        from seeded_inputs import SWEEP_LAYERS, SWEEP_STEPS, WORKLOADS, randn_bf16

        self.nm, self.torch = nm, torch
        w = self.w = WORKLOADS["720p"]
        dev = "cuda"
        ns, nt = w.n_seg, w.n_text
        self.layers, self.steps_per_segment = SWEEP_LAYERS, SWEEP_STEPS
        self.layout = nm.SegLayout(w.frames, w.grid_h, w.grid_w, w.t0, nt)
        self.cfg = nm.RopeConfig(*w.rope_split, w.rope_theta)
        self.cache = []
        for l in range(self.layers):
            k = randn_bf16((w.n_cache + nt, 16, 128), seed * 1000 + 2 * l, dev)
            v = randn_bf16((w.n_cache + nt, 16, 128), seed * 1000 + 2 * l + 1, dev)
            self.cache.append((k, v))
        self.inputs = [tuple(randn_bf16((w.n_q if i == 0 else ns, 16, 128),
                                        seed * 100000 + 3 * s + i, dev) for i in range(3))
                       for s in range(self.steps_per_segment)]
        self.q_rot = torch.empty((w.n_q, 16, 128), dtype=torch.bfloat16, device=dev)
        self.k_rot = torch.empty((ns, 16, 128), dtype=torch.bfloat16, device=dev)
        self.o = torch.empty_like(self.q_rot)
        self.err = torch.zeros(1, dtype=torch.int32, device=dev)
        self.i = 0
        self.launches_per_step = 3 * self.layers

    def flops(self) -> float:
        return self.w.attention_flops() * self.layers

    def run(self, ev=None):
        nm, w = self.nm, self.w
        ns, nt = w.n_seg, w.n_text
        q, k, v = self.inputs[self.i % self.steps_per_segment]
        self.i += 1
        # text rows of Q are copied by the RoPE pass; text K/V live with each layer
        lay_q = nm.SegLayout(w.frames, w.grid_h, w.grid_w, w.t0, nt)
        lay_k = nm.SegLayout(w.frames, w.grid_h, w.grid_w, w.t0, 0)
        if ev is not None:
            ev[0].record()
        for l in range(self.layers):
            ck, cv = self.cache[l]
            nm.rope3d_qk(q, None, self.q_rot, None, lay_q, self.cfg)
            nm.rope3d_qk(k, None, self.k_rot, None, lay_k, self.cfg)
            spans = [(ck[:w.n_cache], cv[:w.n_cache]), (ck[w.n_cache:], cv[w.n_cache:]),
                     (self.k_rot, v)]
            nm.segment_attention(self.q_rot, spans, o=self.o, dev_err=self.err)
        if ev is not None:
            ev[1].record()


def max_over_ranks(values, world: int, device):
    """Element-wise max of per-rank floats over all ranks (identity at world 1)."""
    if world <= 1:
        return [float(x) for x in values]
    import torch
    import torch.distributed as dist

    t = torch.tensor([float(x) for x in values], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(x) for x in t.tolist()]


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
        rows = np.sort(rng.integers(0, ns, rows_per_chunk))
        q_rows = oracle.rope3d(f64(q_all[torch.as_tensor(rows)]), rows.size, t[rows], h[rows],
                               ww[rows])
        refs.append((rows, oracle.attention(q_rows, spans)))
        done += rows.size
        elapsed = time.perf_counter() - t0
    flops = 4.0 * done * w.n_k * 128 * 16
    # parity of the step's output on the sampled rows (outside the timing)
    err_o = np.concatenate([np.abs(f64(step.o[torch.as_tensor(r)]) - o).ravel()
                            for r, (o, _) in refs])
    lse_gpu = step.lse.view(16, w.n_q).cpu().numpy().astype(np.float64)
    err_l = np.concatenate([np.abs(lse_gpu[:, r] - lse).ravel() for r, (_, lse) in refs])
    parity = {"rows": done, "max_abs_o": float(err_o.max()), "mean_abs_o": float(err_o.mean()),
              "max_abs_lse": float(err_l.max()), "bar_max_abs": 2e-2, "bar_mean_abs": 2e-3}
    parity["pass"] = bool(parity["max_abs_o"] <= 2e-2 and parity["mean_abs_o"] <= 2e-3
                          and parity["max_abs_lse"] <= 2e-2)
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


def make_step(args, rank):
    if args.workload == "sweep":
        return SweepStep(seed=1 + rank)
    if args.int8:
        return LayerStepI8(args.workload, seed=1 + rank)
    step = LayerStep(args.workload, seed=1 + rank)
    if args.sparse > 0:
        step.use_sparse(args.sparse, seed=1 + rank)
    if args.key_shards > 0:
        if args.sparse > 0:
            raise SystemExit("--key-shards and --sparse are exclusive")
        step.use_key_shards(args.key_shards)
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
    extra = " (INT8 history cache)" if args.int8 else ""
    if getattr(step, "kv_splits", 1) > 1:
        extra += f" (keys split {step.kv_splits} ways per query block, partials merged)"
    if getattr(args, "key_shards", 0) > 0:
        extra += (f" (keys split into {args.key_shards} contiguous shards, partial results "
                  f"merged)")
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
    step = make_step(args, rank)
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

    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(args.steps)]
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
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

    merge_ms = 0.0
    n_shards = getattr(step, "shards", 0)
    if n_shards:
        merge_ms = statistics.mean(a.elapsed_time(b) for a, b in step.merge_ev[:args.steps])
    ms, attn_ms, merge_ms = max_over_ranks(
        [start.elapsed_time(stop), statistics.mean(a.elapsed_time(b) for a, b in evs), merge_ms],
        world, "cuda")
    attn_ms -= merge_ms  # attention launches only
    ms_per_step = ms / args.steps
    flops = step.flops()
    value = flops * args.steps * world / (ms / 1e3) / 1e12
    attn_tflops = flops / (attn_ms / 1e3) / 1e12

    # ---- end to end through the public API with host buffers: every step
    # copies its inputs from pinned host memory and reads its output back;
    # two buffer sets and two copy streams overlap step i+1's upload and step
    # i-1's download with step i's kernels.
    e2e = None
    if not args.no_e2e and args.workload != "sweep":
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
               "sample": f"fp64 oracle RoPE + attention of {rows} sampled segment query rows "
                         f"x 16 heads over all {step.w.n_k} keys ({secs:.1f} s)"}
        if step.sparse is not None:
            parity = None  # the oracle above is dense attention

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
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {
            "workload": workload_text(args, step),
            "n_q": w.n_q, "n_k": w.n_k, "heads": 16, "head_dim": 128,
            "attention_flops_per_step": flops,
            "step": ("per layer: rope3d_qk x2 + segment attention" if args.workload == "sweep"
                     else "rope3d_qk + int8 append + int8 select + segment attention" if args.int8
                     else "fused rope3d+append" + (" + select" if w.select_frames else "")
                     + " + segment attention"),
            "l2": "inputs larger than L2: each step reads "
                  f"{attn_per_step * (w.n_q * 3 + w.n_k * 2) * 4096 / 1e9:.2f} GB > 126 MB",
            "parallelism": f"independent layer-step per GPU x{world}",
        },
        # per GPU: value is the whole job's aggregate over `world` GPUs
        "pct_of_measured_bf16_peak": 100.0 * value / world / peak,
        "pct_of_datasheet_bf16_peak": 100.0 * value / world / DATASHEET_BF16_TFLOPS,
        "attention_ms": attn_ms / attn_per_step,
        "roofline": {"kernel": "attention_kernel", "bound": "tensor",
                     "achieved": attn_tflops, "peak": peak, "unit": "TFLOP/s",
                     "frac": attn_tflops / peak, "peak_source": f"{peak_src} bf16 {peak_kind}",
                     "traffic": recorded_traffic(args.workload)},
        "cpu_baseline": cpu, "e2e": e2e, "parity": parity,
        "gpu_launches": step.launches_per_step * args.steps * world,  # all ranks
        "clocks": clocks,
    }
    if n_shards:
        # merge: R partial O rows (+ LSE) read, one O row (+ LSE) written per query row
        mbytes = (n_shards + 1) * w.n_q * (16 * 128 * 2 + 16 * 4)
        hbm = peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"])
        out["config"]["key_shards"] = n_shards
        out["merge"] = {"kernel": "merge_kernel", "bound": "hbm", "ms": merge_ms,
                        "bytes": mbytes, "achieved": mbytes / (merge_ms / 1e3) / 1e9,
                        "peak": hbm, "unit": "GB/s",
                        "frac": mbytes / (merge_ms / 1e3) / 1e9 / hbm}
    if args.workload == "sweep":
        out["ms_per_segment"] = ms_per_step * step.steps_per_segment
        out["roofline"]["note"] = "per-step average over the 54 layers (rope3d_qk launches included)"
    print(json.dumps(out), flush=True)


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
        rows = np.sort(rng.integers(0, ns, rows_per_step))
        q_rows = oracle.rope3d(f64(q_all[torch.as_tensor(rows)]), rows.size, t[rows], h[rows],
                               ww[rows])
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
        # the same workload as the CUDA arm's line; what was sampled is in
        # cpu_baseline.sample
        "config": {"workload": workload_text(args, types.SimpleNamespace(w=w, kv_splits=1)),
                   "n_q": w.n_q, "n_k": w.n_k, "heads": 16, "head_dim": 128,
                   "attention_flops_per_step": w.attention_flops(),
                   "step": "fused rope3d+append" + (" + select" if w.select_frames else "")
                           + " + segment attention",
                   "l2": "host memory (the oracle runs on the CPU)",
                   "parallelism": "one process on the host cores"},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle",
                         "host": cpu_model(),
                         "sample": f"fp64 oracle RoPE + attention of {rows_per_step} sampled "
                                   f"segment query rows per step x 16 heads over all {w.n_k} "
                                   f"keys, {args.steps} steps"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(out), flush=True)


if __name__ == "__main__":
    main()
