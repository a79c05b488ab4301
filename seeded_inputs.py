"""Seeded synthetic inputs for the segment-over-cache attention path.

This module is the only code shared by the fp64 oracle (``oracle/``) and the
CUDA path (``kv_cached_segment_b200``).  It holds workload shapes and random
number generation and nothing of the method's arithmetic: no rotary angles, no
softmax, no index copies.

Shapes follow the token grid of the segment-autoregressive world model
described in "Hy-Nomas: an 8.6B world model whose memory is a KV cache"
(ai.thesatyajit.com), section "How one segment is made" (16 heads of 128, one
token per latent grid cell, 30 latent frames per five-second segment) and the
five synthetic workloads this library is measured on.  Every tensor is
N(0, 1) rounded to bf16, row layout ``[tokens][heads][head_dim]``.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np
import torch

HEADS = 16
HEAD_DIM = 128


@dataclass(frozen=True)
class Workload:
    """One segment-over-cache layer-step.

    Video rows of the segment come first (``frames * grid_h * grid_w`` of
    them, frame-major then row-major over the latent grid), then ``n_text``
    text rows.  ``cache_frames`` latent frames of earlier segments are already
    resident in the KV cache; the first segment frame has temporal position
    ``t0``.  ``select_frames > 0`` means the attention reads a window of that
    many frames gathered from the cache instead of the whole cache.
    """

    name: str
    n_text: int
    frames: int
    grid_h: int
    grid_w: int
    cache_frames: int
    t0: int
    select_frames: int = 0
    heads: int = HEADS
    head_dim: int = HEAD_DIM
    rope_split: tuple = (32, 48, 48)
    rope_theta: float = 10000.0
    notes: str = field(default="", compare=False)

    @property
    def tokens_per_frame(self) -> int:
        return self.grid_h * self.grid_w

    @property
    def n_seg(self) -> int:
        return self.frames * self.tokens_per_frame

    @property
    def n_q(self) -> int:
        return self.n_seg + self.n_text

    @property
    def n_cache(self) -> int:
        return self.cache_frames * self.tokens_per_frame

    @property
    def n_window(self) -> int:
        return self.select_frames * self.tokens_per_frame

    @property
    def n_k(self) -> int:
        hist = self.n_window if self.select_frames else self.n_cache
        return hist + self.n_text + self.n_seg

    def attention_flops(self) -> float:
        """4 * Nq * Nk * D * H: two matmuls (QK^T and PV) of 2 flops per MAC."""
        return 4.0 * self.n_q * self.n_k * self.head_dim * self.heads


WORKLOADS = {
    # Tiny: 2 latent frames of 4x6, 64 text tokens, 2 cached frames.
    "tiny": Workload("tiny", n_text=64, frames=2, grid_h=4, grid_w=6,
                     cache_frames=2, t0=2),
    # Mid: 8 frames of 12x20, 256 text tokens, 3 prior segments (24 frames).
    "mid": Workload("mid", n_text=256, frames=8, grid_h=12, grid_w=20,
                    cache_frames=24, t0=24),
    # 720p-shaped: 30 frames of 23x40, 512 text tokens, 2 prior segments.
    "720p": Workload("720p", n_text=512, frames=30, grid_h=23, grid_w=40,
                     cache_frames=60, t0=60),
    # Profiling-sized 720p grid: 8 frames over 15 cached frames (K/V 178 MB,
    # above the 126 MB L2, so DRAM counters stay meaningful).
    "short": Workload("short", n_text=512, frames=8, grid_h=23, grid_w=40,
                      cache_frames=15, t0=15),
    # Bounded active history: 8 prior segments (240 frames) in the cache; a
    # 63-frame list is gathered into a window before the 720p attention.
    "bounded": Workload("bounded", n_text=512, frames=30, grid_h=23, grid_w=40,
                        cache_frames=240, t0=240, select_frames=63),
    # the other reading of the bounded history: all 30 frames of the first
    # segment plus the last 60 cached frames (90 frames, 82,800 tokens)
    "bounded90": Workload("bounded90", n_text=512, frames=30, grid_h=23, grid_w=40,
                          cache_frames=240, t0=240, select_frames=90),
}
# Full segment sweep: 54 layers x 8 denoising steps of the 720p workload.
SWEEP_LAYERS = 54
SWEEP_STEPS = 8


def randn_bf16(shape, seed: int, device="cpu") -> torch.Tensor:
    """N(0,1) samples rounded to bf16 from a seeded torch generator."""
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    x = torch.randn(tuple(shape), generator=g, dtype=torch.float32, device=device)
    return x.to(torch.bfloat16)


def layer_inputs(w: Workload, seed: int, device="cpu") -> dict:
    """Q/K/V of one layer-step plus the resident cache contents.

    Returns bf16 tensors: ``q``, ``k``, ``v`` of ``[n_q][H][D]`` (segment
    rows then text rows) and ``cache_k``, ``cache_v`` of
    ``[n_cache][H][D]``.  Each tensor has its own sub-seed so that any one of
    them can be regenerated alone.
    """
    h, d = w.heads, w.head_dim
    return {
        "q": randn_bf16((w.n_q, h, d), seed * 16 + 1, device),
        "k": randn_bf16((w.n_q, h, d), seed * 16 + 2, device),
        "v": randn_bf16((w.n_q, h, d), seed * 16 + 3, device),
        "cache_k": randn_bf16((w.n_cache, h, d), seed * 16 + 4, device),
        "cache_v": randn_bf16((w.n_cache, h, d), seed * 16 + 5, device),
    }


def bounded_frame_list(w: Workload, seed: int) -> np.ndarray:
    """Frame list for the bounded-history workload.

    Keeps ``select_frames - 60`` frames of the first segment (the first ones
    of a seeded permutation of frames 0..29) plus the last 60 cached frames,
    then shuffles the whole list with the same seed so the gather is not
    monotone.  Returns int32.
    """
    rng = np.random.default_rng(seed)
    n_first = w.select_frames - 60
    first_seg = rng.permutation(30)[:n_first]
    recent = np.arange(w.cache_frames - 60, w.cache_frames)
    idx = np.concatenate([first_seg, recent]).astype(np.int32)
    return idx[rng.permutation(idx.size)]


def random_frame_list(n_src_frames: int, n: int, seed: int) -> np.ndarray:
    """Uniform random frame indices in [0, n_src_frames), repeats allowed."""
    rng = np.random.default_rng(seed)
    return rng.integers(0, n_src_frames, size=n).astype(np.int32)


def sparse_tile_lists(n_q: int, span_lens, keep_spans, candidate_spans, fraction: float,
                      seed: int, heads: int = HEADS, block_q: int = 256, block_k: int = 128):
    """Seeded block-sparse selection: per (query block, head), every key tile
    of the spans in ``keep_spans`` plus a random ``fraction`` of the tiles of
    ``candidate_spans``.  Returns (lists [blocks][heads][max] int32 padded
    with -1, counts [blocks][heads] int32).  The pages give no selection
    rule; this only produces inputs of the right shape and density."""
    rng = np.random.default_rng(seed)
    first, span_tiles = [], []
    t = 0
    for n in span_lens:
        k = (int(n) + block_k - 1) // block_k
        first.append(t)
        span_tiles.append(k)
        t += k
    keep = [first[s] + i for s in keep_spans for i in range(span_tiles[s])]
    cand = np.array([first[s] + i for s in candidate_spans for i in range(span_tiles[s])],
                    dtype=np.int64)
    n_pick = int(round(fraction * cand.size))
    n_blocks = (n_q + block_q - 1) // block_q
    max_tiles = len(keep) + n_pick
    lists = np.full((n_blocks, heads, max(1, max_tiles)), -1, dtype=np.int32)
    counts = np.zeros((n_blocks, heads), dtype=np.int32)
    for b in range(n_blocks):
        for h in range(heads):
            pick = np.sort(rng.choice(cand, size=n_pick, replace=False)) if n_pick else []
            sel = sorted(keep + [int(x) for x in pick])
            lists[b, h, :len(sel)] = sel
            counts[b, h] = len(sel)
    return lists, counts
