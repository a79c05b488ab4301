"""fp64 oracle functions (test infrastructure; see the package docstring).

Pages cited:
  [KV]  "Hy-Nomas: an 8.6B world model whose memory is a KV cache"
        (ai.thesatyajit.com)
  [4090] "Hy-Nomas en una RTX 4090: un mundo en vídeo que recuerda"
        (inferencekey.com)
  [IT]  "Hy-Nomas: cosa fa davvero il modello del mondo interattivo a forma
        libera di Tencent" (orcarouter.ai)

Readings taken where the pages leave a step open are stated at each function.
"""
from __future__ import annotations

import math

import numpy as np


# ---------------------------------------------------------------------------
# bf16 widening
# ---------------------------------------------------------------------------
def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns (uint16) to float64.

    A bf16 value is the upper half of the float32 with the same bits, so
    shifting the pattern left by 16 and reinterpreting gives the float32
    exactly; float32 -> float64 is exact.
    """
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return b.view(np.float32).astype(np.float64)


# ---------------------------------------------------------------------------
# 3D rotary positions
# ---------------------------------------------------------------------------
def video_positions(frames: int, grid_h: int, grid_w: int, t0: int):
    """(t, h, w) of every video row of a segment.

    [KV] "How one segment is made": patch size 1x1x1, so every cell of the
    latent grid of every latent frame is one token.  Reading (the pages fix no
    order): rows are frame-major, then row-major over the grid; h and w count
    from 0 inside a frame; t counts latent frames of the whole history, so the
    segment's first frame sits at ``t0`` = latent frames already written.
    """
    n = frames * grid_h * grid_w
    r = np.arange(n, dtype=np.int64)
    f = r // (grid_h * grid_w)
    y = (r // grid_w) % grid_h
    x = r % grid_w
    return (t0 + f), y, x


def rope_frequencies(d_axis: int, theta: float) -> np.ndarray:
    """Angular frequency of each rotation pair of one axis chunk.

    Standard rotary embedding applied per axis: pair j of a chunk of width
    ``d_axis`` turns by ``theta ** (-2 j / d_axis)`` radians per unit of
    position ([KV] "How one segment is made", item "The blocks": 3D RoPE with
    a per-axis split of the head dimension and a base theta).
    """
    j = np.arange(d_axis // 2, dtype=np.float64)
    return np.power(float(theta), -2.0 * j / d_axis)


def rope3d(x: np.ndarray, n_video: int, pos_t, pos_h, pos_w,
           split=(32, 48, 48), theta: float = 10000.0) -> np.ndarray:
    """Apply 3D RoPE to the first ``n_video`` rows of ``x`` ([N][H][D] f64).

    [KV] "How one segment is made", item "The blocks" (3D RoPE, split of the
    head dimension over t/h/w, base theta); [IT] release overview (3D RoPE);
    [4090] "Modelo y ficheros" (3D RoPE).  Head dims ``[0, d_t)`` rotate by
    the temporal position, ``[d_t, d_t + d_h)`` by the grid row and the rest
    by the grid column.  Readings: pairs are adjacent elements (2j, 2j+1)
    inside each axis chunk; the pair (a, b) at angle phi becomes
    (a cos phi - b sin phi, a sin phi + b cos phi); text rows (row index
    ``>= n_video``) carry no 3D position and are returned unchanged.
    """
    x = np.array(x, dtype=np.float64, copy=True)
    d_t, d_h, d_w = split
    assert d_t + d_h + d_w == x.shape[2]
    chunks = ((0, d_t, pos_t), (d_t, d_h, pos_h), (d_t + d_h, d_w, pos_w))
    for off, d_a, pos in chunks:
        omega = rope_frequencies(d_a, theta)
        pos = np.asarray(pos, dtype=np.float64)[:n_video]
        for j in range(d_a // 2):
            phi = pos * omega[j]                       # [n_video]
            c = np.cos(phi)[:, None]
            s = np.sin(phi)[:, None]
            a = x[:n_video, :, off + 2 * j].copy()
            b = x[:n_video, :, off + 2 * j + 1].copy()
            x[:n_video, :, off + 2 * j] = a * c - b * s
            x[:n_video, :, off + 2 * j + 1] = a * s + b * c
    return x


# ---------------------------------------------------------------------------
# Lifelong KV cache: append and frame select
# ---------------------------------------------------------------------------
def kvcache_append(cache_k, cache_v, length: int, k_new, v_new):
    """Write a segment's K/V at the end of the cache.

    [KV] "Writing the segment into memory" and "What 'world memory' stores":
    after a segment is finished its keys and values are stored in the cache,
    which grows by one segment per step.  Returns new arrays: rows
    ``[length, length + n)`` hold the segment, every other row is unchanged,
    and the new length.
    """
    n = k_new.shape[0]
    if length + n > cache_k.shape[0]:
        raise ValueError("cache capacity exceeded")
    out_k = np.array(cache_k, copy=True)
    out_v = np.array(cache_v, copy=True)
    for i in range(n):
        out_k[length + i] = k_new[i]
        out_v[length + i] = v_new[i]
    return out_k, out_v, length + n


def kvcache_select(src, frame_idx, tokens_per_frame: int):
    """Gather whole latent frames of the cache into a contiguous window.

    [KV] "The 4090 preset": before each segment only a list of past latent
    frames is restored to the GPU.  The window holds frame ``frame_idx[j]``
    at rows ``[j * P, (j + 1) * P)``, P = tokens per frame.  Repeated indices
    are allowed (a plain gather); an index outside the cache is an error.
    """
    p = tokens_per_frame
    n_src_frames = src.shape[0] // p
    out = np.empty((len(frame_idx) * p,) + src.shape[1:], dtype=src.dtype)
    for j, f in enumerate(frame_idx):
        f = int(f)
        if not 0 <= f < n_src_frames:
            raise IndexError(f"frame {f} outside [0, {n_src_frames})")
        out[j * p:(j + 1) * p] = src[f * p:(f + 1) * p]
    return out


# ---------------------------------------------------------------------------
# Segment-over-cache attention
# ---------------------------------------------------------------------------
def attention_rows(q, rows, spans, scale=None):
    """Softmax attention of the query rows ``rows`` over all keys of ``spans``.

    [KV] "How one segment is made" (joint attention of text and video tokens,
    16 heads of 128; attention is causal across segments, so the current
    segment reads earlier ones from the cache) and "What 'world memory'
    stores" (queries of segment k attend over the cache).  Reading: the
    queries are the current segment's video rows and the text rows; the keys
    are the union of the spans (cache or window, text, segment) in that order;
    no mask applies among them, so every query sees every key.  The scale is
    1/sqrt(head_dim) unless given.

    For each head h and row i: s_j = scale * <q_i, k_j>,
    O_i = sum_j exp(s_j - m) v_j / sum_j exp(s_j - m) with m = max_j s_j
    (two passes: the max, then the sums), LSE_i = m + ln(sum_j exp(s_j - m)).

    q: [Nq][H][D] float64; spans: list of (k, v), each [Nj][H][D] float64.
    Returns O [len(rows)][H][D] and LSE [H][len(rows)], float64.
    """
    k = np.concatenate([np.asarray(s[0], dtype=np.float64) for s in spans], axis=0)
    v = np.concatenate([np.asarray(s[1], dtype=np.float64) for s in spans], axis=0)
    rows = np.asarray(rows, dtype=np.int64)
    n_heads, d = q.shape[1], q.shape[2]
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    out = np.zeros((rows.size, n_heads, d), dtype=np.float64)
    lse = np.zeros((n_heads, rows.size), dtype=np.float64)
    if k.shape[0] == 0:
        # No keys: the sums are empty.  Reading: O = 0 and LSE = -inf.
        lse[:] = -np.inf
        return out, lse
    block = 256
    for h in range(n_heads):
        kh = k[:, h, :]
        vh = v[:, h, :]
        for b0 in range(0, rows.size, block):
            r = rows[b0:b0 + block]
            s = (np.asarray(q[r, h, :], dtype=np.float64) @ kh.T) * scale
            m = s.max(axis=1, keepdims=True)          # pass 1: row max
            e = np.exp(s - m)
            l_sum = e.sum(axis=1, keepdims=True)      # pass 2: row sum
            out[b0:b0 + block, h, :] = (e @ vh) / l_sum
            lse[h, b0:b0 + block] = (m + np.log(l_sum))[:, 0]
    return out, lse


def attention(q, spans, scale=None):
    """``attention_rows`` over every query row."""
    return attention_rows(q, np.arange(q.shape[0]), spans, scale)


# ---------------------------------------------------------------------------
# Power-spaced history frame picker
# ---------------------------------------------------------------------------
def temporal_context_frame_indices(n_past: int, budget: int = 18,
                                   gamma: float = 2.0) -> np.ndarray:
    """Past latent frames kept resident by the single-GPU preset.

    [KV] "The 4090 preset", the distance formula there:
    N = min(budget, T), u_i = i / (N - 1), d_i = i + rint((T - N) u_i^gamma)
    for i < N, and the kept frames are T - 1 - d_i.  ``rint`` rounds half to
    even (numpy's rint).  Reading for N = 1, where u_0 is 0/0: u_0 = 0, so
    the only kept frame is T - 1 (= 0, since N = 1 implies T = 1 when the
    budget is above 1).  Returned in ascending frame order, as the page
    prints its example.
    """
    t = int(n_past)
    n = min(int(budget), t)
    if n <= 0:
        return np.zeros(0, dtype=np.int64)
    kept = []
    for i in range(n):
        u = i / (n - 1) if n > 1 else 0.0
        d = i + int(np.rint((t - n) * u ** gamma))
        kept.append(t - 1 - d)
    return np.array(sorted(kept), dtype=np.int64)


# ---------------------------------------------------------------------------
# INT8 KV cache
# ---------------------------------------------------------------------------
def f32_to_bf16_bits(x) -> np.ndarray:
    """Round float32 values to bf16 (round to nearest, ties to even); bits.

    bf16 keeps the upper 16 bits of a float32; rounding adds half of the
    dropped part, plus one when the kept part is odd and the dropped part is
    exactly half (ties to even).  Inputs are finite here.
    """
    b = np.asarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    lsb = (b >> np.uint64(16)) & np.uint64(1)
    rounded = (b + np.uint64(0x7FFF) + lsb) >> np.uint64(16)
    return rounded.astype(np.uint16)


def quantize_int8(x_bits):
    """Symmetric INT8 quantisation per (token, head) of a bf16 [N][H][D] tensor.

    [KV] "The 4090 preset": the cache is quantised once per segment to one
    byte per value plus an FP32 scale per token and head (4,224 B per token
    per layer for K and V together).  Reading (the page gives no formula):
    absmax scaling, a = max_d |x_d|; the stored scale is a / 127 rounded to
    the nearest float32, and the code is the integer nearest to the exact
    quotient 127 x_d / a, ties to even.  An all-zero (token, head) gets scale
    0 and codes 0.  Returns int8 codes [N][H][D] and float32 scales [N][H].

    The quotient is formed in float64 from the exactly widened inputs: 127 x
    is exact, and the one rounding of the division cannot move a quotient
    onto or across a half-integer (x and a carry 8 significant bits, so a
    quotient that is not itself a tie stays more than 2^-17 away from one).
    """
    x = bf16_bits_to_f64(x_bits)                               # exact
    amax = np.max(np.abs(x), axis=2)                           # exact
    scale = (amax.astype(np.float32) / np.float32(127.0)).astype(np.float32)
    zero = amax == 0
    safe = np.where(zero, 1.0, amax)
    codes = np.rint(127.0 * x / safe[:, :, None])              # half to even
    codes = np.clip(codes, -127, 127).astype(np.int8)          # |x| <= a
    codes[zero] = 0
    return codes, scale


def round_to_bf16_bits(x) -> np.ndarray:
    """Round float64 values to the nearest bf16, ties to even, in one step; bits.

    bf16 keeps 8 significant bits: a normal value in [2^e, 2^(e+1)) lies on
    the grid of step 2^(e-7), and below 2^-126 the step is 2^-133 (the bf16
    subnormals).  The value is divided by its step (exact: a power of two),
    rounded to an integer half to even, and multiplied back.  Inputs are
    finite and inside the bf16 range.
    """
    x = np.asarray(x, dtype=np.float64)
    _, e = np.frexp(x)                       # |x| in [2^(e-1), 2^e)
    step_exp = np.maximum(e - 1 - 7, -133)
    step = np.ldexp(1.0, step_exp)
    r = np.rint(x / step) * step             # exact in float64
    return f32_to_bf16_bits(r.astype(np.float32))   # r is a bf16 value: exact


def dequantize_int8_f64(codes, scales) -> np.ndarray:
    """Dequantised values code * scale, exact in float64 ([KV] "The 4090
    preset": a stored value is its code times its token and head's scale)."""
    return (np.asarray(codes, dtype=np.float64) *
            np.asarray(scales, dtype=np.float32).astype(np.float64)[:, :, None])


def dequantize_int8(codes, scales) -> np.ndarray:
    """bf16 bits of code * scale: the exact product rounded once to the
    nearest bf16, ties to even (the restored window is bf16)."""
    return round_to_bf16_bits(dequantize_int8_f64(codes, scales))


# ---------------------------------------------------------------------------
# Block-sparse segment attention
# ---------------------------------------------------------------------------
def key_tiles(span_lens, block_k: int = 128):
    """Key tiles of the concatenated spans: (span, first key, end key) each.

    Tiles never straddle spans: span s contributes ceil(len_s / block_k) tiles,
    the last one short.  A tile's global id is its index in this list.
    """
    tiles = []
    for s, n in enumerate(span_lens):
        for a in range(0, int(n), block_k):
            tiles.append((s, a, min(int(n), a + block_k)))
    return tiles


def block_sparse_attention(q, spans, tile_lists, block_q: int = 256, block_k: int = 128,
                           scale=None):
    """Attention where each (query block, head) sees only listed key tiles.

    [4090] "El preset de una GPU": the single-GPU preset's attention is dense
    on the first two denoising steps and then keeps 25% of the candidate
    video key blocks; the pages do not state the selection rule, so the
    selection is an input here:
    ``tile_lists[b][h]`` lists the global tile ids (see ``key_tiles``) that
    query rows [b * block_q, (b + 1) * block_q) of head h attend to.  Within
    that key set the result is the plain softmax attention of
    ``attention_rows``.  Each listed tile contributes its keys once per
    listing; ids outside the tile list are ignored; an empty set gives O = 0
    and LSE = -inf.
    """
    nq, n_heads, d = q.shape
    tiles = key_tiles([s[0].shape[0] for s in spans], block_k)
    out = np.zeros((nq, n_heads, d), dtype=np.float64)
    lse = np.full((n_heads, nq), -np.inf, dtype=np.float64)
    for b in range(len(tile_lists)):
        rows = np.arange(b * block_q, min(nq, (b + 1) * block_q))
        if rows.size == 0:
            continue
        for h in range(n_heads):
            sel = [tiles[g] for g in tile_lists[b][h] if 0 <= g < len(tiles)]
            if not sel:
                continue
            kh = np.concatenate([spans[s][0][a:e, h:h + 1] for s, a, e in sel])
            vh = np.concatenate([spans[s][1][a:e, h:h + 1] for s, a, e in sel])
            o_h, l_h = attention_rows(q[:, h:h + 1], rows, [(kh, vh)], scale)
            out[rows, h] = o_h[:, 0]
            lse[h, rows] = l_h[0]
    return out, lse


# ---------------------------------------------------------------------------
# Sharded keys: merging partial results
# ---------------------------------------------------------------------------
def merge_partials(o_parts, lse_parts):
    """Combine attention results computed over disjoint key subsets.

    [KV] "What 'world memory' stores" (the standard preset spreads the cache
    over eight GPUs, sp_size 8): each GPU attends over its part of the keys.
    With LSE_r = ln sum_{j in part r} e^{s_j} and O_r the softmax-weighted V
    of part r, the whole is LSE = ln sum_r e^{LSE_r} and
    O = sum_r e^{LSE_r - LSE} O_r (the sums over parts regroup the sums over
    keys).  Parts with LSE = -inf (no keys) contribute nothing; if every part
    is empty, O = 0 and LSE = -inf.
    o_parts: [R][Nq][H][D], lse_parts: [R][H][Nq] (natural log).
    """
    o_parts = np.asarray(o_parts, dtype=np.float64)
    lse_parts = np.asarray(lse_parts, dtype=np.float64)
    m = lse_parts.max(axis=0)                                   # [H][Nq]
    safe_m = np.where(np.isfinite(m), m, 0.0)
    w = np.exp(lse_parts - safe_m[None])                        # [R][H][Nq]
    total = w.sum(axis=0)
    lse = np.where(total > 0, safe_m + np.log(np.where(total > 0, total, 1.0)), -np.inf)
    wn = np.where(total[None] > 0, w / np.where(total > 0, total, 1.0)[None], 0.0)
    out = np.einsum("rhq,rqhd->qhd", wn, o_parts)
    return out, lse
