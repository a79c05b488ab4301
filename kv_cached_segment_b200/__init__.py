"""Python binding of libnomas (segment-over-cache attention for B200).

Argument marshalling only: every step of the path runs in the library's CUDA
kernels behind the C ABI declared in ``include/nomas.h``.  PyTorch provides
device memory and streams.  There is no CPU fallback: if the compiled
library is missing, importing the binding's entry points raises.

Entry points (same names as the C ABI, without the ``nomas_`` prefix):

- ``rope3d_qk``: 3D RoPE of a segment's Q (and K) rows;
- ``kvcache_append`` / ``kvcache_append_i8``: rotate the segment's K into a
  bf16 or INT8 cache (V copied or quantised), optionally Q too;
- ``kvcache_select``: gather latent frames of a bf16 or INT8 cache into a
  bf16 window, or of an INT8 cache into an INT8 window;
- ``segment_attention`` / ``segment_attention_sparse``: attention of the
  query rows over up to four key/value spans, all tiles or listed tiles; a
  first span that is an INT8 ``I8Span`` (``KVCacheI8.span()``) is read as
  codes and scales and dequantised inside the kernel;
- ``attention_merge``: combine partial (O, LSE) over disjoint key shards;
- ``temporal_context_frames``: the power-spaced history frame picker (host).

Holders: ``KVCache`` and ``KVCacheI8`` (caller-owned device buffers plus
``len``), ``RopeConfig`` and ``SegLayout``.

Head-sharded attention over several GPUs (``head_sharded_segment_attention``:
all-to-all of the query and key rows by heads, attention over 16/world heads,
all-to-all back).  Key-sharded attention over several GPUs, in three forms:
``sharded_segment_attention`` (partial attention per rank, NCCL all-gather of
the partials, merge); ``peer_partial_attention`` + ``peer_merge_owned_rows``
(the all-gather replaced by a merge that reads the owned rows of every GPU's
partial over peer memory and writes every GPU's output,
``attention_merge_peers``); and ``sharded_segment_attention_routed``
(``peer_attention_to_owners`` stores the partial rows into their owners'
buffers from the attention kernel itself, then ``peer_merge_inbox``).
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import torch

from . import _build

HEADS = 16
HEAD_DIM = 128

NOMAS_OK = 0
NOMAS_ERR_INVALID_ARG = 1
NOMAS_ERR_CAPACITY = 2
NOMAS_ERR_INDEX = 3
NOMAS_ERR_UNSUPPORTED = 4
NOMAS_ERR_CUDA = 5
DEVERR_BAD_FRAME_INDEX = 0x1
DEVERR_WAIT_TIMEOUT = 0x2
MAX_SPANS = 4
# Attention kernel schedules (NOMAS_ATTN_PIPELINE_* in nomas.h); 0 = default.
PIPELINE_TWO_TILE = 1
PIPELINE_ONE_TILE = 2
PIPELINE_PAIR = 3
MAX_MERGE_PARTS = 32
MAX_MERGE_OUTPUTS = 32

EXPORTED_SYMBOLS = (
    "nomas_last_error",
    "nomas_version",
    "nomas_rope3d_qk",
    "nomas_kvcache_append",
    "nomas_kvcache_select",
    "nomas_segment_attention",
    "nomas_segment_attention_ex",
    "nomas_temporal_context_frames",
    "nomas_kvcache_append_i8",
    "nomas_kvcache_select_i8",
    "nomas_segment_attention_sparse",
    "nomas_attention_merge",
    "nomas_segment_attention_split",
    "nomas_segment_attention_scratch_bytes",
    "nomas_attention_merge_peers",
    "nomas_segment_attention_to_owners",
    "nomas_kvcache_select_i8_codes",
    "nomas_segment_attention_i8",
    "nomas_set_attention_pipeline",
)
SPARSE_BLOCK_Q = 256
SPARSE_BLOCK_K = 128
DEVERR_BAD_TILE_INDEX = 0x4


class NomasError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"nomas status {status}: {message}")
        self.status = status


class _RopeCfg(ctypes.Structure):
    _fields_ = [("d_t", ctypes.c_int32), ("d_h", ctypes.c_int32), ("d_w", ctypes.c_int32),
                ("theta", ctypes.c_float)]


class _SegLayout(ctypes.Structure):
    _fields_ = [("frames", ctypes.c_int32), ("grid_h", ctypes.c_int32),
                ("grid_w", ctypes.c_int32), ("t0", ctypes.c_int32), ("n_text", ctypes.c_int32)]


class _KVCache(ctypes.Structure):
    _fields_ = [("k", ctypes.c_void_p), ("v", ctypes.c_void_p), ("capacity", ctypes.c_int64),
                ("len", ctypes.c_int64), ("tokens_per_frame", ctypes.c_int32),
                ("heads", ctypes.c_int32), ("head_dim", ctypes.c_int32)]


class _KVCacheI8(ctypes.Structure):
    _fields_ = [("k", ctypes.c_void_p), ("v", ctypes.c_void_p), ("k_scale", ctypes.c_void_p),
                ("v_scale", ctypes.c_void_p), ("capacity", ctypes.c_int64),
                ("len", ctypes.c_int64), ("tokens_per_frame", ctypes.c_int32),
                ("heads", ctypes.c_int32), ("head_dim", ctypes.c_int32)]


class _KVSpan(ctypes.Structure):
    _fields_ = [("k", ctypes.c_void_p), ("v", ctypes.c_void_p), ("len", ctypes.c_int64)]


class _KVSpanI8(ctypes.Structure):
    _fields_ = [("k", ctypes.c_void_p), ("v", ctypes.c_void_p), ("k_scale", ctypes.c_void_p),
                ("v_scale", ctypes.c_void_p), ("len", ctypes.c_int64)]


class _AttnOpts(ctypes.Structure):
    _fields_ = [("wait_limit_ns", ctypes.c_uint64), ("testing_skip_kv_load", ctypes.c_int32),
                ("pipeline", ctypes.c_int32)]


_lib = None


def library_path() -> str:
    return _build.LIB_PATH


def load_library(path: str | None = None) -> ctypes.CDLL:
    """Loads libnomas.so (built in-tree by ``_build.build``); raises if absent."""
    global _lib
    if _lib is not None:
        return _lib
    path = path or _build.LIB_PATH
    if not os.path.exists(path):
        raise ImportError(f"{path} is missing: build it with "
                          "`python -m kv_cached_segment_b200._build` (no CPU fallback exists)")
    lib = ctypes.CDLL(path)
    P, I32, I64, F32 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_float
    lib.nomas_last_error.restype = ctypes.c_char_p
    lib.nomas_last_error.argtypes = []
    lib.nomas_version.restype = ctypes.c_char_p
    lib.nomas_version.argtypes = []
    lib.nomas_rope3d_qk.restype = ctypes.c_int
    lib.nomas_rope3d_qk.argtypes = [P, P, P, P, ctypes.POINTER(_SegLayout),
                                    ctypes.POINTER(_RopeCfg), I32, I32, P]
    lib.nomas_kvcache_append.restype = ctypes.c_int
    lib.nomas_kvcache_append.argtypes = [ctypes.POINTER(_KVCache), P, P, I64, P, P,
                                         ctypes.POINTER(_SegLayout), ctypes.POINTER(_RopeCfg), P]
    lib.nomas_kvcache_select.restype = ctypes.c_int
    lib.nomas_kvcache_select.argtypes = [ctypes.POINTER(_KVCache), P, I32, I32,
                                         ctypes.POINTER(_KVCache), P, P]
    lib.nomas_segment_attention.restype = ctypes.c_int
    lib.nomas_segment_attention.argtypes = [P, I64, ctypes.POINTER(_KVSpan), I32, P, P, F32,
                                            I32, I32, P, P]
    lib.nomas_segment_attention_ex.restype = ctypes.c_int
    lib.nomas_segment_attention_ex.argtypes = [P, I64, ctypes.POINTER(_KVSpan), I32, P, P, F32,
                                               I32, I32, P, ctypes.POINTER(_AttnOpts), P]
    lib.nomas_kvcache_append_i8.restype = ctypes.c_int
    lib.nomas_kvcache_append_i8.argtypes = [ctypes.POINTER(_KVCacheI8), P, P, I64, P, P,
                                            ctypes.POINTER(_SegLayout), ctypes.POINTER(_RopeCfg),
                                            P]
    lib.nomas_kvcache_select_i8.restype = ctypes.c_int
    lib.nomas_kvcache_select_i8.argtypes = [ctypes.POINTER(_KVCacheI8), P, I32, I32,
                                            ctypes.POINTER(_KVCache), P, P]
    lib.nomas_segment_attention_sparse.restype = ctypes.c_int
    lib.nomas_segment_attention_sparse.argtypes = [P, I64, ctypes.POINTER(_KVSpan), I32, P, P, I32,
                                                   P, P, F32, I32, I32, P, P]
    lib.nomas_attention_merge.restype = ctypes.c_int
    lib.nomas_attention_merge.argtypes = [P, P, I32, I64, P, P, I32, I32, P]
    lib.nomas_segment_attention_split.restype = ctypes.c_int
    lib.nomas_segment_attention_split.argtypes = [P, I64, ctypes.POINTER(_KVSpan), I32, P, P, F32,
                                                  I32, I32, I32, P, I64, P, P]
    lib.nomas_segment_attention_scratch_bytes.restype = I64
    lib.nomas_segment_attention_scratch_bytes.argtypes = [I64, I32]
    lib.nomas_attention_merge_peers.restype = ctypes.c_int
    lib.nomas_attention_merge_peers.argtypes = [P, P, I32, I64, I64, I64, P, P, I32, I32, I32, P]
    lib.nomas_segment_attention_to_owners.restype = ctypes.c_int
    lib.nomas_segment_attention_to_owners.argtypes = [P, I64, ctypes.POINTER(_KVSpan), I32, I32, P,
                                                      P, P, I32, F32, I32, I32, P, P]
    lib.nomas_kvcache_select_i8_codes.restype = ctypes.c_int
    lib.nomas_kvcache_select_i8_codes.argtypes = [ctypes.POINTER(_KVCacheI8), P, I32, I32,
                                                  ctypes.POINTER(_KVCacheI8), P, P]
    lib.nomas_set_attention_pipeline.restype = ctypes.c_int
    lib.nomas_set_attention_pipeline.argtypes = [I32]
    lib.nomas_segment_attention_i8.restype = ctypes.c_int
    lib.nomas_segment_attention_i8.argtypes = [P, I64, ctypes.POINTER(_KVSpanI8),
                                               ctypes.POINTER(_KVSpan), I32, P, P, F32, I32, I32,
                                               P, ctypes.POINTER(_AttnOpts), P]
    lib.nomas_temporal_context_frames.restype = ctypes.c_int
    lib.nomas_temporal_context_frames.argtypes = [I32, I32, F32, P, I32, P]
    _lib = lib
    return lib


def _check(status: int) -> None:
    if status != NOMAS_OK:
        raise NomasError(status, load_library().nomas_last_error().decode())


@dataclass
class RopeConfig:
    """3D rotary split of the head dimension over (t, h, w) and its base."""
    d_t: int = 32
    d_h: int = 48
    d_w: int = 48
    theta: float = 10000.0

    def _c(self):
        return _RopeCfg(self.d_t, self.d_h, self.d_w, self.theta)


@dataclass
class SegLayout:
    """Video rows (frames x grid_h x grid_w, first latent frame at t0), then text rows."""
    frames: int
    grid_h: int
    grid_w: int
    t0: int
    n_text: int

    @property
    def n_video(self) -> int:
        return self.frames * self.grid_h * self.grid_w

    def _c(self):
        return _SegLayout(self.frames, self.grid_h, self.grid_w, self.t0, self.n_text)


def _ptr(t: torch.Tensor | None) -> int | None:
    return None if t is None else t.data_ptr()


def _rows(t: torch.Tensor, name: str, heads: int = HEADS) -> int:
    if t.dtype != torch.bfloat16 or not t.is_cuda or not t.is_contiguous():
        raise TypeError(f"{name} must be a contiguous CUDA bf16 tensor")
    if t.dim() != 3 or t.shape[1] != heads or t.shape[2] != HEAD_DIM:
        raise ValueError(f"{name} must have shape [N][{heads}][{HEAD_DIM}], got {tuple(t.shape)}")
    return t.shape[0]


def _stream(stream) -> int | None:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


class KVCache:
    """One layer's KV cache: caller-owned K/V buffers of ``capacity`` rows, ``len`` valid."""

    def __init__(self, k: torch.Tensor, v: torch.Tensor, length: int, tokens_per_frame: int):
        _rows(k, "cache k")
        _rows(v, "cache v")
        if k.shape != v.shape:
            raise ValueError("cache k and v differ in shape")
        self.k, self.v = k, v
        self._c = _KVCache(k.data_ptr(), v.data_ptr(), k.shape[0], int(length),
                           int(tokens_per_frame), HEADS, HEAD_DIM)

    @classmethod
    def empty(cls, capacity: int, tokens_per_frame: int, device="cuda"):
        k = torch.empty((capacity, HEADS, HEAD_DIM), dtype=torch.bfloat16, device=device)
        v = torch.empty_like(k)
        return cls(k, v, 0, tokens_per_frame)

    @property
    def len(self) -> int:
        return self._c.len

    @len.setter
    def len(self, n: int) -> None:
        self._c.len = int(n)

    @property
    def capacity(self) -> int:
        return self._c.capacity

    @property
    def tokens_per_frame(self) -> int:
        return self._c.tokens_per_frame

    def span(self, start: int = 0, stop: int | None = None):
        """(k, v) views of rows [start, stop) (default: the valid rows)."""
        stop = self.len if stop is None else stop
        return self.k[start:stop], self.v[start:stop]


class KVCacheI8:
    """INT8 layer cache: int8 codes [capacity][16][128] and fp32 scales [capacity][16] for K and V."""

    def __init__(self, k, v, k_scale, v_scale, length: int, tokens_per_frame: int):
        for t, name in ((k, "k"), (v, "v")):
            if t.dtype != torch.int8 or not t.is_cuda or not t.is_contiguous() or \
                    t.dim() != 3 or t.shape[1:] != (HEADS, HEAD_DIM):
                raise TypeError(f"INT8 cache {name} must be contiguous CUDA int8 [N][16][128]")
        for t, name in ((k_scale, "k_scale"), (v_scale, "v_scale")):
            if t.dtype != torch.float32 or not t.is_cuda or not t.is_contiguous() or \
                    t.shape != (k.shape[0], HEADS):
                raise TypeError(f"INT8 cache {name} must be contiguous CUDA fp32 [N][16]")
        self.k, self.v, self.k_scale, self.v_scale = k, v, k_scale, v_scale
        self._c = _KVCacheI8(k.data_ptr(), v.data_ptr(), k_scale.data_ptr(), v_scale.data_ptr(),
                             k.shape[0], int(length), int(tokens_per_frame), HEADS, HEAD_DIM)

    @classmethod
    def empty(cls, capacity: int, tokens_per_frame: int, device="cuda"):
        k = torch.empty((capacity, HEADS, HEAD_DIM), dtype=torch.int8, device=device)
        s = torch.empty((capacity, HEADS), dtype=torch.float32, device=device)
        return cls(k, torch.empty_like(k), s, torch.empty_like(s), 0, tokens_per_frame)

    @property
    def len(self) -> int:
        return self._c.len

    @len.setter
    def len(self, n: int) -> None:
        self._c.len = int(n)

    @property
    def capacity(self) -> int:
        return self._c.capacity

    @property
    def tokens_per_frame(self) -> int:
        return self._c.tokens_per_frame

    def span(self, start: int = 0, stop: int | None = None) -> "I8Span":
        """Rows [start, stop) (default: all valid rows) as an INT8 key/value span."""
        stop = self.len if stop is None else stop
        return I8Span(self.k[start:stop], self.v[start:stop], self.k_scale[start:stop],
                      self.v_scale[start:stop])


@dataclass
class I8Span:
    """INT8 rows of keys and values: codes [N][16][128] int8, scales [N][16] fp32."""

    k: torch.Tensor
    v: torch.Tensor
    k_scale: torch.Tensor
    v_scale: torch.Tensor

    def _c(self) -> _KVSpanI8:
        n = self.k.shape[0]
        for t, name in ((self.k, "k"), (self.v, "v")):
            if t.dtype != torch.int8 or not t.is_cuda or not t.is_contiguous() or \
                    t.dim() != 3 or t.shape != (n, HEADS, HEAD_DIM):
                raise TypeError(f"INT8 span {name} must be contiguous CUDA int8 [N][16][128]")
        for t, name in ((self.k_scale, "k_scale"), (self.v_scale, "v_scale")):
            if t.dtype != torch.float32 or not t.is_cuda or not t.is_contiguous() or \
                    t.shape != (n, HEADS):
                raise TypeError(f"INT8 span {name} must be contiguous CUDA fp32 [N][16]")
        ptr = (lambda t: t.data_ptr() if n else None)  # noqa: E731
        return _KVSpanI8(ptr(self.k), ptr(self.v), ptr(self.k_scale), ptr(self.v_scale), n)


def kvcache_append_i8(cache: KVCacheI8, k_seg, v_seg, q_in=None, q_out=None,
                      layout: SegLayout | None = None, cfg: RopeConfig | None = None,
                      stream=None) -> None:
    """kvcache_append into an INT8 cache (keys rotated, then K and V quantised)."""
    lib = load_library()
    n = _rows(k_seg, "k_seg")
    if _rows(v_seg, "v_seg") != n:
        raise ValueError("k_seg and v_seg differ in rows")
    if q_in is not None:
        _rows(q_in, "q_in")
        _rows(q_out, "q_out")
    lay = layout._c() if layout is not None else None
    c = cfg._c() if cfg is not None else None
    _check(lib.nomas_kvcache_append_i8(ctypes.byref(cache._c), _ptr(k_seg), _ptr(v_seg), n,
                                       _ptr(q_in), _ptr(q_out),
                                       ctypes.byref(lay) if lay is not None else None,
                                       ctypes.byref(c) if c is not None else None,
                                       _stream(stream)))


def rope3d_qk(q, k, q_out, k_out, layout: SegLayout, cfg: RopeConfig, stream=None) -> None:
    """3D RoPE on Q (and K): video rows rotated, text rows copied."""
    lib = load_library()
    n = _rows(q, "q")
    _rows(q_out, "q_out")
    if k is not None:
        _rows(k, "k")
        _rows(k_out, "k_out")
    if n != layout.n_video + layout.n_text:
        raise ValueError("q rows != video rows + text rows")
    lay, c = layout._c(), cfg._c()
    _check(lib.nomas_rope3d_qk(_ptr(q), _ptr(k), _ptr(q_out), _ptr(k_out), ctypes.byref(lay),
                               ctypes.byref(c), HEADS, HEAD_DIM, _stream(stream)))


def kvcache_append(cache: KVCache, k_seg, v_seg, q_in=None, q_out=None,
                   layout: SegLayout | None = None, cfg: RopeConfig | None = None,
                   stream=None) -> None:
    """Rotates the segment's K into the cache (V copied), optionally Q too; advances len."""
    lib = load_library()
    n = _rows(k_seg, "k_seg")
    if _rows(v_seg, "v_seg") != n:
        raise ValueError("k_seg and v_seg differ in rows")
    if q_in is not None:
        _rows(q_in, "q_in")
        _rows(q_out, "q_out")
    lay = layout._c() if layout is not None else None
    c = cfg._c() if cfg is not None else None
    _check(lib.nomas_kvcache_append(ctypes.byref(cache._c), _ptr(k_seg), _ptr(v_seg), n,
                                    _ptr(q_in), _ptr(q_out),
                                    ctypes.byref(lay) if lay is not None else None,
                                    ctypes.byref(c) if c is not None else None,
                                    _stream(stream)))


def temporal_context_frames(n_past: int, budget: int = 18, gamma: float = 2.0) -> list:
    """Past latent frames to keep resident (power-spaced back from the newest)."""
    lib = load_library()
    n = max(0, min(int(budget), int(n_past)))
    out = (ctypes.c_int32 * max(1, n))()
    n_out = ctypes.c_int32(0)
    _check(lib.nomas_temporal_context_frames(int(n_past), int(budget), float(gamma),
                                             ctypes.cast(out, ctypes.c_void_p), max(1, n),
                                             ctypes.byref(n_out)))
    return [int(out[i]) for i in range(n_out.value)]


def kvcache_select(src, frame_idx, window, dev_err=None, stream=None) -> None:
    """Gathers the listed latent frames of ``src`` into ``window``.

    A bf16 ``src`` is copied bit for bit into a bf16 window.  An INT8 ``src``
    (KVCacheI8) is either dequantised into a bf16 window (code * scale,
    rounded once to bf16) or, into an INT8 window, copied as codes and
    scales bit for bit.
    """
    lib = load_library()
    if isinstance(frame_idx, torch.Tensor) and frame_idx.is_cuda:
        if frame_idx.dtype != torch.int32 or not frame_idx.is_contiguous():
            raise TypeError("device frame_idx must be contiguous int32")
        n, on_dev, keep = frame_idx.numel(), 1, frame_idx
        ptr = frame_idx.data_ptr()
    else:
        arr = (ctypes.c_int32 * len(frame_idx))(*[int(x) for x in frame_idx])
        n, on_dev, keep = len(frame_idx), 0, arr
        ptr = ctypes.cast(arr, ctypes.c_void_p).value
    if dev_err is not None and (dev_err.dtype != torch.int32 or not dev_err.is_cuda):
        raise TypeError("dev_err must be a CUDA int32 tensor")
    if isinstance(window, KVCacheI8):
        if not isinstance(src, KVCacheI8):
            raise TypeError("an INT8 window needs an INT8 source cache")
        fn = lib.nomas_kvcache_select_i8_codes
    else:
        fn = lib.nomas_kvcache_select_i8 if isinstance(src, KVCacheI8) else lib.nomas_kvcache_select
    _check(fn(ctypes.byref(src._c), ptr, n, on_dev, ctypes.byref(window._c), _ptr(dev_err),
              _stream(stream)))
    del keep


def auto_kv_splits(n_q: int, span_lens, sm_count: int = 148, max_splits: int = 8,
                   heads: int = HEADS) -> int:
    """Key splits for ``segment_attention(kv_splits="auto")``.

    Minimises a simple time model of the launch, in units of one CTA's time
    per 128-key tile: ceil(CTAs x S / SMs) waves, each as long as one CTA's
    share of the tiles plus about 3 tiles of fixed cost, plus the merge of
    the S partial rows (read at ~5.5 TB/s, one tile taking ~1.5 us).  A
    split must leave at least 4 tiles per CTA and gain at least 2%."""
    tiles = sum((int(n) + 127) // 128 for n in span_lens)
    ctas = (int(n_q) + 255) // 256 * int(heads)
    if tiles == 0 or ctas == 0:
        return 1
    best, best_t = 1, None
    for s in range(1, max_splits + 1):
        if tiles / s < 4:
            break
        t = -(-ctas * s // sm_count) * (tiles / s + 3.0)
        if s > 1:
            t += (s + 1) * n_q * heads * (128 * 2 + 4) / 5.5e12 / 1.5e-6 + 3.0
        if best_t is None or t < 0.98 * best_t:
            best, best_t = s, t
    return best


def segment_attention(q, spans, o=None, lse=None, softmax_scale: float = 0.0, dev_err=None,
                      stream=None, wait_limit_ns: int = 0, testing_skip_kv_load: int = -1,
                      kv_splits=1, pipeline: int = 0):
    """Attention of every row of q over all keys of ``spans`` (list of (k, v)); returns o.

    ``wait_limit_ns`` bounds every pipeline wait in the kernel (0: default);
    ``testing_skip_kv_load`` is for tests of the timeout path only.
    ``pipeline`` picks the kernel schedule (``PIPELINE_*``; 0: the default,
    see ``set_attention_pipeline``).
    ``kv_splits`` > 1 (or "auto", see ``auto_kv_splits``) cuts the key tiles
    into that many ranges computed by separate CTAs and merged, for shapes
    whose query blocks alone do not fill the GPU; the scratch for the
    partial results is allocated here, through PyTorch.
    """
    lib = load_library()
    # Heads per row: 16, or 1, 2, 4 or 8 for a head-sharded dense call.
    heads = int(q.shape[1]) if q.dim() == 3 else HEADS
    if heads not in (1, 2, 4, 8, HEADS):
        raise ValueError(f"q must have 16 heads (or 1, 2, 4 or 8), got {tuple(q.shape)}")
    n_q = _rows(q, "q", heads)
    if o is None:
        o = torch.empty_like(q)
    _rows(o, "o", heads)
    if lse is not None and (lse.dtype != torch.float32 or not lse.is_cuda or
                            lse.numel() != heads * n_q or not lse.is_contiguous()):
        raise ValueError("lse must be a contiguous CUDA fp32 tensor of heads * n_q elements")
    if len(spans) > MAX_SPANS:
        raise ValueError(f"at most {MAX_SPANS} spans")
    history = None
    if spans and isinstance(spans[0], I8Span):
        history, spans = spans[0]._c(), list(spans[1:])
        if kv_splits not in (1, "1"):
            raise ValueError("an INT8 history span takes kv_splits=1")
    if heads != HEADS and history is not None:
        raise ValueError("fewer than 16 heads: dense bf16 spans only")
    arr = (_KVSpan * max(1, len(spans)))()
    for i, (k, v) in enumerate(spans):
        nk = _rows(k, f"span {i} k", heads)
        if _rows(v, f"span {i} v", heads) != nk:
            raise ValueError(f"span {i}: k and v differ in rows")
        arr[i] = _KVSpan(k.data_ptr() if nk else None, v.data_ptr() if nk else None, nk)
    if dev_err is not None and (dev_err.dtype != torch.int32 or not dev_err.is_cuda):
        raise TypeError("dev_err must be a CUDA int32 tensor")
    if kv_splits == "auto":
        sm = torch.cuda.get_device_properties(q.device).multi_processor_count
        kv_splits = auto_kv_splits(n_q, [int(k.shape[0]) for k, _ in spans], sm, heads=heads)
    kv_splits = int(kv_splits)
    if history is not None:
        opts = _AttnOpts(int(wait_limit_ns), int(testing_skip_kv_load), int(pipeline))
        _check(lib.nomas_segment_attention_i8(_ptr(q), n_q, ctypes.byref(history), arr, len(spans),
                                              _ptr(o), _ptr(lse), float(softmax_scale), HEADS,
                                              HEAD_DIM, _ptr(dev_err), ctypes.byref(opts),
                                              _stream(stream)))
    elif kv_splits > 1:
        if wait_limit_ns or testing_skip_kv_load != -1 or pipeline:
            raise ValueError("kv_splits > 1 takes no wait_limit_ns / testing_skip_kv_load / "
                             "pipeline (set_attention_pipeline sets the default)")
        if stream is not None and not isinstance(stream, torch.cuda.Stream):
            raise TypeError("kv_splits > 1 takes stream=None or a torch.cuda.Stream")
        nbytes = lib.nomas_segment_attention_scratch_bytes(n_q, kv_splits)
        scratch = torch.empty(max(nbytes, 16), dtype=torch.uint8, device=q.device)
        _check(lib.nomas_segment_attention_split(_ptr(q), n_q, arr, len(spans), _ptr(o), _ptr(lse),
                                                 float(softmax_scale), heads, HEAD_DIM, kv_splits,
                                                 _ptr(scratch), nbytes, _ptr(dev_err),
                                                 _stream(stream)))
        # allocated on the current stream; when the kernels run on another
        # one, the allocator must not hand the scratch out before they end
        if stream is not None:
            scratch.record_stream(stream)
    elif wait_limit_ns or testing_skip_kv_load != -1 or pipeline:
        opts = _AttnOpts(int(wait_limit_ns), int(testing_skip_kv_load), int(pipeline))
        _check(lib.nomas_segment_attention_ex(_ptr(q), n_q, arr, len(spans), _ptr(o), _ptr(lse),
                                              float(softmax_scale), heads, HEAD_DIM,
                                              _ptr(dev_err), ctypes.byref(opts), _stream(stream)))
    else:
        _check(lib.nomas_segment_attention(_ptr(q), n_q, arr, len(spans), _ptr(o), _ptr(lse),
                                           float(softmax_scale), heads, HEAD_DIM, _ptr(dev_err),
                                           _stream(stream)))
    return o


def set_attention_pipeline(pipeline: int) -> None:
    """Sets the schedule of later attention calls that name none (0: built-in)."""
    _check(load_library().nomas_set_attention_pipeline(int(pipeline)))


def segment_attention_sparse(q, spans, tile_list, tile_count, o=None, lse=None,
                             softmax_scale: float = 0.0, dev_err=None, stream=None):
    """Block-sparse attention: query block b (256 rows) of head h attends to the
    128-key tiles tile_list[b, h, :tile_count[b, h]] (tiles numbered over the
    spans in order).  tile_list: CUDA int32 [blocks][16][max_tiles];
    tile_count: CUDA int32 [blocks][16]; dev_err: CUDA int32 word (required)."""
    lib = load_library()
    n_q = _rows(q, "q")
    if o is None:
        o = torch.empty_like(q)
    _rows(o, "o")
    n_blocks = (n_q + SPARSE_BLOCK_Q - 1) // SPARSE_BLOCK_Q
    for t, name in ((tile_list, "tile_list"), (tile_count, "tile_count")):
        if t.dtype != torch.int32 or not t.is_cuda or not t.is_contiguous():
            raise TypeError(f"{name} must be a contiguous CUDA int32 tensor")
    if tile_list.dim() != 3 or tile_list.shape[:2] != (n_blocks, HEADS):
        raise ValueError(f"tile_list must have shape [{n_blocks}][{HEADS}][max_tiles]")
    if tuple(tile_count.shape) != (n_blocks, HEADS):
        raise ValueError(f"tile_count must have shape [{n_blocks}][{HEADS}]")
    if dev_err is None or dev_err.dtype != torch.int32 or not dev_err.is_cuda:
        raise TypeError("dev_err must be a CUDA int32 tensor")
    if lse is not None and (lse.dtype != torch.float32 or not lse.is_cuda or
                            lse.numel() != HEADS * n_q or not lse.is_contiguous()):
        raise ValueError("lse must be a contiguous CUDA fp32 tensor of heads * n_q elements")
    arr = (_KVSpan * max(1, len(spans)))()
    for i, (k, v) in enumerate(spans):
        nk = _rows(k, f"span {i} k")
        if _rows(v, f"span {i} v") != nk:
            raise ValueError(f"span {i}: k and v differ in rows")
        arr[i] = _KVSpan(k.data_ptr() if nk else None, v.data_ptr() if nk else None, nk)
    _check(lib.nomas_segment_attention_sparse(_ptr(q), n_q, arr, len(spans), tile_list.data_ptr(),
                                              tile_count.data_ptr(), tile_list.shape[2], _ptr(o),
                                              _ptr(lse), float(softmax_scale), HEADS, HEAD_DIM,
                                              dev_err.data_ptr(), _stream(stream)))
    return o


def attention_merge(o_parts, lse_parts, o=None, lse=None, stream=None):
    """Combine partial results over disjoint key shards.

    o_parts: CUDA bf16 [R][n_q][16][128]; lse_parts: CUDA fp32 [R][16][n_q].
    Returns o ([n_q][16][128] bf16); fills lse ([16][n_q] fp32) if given."""
    lib = load_library()
    if o_parts.dtype != torch.bfloat16 or o_parts.dim() != 4 or not o_parts.is_contiguous():
        raise TypeError("o_parts must be a contiguous bf16 [R][n_q][16][128] tensor")
    r, n_q = o_parts.shape[0], o_parts.shape[1]
    if lse_parts.dtype != torch.float32 or tuple(lse_parts.shape) != (r, HEADS, n_q) or \
            not lse_parts.is_contiguous():
        raise TypeError("lse_parts must be a contiguous fp32 [R][16][n_q] tensor")
    if o is None:
        o = torch.empty(o_parts.shape[1:], dtype=torch.bfloat16, device=o_parts.device)
    _check(lib.nomas_attention_merge(o_parts.data_ptr(), lse_parts.data_ptr(), r, n_q,
                                     o.data_ptr(), _ptr(lse), HEADS, HEAD_DIM, _stream(stream)))
    return o


def attention_merge_peers(o_parts, lse_parts, o_outs, lse_outs=None, row0: int = 0,
                          n_rows: int | None = None, stream=None):
    """Merge rows [row0, row0 + n_rows) of key-shard partials found through
    lists of tensors, writing the merged rows into every tensor of o_outs
    (and lse_outs).  The tensors may live on other GPUs whose memory this
    process can reach (peer access, IPC or symmetric memory): the exchange
    between GPUs and the merge are one kernel.  The caller orders the call
    after every GPU's partials are complete, and the outputs' readers after
    every GPU's call.

    o_parts: R bf16 [n_q][16][128]; lse_parts: R fp32 [16][n_q] (or flat);
    o_outs: bf16 [n_q][16][128] outputs; lse_outs: fp32 LSE outputs or None."""
    lib = load_library()
    n_parts, n_outs = len(o_parts), len(o_outs)
    if len(lse_parts) != n_parts:
        raise ValueError("o_parts and lse_parts differ in length")
    n_q = _rows(o_parts[0], "o_parts[0]")
    for i, t in enumerate(list(o_parts) + list(o_outs)):
        if _rows(t, f"partial/output {i}") != n_q:
            raise ValueError("every partial and output must have n_q rows")
    for t in list(lse_parts) + list(lse_outs or []):
        if t.dtype != torch.float32 or t.numel() != HEADS * n_q or not t.is_contiguous():
            raise ValueError("LSE tensors must be contiguous fp32 with heads * n_q elements")
    if lse_outs is not None and len(lse_outs) != n_outs:
        raise ValueError("o_outs and lse_outs differ in length")
    n_rows = n_q - row0 if n_rows is None else n_rows
    parts = (ctypes.c_void_p * n_parts)(*[t.data_ptr() for t in o_parts])
    lses = (ctypes.c_void_p * n_parts)(*[t.data_ptr() for t in lse_parts])
    outs = (ctypes.c_void_p * n_outs)(*[t.data_ptr() for t in o_outs])
    louts = (ctypes.c_void_p * n_outs)(*[t.data_ptr() for t in lse_outs]) if lse_outs else None
    _check(lib.nomas_attention_merge_peers(parts, lses, n_parts, n_q, int(row0), int(n_rows), outs,
                                           louts, n_outs, HEADS, HEAD_DIM, _stream(stream)))


def shard_rows(n: int, rank: int, world: int, align: int = 1):
    """Contiguous share [a, b) of n rows for `rank` (boundaries on multiples of align)."""
    units = (n + align - 1) // align
    a = (units * rank) // world * align
    b = min(n, (units * (rank + 1)) // world * align)
    return min(a, n), b


def peer_partial_attention(q, local_spans, part_o, part_lse):
    """Phase 1 of key-sharded attention over peer memory: this GPU's partial
    (O, LSE) over its own key spans, into its slot of the partial buffers."""
    segment_attention(q, local_spans, o=part_o, lse=part_lse.view(-1))


def _span_table(spans):
    arr = (_KVSpan * max(1, len(spans)))()
    for i, (k, v) in enumerate(spans):
        nk = _rows(k, f"span {i} k")
        if _rows(v, f"span {i} v") != nk:
            raise ValueError(f"span {i}: k and v differ in rows")
        arr[i] = _KVSpan(k.data_ptr() if nk else None, v.data_ptr() if nk else None, nk)
    return arr


def owner_rows(n_q: int, world: int):
    """Row boundaries of the owners: world + 1 ints, shares on 16-row steps."""
    return [shard_rows(n_q, r, world, align=16)[0] for r in range(world)] + [n_q]


def peer_attention_to_owners(q, local_spans, inbox_o_peers, inbox_lse_peers, slot: int,
                             dev_err=None, stream=None):
    """Phase 1 of key-sharded attention with the exchange in the attention
    kernel: this GPU's partial (O, LSE) over its own key spans, each query
    row stored into part ``slot`` of its owner's inbox (owner s owns the rows
    of ``owner_rows(n_q, world)``, world = len(inbox_o_peers)).
    inbox_o_peers[s]: bf16 [R][n_q][16][128]; inbox_lse_peers[s]: fp32
    [R][16][n_q] (R > slot); they may live on other GPUs."""
    lib = load_library()
    n_q = _rows(q, "q")
    world = len(inbox_o_peers)
    if len(inbox_lse_peers) != world or world > MAX_MERGE_PARTS:
        raise ValueError("one o and one lse inbox per owner, at most MAX_MERGE_PARTS owners")
    for t in inbox_o_peers:
        if t.dtype != torch.bfloat16 or t.dim() != 4 or t.shape[0] <= slot or \
                t.shape[1] != n_q or not t.is_contiguous():
            raise ValueError("inbox_o_peers must be contiguous bf16 [R][n_q][16][128], R > slot")
    for t in inbox_lse_peers:
        if t.dtype != torch.float32 or t.dim() != 3 or t.shape[0] <= slot or \
                t.shape[2] != n_q or not t.is_contiguous():
            raise ValueError("inbox_lse_peers must be contiguous fp32 [R][16][n_q], R > slot")
    rows = (ctypes.c_int64 * (world + 1))(*owner_rows(n_q, world))
    o_tab = (ctypes.c_void_p * world)(*[t.data_ptr() for t in inbox_o_peers])
    l_tab = (ctypes.c_void_p * world)(*[t.data_ptr() for t in inbox_lse_peers])
    _check(lib.nomas_segment_attention_to_owners(_ptr(q), n_q, _span_table(local_spans),
                                                 len(local_spans), world, rows, o_tab, l_tab,
                                                 int(slot), 0.0, HEADS, HEAD_DIM, _ptr(dev_err),
                                                 _stream(stream)))


def peer_merge_inbox(inbox_o, inbox_lse, o_peers, lse_peers, rank: int, stream=None):
    """Phase 2 with the exchange in the attention kernel: merge this GPU's own
    rows from its inbox (local [R][n_q][16][128] and [R][16][n_q]) and store
    them into every GPU's output."""
    n_q = inbox_o.shape[1]
    a, b = owner_rows(n_q, len(o_peers))[rank:rank + 2]
    attention_merge_peers(list(inbox_o.unbind(0)), list(inbox_lse.unbind(0)), o_peers, lse_peers,
                          row0=a, n_rows=b - a, stream=stream)


def sharded_segment_attention_routed(q, local_spans, inbox_o_peers, inbox_lse_peers, o_peers,
                                     lse_peers, rank: int, barrier=lambda: None, dev_err=None):
    """Key-sharded attention with the exchange in the attention kernel, on
    the GPU of ``rank``: phase 1 (partials stored into the owners' inboxes),
    ``barrier()``, phase 2 (this GPU's rows merged into every output),
    ``barrier()``.  The lists hold every GPU's buffers, mapped into this
    process (peer access, IPC or symmetric memory); ``barrier`` must order
    the streams of all GPUs (a one-element NCCL all-reduce, for example).
    Returns this GPU's output, o_peers[rank]."""
    peer_attention_to_owners(q, local_spans, inbox_o_peers, inbox_lse_peers, slot=rank,
                             dev_err=dev_err)
    barrier()
    peer_merge_inbox(inbox_o_peers[rank], inbox_lse_peers[rank], o_peers, lse_peers, rank)
    barrier()
    return o_peers[rank]


def peer_merge_owned_rows(part_o_peers, part_lse_peers, o_peers, lse_peers, rank: int,
                          world: int):
    """Phase 2: this GPU merges the query rows it owns (a contiguous share,
    on 16-row boundaries) from every GPU's partial and writes them into every
    GPU's output.  Between phase 1 on all GPUs and this call, and after this
    call on all GPUs, the caller needs a cross-GPU barrier in stream order
    (for example a one-element NCCL all-reduce)."""
    n_q = part_o_peers[0].shape[0]
    a, b = shard_rows(n_q, rank, world, align=16)
    attention_merge_peers(part_o_peers, part_lse_peers, o_peers, lse_peers, row0=a, n_rows=b - a)


def _all_to_all_rows(t, send_rows, recv_rows, group):
    """all_to_all_single over dim 0 with per-rank row counts; bf16 moves as
    int16 (a bit copy), so that backends without bf16 collectives work."""
    import torch.distributed as dist

    out = torch.empty((sum(recv_rows),) + tuple(t.shape[1:]), dtype=t.dtype, device=t.device)
    a, b = (out.view(torch.int16), t.view(torch.int16)) if t.dtype == torch.bfloat16 else (out, t)
    dist.all_to_all_single(a, b.contiguous(), output_split_sizes=list(recv_rows),
                           input_split_sizes=list(send_rows), group=group)
    return out


def head_sharded_segment_attention(q, local_spans, group=None, lse=None, attend=None):
    """Attention with the rows of Q and of the keys spread across the ranks of
    `group` (sequence parallel), computed head-parallel (Ulysses-style): one
    all-to-all gives every rank all query and key rows for 16/world of the
    heads, each rank attends over those heads, and a second all-to-all
    returns every rank its own query rows for all 16 heads.

    q: this rank's query rows [n_q_local][16][128]; local_spans: this rank's
    key/value rows (list of (k, v), [n][16][128]); the world size divides 16.
    Returns O for the local query rows; fills lse ([16][n_q_local], fp32) if
    given.  `attend(q_heads, spans, lse_heads)` defaults to segment_attention
    (which takes 16/world heads per row)."""
    import torch.distributed as dist

    world = dist.get_world_size(group) if dist.is_initialized() else 1
    if HEADS % world:
        raise ValueError(f"the world size must divide {HEADS} (got {world})")
    hl = HEADS // world
    attend = attend or (lambda qq, spans, l: segment_attention(qq, spans, lse=l))
    n_q = q.shape[0]
    dev = q.device
    if local_spans:
        k_loc = torch.cat([k for k, _ in local_spans]) if len(local_spans) > 1 else local_spans[0][0]
        v_loc = torch.cat([v for _, v in local_spans]) if len(local_spans) > 1 else local_spans[0][1]
    else:
        k_loc = q.new_empty((0, HEADS, HEAD_DIM))
        v_loc = q.new_empty((0, HEADS, HEAD_DIM))
    n_k = k_loc.shape[0]
    if world == 1:
        rows_q, rows_k = [n_q], [n_k]
    else:
        cnt = torch.tensor([n_q, n_k], dtype=torch.int64,
                           device=dev if dist.get_backend(group) == "nccl" else "cpu")
        allc = [torch.empty_like(cnt) for _ in range(world)]
        dist.all_gather(allc, cnt, group=group)
        rows_q = [int(c[0]) for c in allc]
        rows_k = [int(c[1]) for c in allc]

    def to_heads(t, n_local, rows_all):
        # [n][world][hl][128] -> per destination rank d, this rank's rows of
        # heads d*hl .. d*hl + hl - 1; received in source-rank order.
        send = t.reshape(n_local, world, hl, HEAD_DIM).transpose(0, 1).reshape(
            world * n_local, hl, HEAD_DIM)
        if world == 1:
            return send.contiguous()
        return _all_to_all_rows(send, [n_local] * world, rows_all, group)

    q_h = to_heads(q, n_q, rows_q)
    k_h = to_heads(k_loc, n_k, rows_k)
    v_h = to_heads(v_loc, n_k, rows_k)
    lse_h = torch.empty(hl * sum(rows_q), dtype=torch.float32, device=dev)
    o_h = attend(q_h, [(k_h, v_h)] if k_h.shape[0] else [], lse_h)
    # back: the rows of rank d (rows_q[d] of them, in order) to rank d
    if world == 1:
        o_back = o_h.reshape(1, n_q, hl, HEAD_DIM)
    else:
        o_back = _all_to_all_rows(o_h.contiguous(), rows_q, [n_q] * world, group).reshape(
            world, n_q, hl, HEAD_DIM)
    o = o_back.transpose(0, 1).reshape(n_q, HEADS, HEAD_DIM).contiguous()
    if lse is not None:
        lh = lse_h.view(hl, sum(rows_q)).t().contiguous()  # [rows][hl]
        if world == 1:
            lb = lh.reshape(1, n_q, hl)
        else:
            lb = _all_to_all_rows(lh, rows_q, [n_q] * world, group).reshape(world, n_q, hl)
        lse.view(HEADS, n_q).copy_(lb.permute(0, 2, 1).reshape(HEADS, n_q))
    return o


def sharded_segment_attention(q, local_spans, group=None, lse=None, attend=None, merge=None):
    """Attention over keys spread across the ranks of `group` (cache sequence
    parallelism): every rank attends with all of q over its own key spans,
    the partial (O, LSE) of all ranks are all-gathered, and each rank merges
    them into the full result.  `attend` and `merge` default to this
    library's kernels (segment_attention, attention_merge)."""
    import torch.distributed as dist

    world = dist.get_world_size(group) if dist.is_initialized() else 1
    n_q = q.shape[0]
    attend = attend or (lambda qq, spans, l: segment_attention(qq, spans, lse=l))
    merge = merge or (lambda op, lp, l: attention_merge(op, lp, lse=l))
    part_lse = torch.empty(HEADS * n_q, dtype=torch.float32, device=q.device)
    part_o = attend(q, local_spans, part_lse)
    if world == 1:
        o_parts, lse_parts = part_o[None], part_lse.view(1, HEADS, n_q)
    else:
        o_parts = torch.empty((world,) + tuple(part_o.shape), dtype=part_o.dtype, device=q.device)
        lse_parts = torch.empty((world, HEADS, n_q), dtype=torch.float32, device=q.device)
        dist.all_gather(list(o_parts.unbind(0)), part_o.contiguous(), group=group)
        dist.all_gather(list(lse_parts.unbind(0)), part_lse.view(HEADS, n_q), group=group)
    return merge(o_parts, lse_parts, lse)
