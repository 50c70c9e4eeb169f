"""Workload table: the five problem shapes of absorbed multi-head latent attention
over a sliding-window latent KV ring (VideoMLA, "Core Mechanism"; the MLA concept
page, "Low-rank joint compression" and "The RoPE problem, and the decoupled fix").

Pure data: sizes, positions and the ring history of each workload. No arithmetic of
the method lives here; both the oracle-side tests and the GPU side read this table.

Positions.  A global token index ``g`` belongs to frame ``g // F`` (``F = grid_h *
grid_w`` tokens per frame), row ``(g % F) // grid_w`` and column ``g % grid_w`` of
that frame.  The ring keeps ``S`` token slots per sequence; token ``g`` lives in slot
``g mod S``.
"""

from __future__ import annotations

import dataclasses
import math
from typing import Optional, Tuple


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    dtype: str                 # storage dtype of every tensor: "f32" or "bf16"
    batch: int                 # B, independent sequences
    n_heads: int               # n_h
    d_nope: int                # d_h, per-head content (no-RoPE) query/key width
    d_latent: int              # d_c, shared content latent width
    d_rope: int                # d_R, shared decoupled RoPE key width
    rope_pairs: Tuple[int, int, int]   # rotation pairs on the (t, y, x) axes
    rope_theta: float
    grid_h: int                # frame rows
    grid_w: int                # frame columns
    d_model: int               # hidden width d (0: no cache write in this workload)
    window_frames: int         # W, cached frames visible besides the chunk
    chunk_frames: int          # C, frames of queries in the chunk
    first_chunk_frame: int     # global frame index of the chunk's first frame
    ring_slots: int            # S
    decode: bool = False       # one query per sequence at the last key position
    cache_direct: bool = False # cache rows drawn directly (no cache-write history)

    @property
    def tokens_per_frame(self) -> int:
        return self.grid_h * self.grid_w

    @property
    def row_width(self) -> int:
        """Elements of one cached token row [c_KV || k_R]."""
        return self.d_latent + self.d_rope

    @property
    def n_queries(self) -> int:
        """Query tokens per sequence in one attention call."""
        return 1 if self.decode else self.chunk_frames * self.tokens_per_frame

    @property
    def q_first_tok(self) -> int:
        if self.decode:
            return self.ring_slots - 1
        return self.first_chunk_frame * self.tokens_per_frame

    @property
    def k_first_tok(self) -> int:
        """First global token of the visible window (window frames, then the chunk)."""
        if self.decode:
            return 0
        return (self.first_chunk_frame - self.window_frames) * self.tokens_per_frame

    @property
    def n_keys(self) -> int:
        if self.decode:
            return self.ring_slots
        return (self.window_frames + self.chunk_frames) * self.tokens_per_frame

    @property
    def frames_written(self) -> int:
        """Frames pushed through the cache write, chunk included (0 for decode)."""
        if self.cache_direct:
            return 0
        return self.first_chunk_frame + self.chunk_frames

    @property
    def softmax_scale(self) -> float:
        """1/sqrt(d_h + d_R): the width of the concatenated content+RoPE dot product."""
        return 1.0 / math.sqrt(self.d_nope + self.d_rope)

    @property
    def elem_bytes(self) -> int:
        return 4 if self.dtype == "f32" else 2

    def scaled(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


TINY = Workload(
    name="tiny_f32", dtype="f32", batch=1, n_heads=4, d_nope=32, d_latent=64,
    d_rope=16, rope_pairs=(2, 3, 3), rope_theta=10000.0, grid_h=4, grid_w=4,
    d_model=128, window_frames=3, chunk_frames=1, first_chunk_frame=3, ring_slots=64)

VIDEO_CHUNK = Workload(
    name="video_chunk_bf16", dtype="bf16", batch=1, n_heads=32, d_nope=128,
    d_latent=512, d_rope=64, rope_pairs=(8, 12, 12), rope_theta=10000.0, grid_h=30,
    grid_w=52, d_model=4096, window_frames=3, chunk_frames=1, first_chunk_frame=3,
    ring_slots=4 * 1560)

LONG_WINDOW = Workload(
    name="long_window_bf16", dtype="bf16", batch=1, n_heads=32, d_nope=128,
    d_latent=512, d_rope=64, rope_pairs=(8, 12, 12), rope_theta=10000.0, grid_h=30,
    grid_w=52, d_model=4096, window_frames=21, chunk_frames=3, first_chunk_frame=58,
    ring_slots=24 * 1560)

WIDE_KEY = Workload(
    name="wide_key_bf16", dtype="bf16", batch=4, n_heads=32, d_nope=128,
    d_latent=512, d_rope=512, rope_pairs=(64, 96, 96), rope_theta=10000.0, grid_h=30,
    grid_w=52, d_model=4096, window_frames=9, chunk_frames=1, first_chunk_frame=9,
    ring_slots=10 * 1560)

DECODE = Workload(
    name="decode_bf16", dtype="bf16", batch=64, n_heads=128, d_nope=128,
    d_latent=512, d_rope=64, rope_pairs=(32, 0, 0), rope_theta=10000.0, grid_h=1,
    grid_w=1, d_model=0, window_frames=8191, chunk_frames=1, first_chunk_frame=8191,
    ring_slots=8192, decode=True, cache_direct=True)

ALL = (TINY, VIDEO_CHUNK, LONG_WINDOW, WIDE_KEY, DECODE)
BY_NAME = {w.name: w for w in ALL}


def small_variant(w: Workload) -> Workload:
    """A reduced copy of a bf16 workload that the fp64 oracle finishes in seconds
    while still spanning several 128-row tiles, several key blocks and ragged tails
    (frame sizes that are not multiples of the tile sizes)."""
    if w is DECODE:
        return w.scaled(name="decode_small", batch=3, n_heads=128, ring_slots=700,
                        window_frames=699, first_chunk_frame=699)
    if w is LONG_WINDOW:
        # 3-frame chunk over a window that wraps the ring twice.
        return w.scaled(name="long_window_small", grid_h=5, grid_w=7, window_frames=4,
                        chunk_frames=3, first_chunk_frame=16, ring_slots=7 * 35,
                        d_model=256, n_heads=8)
    if w is WIDE_KEY:
        return w.scaled(name="wide_key_small", batch=2, grid_h=5, grid_w=9,
                        window_frames=3, first_chunk_frame=3, ring_slots=4 * 45,
                        d_model=256, n_heads=8, rope_pairs=(64, 96, 96))
    if w is VIDEO_CHUNK:
        return w.scaled(name="video_chunk_small", grid_h=6, grid_w=11, window_frames=3,
                        first_chunk_frame=3, ring_slots=4 * 66, d_model=512, n_heads=8)
    return w


def check(w: Workload) -> None:
    """Consistency of a workload's own numbers (no arithmetic of the method)."""
    assert sum(w.rope_pairs) * 2 == w.d_rope, w
    assert w.n_keys <= w.ring_slots, w
    if not w.decode:
        assert w.k_first_tok >= 0, w
        assert w.q_first_tok + w.n_queries == w.k_first_tok + w.n_keys, w


for _w in ALL:
    check(_w)
