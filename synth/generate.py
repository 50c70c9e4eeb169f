"""Seeded synthetic inputs, shared by the oracle-side tests and the GPU side.

Every tensor is drawn from its own PCG64 substream ``default_rng([seed, id, index])``
so that a frame, a chunk or one sequence can be regenerated on its own.  Values are
drawn in float64, scaled, and rounded once to the storage dtype (round-to-nearest-even
for bfloat16); both sides consume exactly the rounded values.  Distributions follow
the workloads' statement: hidden states and queries ~ N(0, 1), weights ~ N(0, std =
1/sqrt(fan_in)) with fan_in = d for W_DKV and W_KR and fan_in = d_c for W_UK and W_UV,
and, where the cache is drawn directly, cache rows ~ N(0, 1).

This module holds no arithmetic of the attention method itself.
"""

from __future__ import annotations

import dataclasses
import math
from typing import Dict

import numpy as np

from .configs import Workload

# substream ids, one per tensor
_ID = {"h": 1, "w_dkv": 2, "w_kr": 3, "w_uk": 4, "w_uv": 5, "q_nope": 6, "q_rope": 7,
       "cache": 8}


@dataclasses.dataclass
class Tensor:
    """A synthetic tensor: exact float64 values plus the bits that are uploaded."""
    values: np.ndarray        # float64, exactly representable in the storage dtype
    storage: np.ndarray       # float32 array, or uint16 array of bfloat16 bits
    dtype: str

    @property
    def shape(self):
        return self.values.shape


def bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float64 values to bfloat16 (via float32, nearest-even) -> uint16 bits."""
    u = np.ascontiguousarray(x, dtype=np.float64).astype(np.float32).view(np.uint32)
    u = u.astype(np.uint64)
    r = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return r.astype(np.uint16)


def bf16_bits_to_f64(b: np.ndarray) -> np.ndarray:
    return (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def to_storage(x: np.ndarray, dtype: str) -> Tensor:
    if dtype == "f32":
        s = np.ascontiguousarray(x, dtype=np.float32)
        return Tensor(s.astype(np.float64), s, dtype)
    if dtype == "bf16":
        b = bf16_bits(x)
        return Tensor(bf16_bits_to_f64(b), b, dtype)
    raise ValueError(dtype)


def _normal(seed: int, name: str, index: int, shape, std: float) -> np.ndarray:
    rng = np.random.default_rng([seed, _ID[name], index])
    return rng.standard_normal(shape) * std


def hidden_frame(w: Workload, seed: int, frame: int) -> Tensor:
    """Hidden states h of one frame for every sequence: [B, F, d]."""
    x = _normal(seed, "h", frame, (w.batch, w.tokens_per_frame, w.d_model), 1.0)
    return to_storage(x, w.dtype)


def hidden_frames(w: Workload, seed: int, first: int, count: int) -> Tensor:
    """Hidden states of ``count`` consecutive frames: [B, count*F, d]."""
    parts = [hidden_frame(w, seed, first + i) for i in range(count)]
    return Tensor(np.concatenate([p.values for p in parts], axis=1),
                  np.concatenate([p.storage for p in parts], axis=1), w.dtype)


def weights(w: Workload, seed: int) -> Dict[str, Tensor]:
    """W_DKV [d, d_c], W_KR [d, d_R], W_UK [n_h, d_h, d_c], W_UV [n_h, d_h, d_c]."""
    out = {}
    if w.d_model:
        sd = 1.0 / math.sqrt(w.d_model)
        out["w_dkv"] = to_storage(_normal(seed, "w_dkv", 0, (w.d_model, w.d_latent), sd), w.dtype)
        out["w_kr"] = to_storage(_normal(seed, "w_kr", 0, (w.d_model, w.d_rope), sd), w.dtype)
    sc = 1.0 / math.sqrt(w.d_latent)
    out["w_uk"] = to_storage(_normal(seed, "w_uk", 0, (w.n_heads, w.d_nope, w.d_latent), sc), w.dtype)
    out["w_uv"] = to_storage(_normal(seed, "w_uv", 0, (w.n_heads, w.d_nope, w.d_latent), sc), w.dtype)
    return out


def queries(w: Workload, seed: int) -> Dict[str, Tensor]:
    """Per-head content queries q_nope [B, T, n_h, d_h] and un-rotated RoPE queries
    q_R [B, T, n_h, d_R] for the call's T query tokens (one substream per frame)."""
    if w.decode:
        idx = [0]
        per = 1
    else:
        idx = [w.first_chunk_frame + i for i in range(w.chunk_frames)]
        per = w.tokens_per_frame
    qn = np.concatenate([_normal(seed, "q_nope", f, (w.batch, per, w.n_heads, w.d_nope), 1.0)
                         for f in idx], axis=1)
    qr = np.concatenate([_normal(seed, "q_rope", f, (w.batch, per, w.n_heads, w.d_rope), 1.0)
                         for f in idx], axis=1)
    return {"q_nope": to_storage(qn, w.dtype), "q_rope": to_storage(qr, w.dtype)}


def direct_cache(w: Workload, seed: int, batch_index: int | None = None) -> Tensor:
    """Cache rows drawn directly (decode workload): [B, S, d_c + d_R] ~ N(0, 1).
    With ``batch_index`` only that sequence: [S, d_c + d_R]."""
    if batch_index is not None:
        return to_storage(_normal(seed, "cache", batch_index, (w.ring_slots, w.row_width), 1.0),
                          w.dtype)
    parts = [direct_cache(w, seed, b) for b in range(w.batch)]
    return Tensor(np.stack([p.values for p in parts]), np.stack([p.storage for p in parts]),
                  w.dtype)
