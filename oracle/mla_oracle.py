"""fp64 CPU oracle for multi-head latent attention over a latent KV ring.

TEST INFRASTRUCTURE ONLY.  Only the tests, the package smoke check and the CPU
baseline leg of the benchmark may import this module.  It shares no code with the
CUDA path and the CUDA path never calls it.

Sources, cited by page title and section:

* [MLA concept]   "Multi-Head Latent Attention" (concept page), sections
  "Low-rank joint compression" (joint latent c_t^KV, only it is cached; the
  absorption identity q_t^T k_s = c_t^Q^T (W^UQ^T W^UK) c_s^KV; W^UV folds into the
  output side) and "The RoPE problem, and the decoupled fix" (query and key are the
  concatenation of a content channel and a small decoupled RoPE channel shared across
  heads; the score is the sum of a content term and a positional term; the cache
  holds d_c latent plus the RoPE dims per token).
* [MLA explainer] "Understanding Multi-Head Latent Attention and KV Compression",
  sections "Low-Rank Joint Compression", "On-the-Fly Reconstruction and Matrix
  Absorption" (per-head K and V are reconstructed from the latent with
  up-projections) and "Decoupling Rotary Position Embeddings (RoPE)" (the cache
  stores the latent alongside the RoPE key; the two key parts are concatenated).
* [Irminsul]      the Irminsul abstract on the "Multi-Head Latent Attention" topic page:
  the cached row is a position-free latent plus a RoPE key that a delta-rotation
  re-indexes in closed form when the same tokens move to shifted positions.
* [VideoMLA]      "VideoMLA: Compressing Video Diffusion Memory by 92.7% with
  Low-Rank Latent Attention", sections "The Gap" (sliding-window KV cache,
  next-frame prediction) and "Core Mechanism" (a shared content latent and a
  shared positional key that encodes the 3-D (t, h, w) position with RoPE), and the
  VideoMLA abstract on the "Multi-Head Latent Attention" topic page.

What the pages leave open is fixed by these readings (each one listed with its reason
in the design notes): 3-D RoPE splits d_R into contiguous t, y, x segments and
rotates adjacent pairs (2j, 2j+1) of an axis segment with n_a pairs by
pos_a * theta^(-j/n_a); the RoPE key is rotated with its absolute position when it
is written; a key is visible to a query iff its frame is not later than the query's
frame; the ring keeps token g in slot g mod S; the softmax scale is a caller value.

Every function here is the plain definition: no blocking, fusion or reordering.
"""

from __future__ import annotations

import math
from typing import Iterable, Optional, Sequence, Tuple

import numpy as np

# ----------------------------------------------------------------------------------
# positions and the ring  ([VideoMLA] "The Gap", "Core Mechanism")
# ----------------------------------------------------------------------------------


def token_position(g: int, grid_h: int, grid_w: int) -> Tuple[int, int, int]:
    """(t, y, x) of global token g: frame index, row and column inside the frame."""
    f = grid_h * grid_w
    return g // f, (g % f) // grid_w, g % grid_w


def ring_slot(g: int, ring_slots: int) -> int:
    """Slot of global token g in a sliding-window ring of ``ring_slots`` tokens."""
    return g % ring_slots


# ----------------------------------------------------------------------------------
# 3-D rotary position embedding  ([VideoMLA] "Core Mechanism"; [MLA concept]
# "The RoPE problem, and the decoupled fix")
# ----------------------------------------------------------------------------------


def rope_angles(t: int, y: int, x: int, pairs: Sequence[int], theta: float) -> np.ndarray:
    """Rotation angle of every pair of a d_R-wide RoPE vector at position (t, y, x).

    The vector is split into contiguous segments for the t, y and x axes holding
    pairs[0], pairs[1], pairs[2] rotation pairs.  Pair j of an axis with n pairs turns
    by pos * theta**(-j/n) radians (the rotary embedding with base theta applied to
    that segment alone)."""
    out = []
    for pos, n in zip((t, y, x), pairs):
        for j in range(n):
            out.append(pos * theta ** (-j / n))
    return np.asarray(out, dtype=np.float64)


def rotate_pairs(v: np.ndarray, angles: np.ndarray) -> np.ndarray:
    """Rotate pairs (v[2j], v[2j+1]) of the last axis by angles[..., j]."""
    a = v[..., 0::2]
    b = v[..., 1::2]
    c = np.cos(angles)
    s = np.sin(angles)
    out = np.empty_like(v, dtype=np.float64)
    out[..., 0::2] = a * c - b * s
    out[..., 1::2] = a * s + b * c
    return out


def rope3d(v: np.ndarray, tokens: Sequence[int], grid_h: int, grid_w: int,
           pairs: Sequence[int], theta: float) -> np.ndarray:
    """RoPE of v[..., n_tok, (heads...,) d_R] where axis -2 or the axis matching
    ``tokens`` carries the token: v has shape [n_tok, d_R] or [n_tok, H, d_R]."""
    v = np.asarray(v, dtype=np.float64)
    ang = np.stack([rope_angles(*token_position(g, grid_h, grid_w), pairs, theta)
                    for g in tokens]) if len(tokens) else np.zeros((0, v.shape[-1] // 2))
    if v.ndim == 3:
        ang = ang[:, None, :]
    return rotate_pairs(v, ang)


# ----------------------------------------------------------------------------------
# step a1: cache write  ([MLA concept] "Low-rank joint compression"; [MLA explainer]
# "Decoupling Rotary Position Embeddings (RoPE)")
# ----------------------------------------------------------------------------------


def cache_rows(h: np.ndarray, w_dkv: np.ndarray, w_kr: np.ndarray, first_tok: int,
               wl) -> np.ndarray:
    """Cached rows [c_KV || RoPE(k_R)] of tokens first_tok.. for h [B, n, d].

    c_KV = h W_DKV (the shared content latent); k_R = h W_KR rotated by the token's
    own absolute (t, y, x) position before it is stored."""
    h = np.asarray(h, dtype=np.float64)
    c = h @ np.asarray(w_dkv, dtype=np.float64)
    kr = h @ np.asarray(w_kr, dtype=np.float64)
    toks = list(range(first_tok, first_tok + h.shape[1]))
    kr = np.stack([rope3d(kr[b], toks, wl.grid_h, wl.grid_w, wl.rope_pairs, wl.rope_theta)
                   for b in range(h.shape[0])])
    return np.concatenate([c, kr], axis=-1)


def cache_write(cache: np.ndarray, h: np.ndarray, w_dkv: np.ndarray, w_kr: np.ndarray,
                first_tok: int, wl) -> Tuple[np.ndarray, np.ndarray]:
    """Write the rows of tokens first_tok .. first_tok+n-1 into their ring slots.
    Returns the updated cache [B, S, d_c+d_R] and the slot of every token [B, n]."""
    rows = cache_rows(h, w_dkv, w_kr, first_tok, wl)
    out = np.array(cache, dtype=np.float64, copy=True)
    n = h.shape[1]
    slots = np.empty((h.shape[0], n), dtype=np.int64)
    for b in range(h.shape[0]):
        for i in range(n):
            s = ring_slot(first_tok + i, wl.ring_slots)
            out[b, s] = rows[b, i]
            slots[b, i] = s
    return out, slots


def shift_frames(cache: np.ndarray, first_tok: int, n_tok: int, delta_frames: int,
                 wl) -> np.ndarray:
    """Re-index cached RoPE keys to positions delta_frames frames later ([Irminsul]
    delta-rotation; [VideoMLA] "Core Mechanism" for the 3-D positions).

    A whole-frame shift moves t by delta_frames and leaves y and x alone, so the RoPE
    key of each token g in [first_tok, first_tok + n_tok) (slot g mod S) is turned by
    the angles of position (delta_frames, 0, 0); the latent is position-free and stays.
    Returns a new cache."""
    out = np.array(cache, dtype=np.float64, copy=True)
    d_c = wl.d_latent
    ang = rope_angles(delta_frames, 0, 0, wl.rope_pairs, wl.rope_theta)
    for g in range(first_tok, first_tok + n_tok):
        slot = ring_slot(g, wl.ring_slots)
        out[:, slot, d_c:] = rotate_pairs(out[:, slot, d_c:], ang)
    return out


# ----------------------------------------------------------------------------------
# step a2: query absorption  ([MLA concept] "Low-rank joint compression": W^UK folds
# into the query side; "The RoPE problem, and the decoupled fix")
# ----------------------------------------------------------------------------------


def absorb_q(q_nope: np.ndarray, q_rope: np.ndarray, w_uk: np.ndarray, q_first_tok: int,
             wl) -> np.ndarray:
    """q_abs[b, i, h] = [q_nope[b,i,h] W_UK[h] || RoPE(q_R[b,i,h], pos(q_first_tok+i))].

    W_UK[h] is [d_h, d_c]; the per-head key is k_h = W_UK[h] c, so the content score
    q_nope . k_h equals (q_nope W_UK[h]) . c."""
    q_nope = np.asarray(q_nope, dtype=np.float64)
    w_uk = np.asarray(w_uk, dtype=np.float64)
    q_lat = np.einsum("bihd,hdc->bihc", q_nope, w_uk)
    toks = list(range(q_first_tok, q_first_tok + q_nope.shape[1]))
    q_r = np.stack([rope3d(q_rope[b], toks, wl.grid_h, wl.grid_w, wl.rope_pairs,
                           wl.rope_theta) for b in range(q_nope.shape[0])])
    return np.concatenate([q_lat, q_r], axis=-1)


# ----------------------------------------------------------------------------------
# steps a3/a4: attention.  Two definitions of the same result.
# ----------------------------------------------------------------------------------


def visible_keys(g_query: int, k_first_tok: int, n_keys: int, wl) -> np.ndarray:
    """Global tokens of the window that query g_query may attend to: frame-block-causal,
    every key of its own and earlier frames (next-frame prediction over a sliding
    window, [VideoMLA] "The Gap")."""
    ks = np.arange(k_first_tok, k_first_tok + n_keys, dtype=np.int64)
    f = wl.grid_h * wl.grid_w
    return ks[ks // f <= g_query // f]


def _softmax_lse(scores: np.ndarray):
    m = scores.max(axis=-1, keepdims=True)
    e = np.exp(scores - m)
    s = e.sum(axis=-1, keepdims=True)
    return e / s, (m + np.log(s))[..., 0]


def attend_latent(q_abs: np.ndarray, cache: np.ndarray, q_first_tok: int,
                  k_first_tok: int, n_keys: int, scale: float, wl,
                  queries: Optional[Iterable[Tuple[int, int]]] = None):
    """Absorbed attention in latent space ([MLA concept] "Low-rank joint compression":
    at decode time one attends directly in latent space).

    score(q, s) = scale * (q_lat . c_s + q_rope . k_R,s) over visible keys s, softmax,
    o_lat = sum_s p * c_s.  Returns (o_lat [B,T,n_h,d_c], lse [B,T,n_h]) for all
    queries, or, with ``queries`` = [(b, i), ...], arrays [len, n_h, ...] for those."""
    q_abs = np.asarray(q_abs, dtype=np.float64)
    cache = np.asarray(cache, dtype=np.float64)
    d_c = wl.d_latent
    sel = list(queries) if queries is not None else [
        (b, i) for b in range(q_abs.shape[0]) for i in range(q_abs.shape[1])]
    o = np.zeros((len(sel), q_abs.shape[2], d_c))
    lse = np.zeros((len(sel), q_abs.shape[2]))
    for n, (b, i) in enumerate(sel):
        g_q = q_first_tok + i
        keys = visible_keys(g_q, k_first_tok, n_keys, wl)
        rows = cache[b, keys % wl.ring_slots]                  # [L, d_c + d_R]
        sc = scale * (q_abs[b, i] @ rows.T)                    # [n_h, L]
        p, lse[n] = _softmax_lse(sc)
        o[n] = p @ rows[:, :d_c]
    if queries is None:
        B, T = q_abs.shape[0], q_abs.shape[1]
        return o.reshape(B, T, *o.shape[1:]), lse.reshape(B, T, -1)
    return o, lse


def attend_latent_part(q_abs: np.ndarray, cache: np.ndarray, q_first_tok: int,
                       k_first_tok: int, n_keys: int, scale: float, wl, key_lo: int,
                       key_hi: int, queries: Optional[Iterable[Tuple[int, int]]] = None):
    """One piece of a key range cut between workers: ``attend_latent`` over the visible keys
    g with key_lo <= g < key_hi only (the cross-instance MLA abstract on the topic page
    computes attention where the blocks live and merges the partial results).  Returns
    (o_lat normalised over the piece, lse of the piece); a query without a visible key in
    the piece gets o_lat = 0 and lse = -inf."""
    q_abs = np.asarray(q_abs, dtype=np.float64)
    cache = np.asarray(cache, dtype=np.float64)
    d_c = wl.d_latent
    sel = list(queries) if queries is not None else [
        (b, i) for b in range(q_abs.shape[0]) for i in range(q_abs.shape[1])]
    o = np.zeros((len(sel), q_abs.shape[2], d_c))
    lse = np.full((len(sel), q_abs.shape[2]), -np.inf)
    for n, (b, i) in enumerate(sel):
        keys = visible_keys(q_first_tok + i, k_first_tok, n_keys, wl)
        keys = keys[(keys >= key_lo) & (keys < key_hi)]
        if keys.size == 0:
            continue
        rows = cache[b, keys % wl.ring_slots]
        p, lse[n] = _softmax_lse(scale * (q_abs[b, i] @ rows.T))
        o[n] = p @ rows[:, :d_c]
    if queries is None:
        B, T = q_abs.shape[0], q_abs.shape[1]
        return o.reshape(B, T, *o.shape[1:]), lse.reshape(B, T, -1)
    return o, lse


def merge_partials(parts):
    """Merge pieces (o_p, lse_p) of one softmax attention over disjoint key sets:
    lse = log sum_p exp(lse_p) and o = sum_p exp(lse_p - lse) o_p (a piece with
    lse_p = -inf has weight 0)."""
    lses = np.stack([np.asarray(l, dtype=np.float64) for _, l in parts])      # [P, ...]
    top = lses.max(axis=0)
    safe = np.where(np.isfinite(top), top, 0.0)
    w = np.exp(lses - safe)                                                    # [P, ...]
    tot = w.sum(axis=0)
    lse = np.where(tot > 0, safe + np.log(np.where(tot > 0, tot, 1.0)), -np.inf)
    o = sum(w[k][..., None] * np.asarray(op, dtype=np.float64) for k, (op, _) in enumerate(parts))
    o = o / np.where(tot > 0, tot, 1.0)[..., None]
    return o, lse


def attend_materialised(q_nope: np.ndarray, q_rope: np.ndarray, cache: np.ndarray,
                        w_uk: np.ndarray, w_uv: np.ndarray, q_first_tok: int,
                        k_first_tok: int, n_keys: int, scale: float, wl,
                        queries: Optional[Iterable[Tuple[int, int]]] = None):
    """Non-absorbed attention: per-head keys and values are rebuilt from the latent
    ([MLA explainer] "On-the-Fly Reconstruction and Matrix Absorption"), query and key
    are the concatenation of the content and RoPE channels ([MLA explainer]
    "Decoupling Rotary Position Embeddings (RoPE)"; [MLA concept] "The RoPE problem,
    and the decoupled fix").

    K_h[s] = W_UK[h] c_s, V_h[s] = W_UV[h] c_s,
    score_h(q, s) = scale * ([q_nope,h || RoPE(q_R,h)] . [K_h[s] || k_R,s]),
    o_h(q) = sum_s p_h(q, s) V_h[s].
    Returns (o [.., n_h, d_h], o_lat [.., n_h, d_c], lse [.., n_h]) in the layout of
    ``attend_latent``."""
    q_nope = np.asarray(q_nope, dtype=np.float64)
    cache = np.asarray(cache, dtype=np.float64)
    w_uk = np.asarray(w_uk, dtype=np.float64)
    w_uv = np.asarray(w_uv, dtype=np.float64)
    d_c = wl.d_latent
    n_h = q_nope.shape[2]
    sel = list(queries) if queries is not None else [
        (b, i) for b in range(q_nope.shape[0]) for i in range(q_nope.shape[1])]
    o = np.zeros((len(sel), n_h, wl.d_nope))
    o_lat = np.zeros((len(sel), n_h, d_c))
    lse = np.zeros((len(sel), n_h))
    for n, (b, i) in enumerate(sel):
        g_q = q_first_tok + i
        keys = visible_keys(g_q, k_first_tok, n_keys, wl)
        rows = cache[b, keys % wl.ring_slots]
        c = rows[:, :d_c]
        k_r = rows[:, d_c:]
        q_r = rope3d(np.asarray(q_rope, dtype=np.float64)[b, i][None], [g_q], wl.grid_h,
                     wl.grid_w, wl.rope_pairs, wl.rope_theta)[0]          # [n_h, d_R]
        for h in range(n_h):
            k_h = c @ w_uk[h].T                                 # [L, d_h]
            v_h = c @ w_uv[h].T                                 # [L, d_h]
            q_cat = np.concatenate([q_nope[b, i, h], q_r[h]])
            k_cat = np.concatenate([k_h, k_r], axis=1)
            sc = scale * (k_cat @ q_cat)                        # [L]
            p, l = _softmax_lse(sc[None])
            p = p[0]
            lse[n, h] = l[0]
            o[n, h] = p @ v_h
            o_lat[n, h] = p @ c
    if queries is None:
        B, T = q_nope.shape[0], q_nope.shape[1]
        return (o.reshape(B, T, n_h, -1), o_lat.reshape(B, T, n_h, -1),
                lse.reshape(B, T, n_h))
    return o, o_lat, lse


# ----------------------------------------------------------------------------------
# step a5: W_UV up-projection ([MLA concept] "Low-rank joint compression": the same
# trick folds W^UV into the output side)
# ----------------------------------------------------------------------------------


def up_v(o_lat: np.ndarray, w_uv: np.ndarray) -> np.ndarray:
    """out[..., h, :] = W_UV[h] o_lat[..., h, :]  (W_UV[h] is [d_h, d_c])."""
    return np.einsum("hdc,...hc->...hd", np.asarray(w_uv, dtype=np.float64),
                     np.asarray(o_lat, dtype=np.float64))


# ----------------------------------------------------------------------------------
# closed forms: cache bytes per token ([MLA concept] "The RoPE problem, and the
# decoupled fix": d_c latent dims plus the RoPE dims, not 2 n_h d_h) and work counts
# ----------------------------------------------------------------------------------


def mla_bytes_per_token(d_latent: int, d_rope: int, elem_bytes: int) -> int:
    return (d_latent + d_rope) * elem_bytes


def mha_bytes_per_token(n_heads: int, d_head: int, elem_bytes: int) -> int:
    return 2 * n_heads * d_head * elem_bytes


def visible_pairs(wl) -> int:
    """Number of (query, key) pairs the mask leaves visible, summed over the batch."""
    total = 0
    counted = {}
    f = wl.grid_h * wl.grid_w
    for i in range(wl.n_queries):
        fq = (wl.q_first_tok + i) // f
        if fq not in counted:
            counted[fq] = len(visible_keys(wl.q_first_tok + i, wl.k_first_tok, wl.n_keys, wl))
        total += counted[fq]
    return total * wl.batch


def attention_flops(wl) -> int:
    """Absorbed attention flops: per visible (query, key, head) triple a dot product
    over d_c + d_R and an accumulation over d_c (2 flops per multiply-add)."""
    per = 2 * (wl.d_latent + wl.d_rope) + 2 * wl.d_latent
    return visible_pairs(wl) * wl.n_heads * per
