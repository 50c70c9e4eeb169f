"""Pins of the fp64 oracle against facts that do not come from the oracle itself.

Each ``pin_*`` function raises AssertionError when the oracle disagrees with:
the absorption identity, the geometry of rotary embeddings, a pure-Python brute-force
evaluation, textbook or library routines in special cases, the causal-frame mask,
the ring closed form, or the cache-size closed forms.  The functions are plain so
that ``test_oracle_mutations`` can plant mistakes in the oracle and check that some
pin fails.
"""

from __future__ import annotations

import cmath
import json
import math
import os

import numpy as np
import torch

import oracle.mla_oracle as O
from synth import configs as C
from synth import generate as G

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")

# A miniature workload whose ring wraps, with a 2-frame chunk, odd widths and all
# three RoPE axes active; small enough for pure-Python brute force.
MINI = C.Workload(
    name="mini", dtype="f32", batch=2, n_heads=2, d_nope=4, d_latent=6, d_rope=6,
    rope_pairs=(1, 1, 1), rope_theta=10000.0, grid_h=2, grid_w=2, d_model=5,
    window_frames=2, chunk_frames=2, first_chunk_frame=5, ring_slots=16)

# TINY-shaped workload with a 2-frame chunk so that the frame mask bites.
SMALL = C.TINY.scaled(name="small", chunk_frames=2, first_chunk_frame=4, window_frames=2,
                      ring_slots=64, grid_h=2, grid_w=5, batch=2)


def build_state(wl, seed=0):
    """Push every frame of the workload's history through the oracle cache write."""
    wt = G.weights(wl, seed)
    w = {k: v.values for k, v in wt.items()}
    cache = np.zeros((wl.batch, wl.ring_slots, wl.row_width))
    F = wl.tokens_per_frame
    for f in range(wl.frames_written):
        h = G.hidden_frame(wl, seed, f).values
        cache, _ = O.cache_write(cache, h, w["w_dkv"], w["w_kr"], f * F, wl)
    q = G.queries(wl, seed)
    return w, cache, q["q_nope"].values, q["q_rope"].values


def rel(a, b):
    return float(np.linalg.norm(np.asarray(a) - np.asarray(b)) / max(np.linalg.norm(b), 1e-300))


# ---------------------------------------------------------------- I1 absorption


def pin_absorption_identity():
    """Absorbed scores/outputs equal the materialised ones (the associativity
    identity of weight absorption)."""
    for wl in (SMALL, MINI):
        w, cache, qn, qr = build_state(wl, 1)
        q_abs = O.absorb_q(qn, qr, w["w_uk"], wl.q_first_tok, wl)
        o_lat, lse = O.attend_latent(q_abs, cache, wl.q_first_tok, wl.k_first_tok,
                                     wl.n_keys, wl.softmax_scale, wl)
        out = O.up_v(o_lat, w["w_uv"])
        o_m, o_lat_m, lse_m = O.attend_materialised(
            qn, qr, cache, w["w_uk"], w["w_uv"], wl.q_first_tok, wl.k_first_tok,
            wl.n_keys, wl.softmax_scale, wl)
        assert rel(o_lat, o_lat_m) < 1e-12, rel(o_lat, o_lat_m)
        assert rel(out, o_m) < 1e-12, rel(out, o_m)
        assert rel(lse, lse_m) < 1e-12


# ---------------------------------------------------------------- I2 rotary geometry


def _rope_at(v, pos, pairs, theta):
    return O.rotate_pairs(np.asarray(v, dtype=np.float64),
                          O.rope_angles(*pos, pairs, theta))


def pin_rope_relative():
    """<R(p) q, R(s) k> depends on p - s only, per axis; rotations keep norms and
    compose additively."""
    rng = np.random.default_rng(7)
    pairs = (8, 12, 12)
    for _ in range(20):
        q = rng.standard_normal(64)
        k = rng.standard_normal(64)
        p = rng.integers(0, 60, 3)
        s = rng.integers(0, 60, 3)
        base = _rope_at(q, p, pairs, 1e4) @ _rope_at(k, s, pairs, 1e4)
        for axis in range(3):
            d = np.zeros(3, dtype=int)
            d[axis] = rng.integers(1, 40)
            sh = _rope_at(q, p + d, pairs, 1e4) @ _rope_at(k, s + d, pairs, 1e4)
            assert abs(sh - base) < 1e-9 * (1 + abs(base)), (axis, sh, base)
        # R(p)^T R(s) = R(s - p): <R(p)q, R(s)k> = <q, R(s-p)k>
        rel_form = q @ _rope_at(k, s - p, pairs, 1e4)
        assert abs(rel_form - base) < 1e-9 * (1 + abs(base))
        assert abs(np.linalg.norm(_rope_at(q, p, pairs, 1e4)) - np.linalg.norm(q)) < 1e-12 * 64
        comp = _rope_at(_rope_at(q, p, pairs, 1e4), s, pairs, 1e4)
        assert np.allclose(comp, _rope_at(q, p + s, pairs, 1e4), atol=1e-9)


def pin_rope_textbook_1d():
    """With all pairs on one axis the rotation is the 1-D rotary embedding written as
    complex multiplication z_j * exp(i m base^(-2j/d)) on z_j = v_2j + i v_2j+1."""
    rng = np.random.default_rng(3)
    for d, m in ((4, 5), (16, 37), (64, 8191)):
        v = rng.standard_normal(d)
        got = _rope_at(v, (m, 0, 0), (d // 2, 0, 0), 10000.0)
        for j in range(d // 2):
            z = complex(v[2 * j], v[2 * j + 1]) * cmath.exp(1j * m * 10000.0 ** (-2 * j / d))
            assert abs(got[2 * j] - z.real) < 1e-9 and abs(got[2 * j + 1] - z.imag) < 1e-9
    # textbook values: the first pair turns by exactly one radian per step, and for
    # d = 4 with base 10^4 the second pair turns by 10^-2 radian per step.
    got = _rope_at(np.array([1.0, 0.0, 1.0, 0.0]), (1, 0, 0), (2, 0, 0), 10000.0)
    assert np.allclose(got, [math.cos(1), math.sin(1), math.cos(0.01), math.sin(0.01)],
                       atol=1e-15)


def pin_rope_axes():
    """The t, y, x axes own contiguous segments in that order; moving along one axis
    leaves the other two segments untouched; token positions read frames row-major."""
    pairs = (2, 3, 3)
    v = np.arange(1.0, 17.0)
    for axis, (lo, hi) in enumerate(((0, 4), (4, 10), (10, 16))):
        pos = [0, 0, 0]
        pos[axis] = 3
        got = _rope_at(v, pos, pairs, 1e4)
        mask = np.zeros(16, dtype=bool)
        mask[lo:hi] = True
        assert np.array_equal(got[~mask], v[~mask]), axis
        assert not np.allclose(got[mask], v[mask]), axis
    # 30 x 52 frame: token 3*1560 + 2*52 + 5 is frame 3, row 2, column 5
    assert O.token_position(3 * 1560 + 2 * 52 + 5, 30, 52) == (3, 2, 5)
    assert O.token_position(1559, 30, 52) == (0, 29, 51)
    assert O.token_position(1560, 30, 52) == (1, 0, 0)


def pin_rope_in_cache_and_query():
    """Cached k_R is rotated with the key's absolute position and q_R with the
    query's: the positional score then depends on the position difference only.
    Shifting every token of a sequence by whole frames leaves the scores unchanged."""
    wl = MINI
    rng = np.random.default_rng(11)
    h = rng.standard_normal((1, 3, wl.d_model))
    w_dkv = rng.standard_normal((wl.d_model, wl.d_latent))
    w_kr = rng.standard_normal((wl.d_model, wl.d_rope))
    qr = rng.standard_normal((1, 1, wl.n_heads, wl.d_rope))
    qn = np.zeros((1, 1, wl.n_heads, wl.d_nope))
    w_uk = rng.standard_normal((wl.n_heads, wl.d_nope, wl.d_latent))
    F = wl.tokens_per_frame
    scores = []
    for shift in (0, 3 * F):
        rows = O.cache_rows(h, w_dkv, w_kr, 4 + shift, wl)
        qa = O.absorb_q(qn, qr, w_uk, 6 + shift, wl)
        scores.append(qa[0, 0] @ rows[0].T)
    assert np.allclose(scores[0], scores[1], atol=1e-10)
    # the unrotated content part is position free
    rows0 = O.cache_rows(h, w_dkv, w_kr, 4, wl)
    rows1 = O.cache_rows(h, w_dkv, w_kr, 40, wl)
    assert np.array_equal(rows0[..., :wl.d_latent], rows1[..., :wl.d_latent])


# ---------------------------------------------------------------- I3 brute force


def _brute(wl, seed):
    """Pure-Python loops over tokens, heads and keys with math.exp; no numpy
    arithmetic and no oracle function."""
    wt = G.weights(wl, seed)
    Wdkv = wt["w_dkv"].values.tolist()
    Wkr = wt["w_kr"].values.tolist()
    Wuk = wt["w_uk"].values.tolist()
    Wuv = wt["w_uv"].values.tolist()
    F = wl.grid_h * wl.grid_w
    S = wl.ring_slots

    def rot(vec, g):
        t, rem = divmod(g, F)
        y, x = divmod(rem, wl.grid_w)
        out = list(vec)
        off = 0
        for pos, n in zip((t, y, x), wl.rope_pairs):
            for j in range(n):
                z = complex(vec[off + 2 * j], vec[off + 2 * j + 1]) * cmath.exp(
                    1j * pos * wl.rope_theta ** (-2 * j / (2 * n)))
                out[off + 2 * j], out[off + 2 * j + 1] = z.real, z.imag
            off += 2 * n
        return out

    ring = [[None] * S for _ in range(wl.batch)]
    for f in range(wl.frames_written):
        hf = G.hidden_frame(wl, seed, f).values.tolist()
        for b in range(wl.batch):
            for i in range(F):
                g = f * F + i
                hv = hf[b][i]
                c = [sum(hv[k] * Wdkv[k][j] for k in range(wl.d_model)) for j in range(wl.d_latent)]
                kr = [sum(hv[k] * Wkr[k][j] for k in range(wl.d_model)) for j in range(wl.d_rope)]
                ring[b][g % S] = (g, c, rot(kr, g))
    q = G.queries(wl, seed)
    qn = q["q_nope"].values.tolist()
    qr = q["q_rope"].values.tolist()
    outs, lats, lses = [], [], []
    for b in range(wl.batch):
        for i in range(wl.n_queries):
            gq = wl.q_first_tok + i
            for hh in range(wl.n_heads):
                qrot = rot(qr[b][i][hh], gq)
                sc, vs, cs = [], [], []
                for gk in range(wl.k_first_tok, wl.k_first_tok + wl.n_keys):
                    if gk // F > gq // F:
                        continue
                    g_st, c, kr = ring[b][gk % S]
                    assert g_st == gk
                    kh = [sum(Wuk[hh][d][j] * c[j] for j in range(wl.d_latent)) for d in range(wl.d_nope)]
                    vh = [sum(Wuv[hh][d][j] * c[j] for j in range(wl.d_latent)) for d in range(wl.d_nope)]
                    s = sum(a * k for a, k in zip(qn[b][i][hh], kh)) + sum(a * k for a, k in zip(qrot, kr))
                    sc.append(s * wl.softmax_scale)
                    vs.append(vh)
                    cs.append(c)
                m = max(sc)
                e = [math.exp(s - m) for s in sc]
                z = sum(e)
                outs.append([sum(e[n] * vs[n][d] for n in range(len(e))) / z for d in range(wl.d_nope)])
                lats.append([sum(e[n] * cs[n][j] for n in range(len(e))) / z for j in range(wl.d_latent)])
                lses.append(m + math.log(z))
    shp = (wl.batch, wl.n_queries, wl.n_heads)
    return (np.array(outs).reshape(*shp, -1), np.array(lats).reshape(*shp, -1),
            np.array(lses).reshape(shp))


def pin_brute_force():
    """Oracle (both attention definitions) against the pure-Python evaluation."""
    wl = MINI
    o_b, lat_b, lse_b = _brute(wl, 5)
    w, cache, qn, qr = build_state(wl, 5)
    o_m, lat_m, lse_m = O.attend_materialised(qn, qr, cache, w["w_uk"], w["w_uv"],
                                              wl.q_first_tok, wl.k_first_tok, wl.n_keys,
                                              wl.softmax_scale, wl)
    assert rel(o_m, o_b) < 1e-12 and rel(lat_m, lat_b) < 1e-12 and rel(lse_m, lse_b) < 1e-12
    q_abs = O.absorb_q(qn, qr, w["w_uk"], wl.q_first_tok, wl)
    lat_a, lse_a = O.attend_latent(q_abs, cache, wl.q_first_tok, wl.k_first_tok, wl.n_keys,
                                   wl.softmax_scale, wl)
    assert rel(lat_a, lat_b) < 1e-12 and rel(lse_a, lse_b) < 1e-12
    assert rel(O.up_v(lat_a, w["w_uv"]), o_b) < 1e-12


# ---------------------------------------------------------------- I4 special cases


def _mask_bool(wl):
    F = wl.tokens_per_frame
    gq = np.arange(wl.q_first_tok, wl.q_first_tok + wl.n_queries)
    gk = np.arange(wl.k_first_tok, wl.k_first_tok + wl.n_keys)
    return (gk[None, :] // F) <= (gq[:, None] // F)


def pin_library_sdpa():
    """Materialised attention equals torch's scaled_dot_product_attention (fp64, CPU)
    fed with explicitly built per-head keys [K_h || k_R] and values V_h and the frame
    mask; with d_R = 0 and W_UK = W_UV = I it is multi-query attention with K = V = c."""
    wl = SMALL
    w, cache, qn, qr = build_state(wl, 2)
    F = wl.tokens_per_frame
    gk = np.arange(wl.k_first_tok, wl.k_first_tok + wl.n_keys)
    rows = cache[:, gk % wl.ring_slots]                          # [B, L, dc+dR]
    c, kr = rows[..., :wl.d_latent], rows[..., wl.d_latent:]
    qrot = np.stack([np.stack([_rope_at(qr[b, i, h], O.token_position(wl.q_first_tok + i, wl.grid_h, wl.grid_w),
                                        wl.rope_pairs, wl.rope_theta)
                               for h in range(wl.n_heads)]) for b in range(wl.batch)
                     for i in range(wl.n_queries)]).reshape(qr.shape)
    Q = torch.from_numpy(np.concatenate([qn, qrot], -1)).permute(0, 2, 1, 3)        # B,H,T,D
    K = torch.from_numpy(np.concatenate([
        np.einsum("blc,hdc->bhld", c, w["w_uk"]),
        np.broadcast_to(kr[:, None], (wl.batch, wl.n_heads) + kr.shape[1:])], -1))
    V = torch.from_numpy(np.einsum("blc,hdc->bhld", c, w["w_uv"]))
    mask = torch.from_numpy(_mask_bool(wl))
    ref = torch.nn.functional.scaled_dot_product_attention(
        Q, K, V, attn_mask=mask, scale=wl.softmax_scale).permute(0, 2, 1, 3).numpy()
    o_m, _, _ = O.attend_materialised(qn, qr, cache, w["w_uk"], w["w_uv"], wl.q_first_tok,
                                      wl.k_first_tok, wl.n_keys, wl.softmax_scale, wl)
    assert rel(o_m, ref) < 1e-12, rel(o_m, ref)

    # MQA special case: no RoPE channel, identity up-projections.
    mq = wl.scaled(name="mqa", d_rope=0, rope_pairs=(0, 0, 0), d_nope=wl.d_latent)
    w2, cache2, qn2, qr2 = build_state(mq, 3)
    eye = np.broadcast_to(np.eye(mq.d_latent), (mq.n_heads, mq.d_latent, mq.d_latent))
    rows2 = cache2[:, gk % mq.ring_slots]
    Q2 = torch.from_numpy(qn2).permute(0, 2, 1, 3)
    K2 = torch.from_numpy(rows2)[:, None].expand(-1, mq.n_heads, -1, -1)
    ref2 = torch.nn.functional.scaled_dot_product_attention(
        Q2, K2, K2, attn_mask=mask, scale=0.3).permute(0, 2, 1, 3).numpy()
    qa = O.absorb_q(qn2, qr2, eye, mq.q_first_tok, mq)
    lat, _ = O.attend_latent(qa, cache2, mq.q_first_tok, mq.k_first_tok, mq.n_keys, 0.3, mq)
    assert rel(lat, ref2) < 1e-12
    o2, _, _ = O.attend_materialised(qn2, qr2, cache2, eye, eye, mq.q_first_tok,
                                     mq.k_first_tok, mq.n_keys, 0.3, mq)
    assert rel(o2, ref2) < 1e-12


def pin_degenerate_cases():
    """One visible key gives its value; a zero query averages the visible values;
    one-token frames give token-causal attention."""
    wl = C.TINY.scaled(name="causal", grid_h=1, grid_w=1, window_frames=5, chunk_frames=3,
                       first_chunk_frame=5, ring_slots=8, rope_pairs=(8, 0, 0))
    w, cache, qn, qr = build_state(wl, 4)
    # one visible key: query at the window's first token, keys starting there
    o, lat, _ = O.attend_materialised(qn[:, :1], qr[:, :1], cache, w["w_uk"], w["w_uv"],
                                      0, 0, 8, wl.softmax_scale, wl)
    c0 = cache[:, 0, :wl.d_latent]
    assert np.allclose(lat[:, 0], np.broadcast_to(c0[:, None], lat[:, 0].shape), atol=1e-12)
    assert np.allclose(o[:, 0], np.einsum("hdc,bc->bhd", w["w_uv"], c0), atol=1e-12)
    # zero query: uniform weights over the visible keys
    z = np.zeros_like(qn)
    zr = np.zeros_like(qr)
    _, lat, lse = O.attend_materialised(z, zr, cache, w["w_uk"], w["w_uv"], wl.q_first_tok,
                                        wl.k_first_tok, wl.n_keys, wl.softmax_scale, wl)
    for i in range(wl.n_queries):
        n_vis = wl.q_first_tok + i - wl.k_first_tok + 1       # token-causal
        keys = np.arange(wl.k_first_tok, wl.k_first_tok + n_vis) % wl.ring_slots
        mean = cache[:, keys, :wl.d_latent].mean(axis=1)
        assert np.allclose(lat[:, i], mean[:, None], atol=1e-12)
        assert np.allclose(lse[:, i], math.log(n_vis), atol=1e-12)


# ---------------------------------------------------------------- I5 mask


def pin_mask_isolation():
    """Perturbing keys of later frames, or ring slots outside the window, changes
    nothing; perturbing a visible key changes the output."""
    wl = SMALL
    w, cache, qn, qr = build_state(wl, 6)
    args = (qn, qr)
    base = O.attend_materialised(*args, cache, w["w_uk"], w["w_uv"], wl.q_first_tok,
                                 wl.k_first_tok, wl.n_keys, wl.softmax_scale, wl)[0]
    F = wl.tokens_per_frame
    last = wl.first_chunk_frame + wl.chunk_frames - 1
    pert = cache.copy()
    later = np.arange(last * F, (last + 1) * F) % wl.ring_slots
    pert[:, later] += 100.0
    o = O.attend_materialised(*args, pert, w["w_uk"], w["w_uv"], wl.q_first_tok,
                              wl.k_first_tok, wl.n_keys, wl.softmax_scale, wl)[0]
    nq_first = F  # queries of the chunk's first frame do not see its last frame
    assert np.array_equal(o[:, :nq_first], base[:, :nq_first])
    assert not np.allclose(o[:, nq_first:], base[:, nq_first:])
    outside = sorted(set(range(wl.ring_slots)) -
                     set(np.arange(wl.k_first_tok, wl.k_first_tok + wl.n_keys) % wl.ring_slots))
    if outside:
        pert = cache.copy()
        pert[:, outside] = 1e6
        o = O.attend_materialised(*args, pert, w["w_uk"], w["w_uv"], wl.q_first_tok,
                                  wl.k_first_tok, wl.n_keys, wl.softmax_scale, wl)[0]
        assert np.array_equal(o, base)


# ---------------------------------------------------------------- I6 ring


def pin_ring_slots():
    """Slot of token g is g mod S; after the ring wraps every slot holds the row of
    its most recent writer."""
    wl = C.small_variant(C.LONG_WINDOW).scaled(d_model=16, d_latent=8, d_rope=64, n_heads=2)
    w = {k: v.values for k, v in G.weights(wl, 0).items()}
    cache = np.full((wl.batch, wl.ring_slots, wl.row_width), np.nan)
    F = wl.tokens_per_frame
    for f in range(wl.frames_written):
        h = G.hidden_frame(wl, 0, f).values
        cache, slots = O.cache_write(cache, h, w["w_dkv"], w["w_kr"], f * F, wl)
        g = np.arange(f * F, (f + 1) * F)
        assert np.array_equal(slots[0], g - (g // wl.ring_slots) * wl.ring_slots)
    n_tok = wl.frames_written * F
    assert n_tok > 2 * wl.ring_slots
    for s in range(wl.ring_slots):
        last = max(g for g in range(n_tok) if g % wl.ring_slots == s)
        f, i = divmod(last, F)
        h = G.hidden_frame(wl, 0, f).values[:, i:i + 1]
        assert np.array_equal(cache[:, s], O.cache_rows(h, w["w_dkv"], w["w_kr"], last, wl)[:, 0])


def pin_split_key_merge():
    """Attention over the visible keys cut into disjoint pieces at arbitrary points, each
    piece normalised on its own and merged by log-sum-exp, equals the attention over all
    of them; pieces past a query's last visible key carry no weight."""
    for wl in (MINI, SMALL):
        w, cache, qn, qr = build_state(wl, 0)
        qa = O.absorb_q(qn, qr, w["w_uk"], wl.q_first_tok, wl)
        full_o, full_l = O.attend_latent(qa, cache, wl.q_first_tok, wl.k_first_tok, wl.n_keys,
                                         wl.softmax_scale, wl)
        lo, hi = wl.k_first_tok, wl.k_first_tok + wl.n_keys
        rng = np.random.default_rng(7)
        for n_cut in (1, 2, 3):
            cuts = sorted(set(rng.integers(lo + 1, hi, n_cut).tolist()))
            edges = [lo] + cuts + [hi]
            parts = [O.attend_latent_part(qa, cache, wl.q_first_tok, wl.k_first_tok, wl.n_keys,
                                          wl.softmax_scale, wl, a, b)
                     for a, b in zip(edges[:-1], edges[1:])]
            o, l = O.merge_partials(parts)
            assert rel(o, full_o) < 1e-12 and rel(l, full_l) < 1e-12, (wl.name, edges)
        # the chunk's last frame as its own piece: earlier chunk frames see none of it
        F = wl.tokens_per_frame
        parts = [O.attend_latent_part(qa, cache, wl.q_first_tok, wl.k_first_tok, wl.n_keys,
                                      wl.softmax_scale, wl, a, b)
                 for a, b in ((lo, hi - F), (hi - F, hi))]
        assert np.isneginf(parts[1][1][:, :F]).all()
        o, l = O.merge_partials(parts)
        assert rel(o, full_o) < 1e-12 and rel(l, full_l) < 1e-12


def pin_frame_shift():
    """Re-indexing cached RoPE keys by whole frames equals writing the same hidden states
    at the shifted positions (rotations compose: R(p + d) = R(d) R(p), and a shift by
    whole frames changes t only), leaves the latent untouched, and shifting back
    restores the rows."""
    wl = SMALL
    w = {k: v.values for k, v in G.weights(wl, 0).items()}
    F = wl.tokens_per_frame
    h = G.hidden_frame(wl, 0, 1).values                   # one frame of hidden states
    first = 1 * F
    for delta in (2, -1, 5):
        cache = np.zeros((wl.batch, wl.ring_slots, wl.row_width))
        cache, _ = O.cache_write(cache, h, w["w_dkv"], w["w_kr"], first, wl)
        shifted = O.shift_frames(cache, first, F, delta, wl)
        direct = O.cache_rows(h, w["w_dkv"], w["w_kr"], first + delta * F, wl)
        slots = [g % wl.ring_slots for g in range(first, first + F)]
        assert rel(shifted[:, slots], direct) < 1e-12, delta
        assert np.array_equal(shifted[:, slots, :wl.d_latent], cache[:, slots, :wl.d_latent])
        back = O.shift_frames(shifted, first, F, -delta, wl)
        assert rel(back, cache) < 1e-12
        others = [s for s in range(wl.ring_slots) if s not in slots]
        assert np.array_equal(shifted[:, others], cache[:, others])


# ---------------------------------------------------------------- C1, C2 closed forms


def pin_cache_bytes():
    """Per-token cache bytes: (d_c + d_R) b for the latent ring against 2 n_h d_h b for
    a per-head cache; the ring array holds exactly that many bytes per slot."""
    g = json.load(open(os.path.join(GOLDEN, "videomla_cache_dims.json")))
    mla = O.mla_bytes_per_token(g["mla_content_latent"], g["mla_positional_key"], 2)
    mha = O.mha_bytes_per_token(g["mha_heads"], g["mha_head_dim"], 2)
    assert mla == 2 * g["mla_dims_per_token_printed"]
    assert abs(1 - mla / mha - 0.875) < 1e-12          # the printed dims give 87.5 %
    assert abs(1 - mla / mha - g["headline_reduction_percent"] / 100) > 0.04
    expect = {"tiny_f32": (320, 1024), "video_chunk_bf16": (1152, 16384),
              "long_window_bf16": (1152, 16384), "wide_key_bf16": (2048, 16384),
              "decode_bf16": (1152, 65536)}
    for wl in C.ALL:
        b = wl.elem_bytes
        assert (O.mla_bytes_per_token(wl.d_latent, wl.d_rope, b),
                O.mha_bytes_per_token(wl.n_heads, wl.d_nope, b)) == expect[wl.name]
    wl = SMALL
    _, cache, _, _ = build_state(wl, 0)
    cache32 = cache.astype(np.float32)
    assert cache32.nbytes // (wl.batch * wl.ring_slots) == O.mla_bytes_per_token(
        wl.d_latent, wl.d_rope, 4)


def pin_flop_counts():
    """Visible (query, key) pairs and absorbed-attention flops against explicit
    enumeration and against the dense-chunk closed forms."""
    for wl in (MINI, SMALL, C.small_variant(C.LONG_WINDOW)):
        F = wl.tokens_per_frame
        n = 0
        for i in range(wl.n_queries):
            for gk in range(wl.k_first_tok, wl.k_first_tok + wl.n_keys):
                n += gk // F <= (wl.q_first_tok + i) // F
        assert O.visible_pairs(wl) == n * wl.batch
    wl = C.VIDEO_CHUNK      # a one-frame chunk sees the whole window
    assert O.attention_flops(wl) == 1560 * 6240 * 32 * (2 * 576 + 2 * 512)
    wl = C.LONG_WINDOW      # chunk frame k sees 22 + k frames
    pairs = sum(1560 * (22 + k) * 1560 for k in range(3))
    assert O.attention_flops(wl) == pairs * 32 * 2176
    assert O.attention_flops(C.DECODE) == 64 * 8192 * 128 * 2176


ALL_PINS = [pin_absorption_identity, pin_rope_relative, pin_rope_textbook_1d,
            pin_rope_axes, pin_rope_in_cache_and_query, pin_brute_force,
            pin_library_sdpa, pin_degenerate_cases, pin_mask_isolation,
            pin_ring_slots, pin_split_key_merge, pin_frame_shift, pin_cache_bytes,
            pin_flop_counts]
