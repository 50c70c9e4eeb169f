"""Plant plausible mistakes in the oracle (on the CPU) and check that the pins catch
every one of them: a pin set that passes a wrong oracle pins nothing."""

import numpy as np
import pytest

import oracle.mla_oracle as O
from tests import oracle_pins as P

_orig = {n: getattr(O, n) for n in (
    "rotate_pairs", "rope_angles", "token_position", "visible_keys", "attend_latent",
    "attend_materialised", "absorb_q", "ring_slot", "up_v", "cache_rows", "_softmax_lse",
    "mla_bytes_per_token", "rope3d", "shift_frames", "merge_partials")}


def _rot_sign(v, angles):
    return _orig["rotate_pairs"](v, -np.asarray(angles))


def _angles_exp(t, y, x, pairs, theta):
    out = []
    for pos, n in zip((t, y, x), pairs):
        out += [pos * theta ** (-2 * j / n) for j in range(n)]
    return np.asarray(out, dtype=np.float64)


def _angles_axis_order(t, y, x, pairs, theta):
    return _orig["rope_angles"](x, y, t, pairs, theta)


def _pos_colmajor(g, grid_h, grid_w):
    f = grid_h * grid_w
    return g // f, (g % f) % grid_h, (g % f) // grid_h


def _visible_strict(g_query, k_first_tok, n_keys, wl):
    ks = np.arange(k_first_tok, k_first_tok + n_keys, dtype=np.int64)
    f = wl.grid_h * wl.grid_w
    keep = ks // f < g_query // f
    keep[ks == g_query] = True
    return ks[keep]


def _latent_no_rope(q_abs, cache, qf, kf, nk, scale, wl, queries=None):
    q = np.array(q_abs, dtype=np.float64, copy=True)
    q[..., wl.d_latent:] = 0.0
    return _orig["attend_latent"](q, cache, qf, kf, nk, scale, wl, queries)


def _mat_no_rope(q_nope, q_rope, *a, **k):
    return _orig["attend_materialised"](q_nope, np.zeros_like(q_rope), *a, **k)


def _absorb_heads_swapped(q_nope, q_rope, w_uk, q_first_tok, wl):
    return _orig["absorb_q"](q_nope, q_rope, np.asarray(w_uk)[::-1], q_first_tok, wl)


def _slot_off(g, s):
    return (g + 1) % s


def _latent_no_scale(q_abs, cache, qf, kf, nk, scale, wl, queries=None):
    return _orig["attend_latent"](q_abs, cache, qf, kf, nk, 1.0, wl, queries)


def _upv_heads_swapped(o_lat, w_uv):
    return _orig["up_v"](o_lat, np.asarray(w_uv)[::-1])


def _rows_one_position(h, w_dkv, w_kr, first_tok, wl):
    h = np.asarray(h, dtype=np.float64)
    c = h @ w_dkv
    kr = h @ w_kr
    toks = [first_tok] * h.shape[1]
    kr = np.stack([_orig["rope3d"](kr[b], toks, wl.grid_h, wl.grid_w, wl.rope_pairs,
                                   wl.rope_theta) for b in range(h.shape[0])])
    return np.concatenate([c, kr], axis=-1)


def _lse_no_max(scores):
    p, lse = _orig["_softmax_lse"](scores)
    return p, lse - scores.max(axis=-1)


def _bytes_no_rope(d_latent, d_rope, elem_bytes):
    return d_latent * elem_bytes


def _merge_unweighted(parts):
    # the plain mean of the pieces, ignoring how much of the softmax mass each holds
    o = sum(np.asarray(op, dtype=np.float64) for op, _ in parts) / len(parts)
    return o, _orig["merge_partials"](parts)[1]


def _merge_lse_max(parts):
    # the largest piece's log-sum-exp instead of the log of the summed masses
    o, _ = _orig["merge_partials"](parts)
    return o, np.max(np.stack([l for _, l in parts]), axis=0)


def _shift_row_axis(cache, first_tok, n_tok, delta_frames, wl):
    # turns the y pairs instead of the t pairs
    out = np.array(cache, dtype=np.float64, copy=True)
    ang = O.rope_angles(0, delta_frames, 0, wl.rope_pairs, wl.rope_theta)
    for g in range(first_tok, first_tok + n_tok):
        s = g % wl.ring_slots
        out[:, s, wl.d_latent:] = O.rotate_pairs(out[:, s, wl.d_latent:], ang)
    return out


def _shift_backwards(cache, first_tok, n_tok, delta_frames, wl):
    return _orig["shift_frames"](cache, first_tok, n_tok, -delta_frames, wl)


MUTATIONS = {
    "rotation_sign": ("rotate_pairs", _rot_sign),
    "rope_frequency_exponent": ("rope_angles", _angles_exp),
    "rope_axis_order": ("rope_angles", _angles_axis_order),
    "frame_column_major": ("token_position", _pos_colmajor),
    "mask_strict_frames": ("visible_keys", _visible_strict),
    "latent_drops_rope_term": ("attend_latent", _latent_no_rope),
    "materialised_drops_rope_term": ("attend_materialised", _mat_no_rope),
    "absorb_wrong_head": ("absorb_q", _absorb_heads_swapped),
    "ring_slot_off_by_one": ("ring_slot", _slot_off),
    "softmax_scale_ignored": ("attend_latent", _latent_no_scale),
    "up_v_wrong_head": ("up_v", _upv_heads_swapped),
    "k_rope_single_position": ("cache_rows", _rows_one_position),
    "lse_missing_max": ("_softmax_lse", _lse_no_max),
    "cache_bytes_drop_rope": ("mla_bytes_per_token", _bytes_no_rope),
    "shift_turns_row_axis": ("shift_frames", _shift_row_axis),
    "shift_backwards": ("shift_frames", _shift_backwards),
    "merge_unweighted": ("merge_partials", _merge_unweighted),
    "merge_lse_max": ("merge_partials", _merge_lse_max),
}


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_planted_mistake_is_caught(name, monkeypatch):
    attr, bad = MUTATIONS[name]
    monkeypatch.setattr(O, attr, bad)
    caught = []
    for pin in P.ALL_PINS:
        try:
            pin()
        except AssertionError:
            caught.append(pin.__name__)
    assert caught, f"no pin catches the planted mistake {name}"
