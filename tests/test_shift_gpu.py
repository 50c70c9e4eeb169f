"""Whole-frame re-indexing of cached RoPE keys (mla_cache_shift_frames) against the oracle.

Row parity: the shifted ring against the oracle's shift of the same ring (the latent and
the untouched y, x pairs bit-exact).  End to end, at small and full sizes: shifting every
window key by as many frames as the ring holds, and moving the queries by the same
amount, leaves the attention output unchanged (rotary relative invariance; the slots
coincide because the shift is a whole ring)."""

import numpy as np
import pytest
import torch

import latent_kv_cache_write_b200 as mla
import oracle.mla_oracle as O
from synth import configs as C
from tests import gpu_path as P

pytestmark = pytest.mark.gpu

SMALL = [C.TINY] + [C.small_variant(w) for w in (C.VIDEO_CHUNK, C.LONG_WINDOW, C.WIDE_KEY)]


@pytest.mark.parametrize("wl", SMALL, ids=lambda w: w.name)
@pytest.mark.parametrize("delta", [3, -1])
def test_rows_against_oracle(wl, delta, cuda_ok):
    r = P.populate(wl, seed=0)
    F = wl.tokens_per_frame
    first = wl.k_first_tok + F                         # the window past its first frame
    n = wl.n_keys - F
    before = P.download(r.cache)
    mla.mla_cache_shift_frames(r.shape, r.cache, first, n, delta)
    after = P.download(r.cache)
    ref = O.shift_frames(before, first, n, delta, wl)
    P.tol_check(after, ref, wl.dtype, "shifted ring")
    d_c, n_t = wl.d_latent, wl.rope_pairs[0]
    assert np.array_equal(after[..., :d_c], before[..., :d_c])          # latent untouched
    assert np.array_equal(after[..., d_c + 2 * n_t:], before[..., d_c + 2 * n_t:])   # y, x
    slots = {g % wl.ring_slots for g in range(first, first + n)}
    others = [s for s in range(wl.ring_slots) if s not in slots]
    assert np.array_equal(after[:, others], before[:, others], equal_nan=True)


def _attend(r, wl, q_first, k_first):
    T = wl.n_queries
    o = P.empty(wl, (wl.batch, T, wl.n_heads, wl.d_latent))
    nws = mla.mla_attend_workspace_size(r.shape, T, wl.n_keys)
    ws = torch.empty(max(nws, 16), dtype=torch.uint8, device=P.DEV)
    mla.mla_attend(r.shape, r.q_abs, T, q_first, r.cache, k_first, wl.n_keys,
                   wl.softmax_scale, o, None, ws, nws)
    return P.download(o)


@pytest.mark.parametrize("wl", [C.small_variant(C.VIDEO_CHUNK), C.VIDEO_CHUNK],
                         ids=lambda w: w.name)
def test_shifted_window_and_queries_attend_alike(wl, cuda_ok):
    F, S = wl.tokens_per_frame, wl.ring_slots
    assert S % F == 0
    ring_frames = S // F
    r = P.run_chunk(P.populate(wl, seed=1), with_lse=False)
    base = _attend(r, wl, wl.q_first_tok, wl.k_first_tok)
    # queries move by a whole ring as well: their RoPE'd part comes from the absorption
    q_first = wl.q_first_tok + S
    mla.mla_absorb_q(r.shape, P.upload(r.q["q_nope"]), P.upload(r.q["q_rope"]), wl.n_queries,
                     q_first, r.wd["w_uk"], r.q_abs)
    mla.mla_cache_shift_frames(r.shape, r.cache, wl.k_first_tok, wl.n_keys, ring_frames)
    moved = _attend(r, wl, q_first, wl.k_first_tok + S)
    P.tol_check(moved, base, wl.dtype, "attention after a whole-ring shift")
