"""The non-absorbed path (mla_attend_materialised) against the fp64 oracle.

Small workloads (several query blocks and heads, ragged query tails, a ring that wraps, a
ring whose unwritten slots hold NaN) are compared in full with the oracle's materialised
definition, which rebuilds every head's keys and values from the latent.  At full sizes
that definition is too slow to evaluate per sampled row, so sampled rows are compared
with the oracle's absorbed form followed by its up-projection: both are the oracle, and
the associativity pin ties them to the materialised definition."""

import numpy as np
import pytest
import torch

import latent_kv_cache_write_b200 as mla
import oracle.mla_oracle as O
from synth import configs as C
from tests import gpu_path as P

pytestmark = pytest.mark.gpu

# several 128-query blocks with a ragged tail, several sequences, a wrapped ring
SMALL = [C.small_variant(C.VIDEO_CHUNK), C.small_variant(C.LONG_WINDOW),
         C.small_variant(C.VIDEO_CHUNK).scaled(name="mat_ragged", batch=3, n_heads=5,
                                               window_frames=5, chunk_frames=2,
                                               first_chunk_frame=9, ring_slots=7 * 66),
         # 66 ring slots never written (NaN): the last key block's box reaches into them
         C.small_variant(C.VIDEO_CHUNK).scaled(name="mat_spare_slots", ring_slots=5 * 66),
         # the wide positional key (d_R = 512: 32-key blocks): two sequences, a ragged
         # 45-query tile; and three chunk frames (135 queries: two query blocks) over a
         # ring the history wraps
         C.small_variant(C.WIDE_KEY),
         C.small_variant(C.WIDE_KEY).scaled(name="mat_wide_wrapped", chunk_frames=3,
                                            window_frames=4, first_chunk_frame=9,
                                            ring_slots=8 * 45)]
WIDE_SMALL = SMALL[4]


def run_materialised(r, with_lse=True):
    wl = r.wl
    T = wl.n_queries
    out = P.empty(wl, (wl.batch, T, wl.n_heads, wl.d_nope))
    lse = torch.empty((wl.batch, T, wl.n_heads), dtype=torch.float32, device=P.DEV) \
        if with_lse else None
    nws = mla.mla_attend_materialised_workspace_size(r.shape)
    assert nws == 2 * wl.batch * wl.ring_slots * wl.n_heads * wl.d_nope * 2
    ws = torch.empty(nws, dtype=torch.uint8, device=P.DEV)
    mla.mla_attend_materialised(r.shape, P.upload(r.q["q_nope"]), P.upload(r.q["q_rope"]), T,
                                wl.q_first_tok, r.cache, wl.k_first_tok, wl.n_keys,
                                wl.softmax_scale, r.wd["w_uk"], r.wd["w_uv"], out, lse, ws)
    assert mla.mla_device_error() == 0
    return out, lse


@pytest.mark.parametrize("wl", SMALL, ids=lambda w: w.name)
def test_small_against_materialised_definition(wl, cuda_ok):
    r = P.populate(wl, seed=0)          # unwritten ring slots hold NaN
    out, lse = run_materialised(r)
    cache = P.download(r.cache)
    o, _, lse_ref = O.attend_materialised(
        r.q["q_nope"].values, r.q["q_rope"].values, cache, r.w["w_uk"].values,
        r.w["w_uv"].values, wl.q_first_tok, wl.k_first_tok, wl.n_keys, wl.softmax_scale, wl)
    P.tol_check(P.download(out), o, wl.dtype, "out")
    assert np.abs(lse.cpu().numpy() - lse_ref).max() < 2e-2


@pytest.mark.parametrize("wl", [SMALL[2], WIDE_SMALL], ids=lambda w: w.name)
def test_small_matches_absorbed_path(wl, cuda_ok):
    """Both forms of the same attention on the GPU agree to bf16 rounding."""
    r = P.run_chunk(P.populate(wl, seed=0))
    out, lse = run_materialised(r)
    P.tol_check(P.download(out), P.download(r.out), wl.dtype, "materialised vs absorbed")
    assert torch.max(torch.abs(lse - r.lse)).item() < 2e-2


def test_without_lse(cuda_ok):
    wl = SMALL[0]
    r = P.populate(wl, seed=0)
    out_a, _ = run_materialised(r, with_lse=True)
    out_b, _ = run_materialised(r, with_lse=False)
    assert torch.equal(out_a, out_b)


@pytest.mark.parametrize("wl", [C.VIDEO_CHUNK, C.LONG_WINDOW, C.WIDE_KEY], ids=lambda w: w.name)
def test_full_sampled_rows(wl, cuda_ok):
    r = P.populate(wl, seed=0)
    out, lse = run_materialised(r)
    rng = np.random.default_rng(3)
    T, F = wl.n_queries, wl.tokens_per_frame
    qs = {0, 1, 127, 128, 129, T - 1} | {f * F + d for f in range(wl.chunk_frames)
                                          for d in (-1, 0, 1)}
    qs |= set(rng.integers(0, T, 6).tolist())
    sel = [(0, i) for i in sorted(q for q in qs if 0 <= q < T)]
    cache = P.download(r.cache)
    qn, qr = r.q["q_nope"].values, r.q["q_rope"].values
    qa = np.zeros((wl.batch, T, wl.n_heads, wl.row_width))
    for b, i in sel:
        qa[b, i] = O.absorb_q(qn[b:b + 1, i:i + 1], qr[b:b + 1, i:i + 1], r.w["w_uk"].values,
                              wl.q_first_tok + i, wl)[0, 0]
    lat, lse_ref = O.attend_latent(qa, cache, wl.q_first_tok, wl.k_first_tok, wl.n_keys,
                                   wl.softmax_scale, wl, queries=sel)
    ref = O.up_v(lat, r.w["w_uv"].values)
    idx = torch.tensor([i for _, i in sel], device=P.DEV)
    P.tol_check(P.download(out[0, idx]), ref, wl.dtype, "out sampled")
    assert np.abs(lse[0, idx].cpu().numpy() - lse_ref).max() < 2e-2
    del r, out, lse
    torch.cuda.empty_cache()
