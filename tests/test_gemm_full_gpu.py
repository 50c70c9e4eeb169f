"""The absorption and the up-projection on calls with many 128-row tiles per head, against
the oracle on every output element.

The row count leaves the last tile of every head partly out of range (1300 rows: ten full
128-row tiles and one of 20 rows), the persistent CTAs walk more tiles than there are SMs,
and the wide positional key (d_R = 512) gives the absorption 256 RoPE pairs per row, shared
out over its column tiles."""

import numpy as np
import pytest
import torch

import latent_kv_cache_write_b200 as mla
import oracle.mla_oracle as O
from synth import configs as C
from synth import generate as G
from tests import gpu_path as P

pytestmark = pytest.mark.gpu

SHAPES = [C.VIDEO_CHUNK.scaled(name="chunk_1300_rows", grid_h=25),
          C.WIDE_KEY.scaled(name="wide_1300_rows", batch=1, grid_h=25, ring_slots=10 * 1300)]


def _lat(wl, seed):
    rng = np.random.default_rng([seed, 77])
    x = rng.standard_normal((wl.batch, wl.n_queries, wl.n_heads, wl.d_latent)) * 0.5
    return G.to_storage(x, wl.dtype)


@pytest.mark.parametrize("wl", SHAPES, ids=lambda w: w.name)
def test_absorb_all_elements(cuda_ok, wl):
    shape = mla.make_shape(wl)
    w = G.weights(wl, 3)
    q = G.queries(wl, 3)
    T = wl.n_queries
    q_abs = P.empty(wl, (wl.batch, T, wl.n_heads, wl.row_width)).fill_(float("nan"))
    mla.mla_absorb_q(shape, P.upload(q["q_nope"]), P.upload(q["q_rope"]), T, wl.q_first_tok,
                     P.upload(w["w_uk"]), q_abs)
    torch.cuda.synchronize()
    assert mla.mla_device_error() == 0
    ref = O.absorb_q(q["q_nope"].values, q["q_rope"].values, w["w_uk"].values,
                     wl.q_first_tok, wl)
    got = P.download(q_abs)
    P.tol_check(got[..., :wl.d_latent], ref[..., :wl.d_latent], wl.dtype, "q_lat")
    P.tol_check(got[..., wl.d_latent:], ref[..., wl.d_latent:], wl.dtype, "RoPE(q_R)")
    # the last (ragged) block of the last head, row by row
    P.tol_check(got[:, -20:, -1], ref[:, -20:, -1], wl.dtype, "last rows of the last head")


@pytest.mark.parametrize("wl", SHAPES, ids=lambda w: w.name)
def test_up_v_all_elements(cuda_ok, wl):
    shape = mla.make_shape(wl)
    w = G.weights(wl, 5)
    lat = _lat(wl, 5)
    T = wl.n_queries
    out = P.empty(wl, (wl.batch, T, wl.n_heads, wl.d_nope)).fill_(float("nan"))
    mla.mla_up_v(shape, P.upload(lat), T, P.upload(w["w_uv"]), out)
    torch.cuda.synchronize()
    assert mla.mla_device_error() == 0
    ref = O.up_v(lat.values, w["w_uv"].values)
    got = P.download(out)
    P.tol_check(got, ref, wl.dtype, "out")
    P.tol_check(got[:, -20:, -1], ref[:, -20:, -1], wl.dtype, "last rows of the last head")
    # the same call twice gives the same bits (fixed unit ranges, no atomics)
    out2 = torch.empty_like(out)
    mla.mla_up_v(shape, P.upload(lat), T, P.upload(w["w_uv"]), out2)
    torch.cuda.synchronize()
    assert torch.equal(out.view(torch.int16), out2.view(torch.int16))
