"""Absorbed attention at large score magnitudes, against the fp64 oracle.

The score is a content term plus a positional term ("Multi-Head Latent Attention" concept
page, "The RoPE problem, and the decoupled fix") at any magnitude.  The tensor-core kernel
splits each score between the two CTAs of a cluster and swaps the partial sums; these
tests scale q_abs and the cached rows by powers of two (exact in bf16) so that raw partial
scores reach 1e5 and more, beyond the fp16 range, and check every row under the bf16
tolerance: on the chunk shapes (d_R = 64 and the wide d_R = 512 variant), decode, and a
schedule that splits tiles between clusters; with every row scaled, and with only some
queries (or sequences) scaled so that blocks with and without large partials meet in one
launch."""

import numpy as np
import pytest
import torch

import oracle.mla_oracle as O
from synth import configs as C
from tests import gpu_path as P

pytestmark = pytest.mark.gpu

SPLIT_DECODE = C.small_variant(C.DECODE).scaled(
    name="decode_split", batch=8, ring_slots=4096, window_frames=4095, first_chunk_frame=4095)

SHAPES = [C.small_variant(C.VIDEO_CHUNK), C.small_variant(C.LONG_WINDOW),
          C.small_variant(C.WIDE_KEY), C.small_variant(C.DECODE), SPLIT_DECODE]


def _attend(r, wl, q_abs, cache):
    import latent_kv_cache_write_b200 as mla
    T = wl.n_queries
    o = torch.full((wl.batch, T, wl.n_heads, wl.d_latent), float("nan"), dtype=torch.bfloat16,
                   device=P.DEV)
    lse = torch.full((wl.batch, T, wl.n_heads), float("nan"), dtype=torch.float32, device=P.DEV)
    nws = mla.mla_attend_workspace_size(r.shape, T, wl.n_keys)
    ws = torch.empty(max(nws, 16), dtype=torch.uint8, device=P.DEV)
    mla.mla_attend(r.shape, q_abs, T, wl.q_first_tok, cache, wl.k_first_tok, wl.n_keys,
                   wl.softmax_scale, o, lse, ws, nws)
    torch.cuda.synchronize()
    assert mla.mla_device_error() == 0
    return P.download(o), lse.cpu().numpy()


@pytest.mark.parametrize("wl", SHAPES, ids=lambda w: w.name)
@pytest.mark.parametrize("mode", ["all_rows", "some_rows"])
def test_large_partial_scores(cuda_ok, wl, mode):
    r = P.run_chunk(P.populate(wl, seed=11), with_lse=False)
    q = r.q_abs.clone()
    c = r.cache.clone()
    if mode == "all_rows":
        q.mul_(64.0)                 # raw scores x 4096: partials of 1e4 .. 2e5
        c.mul_(64.0)
    elif wl.decode:
        q[1::2].mul_(256.0)          # every other sequence
    else:
        q[:, wl.n_queries // 2:].mul_(256.0)    # the later half of the chunk's queries
    lat, lse = O.attend_latent(P.download(q), P.download(c), wl.q_first_tok, wl.k_first_tok,
                               wl.n_keys, wl.softmax_scale, wl)
    if mode == "all_rows":
        # the largest raw score the rows reach (lse is at least the scaled maximum)
        assert float(np.max(lse)) / wl.softmax_scale > 1e5
    got, got_lse = _attend(r, wl, q, c)
    P.tol_check(got, lat, wl.dtype, f"o_lat {mode}")
    np.testing.assert_allclose(got_lse, lse, rtol=1e-5, atol=2e-2)
