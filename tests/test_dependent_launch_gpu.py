"""Ordering of back-to-back calls.  The library's GEMM, attention and merge kernels are
launched so that each may start while the previous kernel on the stream finishes; each
waits for it (griddepcontrol.wait) before its first global access.

Three chunk steps run back to back with no synchronisation between calls.  Each step is
cache write, absorption, attention (split between clusters, so a merge kernel follows)
and up-projection.  Every step brings a different chunk frame and different queries, and
the steps share the ring, q_abs and o_lat.  So each call reads what the call before it
wrote (read after write), and overwrites what the previous step's calls read (write after
read).  The outputs must equal, bit for bit, those of the same calls with a device
synchronisation after each one."""

import pytest
import torch

from synth import configs as C
from synth import generate as G
from tests import gpu_path as P

pytestmark = pytest.mark.gpu

# many key blocks per tile, about as many tiles as SM pairs: the schedule splits tiles
SPLIT_CHUNK = C.small_variant(C.VIDEO_CHUNK).scaled(
    name="video_chunk_split", batch=5, n_heads=32, chunk_frames=1, window_frames=38,
    first_chunk_frame=38, ring_slots=39 * 66)
STEPS = 3


def _run(wl, sync_each):
    import latent_kv_cache_write_b200 as mla
    r = P.populate(wl, seed=11)
    T, F = wl.n_queries, wl.tokens_per_frame
    ins = [(P.upload(G.hidden_frame(wl, 100 + i, wl.first_chunk_frame)),
            {k: P.upload(v) for k, v in G.queries(wl, 100 + i).items()}) for i in range(STEPS)]
    q_abs = P.empty(wl, (wl.batch, T, wl.n_heads, wl.row_width))
    o_lat = P.empty(wl, (wl.batch, T, wl.n_heads, wl.d_latent))
    outs = [P.empty(wl, (wl.batch, T, wl.n_heads, wl.d_nope)) for _ in range(STEPS)]
    nws = mla.mla_attend_workspace_size(r.shape, T, wl.n_keys)
    ws = torch.empty(max(nws, 16), dtype=torch.uint8, device=P.DEV)
    sync = torch.cuda.synchronize if sync_each else (lambda: None)
    torch.cuda.synchronize()
    n0 = mla.mla_kernel_launches()
    for i, (h, q) in enumerate(ins):
        mla.mla_cache_write(r.shape, h, wl.d_model, F, wl.first_chunk_frame * F, r.wd["w_dkv"],
                            r.wd["w_kr"], r.cache)
        sync()
        mla.mla_absorb_q(r.shape, q["q_nope"], q["q_rope"], T, wl.q_first_tok, r.wd["w_uk"], q_abs)
        sync()
        mla.mla_attend(r.shape, q_abs, T, wl.q_first_tok, r.cache, wl.k_first_tok, wl.n_keys,
                       wl.softmax_scale, o_lat, None, ws, nws)
        sync()
        mla.mla_up_v(r.shape, o_lat, T, r.wd["w_uv"], outs[i])
        sync()
    torch.cuda.synchronize()
    launches = mla.mla_kernel_launches() - n0
    assert mla.mla_device_error() == 0
    return [o.view(torch.int16).cpu() for o in outs], launches


def test_back_to_back_steps_match_synchronised(cuda_ok):
    free, n_free = _run(SPLIT_CHUNK, sync_each=False)
    synced, n_synced = _run(SPLIT_CHUNK, sync_each=True)
    assert n_free == n_synced == 5 * STEPS          # the merge ran in every step
    for i in range(STEPS):
        assert torch.equal(free[i], synced[i]), f"step {i}"
    # the steps differ (each read its own frame and queries)
    assert not torch.equal(free[0], free[1]) and not torch.equal(free[1], free[2])
