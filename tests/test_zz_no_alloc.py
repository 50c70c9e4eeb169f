"""mla_attend_fixed_scratch: attention whose split-key scratch is the library's static
device array instead of a caller workspace, for callers that cannot allocate device
memory (a host holding only the tensors it was handed, or a serving loop that must not
call the allocator between steps).

The shapes are ones on which the schedule cuts tiles between clusters, so the kernel
writes partial outputs into the array and the merge kernel reads them back: each call
launches two kernels.  Results must equal mla_attend's with a full workspace bit for bit,
on two calls in a row (the second overwrites what the first left in the array).
Collected last (file name), so it runs both on its own and after every other test has
used the device."""

import numpy as np
import pytest
import torch

from synth import configs as C
from tests import gpu_path as P

pytestmark = pytest.mark.gpu

# many key blocks per tile, about as many tiles as SM pairs: the schedule splits tiles
SPLIT_CHUNK = C.small_variant(C.VIDEO_CHUNK).scaled(
    name="video_chunk_split", batch=5, n_heads=32, chunk_frames=1, window_frames=38,
    first_chunk_frame=38, ring_slots=39 * 66)
SPLIT_DECODE = C.small_variant(C.DECODE).scaled(
    name="decode_split", batch=8, ring_slots=4096, window_frames=4095, first_chunk_frame=4095)
# one sequence's 8192 keys form one tile, cut across every cluster
DECODE_ONE = C.DECODE.scaled(name="decode_one_sequence", batch=1)


def _bits(t):
    return t.view(torch.int16).cpu().numpy()


@pytest.mark.parametrize("wl", [SPLIT_CHUNK, SPLIT_DECODE, DECODE_ONE], ids=lambda w: w.name)
def test_fixed_scratch_matches_workspace(cuda_ok, wl):
    import latent_kv_cache_write_b200 as mla
    r = P.populate(wl, seed=7)
    T = wl.n_queries
    nws = mla.mla_attend_workspace_size(r.shape, T, wl.n_keys)
    assert 0 < nws <= mla.MLA_FIXED_SCRATCH_BYTES   # fits the static array on this device
    n0 = mla.mla_kernel_launches()
    r = P.run_chunk(r)                               # mla_attend with a full workspace
    # absorption, attention, merge, up-projection: the workspace call splits tiles
    assert mla.mla_kernel_launches() - n0 == 4
    outs = []
    for _ in range(2):
        o = torch.full((wl.batch, T, wl.n_heads, wl.d_latent), float("nan"),
                       dtype=torch.bfloat16, device=P.DEV)
        lse = torch.full((wl.batch, T, wl.n_heads), float("nan"), dtype=torch.float32,
                         device=P.DEV)
        n0 = mla.mla_kernel_launches()
        mla.mla_attend_fixed_scratch(r.shape, r.q_abs, T, wl.q_first_tok, r.cache,
                                     wl.k_first_tok, wl.n_keys, wl.softmax_scale, o, lse)
        # the attention kernel wrote partials into the array and the merge read them
        assert mla.mla_kernel_launches() - n0 == 2
        torch.cuda.synchronize()
        assert mla.mla_device_error() == 0
        outs.append((o, lse))
    for o, lse in outs:
        # same kernels, same schedule, same merge order: bit-identical to the workspace call
        np.testing.assert_array_equal(_bits(o), _bits(r.o_lat))
        np.testing.assert_array_equal(lse.cpu().numpy(), r.lse.cpu().numpy())
