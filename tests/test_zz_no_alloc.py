"""mla_attend_fixed_scratch: attention with the split-key scratch in the library's static
device array instead of a caller workspace.  Collected last (file name), so it runs
both on its own and after every other test has used the device.  Its results must equal
those of mla_attend with a full workspace, on two calls in a row (the second call
reuses the array the first one wrote)."""

import numpy as np
import pytest
import torch

from synth import configs as C
from tests import gpu_path as P

pytestmark = pytest.mark.gpu


def _bits(t):
    return t.view(torch.int16).cpu().numpy()


@pytest.mark.parametrize("wl", [C.DECODE, C.small_variant(C.VIDEO_CHUNK),
                                C.small_variant(C.LONG_WINDOW)], ids=lambda w: w.name)
def test_fixed_scratch_matches_workspace(cuda_ok, wl):
    import latent_kv_cache_write_b200 as mla
    r = P.run_chunk(P.populate(wl, seed=7))       # mla_attend with a full workspace
    T = wl.n_queries
    nws = mla.mla_attend_workspace_size(r.shape, T, wl.n_keys)
    assert nws <= 40 * 1024 * 1024                # fits the static array on this device
    outs = []
    for _ in range(2):
        o = torch.full((wl.batch, T, wl.n_heads, wl.d_latent), float("nan"),
                       dtype=torch.bfloat16, device=P.DEV)
        lse = torch.full((wl.batch, T, wl.n_heads), float("nan"), dtype=torch.float32,
                         device=P.DEV)
        mla.mla_attend_fixed_scratch(r.shape, r.q_abs, T, wl.q_first_tok, r.cache,
                                     wl.k_first_tok, wl.n_keys, wl.softmax_scale, o, lse)
        torch.cuda.synchronize()
        assert mla.mla_device_error() == 0
        outs.append((o, lse))
    for o, lse in outs:
        # same kernels, same schedule: bit-identical to the workspace call
        np.testing.assert_array_equal(_bits(o), _bits(r.o_lat))
        np.testing.assert_array_equal(lse.cpu().numpy(), r.lse.cpu().numpy())
