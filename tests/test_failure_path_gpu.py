"""The library's failure path on the GPU, without a fault: a bounded device-side wait that
nothing satisfies gives up after its limit, the kernel returns, the host reads
MLA_ERR_TIMEOUT with the site that gave up, and the device keeps working."""

import time

import pytest

import latent_kv_cache_write_b200 as mla
from latent_kv_cache_write_b200 import native
from synth import configs as C
from tests import gpu_path as P

pytestmark = pytest.mark.gpu


def test_expired_wait_is_reported_and_the_device_stays_usable(cuda_ok):
    assert mla.mla_device_error() == native.MLA_OK            # nothing pending
    t0 = time.monotonic()
    mla.mla_check_wait_timeout()
    assert mla.mla_device_error() == native.MLA_ERR_TIMEOUT
    waited = time.monotonic() - t0
    assert 1.0 < waited < 60.0, waited                          # the wait's limit is ~2 s
    info = mla.mla_device_error_info()
    assert info[0] & 1 and info[1] == 0x7FF, info
    assert mla.mla_device_error() == native.MLA_OK              # the word was cleared
    # the same process and device still run the path correctly
    wl = C.small_variant(C.VIDEO_CHUNK)
    r = P.run_chunk(P.populate(wl, seed=0))
    assert mla.mla_device_error() == native.MLA_OK
    assert bool((r.out.float().abs() < 1e4).all())
