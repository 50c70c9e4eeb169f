"""Two host threads drive the library at once, each on its own CUDA stream with its own
workspace and outputs (the state the library keeps is per-device caches behind locks): the
results equal those of one thread calling alone, bit for bit."""

import threading

import pytest
import torch

import latent_kv_cache_write_b200 as mla
from synth import configs as C
from tests import gpu_path as P

pytestmark = pytest.mark.gpu


def _attend(r, wl, stream, out):
    T = wl.n_queries
    nws = mla.mla_attend_workspace_size(r.shape, T, wl.n_keys)
    ws = torch.empty(max(nws, 16), dtype=torch.uint8, device=P.DEV)
    with torch.cuda.stream(stream):
        for _ in range(5):
            mla.mla_attend(r.shape, r.q_abs, T, wl.q_first_tok, r.cache, wl.k_first_tok,
                           wl.n_keys, wl.softmax_scale, out, None, ws, nws, stream=stream)
    stream.synchronize()


def test_two_threads_two_streams(cuda_ok):
    runs = [(C.small_variant(C.VIDEO_CHUNK), 0), (C.small_variant(C.LONG_WINDOW), 1)]
    rs = [P.run_chunk(P.populate(wl, seed=s), with_lse=False) for wl, s in runs]
    alone = []
    for (wl, _), r in zip(runs, rs):
        o = P.empty(wl, (wl.batch, wl.n_queries, wl.n_heads, wl.d_latent))
        _attend(r, wl, torch.cuda.Stream(), o)
        alone.append(o.clone())
    outs = [torch.zeros_like(a) for a in alone]
    streams = [torch.cuda.Stream() for _ in runs]
    errors = []

    def work(k):
        try:
            torch.cuda.set_device(0)
            _attend(rs[k], runs[k][0], streams[k], outs[k])
        except Exception as e:  # noqa: BLE001 - reported below
            errors.append(e)

    threads = [threading.Thread(target=work, args=(k,)) for k in range(len(runs))]
    for t in threads:
        t.start()
    for t in threads:
        t.join(timeout=120)
    assert not errors, errors
    torch.cuda.synchronize()
    assert mla.mla_device_error() == 0
    for a, o in zip(alone, outs):
        assert torch.equal(a, o)
