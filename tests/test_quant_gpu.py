"""The low-bit latent ring (mla_cache_quantise / mla_cache_dequantise) against the oracle.

Codes and scales are integer and byte results decided by float32 arithmetic, so they are
compared bit-exactly with the oracle's quantiser taking the same decision in float32 on
the rows the GPU ring holds.  Dequantised rows are compared with the oracle's exact
products within one rounding to the storage type, and attention over a ring dequantised on
the GPU with the oracle's attention over the quantised ring (the bf16 or fp32 tolerance)."""

import numpy as np
import pytest
import torch

import latent_kv_cache_write_b200 as mla
import oracle.latent_quant as QZ
from synth import configs as C
from tests import gpu_path as P

pytestmark = pytest.mark.gpu

SMALL = [C.TINY] + [C.small_variant(w) for w in (C.VIDEO_CHUNK, C.LONG_WINDOW, C.WIDE_KEY)]
BITS = [(4, 4), (2, 4), (8, 8)]


def window_slots(wl):
    return [g % wl.ring_slots for g in range(wl.k_first_tok, wl.k_first_tok + wl.n_keys)]


def quantise(r, wl, cb, rb, first=None, n=None):
    B, S = wl.batch, wl.ring_slots
    qc = torch.zeros((B, S, wl.d_latent * cb // 8), dtype=torch.uint8, device=P.DEV)
    qr = torch.zeros((B, S, wl.d_rope * rb // 8), dtype=torch.uint8, device=P.DEV)
    sc = torch.full((B, S), float("nan"), dtype=torch.float32, device=P.DEV)
    sr = torch.full((B, S), float("nan"), dtype=torch.float32, device=P.DEV)
    mla.mla_cache_quantise(r.shape, r.cache, wl.k_first_tok if first is None else first,
                           wl.n_keys if n is None else n, cb, rb, qc, qr, sc, sr)
    return qc, qr, sc, sr


def host(t):
    return t.cpu().numpy()


@pytest.mark.parametrize("wl", SMALL, ids=lambda w: w.name)
@pytest.mark.parametrize("bits", BITS, ids=lambda b: f"c{b[0]}r{b[1]}")
def test_codes_and_scales_bit_exact(wl, bits, cuda_ok):
    cb, rb = bits
    r = P.populate(wl, seed=0)
    qc, qr, sc, sr = quantise(r, wl, cb, rb)
    cache = P.download(r.cache)
    slots = window_slots(wl)
    pc, pr, s_c, s_r = QZ.quantise_row_paths(cache[:, slots], wl, cb, rb, decide=np.float32)
    assert np.array_equal(host(qc)[:, slots], pc)
    assert np.array_equal(host(qr)[:, slots], pr)
    assert np.array_equal(host(sc)[:, slots], s_c)
    assert np.array_equal(host(sr)[:, slots], s_r)
    others = [s for s in range(wl.ring_slots) if s not in set(slots)]
    assert not host(qc)[:, others].any() and np.isnan(host(sc)[:, others]).all()


@pytest.mark.parametrize("wl", SMALL, ids=lambda w: w.name)
@pytest.mark.parametrize("bits", BITS[:2], ids=lambda b: f"c{b[0]}r{b[1]}")
def test_dequantised_rows(wl, bits, cuda_ok):
    cb, rb = bits
    r = P.populate(wl, seed=1)
    qc, qr, sc, sr = quantise(r, wl, cb, rb)
    back = P.empty(wl, (wl.batch, wl.ring_slots, wl.row_width)).fill_(float("nan"))
    mla.mla_cache_dequantise(r.shape, qc, qr, sc, sr, cb, rb, wl.k_first_tok, wl.n_keys, back)
    slots = window_slots(wl)
    got = P.download(back)[:, slots]
    q = {"bits": np.array([cb, rb]), "content": host(qc), "rope": host(qr),
         "scale_c": host(sc), "scale_r": host(sr)}
    ref = QZ.dequantise_cache(q, wl)[:, slots]
    # one rounding of the float32 product to the storage type
    ulp = 2.0 ** -8 if wl.dtype == "bf16" else 2.0 ** -23
    assert np.all(np.abs(got - ref) <= ulp * np.abs(ref))
    others = [s for s in range(wl.ring_slots) if s not in set(slots)]
    assert np.isnan(P.download(back)[:, others]).all()


@pytest.mark.parametrize("wl", SMALL[1:3], ids=lambda w: w.name)
def test_attention_over_quantised_ring(wl, cuda_ok):
    """Chunk attention over an INT4 ring (dequantised on the GPU) against the oracle's
    attention over the same quantised ring."""
    r = P.run_chunk(P.populate(wl, seed=2), with_lse=False)
    qc, qr, sc, sr = quantise(r, wl, 4, 4)
    back = P.empty(wl, (wl.batch, wl.ring_slots, wl.row_width)).fill_(float("nan"))
    mla.mla_cache_dequantise(r.shape, qc, qr, sc, sr, 4, 4, wl.k_first_tok, wl.n_keys, back)
    T = wl.n_queries
    o = P.empty(wl, (wl.batch, T, wl.n_heads, wl.d_latent))
    nws = mla.mla_attend_workspace_size(r.shape, T, wl.n_keys)
    ws = torch.empty(max(nws, 16), dtype=torch.uint8, device=P.DEV)
    mla.mla_attend(r.shape, r.q_abs, T, wl.q_first_tok, back, wl.k_first_tok, wl.n_keys,
                   wl.softmax_scale, o, None, ws, nws)
    q = {"bits": np.array([4, 4]), "content": host(qc), "rope": host(qr),
         "scale_c": host(sc), "scale_r": host(sr)}
    ref, _ = QZ.attend_quantised(P.download(r.q_abs), q, wl.q_first_tok, wl.k_first_tok,
                                 wl.n_keys, wl.softmax_scale, wl)
    P.tol_check(P.download(o), ref, wl.dtype, "attention over the INT4 ring")
    assert mla.mla_device_error() == 0


def test_partial_range_and_empty(cuda_ok):
    wl = C.small_variant(C.LONG_WINDOW)            # the window straddles the ring's end
    r = P.populate(wl, seed=3)
    first, n = wl.k_first_tok + 37, 101
    qc, qr, sc, sr = quantise(r, wl, 2, 4, first=first, n=n)
    slots = [g % wl.ring_slots for g in range(first, first + n)]
    assert slots[0] > slots[-1]                     # the range wraps around the ring
    cache = P.download(r.cache)
    pc, pr, s_c, s_r = QZ.quantise_row_paths(cache[:, slots], wl, 2, 4, decide=np.float32)
    assert np.array_equal(host(qc)[:, slots], pc) and np.array_equal(host(sr)[:, slots], s_r)
    assert int(np.isfinite(host(sc)).sum()) == wl.batch * n
    before = [host(t).copy() for t in (qc, qr, sc, sr)]
    mla.mla_cache_quantise(r.shape, r.cache, first, 0, 2, 4, qc, qr, sc, sr)
    for a, t in zip(before, (qc, qr, sc, sr)):
        assert np.array_equal(a, host(t), equal_nan=True)


def test_full_video_chunk_window(cuda_ok):
    """Every row of the full video-chunk window, INT4 content and RoPE."""
    wl = C.VIDEO_CHUNK
    r = P.populate(wl, seed=0)
    qc, qr, sc, sr = quantise(r, wl, 4, 4)
    cache = P.download(r.cache)
    pc, pr, s_c, s_r = QZ.quantise_row_paths(cache, wl, 4, 4, decide=np.float32)
    assert np.array_equal(host(qc), pc) and np.array_equal(host(qr), pr)
    assert np.array_equal(host(sc), s_c) and np.array_equal(host(sr), s_r)
    assert qc.numel() + qr.numel() + 4 * (sc.numel() + sr.numel()) == \
        wl.batch * wl.ring_slots * QZ.quant_bytes_per_token(wl.d_latent, wl.d_rope, 4, 4)
    del r
    torch.cuda.empty_cache()
