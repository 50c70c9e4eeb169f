"""Attention over the low-bit ring with the dequantisation inside the kernel
(mla_attend_quantised), against the oracle's attention over the same quantised ring.

The QuantMLA abstract on the "Multi-Head Latent Attention" topic page has the attention
kernel unpack and dequantise the INT4 / INT2 content codes and the INT4 RoPE codes itself.
The ring is written by mla_cache_quantise on the GPU; the oracle dequantises the same codes
and scales exactly (code * scale in float64) and attends over them.  Compared under the
bf16 tolerance on the chunk shapes (one with a ring that wraps), decode, a schedule that
splits tiles between clusters and full-size decode on sampled sequences; also against
mla_attend over the ring mla_cache_dequantise rebuilds."""

import numpy as np
import pytest
import torch

import latent_kv_cache_write_b200 as mla
import oracle.latent_quant as QZ
from synth import configs as C
from tests import gpu_path as P

pytestmark = pytest.mark.gpu

SPLIT_DECODE = C.small_variant(C.DECODE).scaled(
    name="decode_split", batch=8, ring_slots=4096, window_frames=4095, first_chunk_frame=4095)
SHAPES = [C.small_variant(C.VIDEO_CHUNK), C.small_variant(C.LONG_WINDOW),
          C.small_variant(C.DECODE), SPLIT_DECODE]
BITS = [(4, 4), (2, 4)]


def _ring(wl, r, cb, rb):
    B, S = wl.batch, wl.ring_slots
    qc = torch.zeros((B, S, wl.d_latent * cb // 8), dtype=torch.uint8, device=P.DEV)
    qr = torch.zeros((B, S, wl.d_rope * rb // 8), dtype=torch.uint8, device=P.DEV)
    sc = torch.full((B, S), float("nan"), dtype=torch.float32, device=P.DEV)
    sr = torch.full((B, S), float("nan"), dtype=torch.float32, device=P.DEV)
    mla.mla_cache_quantise(r.shape, r.cache, wl.k_first_tok, wl.n_keys, cb, rb, qc, qr, sc, sr)
    return qc, qr, sc, sr


def _host_ring(qc, qr, sc, sr, cb, rb):
    return {"bits": np.array([cb, rb]), "content": qc.cpu().numpy(), "rope": qr.cpu().numpy(),
            "scale_c": sc.cpu().numpy(), "scale_r": sr.cpu().numpy()}


def _attend_q(r, wl, ring, cb, rb, use_ws=True):
    qc, qr, sc, sr = ring
    T = wl.n_queries
    o = torch.full((wl.batch, T, wl.n_heads, wl.d_latent), float("nan"), dtype=torch.bfloat16,
                   device=P.DEV)
    lse = torch.full((wl.batch, T, wl.n_heads), float("nan"), dtype=torch.float32, device=P.DEV)
    ws, nws = None, 0
    if use_ws:
        nws = mla.mla_attend_workspace_size(r.shape, T, wl.n_keys)
        ws = torch.empty(max(nws, 16), dtype=torch.uint8, device=P.DEV)
    n0 = mla.mla_kernel_launches()
    mla.mla_attend_quantised(r.shape, r.q_abs, T, wl.q_first_tok, qc, qr, sc, sr, cb, rb,
                             wl.k_first_tok, wl.n_keys, wl.softmax_scale, o, lse, ws, nws)
    launches = mla.mla_kernel_launches() - n0
    torch.cuda.synchronize()
    assert mla.mla_device_error() == 0
    return o, lse, launches


@pytest.mark.parametrize("wl", SHAPES, ids=lambda w: w.name)
@pytest.mark.parametrize("bits", BITS, ids=lambda b: f"c{b[0]}r{b[1]}")
def test_fused_against_oracle(cuda_ok, wl, bits):
    cb, rb = bits
    r = P.run_chunk(P.populate(wl, seed=4), with_lse=False)
    ring = _ring(wl, r, cb, rb)
    o, lse, launches = _attend_q(r, wl, ring, cb, rb)
    ref, ref_lse = QZ.attend_quantised(P.download(r.q_abs), _host_ring(*ring, cb, rb),
                                       wl.q_first_tok, wl.k_first_tok, wl.n_keys,
                                       wl.softmax_scale, wl)
    P.tol_check(P.download(o), ref, wl.dtype, f"o_lat over the c{cb}r{rb} ring")
    np.testing.assert_allclose(lse.cpu().numpy(), ref_lse, rtol=0, atol=2e-2)
    if wl is SPLIT_DECODE:
        assert launches == 2                       # tiles split: the merge ran
    # the same attention through mla_attend over the ring mla_cache_dequantise rebuilds
    back = P.empty(wl, (wl.batch, wl.ring_slots, wl.row_width)).fill_(float("nan"))
    mla.mla_cache_dequantise(r.shape, *ring, cb, rb, wl.k_first_tok, wl.n_keys, back)
    o2 = torch.empty_like(o)
    nws = mla.mla_attend_workspace_size(r.shape, wl.n_queries, wl.n_keys)
    ws = torch.empty(max(nws, 16), dtype=torch.uint8, device=P.DEV)
    mla.mla_attend(r.shape, r.q_abs, wl.n_queries, wl.q_first_tok, back, wl.k_first_tok,
                   wl.n_keys, wl.softmax_scale, o2, None, ws, nws)
    torch.cuda.synchronize()
    P.tol_check(P.download(o), P.download(o2), wl.dtype, "fused against dequantise + attend")


def test_fused_without_workspace(cuda_ok):
    """Whole-tile schedule (no workspace) gives the same result within rounding."""
    wl = SPLIT_DECODE
    r = P.run_chunk(P.populate(wl, seed=6), with_lse=False)
    ring = _ring(wl, r, 4, 4)
    o1, _, n1 = _attend_q(r, wl, ring, 4, 4, use_ws=True)
    o2, _, n2 = _attend_q(r, wl, ring, 4, 4, use_ws=False)
    assert (n1, n2) == (2, 1)
    err = float(np.linalg.norm(P.download(o1) - P.download(o2)) / np.linalg.norm(P.download(o2)))
    assert err <= 4e-3, err


def test_fused_full_decode_sampled(cuda_ok):
    """The full decode workload (64 sequences x 8192 keys, INT4 ring) on sampled sequences."""
    wl = C.DECODE
    r = P.run_chunk(P.populate(wl, seed=0), with_lse=False)
    ring = _ring(wl, r, 4, 4)
    o, lse, launches = _attend_q(r, wl, ring, 4, 4)
    assert launches in (1, 2)
    rng = np.random.default_rng(3)
    seqs = sorted({0, wl.batch - 1} | set(rng.integers(0, wl.batch, 4).tolist()))
    # the sampled sequences alone (the oracle dequantises whole rings in float64)
    idx = torch.tensor(seqs, device=P.DEV)
    sub = wl.scaled(batch=len(seqs))
    hr = _host_ring(*(t[idx] for t in ring), 4, 4)
    ref, ref_lse = QZ.attend_quantised(P.download(r.q_abs[idx]), hr, sub.q_first_tok,
                                       sub.k_first_tok, sub.n_keys, sub.softmax_scale, sub)
    P.tol_check(P.download(o[idx]), ref, wl.dtype, "o_lat sampled sequences")
    np.testing.assert_allclose(lse[idx].cpu().numpy(), ref_lse, rtol=0, atol=2e-2)
    del r
    torch.cuda.empty_cache()


def test_unsupported_bit_widths(cuda_ok):
    wl = C.small_variant(C.VIDEO_CHUNK)
    r = P.run_chunk(P.populate(wl, seed=1), with_lse=False)
    for cb, rb in ((8, 8), (4, 2), (4, 8)):
        ring = _ring(wl, r, cb, rb)
        with pytest.raises(mla.MlaError) as e:
            _attend_q(r, wl, ring, cb, rb)
        assert e.value.code == 2                     # MLA_ERR_UNSUPPORTED
