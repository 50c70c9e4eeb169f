"""CUDA path against the fp64 oracle, element by element on the same seeded inputs.

Small workloads (the oracle finishes in seconds; several 128-row tiles, several key
blocks, ragged tails, a ring that wraps) are compared in full, kernel by kernel (the
GPU's upstream result, upcast, feeds the oracle's next step) and end to end against
the materialised (non-absorbed) definition.  Full-size workloads run in the launch
configuration the benchmark times and are compared on sampled rows."""

import numpy as np
import pytest
import torch

import oracle.mla_oracle as O
from synth import configs as C
from synth import generate as G
from tests import gpu_path as P

pytestmark = pytest.mark.gpu

SMALL = [C.TINY] + [C.small_variant(w) for w in (C.VIDEO_CHUNK, C.LONG_WINDOW, C.WIDE_KEY,
                                                   C.DECODE)]


def oracle_cache(wl, seed=0):
    w = G.weights(wl, seed)
    cache = np.zeros((wl.batch, wl.ring_slots, wl.row_width))
    F = wl.tokens_per_frame
    for f in range(wl.frames_written):
        h = G.hidden_frame(wl, seed, f).values
        cache, _ = O.cache_write(cache, h, w["w_dkv"].values, w["w_kr"].values, f * F, wl)
    return cache


@pytest.fixture(scope="module", params=SMALL, ids=lambda w: w.name)
def small_run(request, cuda_ok):
    wl = request.param
    return P.run_chunk(P.populate(wl, seed=0))


def test_small_slots_bit_exact(small_run):
    r = small_run
    F = r.wl.tokens_per_frame
    for f, s in enumerate(r.slots):
        g = np.arange(f * F, (f + 1) * F, dtype=np.int64)
        expect = np.broadcast_to(g % r.wl.ring_slots, (r.wl.batch, F)).astype(np.int32)
        assert np.array_equal(s.cpu().numpy(), expect)


def test_small_cache_write(small_run):
    r = small_run
    if r.wl.cache_direct:
        pytest.skip("cache rows drawn directly")
    P.tol_check(P.download(r.cache), oracle_cache(r.wl), r.wl.dtype, "cache")


def test_small_absorb(small_run):
    r = small_run
    ref = O.absorb_q(r.q["q_nope"].values, r.q["q_rope"].values, r.w["w_uk"].values,
                     r.wl.q_first_tok, r.wl)
    P.tol_check(P.download(r.q_abs), ref, r.wl.dtype, "q_abs")


def test_small_attend(small_run):
    r = small_run
    wl = r.wl
    lat, lse = O.attend_latent(P.download(r.q_abs), P.download(r.cache), wl.q_first_tok,
                               wl.k_first_tok, wl.n_keys, wl.softmax_scale, wl)
    P.tol_check(P.download(r.o_lat), lat, wl.dtype, "o_lat")
    P.tol_check(r.lse.cpu().numpy(), lse, wl.dtype, "lse")
    assert np.abs(r.lse.cpu().numpy() - lse).max() < (1e-4 if wl.dtype == "f32" else 2e-2)


def test_small_up_v(small_run):
    r = small_run
    ref = O.up_v(P.download(r.o_lat), r.w["w_uv"].values)
    P.tol_check(P.download(r.out), ref, r.wl.dtype, "out")


def test_small_end_to_end(small_run):
    """GPU output against the materialised definition from the raw inputs."""
    r = small_run
    wl = r.wl
    cache = G.direct_cache(wl, 0).values if wl.cache_direct else oracle_cache(wl)
    o, o_lat, lse = O.attend_materialised(
        r.q["q_nope"].values, r.q["q_rope"].values, cache, r.w["w_uk"].values,
        r.w["w_uv"].values, wl.q_first_tok, wl.k_first_tok, wl.n_keys, wl.softmax_scale, wl)
    P.tol_check(P.download(r.out), o, wl.dtype, "out e2e")
    P.tol_check(P.download(r.o_lat), o_lat, wl.dtype, "o_lat e2e")


# ------------------------------------------------------------------ full sizes


def sample_queries(wl, rng, extra=8):
    T, F = wl.n_queries, wl.tokens_per_frame
    base = {0, 1, 3, 4, 5, T - 1, T - 2}
    for f in range(1, wl.chunk_frames):
        base |= {f * F - 1, f * F, f * F + 1}
    base |= set(rng.integers(0, T, extra).tolist())
    qs = sorted(i for i in base if 0 <= i < T)
    bs = sorted({0, wl.batch - 1} | set(rng.integers(0, wl.batch, 6).tolist())) \
        if wl.decode else list(range(wl.batch))
    return [(b, i) for b in bs for i in qs]


@pytest.fixture(scope="module", params=[C.VIDEO_CHUNK, C.LONG_WINDOW, C.WIDE_KEY, C.DECODE],
                ids=lambda w: w.name)
def full_run(request, cuda_ok):
    wl = request.param
    r = P.run_chunk(P.populate(wl, seed=0))
    yield r
    del r
    torch.cuda.empty_cache()


def test_full_slots_and_cache_rows(full_run):
    r = full_run
    wl = r.wl
    F = wl.tokens_per_frame
    for f, s in enumerate(r.slots):
        g = np.arange(f * F, (f + 1) * F, dtype=np.int64) % wl.ring_slots
        assert np.array_equal(s.cpu().numpy(), np.broadcast_to(g, s.shape).astype(np.int32))
    if wl.cache_direct:
        return
    rng = np.random.default_rng(1)
    first_live = wl.frames_written * F - wl.ring_slots     # oldest token still in the ring
    toks = sorted(set(rng.integers(first_live, wl.frames_written * F, 24).tolist()) |
                  {first_live, wl.frames_written * F - 1})
    w = r.w
    for g in toks:
        f, i = divmod(g, F)
        h = G.hidden_frame(wl, 0, f).values[:, i:i + 1]
        ref = O.cache_rows(h, w["w_dkv"].values, w["w_kr"].values, g, wl)[:, 0]
        got = P.download(r.cache[:, g % wl.ring_slots])
        P.tol_check(got, ref, wl.dtype, f"cache row {g}")


def test_full_sampled_rows(full_run):
    r = full_run
    wl = r.wl
    rng = np.random.default_rng(2)
    sel = sample_queries(wl, rng)
    b_idx = torch.tensor([b for b, _ in sel], device=P.DEV)
    i_idx = torch.tensor([i for _, i in sel], device=P.DEV)
    q_abs_s = P.download(r.q_abs[b_idx, i_idx])                       # [n, H, row]
    # absorption on the sampled queries
    qn = r.q["q_nope"].values
    qr = r.q["q_rope"].values
    ref_q = np.stack([O.absorb_q(qn[b:b + 1, i:i + 1], qr[b:b + 1, i:i + 1], r.w["w_uk"].values,
                                 wl.q_first_tok + i, wl)[0, 0] for b, i in sel])
    P.tol_check(q_abs_s, ref_q, wl.dtype, "q_abs sampled")
    # attention on the sampled rows, fed with the GPU's q_abs and cache
    cache = P.download(r.cache)
    qa = np.zeros((wl.batch, wl.n_queries, wl.n_heads, wl.row_width))
    for n, (b, i) in enumerate(sel):
        qa[b, i] = q_abs_s[n]
    lat, lse = O.attend_latent(qa, cache, wl.q_first_tok, wl.k_first_tok, wl.n_keys,
                               wl.softmax_scale, wl, queries=sel)
    got_lat = P.download(r.o_lat[b_idx, i_idx])
    P.tol_check(got_lat, lat, wl.dtype, "o_lat sampled")
    got_lse = r.lse[b_idx, i_idx].cpu().numpy()
    assert np.abs(got_lse - lse).max() < 2e-2
    # up-projection of the sampled rows
    ref_o = O.up_v(got_lat, r.w["w_uv"].values)
    P.tol_check(P.download(r.out[b_idx, i_idx]), ref_o, wl.dtype, "out sampled")


def test_full_attend_repeatable_and_launches(full_run):
    """A second call gives bit-identical o_lat and lse (fixed schedule and merge order).
    The wide-key workload's four sequences each hold 32 MB of keys, more than a third of
    L2 together, so the call runs one attention launch per sequence (plus any merges);
    the single-sequence chunk shapes and decode run one."""
    r = full_run
    wl = r.wl
    o, lse, launches = _attend(r, wl, True)
    assert np.array_equal(o, P.download(r.o_lat))
    assert np.array_equal(lse, r.lse.cpu().numpy())
    if wl is C.WIDE_KEY:
        assert 4 <= launches <= 8, launches
    else:
        assert launches in (1, 2), launches


# ------------------------------------------------------------------ edge cases


def test_empty_calls_leave_outputs_untouched(cuda_ok):
    import latent_kv_cache_write_b200 as mla
    wl = C.small_variant(C.VIDEO_CHUNK)
    shape = mla.make_shape(wl)
    sentinel = torch.full((wl.batch, 4, wl.n_heads, wl.row_width), 7.0, dtype=torch.bfloat16,
                          device=P.DEV)
    w = {k: P.upload(v) for k, v in G.weights(wl, 0).items()}
    mla.mla_absorb_q(shape, sentinel, sentinel, 0, 0, w["w_uk"], sentinel)
    mla.mla_cache_write(shape, sentinel, wl.d_model, 0, 0, w["w_dkv"], w["w_kr"], sentinel)
    mla.mla_up_v(shape, sentinel, 0, w["w_uv"], sentinel)
    torch.cuda.synchronize()
    assert bool((sentinel == 7.0).all())


def test_single_frame_window_and_last_query(cuda_ok):
    """A chunk with no cached window (its own frame only) and a one-query call at
    the window's last token."""
    wl = C.small_variant(C.VIDEO_CHUNK).scaled(name="no_window", window_frames=0,
                                               first_chunk_frame=1, ring_slots=66)
    r = P.run_chunk(P.populate(wl, seed=3))
    lat, lse = O.attend_latent(P.download(r.q_abs), P.download(r.cache), wl.q_first_tok,
                               wl.k_first_tok, wl.n_keys, wl.softmax_scale, wl)
    P.tol_check(P.download(r.o_lat), lat, wl.dtype, "o_lat")
    import latent_kv_cache_write_b200 as mla
    last = wl.n_queries - 1
    o1 = torch.empty((wl.batch, 1, wl.n_heads, wl.d_latent), dtype=torch.bfloat16, device=P.DEV)
    q1 = r.q_abs[:, last:last + 1].contiguous()
    ws_n = mla.mla_attend_workspace_size(r.shape, 1, wl.n_keys)
    ws = torch.empty(max(ws_n, 16), dtype=torch.uint8, device=P.DEV)
    mla.mla_attend(r.shape, q1, 1, wl.q_first_tok + last, r.cache, wl.k_first_tok, wl.n_keys,
                   wl.softmax_scale, o1, None, ws, ws_n)
    torch.cuda.synchronize()
    P.tol_check(P.download(o1)[:, 0], lat[:, last], wl.dtype, "o_lat one query")


def _attend(r, wl, use_ws):
    """mla_attend with or without a workspace; returns (o_lat, lse, kernels launched)."""
    import latent_kv_cache_write_b200 as mla
    T = wl.n_queries
    o = torch.empty((wl.batch, T, wl.n_heads, wl.d_latent), dtype=torch.bfloat16, device=P.DEV)
    lse = torch.empty((wl.batch, T, wl.n_heads), dtype=torch.float32, device=P.DEV)
    ws, nws = None, 0
    if use_ws:
        nws = mla.mla_attend_workspace_size(r.shape, T, wl.n_keys)
        ws = torch.empty(max(nws, 16), dtype=torch.uint8, device=P.DEV)
    n0 = mla.mla_kernel_launches()
    mla.mla_attend(r.shape, r.q_abs, T, wl.q_first_tok, r.cache, wl.k_first_tok, wl.n_keys,
                   wl.softmax_scale, o, lse, ws, nws)
    launches = mla.mla_kernel_launches() - n0
    torch.cuda.synchronize()
    assert mla.mla_device_error() == 0
    return P.download(o), lse.cpu().numpy(), launches


# Shapes on which the schedule splits tiles (the host prefers it when the balance it buys
# outweighs the extra segment switches and the merge launch): many key blocks per tile,
# about as many tiles as SM pairs, so each cluster walks several segments.
SPLIT_CHUNK = C.small_variant(C.VIDEO_CHUNK).scaled(
    name="video_chunk_split", batch=5, n_heads=32, chunk_frames=1, window_frames=38,
    first_chunk_frame=38, ring_slots=39 * 66)
SPLIT_DECODE = C.small_variant(C.DECODE).scaled(
    name="decode_split", batch=8, ring_slots=4096, window_frames=4095, first_chunk_frame=4095)
# small-batch decode: one sequence's 8192 keys are one tile, spread over every cluster
DECODE_ONE = C.DECODE.scaled(name="decode_one_sequence", batch=1)


@pytest.mark.parametrize("wl", [SPLIT_CHUNK, SPLIT_DECODE, DECODE_ONE], ids=lambda w: w.name)
@pytest.mark.parametrize("use_ws", [True, False], ids=["workspace", "no_workspace"])
def test_schedule_split_and_whole(cuda_ok, wl, use_ws):
    """With a workspace these shapes cut tiles between clusters (the merge kernel runs:
    two launches); without one the cuts fall on tile boundaries (one launch).  Every
    cluster walks several segments (tile switches inside one launch).  All rows against
    the oracle."""
    r = P.run_chunk(P.populate(wl, seed=5))
    lat_ref, lse_ref = O.attend_latent(P.download(r.q_abs), P.download(r.cache), wl.q_first_tok,
                                       wl.k_first_tok, wl.n_keys, wl.softmax_scale, wl)
    o, lse, launches = _attend(r, wl, use_ws)
    assert launches == (2 if use_ws else 1)
    P.tol_check(o, lat_ref, wl.dtype, "o_lat")
    np.testing.assert_allclose(lse, lse_ref, rtol=0, atol=2e-2)


def test_schedule_many_whole_tiles(cuda_ok):
    """136 short tiles (5 key blocks each) on fewer SM pairs: whole-tile segments, several
    per cluster, with or without a workspace."""
    wl = C.small_variant(C.VIDEO_CHUNK).scaled(name="video_chunk_sched", batch=8,
                                               n_heads=32, chunk_frames=1)
    r = P.run_chunk(P.populate(wl, seed=5))
    lat_ref, _ = O.attend_latent(P.download(r.q_abs), P.download(r.cache), wl.q_first_tok,
                                 wl.k_first_tok, wl.n_keys, wl.softmax_scale, wl)
    for use_ws in (True, False):
        o, _, launches = _attend(r, wl, use_ws)
        assert launches == 1
        P.tol_check(o, lat_ref, wl.dtype, "o_lat")


def test_schedule_split_matches_whole(cuda_ok):
    """The split-key and the whole-tile schedules give the same attention, up to the
    rounding of the partial merge."""
    wl = SPLIT_DECODE
    r = P.run_chunk(P.populate(wl, seed=2), with_lse=False)
    o1, l1, n1 = _attend(r, wl, True)
    o2, l2, n2 = _attend(r, wl, False)
    assert (n1, n2) == (2, 1)
    err = float(np.linalg.norm(o1 - o2) / np.linalg.norm(o2))
    assert err <= 4e-3, err
    np.testing.assert_allclose(l1, l2, rtol=0, atol=1e-3)
