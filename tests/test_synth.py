"""Seeded input generator: determinism, storage rounding, workload table."""

import numpy as np
import torch

from synth import configs as C
from synth import generate as G


def test_bf16_rounding_matches_torch():
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.standard_normal(10000) * 10 ** rng.uniform(-3, 3, 10000),
                        [1.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -2.5, 0.0]])
    bits = G.bf16_bits(x)
    ref = torch.from_numpy(x.astype(np.float32)).to(torch.bfloat16).view(torch.int16).numpy()
    assert np.array_equal(bits.view(np.int16), ref)
    assert G.bf16_bits(np.array([1.0 + 2 ** -8]))[0] == 0x3F80       # tie to even
    assert G.bf16_bits(np.array([1.0 + 3 * 2 ** -8]))[0] == 0x3F82
    t = G.to_storage(x, "bf16")
    assert np.array_equal(G.bf16_bits(t.values), t.storage)


def test_generator_is_deterministic_and_substreamed():
    wl = C.small_variant(C.VIDEO_CHUNK)
    a = G.hidden_frame(wl, 0, 2)
    b = G.hidden_frame(wl, 0, 2)
    c = G.hidden_frame(wl, 0, 3)
    assert np.array_equal(a.storage, b.storage)
    assert not np.array_equal(a.storage, c.storage)
    both = G.hidden_frames(wl, 0, 2, 2)
    assert np.array_equal(both.values[:, wl.tokens_per_frame:], c.values)
    w1 = G.weights(wl, 0)
    w2 = G.weights(wl, 1)
    assert not np.array_equal(w1["w_uk"].storage, w2["w_uk"].storage)
    d = C.small_variant(C.DECODE)
    full = G.direct_cache(d, 0)
    assert np.array_equal(full.storage[1], G.direct_cache(d, 0, 1).storage)


def test_weight_scales():
    wl = C.VIDEO_CHUNK.scaled(d_model=1024, n_heads=4)
    w = G.weights(wl, 0)
    assert abs(w["w_dkv"].values.std() - 1 / 32) < 1e-3
    assert abs(w["w_uk"].values.std() - 1 / np.sqrt(512)) < 1e-3


def test_workload_table():
    for w in C.ALL:
        C.check(w)
        C.check(C.small_variant(w))
    lw = C.LONG_WINDOW
    assert lw.frames_written == 61 and lw.k_first_tok == 37 * 1560 and lw.n_keys == lw.ring_slots
    # the window physically straddles the ring's end
    assert lw.k_first_tok % lw.ring_slots + lw.n_keys > lw.ring_slots
    assert C.DECODE.q_first_tok == 8191 and C.DECODE.n_keys == 8192
