"""Pins of the low-bit latent cache oracle (oracle/latent_quant.py) against facts that do
not come from it: exact rational rounding, the half-step error bound of a uniform grid,
grids that quantise without loss, packed bytes built by other means (hand-written fixtures
and Python integers), the independence of the two paths' scales, the convergence of the
attention output as codes get wider, and closed forms of the bytes per token.

Each ``pin_*`` raises AssertionError on a disagreement; ``test_quant_oracle`` also plants
mistakes in the module and checks that some pin fails."""

from __future__ import annotations

import math
from fractions import Fraction

import numpy as np

import oracle.latent_quant as QZ
import oracle.mla_oracle as O
from synth import configs as C
from synth import generate as G
from tests import oracle_pins as P


def _nearest_even(r: Fraction) -> int:
    """The integer nearest to r, ties to the even one (exact rational arithmetic)."""
    k = math.floor(r)
    d = r - k
    if d > Fraction(1, 2):
        return k + 1
    if d < Fraction(1, 2):
        return k
    return k if k % 2 == 0 else k + 1


def pin_quant_brute_force():
    """Every code against an exact rational evaluation: the nearest grid point of x / s,
    ties to even, clipped to [-q, q]; the scale is the float32 nearest to max|x| / q."""
    rng = np.random.default_rng(11)
    for bits in (2, 3, 4, 8):
        q = (1 << (bits - 1)) - 1
        for n in (1, 2, 7, 33):
            x = rng.standard_normal((3, n)) * np.array([[1e-3], [1.0], [250.0]])
            codes, s = QZ.quantise_rows(x, bits)
            for r in range(x.shape[0]):
                amax = max(abs(float(v)) for v in x[r])
                exact = Fraction(amax) / q
                sf = Fraction(float(s[r]))
                # float32 nearest: within half a float32 step of the exact quotient
                step = Fraction(float(np.spacing(np.float32(s[r]))))
                assert abs(sf - exact) <= step / 2
                for i in range(n):
                    ratio = Fraction(float(x[r, i])) / sf
                    want = max(-q, min(q, _nearest_even(ratio)))
                    near_tie = abs(ratio - math.floor(ratio) - Fraction(1, 2)) < Fraction(1, 10**9)
                    assert int(codes[r, i]) == want or near_tie, (bits, n, r, i)
    # exact ties, on a power-of-two scale (s = 1/4, q = 7 from the row maximum 7/4)
    x = np.array([[1.75, 0.625, -0.375, 0.125, -0.125, 0.875, -1.75]])
    codes, s = QZ.quantise_rows(x, 4)
    assert float(s[0]) == 0.25
    assert codes[0].tolist() == [7, 2, -2, 0, 0, 4, -7]       # 2.5->2 -1.5->-2 .5->0 3.5->4


def pin_quant_error_bound():
    """Codes lie in [-q, q], the row's largest magnitude takes code +-q, and every value is
    within half a grid step of its dequantised value (a uniform grid's bound)."""
    rng = np.random.default_rng(12)
    for bits in range(2, 9):
        q = (1 << (bits - 1)) - 1
        for scale in (1e-4, 1.0, 3e3):
            x = rng.standard_normal((16, 96)) * scale
            codes, s = QZ.quantise_rows(x, bits)
            deq = QZ.dequantise_rows(codes, s)
            assert np.all(np.abs(codes) <= q)
            am = np.argmax(np.abs(x), axis=-1)
            rows = np.arange(x.shape[0])
            assert np.array_equal(np.abs(codes[rows, am]), np.full(x.shape[0], q))
            assert np.array_equal(np.sign(codes[rows, am]), np.sign(x[rows, am]))
            half = s.astype(np.float64)[:, None] / 2
            assert np.all(np.abs(x - deq) <= half * (1 + 1e-6))
            # the extreme value comes back to float32 rounding of itself
            assert np.all(np.abs(deq[rows, am] - x[rows, am]) <= 1e-6 * np.abs(x[rows, am]))


def pin_quant_grid_exact():
    """Values already on a grid of a power-of-two step, with some code at +-q, quantise to
    exactly those codes and come back unchanged."""
    rng = np.random.default_rng(13)
    for bits in range(2, 9):
        q = (1 << (bits - 1)) - 1
        for e in (-9, 0, 5):
            k = rng.integers(-q, q + 1, size=(5, 40))
            k[:, 3] = q * np.where(rng.random(5) < 0.5, 1, -1)
            x = k * 2.0 ** e
            codes, s = QZ.quantise_rows(x, bits)
            assert np.array_equal(s, np.full(5, 2.0 ** e, np.float32))
            assert np.array_equal(codes.astype(np.int64), k)
            assert np.array_equal(QZ.dequantise_rows(codes, s), x)
    # a row of zeros and an empty row
    codes, s = QZ.quantise_rows(np.zeros((2, 8)), 4)
    assert not codes.any() and not s.any()
    assert not QZ.dequantise_rows(codes, s).any()
    codes, s = QZ.quantise_rows(np.zeros((3, 0)), 4)
    assert codes.shape == (3, 0) and not s.any()


def pin_pack_layout():
    """Packed bytes against hand-written fixtures and against the row's bit string built
    as a Python integer; unpacking restores every two's-complement code."""
    # INT4: fields 0x1, 0xE, 0x7, 0x9 -> bytes 0xE1 0x97 (element 0 in the low nibble)
    assert QZ.pack_codes(np.array([1, -2, 7, -7]), 4).tolist() == [0xE1, 0x97]
    # INT2: fields 01 11 00 01 | 11 -> 0b01001101, 0b00000011
    assert QZ.pack_codes(np.array([1, -1, 0, 1, -1]), 2).tolist() == [0x4D, 0x03]
    # INT3: fields 101 010 001 -> 0b01010101, then the last field's top bit 0
    assert QZ.pack_codes(np.array([-3, 2, 1]), 3).tolist() == [0x55, 0x00]
    rng = np.random.default_rng(14)
    for bits in range(2, 9):
        lo, hi = -(1 << (bits - 1)), (1 << (bits - 1)) - 1
        for n in (1, 3, 8, 13, 64):
            c = rng.integers(lo, hi + 1, size=(4, n))
            got = QZ.pack_codes(c, bits)
            nb = (n * bits + 7) // 8
            assert got.shape == (4, nb) and QZ.packed_bytes(n, bits) == nb
            for r in range(4):
                v = sum((int(c[r, i]) & ((1 << bits) - 1)) << (bits * i) for i in range(n))
                assert bytes(got[r].tolist()) == v.to_bytes(nb, "little")
            assert np.array_equal(QZ.unpack_codes(got, bits, n).astype(np.int64), c)
        every = np.arange(lo, hi + 1)
        assert np.array_equal(QZ.unpack_codes(QZ.pack_codes(every, bits), bits, every.size),
                              every)


def pin_quant_paths_separate():
    """The content and RoPE parts of a row have scales of their own: scaling one part
    leaves the other's codes and scale untouched, and its own codes unchanged."""
    wl = P.SMALL
    rng = np.random.default_rng(15)
    rows = rng.standard_normal((4, wl.row_width))
    d_c = wl.d_latent
    for cb, rb in ((4, 4), (2, 4)):
        pc, pr, sc, sr = QZ.quantise_row_paths(rows, wl, cb, rb)
        big = rows.copy()
        big[:, d_c:] *= 1024.0
        pc2, pr2, sc2, sr2 = QZ.quantise_row_paths(big, wl, cb, rb)
        assert np.array_equal(pc, pc2) and np.array_equal(sc, sc2)
        assert np.array_equal(pr, pr2) and np.array_equal(sr2, sr * np.float32(1024))
        small = rows.copy()
        small[:, :d_c] /= 64.0
        pc3, pr3, sc3, sr3 = QZ.quantise_row_paths(small, wl, cb, rb)
        assert np.array_equal(pr, pr3) and np.array_equal(sr, sr3)
        assert np.array_equal(pc, pc3) and np.array_equal(sc3, sc / np.float32(64))


def pin_quant_ring_write():
    """Writing a quantised ring frame by frame equals quantising the unquantised ring the
    same frames build, slot for slot; slots that nothing wrote stay unwritten."""
    for wl in (P.MINI, P.SMALL):
        w, cache, _, _ = P.build_state(wl, 3)
        F = wl.tokens_per_frame
        qc = QZ.empty_quant_cache(wl, 4, 4)
        ref = np.full((wl.batch, wl.ring_slots, wl.row_width), np.nan)
        for f in range(wl.frames_written):
            h = G.hidden_frame(wl, 3, f).values
            qc, slots = QZ.quant_cache_write(qc, h, w["w_dkv"], w["w_kr"], f * F, wl)
            ref, slots_ref = O.cache_write(ref, h, w["w_dkv"], w["w_kr"], f * F, wl)
            assert np.array_equal(slots, slots_ref)
        want = QZ.quantise_cache(ref, wl, 4, 4)
        for k in ("content", "rope", "scale_c", "scale_r"):
            assert np.array_equal(qc[k], want[k], equal_nan=True), (wl.name, k)
        written = np.all(np.isfinite(ref), axis=-1)
        assert np.array_equal(np.isfinite(qc["scale_c"]), written)
        deq = QZ.dequantise_cache(qc, wl)
        assert np.array_equal(np.isfinite(deq).all(axis=-1), written)


def pin_quant_attention_converges():
    """Attention over a quantised ring tends to the unquantised attention as the codes get
    wider (about half the error per extra bit), and INT2 content is worse than INT4."""
    wl = P.SMALL
    w, cache, qn, qr = P.build_state(wl, 4)
    q_abs = O.absorb_q(qn, qr, w["w_uk"], wl.q_first_tok, wl)
    o_ref, lse_ref = O.attend_latent(q_abs, cache, wl.q_first_tok, wl.k_first_tok,
                                     wl.n_keys, wl.softmax_scale, wl)
    errs = {}
    for cb, rb in ((2, 4), (3, 3), (4, 4), (6, 6), (8, 8)):
        qc = QZ.quantise_cache(cache, wl, cb, rb)
        o, lse = QZ.attend_quantised(q_abs, qc, wl.q_first_tok, wl.k_first_tok, wl.n_keys,
                                     wl.softmax_scale, wl)
        errs[(cb, rb)] = P.rel(o, o_ref)
        assert np.all(np.isfinite(o)) and np.all(np.isfinite(lse))
    assert errs[(2, 4)] > errs[(4, 4)]
    assert errs[(3, 3)] > errs[(4, 4)] > errs[(6, 6)] > errs[(8, 8)]
    assert 2.0 < errs[(4, 4)] / errs[(6, 6)] < 8.0 and 2.0 < errs[(6, 6)] / errs[(8, 8)] < 8.0
    assert errs[(8, 8)] < 2e-2


def pin_quant_bytes():
    """Bytes per cached token: the packed content and RoPE paths plus one float32 scale
    each, against the unquantised bf16 row of the same shape."""
    assert QZ.quant_bytes_per_token(512, 64, 4, 4) == 256 + 32 + 8
    assert QZ.quant_bytes_per_token(512, 64, 2, 4) == 128 + 32 + 8
    assert QZ.quant_bytes_per_token(512, 512, 4, 4) == 256 + 256 + 8
    assert QZ.quant_bytes_per_token(6, 6, 2, 3, scale_bytes=2) == 2 + 3 + 4
    bf16 = O.mla_bytes_per_token(512, 64, 2)
    assert abs(bf16 / QZ.quant_bytes_per_token(512, 64, 4, 4) - 1152 / 296) < 1e-12
    wl = P.SMALL
    qc = QZ.empty_quant_cache(wl, 2, 4)
    per_slot = sum(qc[k].nbytes for k in ("content", "rope", "scale_c", "scale_r"))
    assert per_slot == wl.batch * wl.ring_slots * QZ.quant_bytes_per_token(
        wl.d_latent, wl.d_rope, 2, 4)


def _video_chunk_window_rows() -> np.ndarray:
    """The 6240 rows of the video-chunk window (frames 0-3 through the oracle's cache
    write), rounded to bf16 as the ring holds them."""
    wl = C.VIDEO_CHUNK
    w = G.weights(wl, 0)
    F = wl.tokens_per_frame
    rows = [O.cache_rows(G.hidden_frame(wl, 0, f).values, w["w_dkv"].values,
                         w["w_kr"].values, f * F, wl)[0] for f in range(4)]
    return G.to_storage(np.concatenate(rows), "bf16").values


DECISION_DIFFS = {}        # (bits, path) -> codes the float32 decision changes, on the window


def pin_quant_float32_decision():
    """x / s evaluated in float32 (as a float32 kernel does) against the exact decision:
    the scale is the same, codes differ by at most one, and only where x / s lies within
    float32 rounding of a half-integer (the division's result within 2^-24 of itself, the
    bf16 x exact in float32).  Counted on every element of the video-chunk window at 2, 4
    and 8 bits (DECISION_DIFFS); then on constructed near-ties where the two do differ."""
    rows = _video_chunk_window_rows()
    d_c = C.VIDEO_CHUNK.d_latent
    for bits in (2, 4, 8):
        for path, x in (("content", rows[:, :d_c]), ("rope", rows[:, d_c:])):
            c64, s64 = QZ.quantise_rows(x, bits)
            c32, s32 = QZ.quantise_rows(x, bits, decide=np.float32)
            assert np.array_equal(s64, s32)
            diff = c64.astype(np.int64) - c32.astype(np.int64)
            assert np.abs(diff).max() <= 1, (bits, path)
            DECISION_DIFFS[(bits, path)] = int(np.count_nonzero(diff))
            for r, i in zip(*np.nonzero(diff)):
                ratio = Fraction(float(x[r, i])) / Fraction(float(s64[r]))
                off = abs(ratio - math.floor(ratio) - Fraction(1, 2))
                assert off <= abs(ratio) * Fraction(1, 2 ** 22), (bits, path, r, i)
    # near-ties: x just above (k + 1/2) s, where the float32 quotient rounds to the tie
    rng = np.random.default_rng(5)
    found = 0
    for _ in range(2000):
        s = float(np.float32(rng.uniform(0.01, 10.0)))
        x = 2.5 * s * (1.0 + 2.0 ** -28)          # exact quotient a hair above 2.5
        row = np.array([[7.0 * s, x]])            # max|x| / 7 = s exactly, so the scale is s
        c64, sc = QZ.quantise_rows(row, 4)
        c32, _ = QZ.quantise_rows(row, 4, decide=np.float32)
        assert float(sc[0]) == s and c64[0, 1] == 3
        if c32[0, 1] != c64[0, 1]:
            assert c32[0, 1] == 2                 # the tie, to even: one code apart
            found += 1
    assert found > 0


ALL_QUANT_PINS = [pin_quant_brute_force, pin_quant_error_bound, pin_quant_grid_exact,
                  pin_pack_layout, pin_quant_paths_separate, pin_quant_ring_write,
                  pin_quant_attention_converges, pin_quant_bytes, pin_quant_float32_decision]
