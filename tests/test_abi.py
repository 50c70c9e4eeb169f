"""The C-ABI library loads, exports every symbol its header declares, and rejects bad
arguments with the documented status before launching anything (no GPU needed)."""

import ctypes
import os
import re

import pytest

from latent_kv_cache_write_b200 import build, native
from synth import configs as C

HEADER = os.path.join(os.path.dirname(os.path.dirname(__file__)), "include", "mla.h")
FAKE = 0x10000          # 16-byte aligned, never dereferenced: validation fails first
ODD = 0x10008           # not 16-byte aligned


@pytest.fixture(scope="module")
def L():
    build.build()
    return native.lib()


def declared_symbols():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"^\s*(?:mla_status|size_t|uint64_t|void|const char\*)\s+(mla_\w+)\s*\(",
                                 text, re.M)))


def test_exports_every_declared_symbol(L):
    syms = declared_symbols()
    assert len(syms) >= 7, syms
    for s in syms:
        assert hasattr(L, s), s
    assert set(syms) == set(native.SIGNATURES), "binding and header disagree"


def test_shape_struct_layout():
    assert ctypes.sizeof(native.MlaShape) == 64
    assert native.MlaShape.rope_theta.offset == 32
    assert native.MlaShape.ring_slots.offset == 48
    text = open(HEADER).read()
    assert "64 bytes, no padding holes" in text


def test_status_strings(L):
    for code, name in enumerate(["MLA_OK", "MLA_ERR_ARG", "MLA_ERR_UNSUPPORTED", "MLA_ERR_ALIGN",
                                 "MLA_ERR_RANGE", "MLA_ERR_CUDA", "MLA_ERR_TIMEOUT"]):
        assert native.status_string(code) == name
    assert native.status_string(99) == "MLA_ERR_UNKNOWN"


def _shape(**kw):
    s = native.make_shape(C.VIDEO_CHUNK)
    for k, v in kw.items():
        if k == "rope_pairs":
            s.rope_pairs[:] = v
        else:
            setattr(s, k, v)
    return s


def _attend(L, s, q=FAKE, n_q=1560, q_first=3 * 1560, cache=FAKE, k_first=0, n_keys=6240,
            scale=0.07, o=FAKE, lse=None, ws=None, ws_bytes=0):
    return L.mla_attend(ctypes.byref(s), q, n_q, q_first, cache, k_first, n_keys, scale, o, lse,
                        ws, ws_bytes, None)


def test_shape_validation(L):
    bad = [dict(batch=0), dict(n_heads=0), dict(d_rope=63), dict(rope_pairs=[8, 12, 11]),
           dict(rope_pairs=[-1, 21, 12]), dict(grid_h=0), dict(ring_slots=0), dict(reserved=1),
           dict(rope_theta=0.0), dict(d_latent=511)]
    for kw in bad:
        assert _attend(L, _shape(**kw)) == native.MLA_ERR_ARG, kw
    assert _attend(L, _shape(dtype=7)) == native.MLA_ERR_UNSUPPORTED
    assert L.mla_attend(None, FAKE, 1, 0, FAKE, 0, 1, 1.0, FAKE, None, None, 0, None) == \
        native.MLA_ERR_ARG


def test_attend_ranges_and_pointers(L):
    s = _shape()
    R = native.MLA_ERR_RANGE
    assert _attend(L, s, n_keys=6241) == R                    # more keys than ring slots
    assert _attend(L, s, n_keys=0) == R
    assert _attend(L, s, k_first=-1) == R
    assert _attend(L, s, q_first=0, k_first=1) == R            # query before the window
    assert _attend(L, s, q_first=3 * 1560 + 1) == R            # query past the window
    assert _attend(L, s, q=None) == native.MLA_ERR_ARG
    assert _attend(L, s, cache=None) == native.MLA_ERR_ARG
    assert _attend(L, s, o=None) == native.MLA_ERR_ARG
    assert _attend(L, s, scale=0.0) == native.MLA_ERR_ARG
    assert _attend(L, s, scale=float("nan")) == native.MLA_ERR_ARG
    assert _attend(L, s, q=ODD) == native.MLA_ERR_ALIGN
    assert _attend(L, s, lse=ODD) == native.MLA_ERR_ALIGN
    assert _attend(L, s, n_q=-1) == native.MLA_ERR_ARG


def test_attend_workspace_check(L):
    s = _shape()
    need = L.mla_attend_workspace_size(ctypes.byref(s), 1560, 6240)
    if need:
        assert _attend(L, s, ws=FAKE, ws_bytes=need - 1) == native.MLA_ERR_ARG
        assert _attend(L, s, ws=None, ws_bytes=need) == native.MLA_ERR_ARG


def test_cache_write_validation(L):
    s = _shape()
    cw = lambda **k: L.mla_cache_write(
        ctypes.byref(s), k.get("h", FAKE), k.get("d", 4096), k.get("n", 1560),
        k.get("first", 0), k.get("wd", FAKE), k.get("wr", FAKE), k.get("cache", FAKE),
        k.get("slots", None), None)
    assert cw(n=6241) == native.MLA_ERR_RANGE
    assert cw(first=-1) == native.MLA_ERR_RANGE
    assert cw(d=0) == native.MLA_ERR_ARG
    assert cw(h=None) == native.MLA_ERR_ARG
    assert cw(wr=None) == native.MLA_ERR_ARG
    assert cw(cache=ODD) == native.MLA_ERR_ALIGN
    assert cw(slots=ODD) == native.MLA_ERR_ALIGN
    assert cw(n=0) == native.MLA_OK                             # empty: nothing to do


def test_absorb_and_up_v_validation(L):
    s = _shape()
    ab = lambda **k: L.mla_absorb_q(ctypes.byref(s), k.get("qn", FAKE), k.get("qr", FAKE),
                                    k.get("n", 1560), k.get("first", 0), k.get("w", FAKE),
                                    k.get("out", FAKE), None)
    assert ab(first=-1) == native.MLA_ERR_RANGE
    assert ab(qn=None) == native.MLA_ERR_ARG
    assert ab(out=ODD) == native.MLA_ERR_ALIGN
    assert ab(n=0) == native.MLA_OK
    uv = lambda **k: L.mla_up_v(ctypes.byref(s), k.get("o", FAKE), k.get("n", 1560),
                                k.get("w", FAKE), k.get("out", FAKE), None)
    assert uv(o=None) == native.MLA_ERR_ARG
    assert uv(w=ODD) == native.MLA_ERR_ALIGN
    assert uv(n=-2) == native.MLA_ERR_ARG
    assert uv(n=0) == native.MLA_OK


def _mat(L, s, qn=FAKE, qr=FAKE, n_q=1560, q_first=3 * 1560, cache=FAKE, k_first=0,
         n_keys=6240, scale=0.07, wuk=FAKE, wuv=FAKE, out=FAKE, lse=None, ws=FAKE,
         ws_bytes=None):
    if ws_bytes is None:
        ws_bytes = L.mla_attend_materialised_workspace_size(ctypes.byref(s))
    return L.mla_attend_materialised(ctypes.byref(s), qn, qr, n_q, q_first, cache, k_first,
                                     n_keys, scale, wuk, wuv, out, lse, ws, ws_bytes, None)


def test_materialised_validation(L):
    s = _shape()
    # per-head keys and values of every ring slot, bf16
    assert L.mla_attend_materialised_workspace_size(ctypes.byref(s)) == 2 * 6240 * 32 * 128 * 2
    # the wide positional key (d_R = 512) is supported; other RoPE widths are not
    wide = native.make_shape(C.WIDE_KEY)
    assert L.mla_attend_materialised_workspace_size(ctypes.byref(wide)) == \
        2 * 4 * 15600 * 32 * 128 * 2
    other = _shape(d_rope=128, rope_pairs=[16, 24, 24])
    assert L.mla_attend_materialised_workspace_size(ctypes.byref(other)) == 0
    assert _mat(L, other, ws_bytes=1 << 30) == native.MLA_ERR_UNSUPPORTED
    assert _mat(L, _shape(dtype=native.MLA_F32), ws_bytes=1 << 30) == native.MLA_ERR_UNSUPPORTED
    assert _mat(L, s, ws=None) == native.MLA_ERR_ARG
    assert _mat(L, s, ws_bytes=1024) == native.MLA_ERR_ARG
    assert _mat(L, s, qr=None) == native.MLA_ERR_ARG
    assert _mat(L, s, wuv=None) == native.MLA_ERR_ARG
    assert _mat(L, s, n_keys=6241) == native.MLA_ERR_RANGE
    assert _mat(L, s, q_first=3 * 1560 + 1) == native.MLA_ERR_RANGE
    assert _mat(L, s, out=ODD) == native.MLA_ERR_ALIGN
    assert _mat(L, s, ws=ODD) == native.MLA_ERR_ALIGN
    assert _mat(L, s, n_q=0, q_first=0) == native.MLA_OK          # empty: nothing to do


def test_shift_frames_validation(L):
    s = _shape()
    sh = lambda **k: L.mla_cache_shift_frames(ctypes.byref(s), k.get("cache", FAKE),
                                              k.get("first", 1560), k.get("n", 1560),
                                              k.get("d", 2), None)
    assert sh(cache=None) == native.MLA_ERR_ARG
    assert sh(n=-1) == native.MLA_ERR_ARG
    assert sh(n=6241) == native.MLA_ERR_RANGE                 # more tokens than slots
    assert sh(first=-1) == native.MLA_ERR_RANGE
    assert sh(cache=ODD) == native.MLA_ERR_ALIGN
    assert sh(n=0) == native.MLA_OK                             # empty: nothing to do


def test_quantise_validation(L):
    s = _shape()
    f32 = _shape(dtype=native.MLA_F32)

    def q(fn="mla_cache_quantise", shape=s, **k):
        ptrs = [k.get("cache", FAKE), k.get("qc", FAKE), k.get("qr", FAKE), k.get("sc", FAKE),
                k.get("sr", FAKE)]
        first, n, cb, rb = k.get("first", 0), k.get("n", 6240), k.get("cb", 4), k.get("rb", 4)
        if fn == "mla_cache_quantise":
            return L.mla_cache_quantise(ctypes.byref(shape), ptrs[0], first, n, cb, rb, *ptrs[1:],
                                        None)
        return L.mla_cache_dequantise(ctypes.byref(shape), ptrs[1], ptrs[2], ptrs[3], ptrs[4],
                                      cb, rb, first, n, ptrs[0], None)

    for fn in ("mla_cache_quantise", "mla_cache_dequantise"):
        for name in ("cache", "qc", "qr", "sc", "sr"):
            assert q(fn, **{name: None}) == native.MLA_ERR_ARG, (fn, name)
            assert q(fn, **{name: ODD}) == native.MLA_ERR_ALIGN, (fn, name)
        assert q(fn, n=-1) == native.MLA_ERR_ARG
        for bad in (0, 1, 3, 5, 16):
            assert q(fn, cb=bad) == native.MLA_ERR_ARG and q(fn, rb=bad) == native.MLA_ERR_ARG
        assert q(fn, n=6241) == native.MLA_ERR_RANGE
        assert q(fn, first=-1) == native.MLA_ERR_RANGE
        assert q(fn, shape=_shape(d_latent=516)) == native.MLA_ERR_UNSUPPORTED
        assert q(fn, shape=_shape(d_latent=2048)) == native.MLA_ERR_UNSUPPORTED
        assert q(fn, n=0) == native.MLA_OK
        assert q(fn, shape=f32, n=0, cb=2, rb=8) == native.MLA_OK


def test_row_counts_beyond_32_bit_coordinates(L):
    U = native.MLA_ERR_UNSUPPORTED
    # batch x ring_slots rows: refused by every call, before anything else is looked at
    huge_ring = _shape(ring_slots=1 << 31)
    assert _attend(L, huge_ring) == U
    assert L.mla_cache_shift_frames(ctypes.byref(huge_ring), FAKE, 0, 1, 1, None) == U
    assert L.mla_cache_quantise(ctypes.byref(_shape(batch=2, ring_slots=1 << 30)), FAKE, 0, 1,
                                4, 4, FAKE, FAKE, FAKE, FAKE, None) == U
    assert L.mla_attend_workspace_size(ctypes.byref(huge_ring), 1, 1) == 0
    # batch x n_q x n_heads query rows
    s = _shape(batch=2, n_heads=32)
    n = 1 << 25                                           # 2 x 2^25 x 32 = 2^31 rows
    assert L.mla_absorb_q(ctypes.byref(s), FAKE, FAKE, n, 0, FAKE, FAKE, None) == U
    assert L.mla_up_v(ctypes.byref(s), FAKE, n, FAKE, FAKE, None) == U
    assert L.mla_absorb_q(ctypes.byref(s), FAKE, FAKE, 0, 0, FAKE, FAKE, None) == native.MLA_OK
    big = _shape(batch=1000, n_heads=65, ring_slots=50000)    # 1000 x 40000 x 65 rows
    assert _attend(L, big, n_q=40000, q_first=0, n_keys=50000) == U
    assert _mat(L, big, n_q=40000, q_first=0, n_keys=50000, ws_bytes=1 << 62) == U


def _fixed(L, s, q=FAKE, n_q=1560, q_first=3 * 1560, cache=FAKE, k_first=0, n_keys=6240,
           scale=0.07, o=FAKE, lse=None):
    return L.mla_attend_fixed_scratch(ctypes.byref(s), q, n_q, q_first, cache, k_first, n_keys,
                                      scale, o, lse, None)


def test_fixed_scratch_validation(L):
    """The no-workspace entry point answers bad arguments exactly as mla_attend does,
    before it looks up its static array or launches anything."""
    s = _shape()
    assert native.MLA_FIXED_SCRATCH_BYTES == 40 * 1024 * 1024
    assert "#define MLA_FIXED_SCRATCH_BYTES (40u * 1024u * 1024u)" in open(HEADER).read()
    R, A = native.MLA_ERR_RANGE, native.MLA_ERR_ARG
    assert _fixed(L, _shape(batch=0)) == A
    assert _fixed(L, _shape(dtype=7)) == native.MLA_ERR_UNSUPPORTED
    assert L.mla_attend_fixed_scratch(None, FAKE, 1, 0, FAKE, 0, 1, 1.0, FAKE, None, None) == A
    assert _fixed(L, s, n_keys=6241) == R
    assert _fixed(L, s, n_keys=0) == R
    assert _fixed(L, s, k_first=-1) == R
    assert _fixed(L, s, q_first=3 * 1560 + 1) == R
    assert _fixed(L, s, q=None) == A
    assert _fixed(L, s, cache=None) == A
    assert _fixed(L, s, o=None) == A
    assert _fixed(L, s, scale=float("nan")) == A
    assert _fixed(L, s, n_q=-1) == A
    assert _fixed(L, s, q=ODD) == native.MLA_ERR_ALIGN
    assert _fixed(L, s, lse=ODD) == native.MLA_ERR_ALIGN
    assert _fixed(L, s, n_q=0) == native.MLA_OK               # empty: nothing to do
    big = _shape(batch=1000, n_heads=65, ring_slots=50000)
    assert _fixed(L, big, n_q=40000, q_first=0, n_keys=50000) == native.MLA_ERR_UNSUPPORTED


def test_attend_quantised_validation(L):
    s = _shape()

    def aq(shape=s, q=FAKE, qc=FAKE, qr=FAKE, sc=FAKE, sr=FAKE, cb=4, rb=4, n_q=1560,
           q_first=3 * 1560, k_first=0, n_keys=6240, o=FAKE, ws=None, ws_bytes=0):
        return L.mla_attend_quantised(ctypes.byref(shape), q, n_q, q_first, qc, qr, sc, sr, cb,
                                      rb, k_first, n_keys, 0.07, o, None, ws, ws_bytes, None)

    A, U = native.MLA_ERR_ARG, native.MLA_ERR_UNSUPPORTED
    for name in ("q", "qc", "qr", "sc", "sr", "o"):
        assert aq(**{name: None}) == A, name
    for name in ("q", "qr", "sc", "sr", "o"):
        assert aq(**{name: ODD}) == native.MLA_ERR_ALIGN, name
    assert aq(cb=3) == A and aq(rb=5) == A              # not a code width at all
    assert aq(cb=8) == U and aq(rb=2) == U and aq(rb=8) == U    # widths the kernel lacks
    assert aq(shape=_shape(dtype=native.MLA_F32)) == U
    assert aq(shape=native.make_shape(C.WIDE_KEY), q_first=9 * 1560, n_keys=15600) == U
    assert aq(n_keys=6241) == native.MLA_ERR_RANGE
    assert aq(q_first=3 * 1560 + 1) == native.MLA_ERR_RANGE
    assert aq(n_q=0, q_first=0) == native.MLA_OK
