"""The low-bit latent cache oracle against its pins, and planted mistakes in it (on the
CPU) that some pin must catch."""

import numpy as np
import pytest

import oracle.latent_quant as QZ
from tests import quant_pins as P

_orig = {n: getattr(QZ, n) for n in (
    "qmax", "quantise_rows", "dequantise_rows", "pack_codes", "unpack_codes",
    "quantise_row_paths", "quant_bytes_per_token")}


@pytest.mark.parametrize("pin", P.ALL_QUANT_PINS, ids=lambda f: f.__name__)
def test_pin(pin):
    pin()


def _qmax_power_of_two(bits):
    return 1 << (bits - 1)


def _round_toward_zero(x, bits, decide=np.float64):
    x = np.asarray(x, dtype=np.float64)
    q = _orig["qmax"](bits)
    _, s = _orig["quantise_rows"](x, bits, decide)
    safe = np.where(s > 0, s, np.float32(1)).astype(np.float64)
    return np.clip(np.trunc(x / safe[..., None]), -q, q).astype(np.int8), s


def _scale_over_two_q(x, bits, decide=np.float64):
    # the full two's-complement span as the grid: s = max|x| / 2^(bits-1)
    x = np.asarray(x, dtype=np.float64)
    q = _orig["qmax"](bits)
    s = (np.max(np.abs(x), axis=-1) / (q + 1)).astype(np.float32)
    safe = np.where(s > 0, s, np.float32(1)).astype(np.float64)
    return np.clip(np.rint(x / safe[..., None]), -q, q).astype(np.int8), s


def _dequant_over_q(codes, scales):
    return _orig["dequantise_rows"](codes, scales) / 2.0


def _pack_high_first(codes, bits):
    # fields filled from the top of each byte down
    codes = np.asarray(codes, dtype=np.int64)
    n = codes.shape[-1]
    out = np.zeros(codes.shape[:-1] + (QZ.packed_bytes(n, bits),), dtype=np.uint8)
    for i in range(n):
        bit = i * bits
        f = codes[..., i] & ((1 << bits) - 1)
        for k in range(bits):
            b = bit + k
            out[..., b // 8] |= (((f >> (bits - 1 - k)) & 1) << (7 - b % 8)).astype(np.uint8)
    return out


def _unpack_unsigned(packed, bits, n):
    c = _orig["unpack_codes"](packed, bits, n).astype(np.int64)
    return (c & ((1 << bits) - 1)).astype(np.int8)


def _shared_scale(rows, wl, cb, rb, decide=np.float64):
    # one scale over the whole row, both paths
    rows = np.asarray(rows, dtype=np.float64)
    d_c = wl.d_latent
    cc, s = QZ.quantise_rows(rows, cb)
    cr, _ = QZ.quantise_rows(rows, rb)
    return (QZ.pack_codes(cc[..., :d_c], cb), QZ.pack_codes(cr[..., d_c:], rb), s, s)


def _bytes_one_scale(d_latent, d_rope, cb, rb, scale_bytes=4):
    return _orig["quant_bytes_per_token"](d_latent, d_rope, cb, rb, scale_bytes) - scale_bytes


MUTATIONS = {
    "qmax_power_of_two": ("qmax", _qmax_power_of_two),
    "round_toward_zero": ("quantise_rows", _round_toward_zero),
    "scale_over_two_q": ("quantise_rows", _scale_over_two_q),
    "dequant_half": ("dequantise_rows", _dequant_over_q),
    "pack_high_bits_first": ("pack_codes", _pack_high_first),
    "unpack_no_sign": ("unpack_codes", _unpack_unsigned),
    "paths_share_scale": ("quantise_row_paths", _shared_scale),
    "bytes_one_scale": ("quant_bytes_per_token", _bytes_one_scale),
}


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_planted_mistake_is_caught(name, monkeypatch):
    attr, bad = MUTATIONS[name]
    monkeypatch.setattr(QZ, attr, bad)
    caught = []
    for pin in P.ALL_QUANT_PINS:
        try:
            pin()
        except (AssertionError, ValueError, IndexError, OverflowError):
            caught.append(pin.__name__)
    assert caught, f"no pin catches the planted mistake {name}"
