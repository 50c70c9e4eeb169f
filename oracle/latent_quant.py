"""fp64 CPU oracle for a low-bit latent cache: plain per-row, per-path scale quantisation.

TEST INFRASTRUCTURE ONLY.  Only the tests, the package smoke check and the CPU baseline
leg of the benchmark may import this module.  It shares no code with the CUDA path.

Source, cited by page title and section:

* [QuantMLA] the QuantMLA abstract on the "Multi-Head Latent Attention" topic page: the
  two cached paths of MLA, the content latent and the decoupled RoPE key, are quantised
  separately, both to INT4, or the content to INT2 with the RoPE key kept at INT4; the
  attention kernel unpacks and dequantises the codes as part of the attention itself.

The learned path-specific transformations of that work are not modelled.  What the
abstract leaves open is fixed by these readings:

* a code is a symmetric signed integer in [-q, q] with q = 2^(bits-1) - 1 (INT4: 7,
  INT2: 1), stored as a two's-complement field of ``bits`` bits;
* every cached row has one scale per path: s = max|x| / q over the row's content dims,
  and another over its RoPE dims; the scale is stored as float32, and a row of zeros has
  s = 0 and all codes 0;
* code = x / s rounded to the nearest integer, ties to even, then clipped to [-q, q];
  the dequantised value is code * s;
* the RoPE key is quantised after its rotation, i.e. the row exactly as the unquantised
  cache would hold it;
* the fields of a row are packed little-endian: element i occupies bits
  [i*bits, (i+1)*bits) of the row's bit string, byte k holding bits [8k, 8k+8); a row
  whose bits do not fill its last byte leaves the rest of that byte zero.

Attention over a quantised ring is attention over its dequantised rows: the quantisation
is the only new arithmetic here.
"""

from __future__ import annotations

from typing import Dict, Iterable, Optional, Tuple

import numpy as np

from . import mla_oracle as O


def qmax(bits: int) -> int:
    """Largest code magnitude of a symmetric signed ``bits``-bit code."""
    if bits < 2 or bits > 8:
        raise ValueError("codes of 2 to 8 bits")
    return (1 << (bits - 1)) - 1


def quantise_rows(x: np.ndarray, bits: int, decide=np.float64) -> Tuple[np.ndarray, np.ndarray]:
    """Per-row scale quantisation along the last axis.

    Returns (codes int8 [..., n], scales float32 [...]).  ``decide`` is the float type in
    which x / s is evaluated before rounding (float64 here; the same decision taken in
    float32 reproduces a float32 kernel's codes)."""
    x = np.asarray(x, dtype=np.float64)
    if not np.all(np.isfinite(x)):
        raise ValueError("rows to quantise must be finite")
    q = qmax(bits)
    amax = np.max(np.abs(x), axis=-1) if x.shape[-1] > 0 else np.zeros(x.shape[:-1])
    s = (amax / q).astype(np.float32)
    safe = np.where(s > 0, s, np.float32(1)).astype(np.float32)
    r = x.astype(decide) / safe[..., None].astype(decide)
    codes = np.clip(np.rint(r), -q, q).astype(np.int8)
    codes[s == 0] = 0
    return codes, s


def dequantise_rows(codes: np.ndarray, scales: np.ndarray) -> np.ndarray:
    """code * s, in float64 (both factors are exact in float64)."""
    return np.asarray(codes, dtype=np.float64) * np.asarray(scales, dtype=np.float64)[..., None]


def packed_bytes(n: int, bits: int) -> int:
    """Bytes of one packed row of n codes."""
    return (n * bits + 7) // 8


def pack_codes(codes: np.ndarray, bits: int) -> np.ndarray:
    """Pack codes [..., n] into bytes [..., packed_bytes(n, bits)] (little-endian fields)."""
    codes = np.asarray(codes, dtype=np.int64)
    n = codes.shape[-1]
    field = codes & ((1 << bits) - 1)                      # two's complement, ``bits`` wide
    out = np.zeros(codes.shape[:-1] + (packed_bytes(n, bits),), dtype=np.uint8)
    for i in range(n):
        bit = i * bits
        byte, off = bit // 8, bit % 8
        out[..., byte] |= ((field[..., i] << off) & 0xFF).astype(np.uint8)
        if off + bits > 8:                                  # a field across a byte edge
            out[..., byte + 1] |= (field[..., i] >> (8 - off)).astype(np.uint8)
    return out


def unpack_codes(packed: np.ndarray, bits: int, n: int) -> np.ndarray:
    """The n signed codes of each packed row [..., packed_bytes(n, bits)]."""
    packed = np.asarray(packed, dtype=np.int64)
    codes = np.zeros(packed.shape[:-1] + (n,), dtype=np.int64)
    for i in range(n):
        bit = i * bits
        byte, off = bit // 8, bit % 8
        v = packed[..., byte] >> off
        if off + bits > 8:
            v = v | (packed[..., byte + 1] << (8 - off))
        v = v & ((1 << bits) - 1)
        codes[..., i] = np.where(v >= (1 << (bits - 1)), v - (1 << bits), v)
    return codes.astype(np.int8)


def quant_bytes_per_token(d_latent: int, d_rope: int, content_bits: int, rope_bits: int,
                          scale_bytes: int = 4) -> int:
    """Bytes of one cached token: the two packed paths and one scale for each."""
    return (packed_bytes(d_latent, content_bits) + packed_bytes(d_rope, rope_bits)
            + 2 * scale_bytes)


def empty_quant_cache(wl, content_bits: int, rope_bits: int) -> Dict[str, np.ndarray]:
    """A quantised ring whose slots are all unwritten (codes 0, scales NaN)."""
    B, S = wl.batch, wl.ring_slots
    return {
        "bits": np.array([content_bits, rope_bits]),
        "content": np.zeros((B, S, packed_bytes(wl.d_latent, content_bits)), np.uint8),
        "rope": np.zeros((B, S, packed_bytes(wl.d_rope, rope_bits)), np.uint8),
        "scale_c": np.full((B, S), np.nan, np.float32),
        "scale_r": np.full((B, S), np.nan, np.float32),
    }


def quantise_row_paths(rows: np.ndarray, wl, content_bits: int, rope_bits: int,
                       decide=np.float64):
    """(packed content, packed rope, scale_c, scale_r) of cached rows [..., d_c + d_R];
    ``decide`` as in quantise_rows."""
    rows = np.asarray(rows, dtype=np.float64)
    d_c = wl.d_latent
    cc, sc = quantise_rows(rows[..., :d_c], content_bits, decide)
    cr, sr = quantise_rows(rows[..., d_c:], rope_bits, decide)
    return pack_codes(cc, content_bits), pack_codes(cr, rope_bits), sc, sr


def quant_cache_write(qc: Dict[str, np.ndarray], h: np.ndarray, w_dkv: np.ndarray,
                      w_kr: np.ndarray, first_tok: int, wl):
    """Write tokens first_tok .. first_tok+n-1 into a quantised ring: the rows of the
    unquantised cache write, quantised per path and stored in their slots g mod S.
    Returns the new ring and the slot of every token [B, n]."""
    cb, rb = (int(v) for v in qc["bits"])
    rows = O.cache_rows(h, w_dkv, w_kr, first_tok, wl)
    pc, pr, sc, sr = quantise_row_paths(rows, wl, cb, rb)
    out = {k: np.array(v, copy=True) for k, v in qc.items()}
    n = rows.shape[1]
    slots = np.empty((rows.shape[0], n), dtype=np.int64)
    for b in range(rows.shape[0]):
        for i in range(n):
            s = O.ring_slot(first_tok + i, wl.ring_slots)
            out["content"][b, s] = pc[b, i]
            out["rope"][b, s] = pr[b, i]
            out["scale_c"][b, s] = sc[b, i]
            out["scale_r"][b, s] = sr[b, i]
            slots[b, i] = s
    return out, slots


def quantise_cache(cache: np.ndarray, wl, content_bits: int, rope_bits: int):
    """Quantise every slot of an unquantised ring; slots holding non-finite values are
    taken as unwritten (codes 0, scales NaN)."""
    cache = np.asarray(cache, dtype=np.float64)
    qc = empty_quant_cache(wl, content_bits, rope_bits)
    ok = np.all(np.isfinite(cache), axis=-1)
    rows = np.where(ok[..., None], cache, 0.0)
    pc, pr, sc, sr = quantise_row_paths(rows, wl, content_bits, rope_bits)
    qc["content"][ok] = pc[ok]
    qc["rope"][ok] = pr[ok]
    qc["scale_c"][ok] = sc[ok]
    qc["scale_r"][ok] = sr[ok]
    return qc


def dequantise_cache(qc: Dict[str, np.ndarray], wl) -> np.ndarray:
    """The float64 rows [B, S, d_c + d_R] a quantised ring stands for (NaN where unwritten)."""
    cb, rb = (int(v) for v in qc["bits"])
    c = dequantise_rows(unpack_codes(qc["content"], cb, wl.d_latent), qc["scale_c"])
    r = dequantise_rows(unpack_codes(qc["rope"], rb, wl.d_rope), qc["scale_r"])
    return np.concatenate([c, r], axis=-1)


def attend_quantised(q_abs: np.ndarray, qc: Dict[str, np.ndarray], q_first_tok: int,
                     k_first_tok: int, n_keys: int, scale: float, wl,
                     queries: Optional[Iterable[Tuple[int, int]]] = None):
    """Absorbed attention over a quantised ring: the keys and values are the dequantised
    rows ([QuantMLA]: dequantisation is part of the attention; the result is that of the
    attention over the dequantised cache)."""
    return O.attend_latent(q_abs, dequantise_cache(qc, wl), q_first_tok, k_first_tok,
                           n_keys, scale, wl, queries)
