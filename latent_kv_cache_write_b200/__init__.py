"""Absorbed multi-head latent attention over a sliding-window latent KV ring on B200.

Python face of ``libmla.so``: the calls of the C ABI under the same names, taking
``torch`` CUDA tensors (or raw device pointers) and enqueuing on the current CUDA
stream unless a stream is given.  PyTorch supplies device memory and streams only;
all arithmetic runs in the library's kernels.

One chunk step (bf16; B sequences, T new tokens of one frame written at token g0, the
chunk's queries attending to the n_keys window tokens starting at k0)::

    import latent_kv_cache_write_b200 as mla
    shape = mla.MlaShape(batch=B, n_heads=H, d_nope=128, d_latent=512, d_rope=64,
                         rope_pairs=(8, 12, 12), rope_theta=1e4, grid_h=gh, grid_w=gw,
                         ring_slots=S, dtype=mla.native.MLA_BF16)
    mla.mla_cache_write(shape, h, d_model, T, g0, w_dkv, w_kr, cache)   # ring [B, S, 576]
    mla.mla_absorb_q(shape, q_nope, q_rope, T, g0, w_uk, q_abs)          # [B, T, H, 576]
    ws = torch.empty(mla.mla_attend_workspace_size(shape, T, n_keys), dtype=torch.uint8,
                     device="cuda")
    mla.mla_attend(shape, q_abs, T, g0, cache, k0, n_keys, scale, o_lat, lse, ws)
    mla.mla_up_v(shape, o_lat, T, w_uv, out)                             # [B, T, H, 128]

``mla_attend_materialised`` replaces the last three calls with the non-absorbed form;
``mla_cache_shift_frames`` re-indexes the window's RoPE keys by whole frames;
``mla_cache_quantise`` / ``mla_cache_dequantise`` convert ring rows to and from the
low-bit ring.  Errors raise ``MlaError`` with the library's status.
"""

from __future__ import annotations

import ctypes
from typing import Optional

from . import native
from .native import MLA_FIXED_SCRATCH_BYTES, MlaError, MlaShape, make_shape  # noqa: F401

__all__ = ["mla_cache_write", "mla_absorb_q", "mla_attend", "mla_attend_workspace_size",
           "mla_attend_fixed_scratch", "mla_attend_materialised", "mla_attend_quantised",
           "mla_cache_shift_frames",
           "mla_cache_quantise", "mla_cache_dequantise",
           "mla_attend_materialised_workspace_size", "mla_up_v", "mla_device_error",
           "mla_kernel_launches", "mla_device_error_info", "mla_check_wait_timeout", "make_shape",
           "MlaShape", "MlaError", "MLA_FIXED_SCRATCH_BYTES"]


def _ptr(t) -> Optional[int]:
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream) -> Optional[int]:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def mla_cache_write(shape: MlaShape, h, d_model: int, n_tok: int, first_tok: int, w_dkv, w_kr,
                    cache, slots_out=None, stream=None) -> None:
    native.check("mla_cache_write", native.lib().mla_cache_write(
        ctypes.byref(shape), _ptr(h), d_model, n_tok, first_tok, _ptr(w_dkv), _ptr(w_kr),
        _ptr(cache), _ptr(slots_out), _stream(stream)))


def mla_absorb_q(shape: MlaShape, q_nope, q_rope, n_q: int, q_first_tok: int, w_uk, q_abs,
                 stream=None) -> None:
    native.check("mla_absorb_q", native.lib().mla_absorb_q(
        ctypes.byref(shape), _ptr(q_nope), _ptr(q_rope), n_q, q_first_tok, _ptr(w_uk),
        _ptr(q_abs), _stream(stream)))


def mla_attend_workspace_size(shape: MlaShape, n_q: int, n_keys: int) -> int:
    return int(native.lib().mla_attend_workspace_size(ctypes.byref(shape), n_q, n_keys))


def mla_attend(shape: MlaShape, q_abs, n_q: int, q_first_tok: int, cache, k_first_tok: int,
               n_keys: int, softmax_scale: float, o_lat, lse=None, workspace=None,
               workspace_bytes: Optional[int] = None, stream=None) -> None:
    if workspace_bytes is None:
        workspace_bytes = 0 if workspace is None else (
            workspace.numel() * workspace.element_size())
    native.check("mla_attend", native.lib().mla_attend(
        ctypes.byref(shape), _ptr(q_abs), n_q, q_first_tok, _ptr(cache), k_first_tok, n_keys,
        softmax_scale, _ptr(o_lat), _ptr(lse), _ptr(workspace), workspace_bytes,
        _stream(stream)))


def mla_attend_fixed_scratch(shape: MlaShape, q_abs, n_q: int, q_first_tok: int, cache,
                             k_first_tok: int, n_keys: int, softmax_scale: float, o_lat,
                             lse=None, stream=None) -> None:
    native.check("mla_attend_fixed_scratch", native.lib().mla_attend_fixed_scratch(
        ctypes.byref(shape), _ptr(q_abs), n_q, q_first_tok, _ptr(cache), k_first_tok, n_keys,
        softmax_scale, _ptr(o_lat), _ptr(lse), _stream(stream)))


def mla_cache_shift_frames(shape: MlaShape, cache, first_tok: int, n_tok: int,
                           delta_frames: int, stream=None) -> None:
    native.check("mla_cache_shift_frames", native.lib().mla_cache_shift_frames(
        ctypes.byref(shape), _ptr(cache), first_tok, n_tok, delta_frames, _stream(stream)))


def mla_cache_quantise(shape: MlaShape, cache, first_tok: int, n_tok: int, content_bits: int,
                       rope_bits: int, q_content, q_rope, scale_c, scale_r,
                       stream=None) -> None:
    native.check("mla_cache_quantise", native.lib().mla_cache_quantise(
        ctypes.byref(shape), _ptr(cache), first_tok, n_tok, content_bits, rope_bits,
        _ptr(q_content), _ptr(q_rope), _ptr(scale_c), _ptr(scale_r), _stream(stream)))


def mla_cache_dequantise(shape: MlaShape, q_content, q_rope, scale_c, scale_r,
                         content_bits: int, rope_bits: int, first_tok: int, n_tok: int, cache,
                         stream=None) -> None:
    native.check("mla_cache_dequantise", native.lib().mla_cache_dequantise(
        ctypes.byref(shape), _ptr(q_content), _ptr(q_rope), _ptr(scale_c), _ptr(scale_r),
        content_bits, rope_bits, first_tok, n_tok, _ptr(cache), _stream(stream)))


def mla_attend_quantised(shape: MlaShape, q_abs, n_q: int, q_first_tok: int, q_content, q_rope,
                         scale_c, scale_r, content_bits: int, rope_bits: int, k_first_tok: int,
                         n_keys: int, softmax_scale: float, o_lat, lse=None, workspace=None,
                         workspace_bytes: Optional[int] = None, stream=None) -> None:
    if workspace_bytes is None:
        workspace_bytes = 0 if workspace is None else (
            workspace.numel() * workspace.element_size())
    native.check("mla_attend_quantised", native.lib().mla_attend_quantised(
        ctypes.byref(shape), _ptr(q_abs), n_q, q_first_tok, _ptr(q_content), _ptr(q_rope),
        _ptr(scale_c), _ptr(scale_r), content_bits, rope_bits, k_first_tok, n_keys,
        softmax_scale, _ptr(o_lat), _ptr(lse), _ptr(workspace), workspace_bytes,
        _stream(stream)))


def mla_attend_materialised_workspace_size(shape: MlaShape) -> int:
    return int(native.lib().mla_attend_materialised_workspace_size(ctypes.byref(shape)))


def mla_attend_materialised(shape: MlaShape, q_nope, q_rope, n_q: int, q_first_tok: int,
                            cache, k_first_tok: int, n_keys: int, softmax_scale: float, w_uk,
                            w_uv, out, lse=None, workspace=None,
                            workspace_bytes: Optional[int] = None, stream=None) -> None:
    if workspace_bytes is None:
        workspace_bytes = 0 if workspace is None else (
            workspace.numel() * workspace.element_size())
    native.check("mla_attend_materialised", native.lib().mla_attend_materialised(
        ctypes.byref(shape), _ptr(q_nope), _ptr(q_rope), n_q, q_first_tok, _ptr(cache),
        k_first_tok, n_keys, softmax_scale, _ptr(w_uk), _ptr(w_uv), _ptr(out), _ptr(lse),
        _ptr(workspace), workspace_bytes, _stream(stream)))


def mla_up_v(shape: MlaShape, o_lat, n_q: int, w_uv, out, stream=None) -> None:
    native.check("mla_up_v", native.lib().mla_up_v(
        ctypes.byref(shape), _ptr(o_lat), n_q, _ptr(w_uv), _ptr(out), _stream(stream)))


def mla_kernel_launches() -> int:
    """Kernels launched by the library so far in this process."""
    return int(native.lib().mla_kernel_launches())


def mla_device_error_info() -> list:
    """[status bits, wait site id, CTA index, (thread << 16 | block)] of the last
    device-side error reported by mla_device_error."""
    buf = (ctypes.c_uint32 * 4)()
    native.lib().mla_device_error_info(buf)
    return list(buf)


def mla_check_wait_timeout(stream=None) -> None:
    """Enqueue the diagnostic whose bounded wait must expire; mla_device_error on the same
    stream then reports MLA_ERR_TIMEOUT."""
    native.check("mla_check_wait_timeout", native.lib().mla_check_wait_timeout(_stream(stream)))


def mla_device_error(stream=None) -> int:
    """Synchronise the stream and return (and clear) the device-side error status."""
    return int(native.lib().mla_device_error(_stream(stream)))
