"""ctypes binding of ``libmla.so`` (declared in ``include/mla.h``).

Argument marshalling only: shapes become an ``MlaShape``, tensors become device
pointers, streams become ``cudaStream_t`` handles.  Every step of the path runs in the
library's CUDA kernels.  If the library has not been built, loading raises; there is
no other implementation to fall back to.
"""

from __future__ import annotations

import ctypes
import os

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libmla.so")

MLA_OK, MLA_ERR_ARG, MLA_ERR_UNSUPPORTED, MLA_ERR_ALIGN, MLA_ERR_RANGE, MLA_ERR_CUDA, \
    MLA_ERR_TIMEOUT = range(7)
MLA_F32, MLA_BF16 = 0, 1
MLA_FIXED_SCRATCH_BYTES = 40 * 1024 * 1024     # the header's static split-key scratch

# Every symbol the header declares, with (restype, argtypes).
_vp, _i32, _i64, _f32, _sz = (ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_float,
                              ctypes.c_size_t)


class MlaShape(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int32), ("n_heads", ctypes.c_int32),
                ("d_nope", ctypes.c_int32), ("d_latent", ctypes.c_int32),
                ("d_rope", ctypes.c_int32), ("rope_pairs", ctypes.c_int32 * 3),
                ("rope_theta", ctypes.c_double), ("grid_h", ctypes.c_int32),
                ("grid_w", ctypes.c_int32), ("ring_slots", ctypes.c_int64),
                ("dtype", ctypes.c_int32), ("reserved", ctypes.c_int32)]


_P = ctypes.POINTER(MlaShape)
SIGNATURES = {
    "mla_cache_write": (_i32, [_P, _vp, _i32, _i64, _i64, _vp, _vp, _vp, _vp, _vp]),
    "mla_absorb_q": (_i32, [_P, _vp, _vp, _i64, _i64, _vp, _vp, _vp]),
    "mla_attend_workspace_size": (_sz, [_P, _i64, _i64]),
    "mla_attend": (_i32, [_P, _vp, _i64, _i64, _vp, _i64, _i64, _f32, _vp, _vp, _vp, _sz, _vp]),
    "mla_attend_fixed_scratch": (_i32, [_P, _vp, _i64, _i64, _vp, _i64, _i64, _f32, _vp, _vp,
                                        _vp]),
    "mla_up_v": (_i32, [_P, _vp, _i64, _vp, _vp, _vp]),
    "mla_cache_shift_frames": (_i32, [_P, _vp, _i64, _i64, _i64, _vp]),
    "mla_cache_quantise": (_i32, [_P, _vp, _i64, _i64, _i32, _i32, _vp, _vp, _vp, _vp, _vp]),
    "mla_cache_dequantise": (_i32, [_P, _vp, _vp, _vp, _vp, _i32, _i32, _i64, _i64, _vp, _vp]),
    "mla_attend_quantised": (_i32, [_P, _vp, _i64, _i64, _vp, _vp, _vp, _vp, _i32, _i32, _i64,
                                    _i64, _f32, _vp, _vp, _vp, _sz, _vp]),
    "mla_attend_materialised_workspace_size": (_sz, [_P]),
    "mla_attend_materialised": (_i32, [_P, _vp, _vp, _i64, _i64, _vp, _i64, _i64, _f32, _vp, _vp,
                                       _vp, _vp, _vp, _sz, _vp]),
    "mla_status_string": (ctypes.c_char_p, [_i32]),
    "mla_device_error": (_i32, [_vp]),
    "mla_check_wait_timeout": (_i32, [_vp]),
    "mla_kernel_launches": (ctypes.c_uint64, []),
    "mla_device_error_info": (None, [ctypes.POINTER(ctypes.c_uint32)]),
}

_lib = None


def lib() -> ctypes.CDLL:
    """Load the library (once).  Raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(_LIB_PATH):
            raise RuntimeError(
                f"{_LIB_PATH} is missing: build it with "
                "`python -m latent_kv_cache_write_b200.build` (nvcc, sm_100a)")
        L = ctypes.CDLL(_LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def status_string(code: int) -> str:
    return lib().mla_status_string(code).decode()


class MlaError(RuntimeError):
    def __init__(self, call: str, code: int):
        super().__init__(f"{call} failed: {status_string(code)}")
        self.code = code


def check(call: str, code: int) -> None:
    if code != MLA_OK:
        raise MlaError(call, code)


def make_shape(wl, dtype=None) -> MlaShape:
    """MlaShape of a workload (anything with the workload table's attributes)."""
    s = MlaShape()
    s.batch, s.n_heads, s.d_nope = wl.batch, wl.n_heads, wl.d_nope
    s.d_latent, s.d_rope = wl.d_latent, wl.d_rope
    s.rope_pairs[:] = list(wl.rope_pairs)
    s.rope_theta = wl.rope_theta
    s.grid_h, s.grid_w = wl.grid_h, wl.grid_w
    s.ring_slots = wl.ring_slots
    d = dtype if dtype is not None else wl.dtype
    s.dtype = MLA_BF16 if d in ("bf16", MLA_BF16) else MLA_F32
    s.reserved = 0
    return s
