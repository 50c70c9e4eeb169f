"""Drive the CUDA path through the Python binding of the C ABI for a workload, and
compare results with the oracle.  Used by the GPU tests only."""

from __future__ import annotations

import dataclasses
from typing import Dict, Optional

import numpy as np
import torch

import latent_kv_cache_write_b200 as mla
from synth import configs as C
from synth import generate as G

DEV = "cuda"


def upload(t: G.Tensor) -> torch.Tensor:
    if t.dtype == "bf16":
        return torch.from_numpy(t.storage.view(np.int16)).to(DEV).view(torch.bfloat16)
    return torch.from_numpy(t.storage).to(DEV)


def download(x: torch.Tensor) -> np.ndarray:
    return x.detach().float().cpu().numpy().astype(np.float64)


def empty(wl, shape, dtype=None):
    dt = dtype or (torch.bfloat16 if wl.dtype == "bf16" else torch.float32)
    return torch.empty(shape, dtype=dt, device=DEV)


@dataclasses.dataclass
class Run:
    wl: C.Workload
    shape: mla.MlaShape
    w: Dict[str, G.Tensor]
    wd: Dict[str, torch.Tensor]
    cache: torch.Tensor
    slots: list
    q: Dict[str, G.Tensor]
    q_abs: Optional[torch.Tensor] = None
    o_lat: Optional[torch.Tensor] = None
    lse: Optional[torch.Tensor] = None
    out: Optional[torch.Tensor] = None


def populate(wl: C.Workload, seed: int = 0, fill: float = float("nan")) -> Run:
    """Allocate the ring and write the workload's whole frame history into it, one
    frame per mla_cache_write call (or upload directly drawn rows for decode)."""
    shape = mla.make_shape(wl)
    w = G.weights(wl, seed)
    wd = {k: upload(v) for k, v in w.items()}
    slots = []
    if wl.cache_direct:
        cache = upload(G.direct_cache(wl, seed))
    else:
        cache = empty(wl, (wl.batch, wl.ring_slots, wl.row_width))
        cache.fill_(fill)
        F = wl.tokens_per_frame
        for f in range(wl.frames_written):
            h = upload(G.hidden_frame(wl, seed, f))
            s = torch.empty((wl.batch, F), dtype=torch.int32, device=DEV)
            mla.mla_cache_write(shape, h, wl.d_model, F, f * F, wd["w_dkv"], wd["w_kr"], cache, s)
            slots.append(s)
    return Run(wl, shape, w, wd, cache, slots, G.queries(wl, seed))


def run_chunk(r: Run, with_lse: bool = True) -> Run:
    wl = r.wl
    T = wl.n_queries
    r.q_abs = empty(wl, (wl.batch, T, wl.n_heads, wl.row_width))
    mla.mla_absorb_q(r.shape, upload(r.q["q_nope"]), upload(r.q["q_rope"]), T, wl.q_first_tok,
                     r.wd["w_uk"], r.q_abs)
    r.o_lat = empty(wl, (wl.batch, T, wl.n_heads, wl.d_latent))
    r.lse = torch.empty((wl.batch, T, wl.n_heads), dtype=torch.float32, device=DEV) \
        if with_lse else None
    nws = mla.mla_attend_workspace_size(r.shape, T, wl.n_keys)
    ws = torch.empty(max(nws, 16), dtype=torch.uint8, device=DEV)
    mla.mla_attend(r.shape, r.q_abs, T, wl.q_first_tok, r.cache, wl.k_first_tok, wl.n_keys,
                   wl.softmax_scale, r.o_lat, r.lse, ws, nws)
    r.out = empty(wl, (wl.batch, T, wl.n_heads, wl.d_nope))
    mla.mla_up_v(r.shape, r.o_lat, T, r.wd["w_uv"], r.out)
    torch.cuda.synchronize()
    assert mla.mla_device_error() == 0
    return r


# ------------------------------------------------------------------ tolerances


def tol_check(got: np.ndarray, ref: np.ndarray, dtype: str, what: str = "") -> float:
    """The workloads' tolerances: float32 relative Frobenius <= 1e-5; bfloat16
    relative Frobenius <= 1e-2 and max-abs <= 3e-2 * max|ref|."""
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, (what, got.shape, ref.shape)
    assert np.all(np.isfinite(got)), f"{what}: non-finite values"
    err = float(np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-300))
    if dtype == "f32":
        assert err <= 1e-5, f"{what}: rel Frobenius {err:.3e} > 1e-5"
    else:
        mx = float(np.abs(got - ref).max()) if got.size else 0.0
        assert err <= 1e-2, f"{what}: rel Frobenius {err:.3e} > 1e-2"
        assert mx <= 3e-2 * float(np.abs(ref).max()), f"{what}: max-abs {mx:.3e}"
    return err
