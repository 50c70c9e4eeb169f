#!/usr/bin/env python3
"""Benchmark of the absorbed-MLA hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One step is one pass of the whole path over the video-chunk workload (batch 1,
n_h=32, d_h=128, d_c=512, d_R=64 3-D RoPE, 30x52-token frames, a 3-frame window plus a
1-frame query chunk, hidden 4096, bf16): the chunk frame's cache write, query
absorption, absorbed attention over the 6240-key window, and the W_UV up-projection.
The ring holds the three window frames before timing starts.  Each rank runs its own
independent sequence (weak scaling, no data-path collective).

Printed metric: algorithmic TFLOP/s of the step (absorbed flops: per visible
(query, key, head) 2(d_c+d_R) + 2 d_c, plus the three GEMMs), with
the dominant kernel's roofline, the decode workload's latent-cache GB/s, an end-to-end
figure through host buffers, and the CPU oracle baseline.
"""

from __future__ import annotations

import argparse
import json
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from synth import configs as C  # noqa: E402
from synth import generate as G  # noqa: E402

WORKLOAD = C.VIDEO_CHUNK            # the default step; --workload picks another
# workloads whose step writes its own cache (decode reads a cache given directly and is
# timed by the decode leg)
LEGS = ("decode", "materialised", "shift", "quant", "fold", "quant_attend", "workloads")
STEP_WORKLOADS = tuple(w.name for w in C.ALL if not w.cache_direct and w.elem_bytes == 2)
L2_FLUSH_BYTES = 256 << 20           # > 126 MB L2: written between timed steps
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# ------------------------------------------------------------------ work accounting


def visible_pairs(wl) -> int:
    """(query, key) pairs the frame-block-causal mask keeps, summed over the batch."""
    F = wl.tokens_per_frame
    k_end = wl.k_first_tok + wl.n_keys
    total = 0
    for i in range(wl.n_queries):
        g = wl.q_first_tok + i
        total += min(k_end, (g // F + 1) * F) - wl.k_first_tok
    return total * wl.batch


def step_flops(wl) -> dict:
    T, B = wl.n_queries, wl.batch
    return {
        "cache_write": 0 if wl.cache_direct else 2 * B * T * wl.d_model * wl.row_width,
        "absorb_q": 2 * B * T * wl.n_heads * wl.d_nope * wl.d_latent,
        "attend": visible_pairs(wl) * wl.n_heads * (2 * wl.row_width + 2 * wl.d_latent),
        "up_v": 2 * B * T * wl.n_heads * wl.d_latent * wl.d_nope,
    }


def step_bytes(wl) -> dict:
    """Algorithmic HBM bytes of each call of the step: every operand read once, every
    result written once (the attention reads the window's cached rows once)."""
    e, T, B, H = wl.elem_bytes, wl.n_queries, wl.batch, wl.n_heads
    return {
        "cache_write": (B * T * wl.d_model + wl.d_model * wl.row_width + B * T * wl.row_width) * e,
        "absorb_q": (B * T * H * (wl.d_nope + wl.d_rope) + H * wl.d_nope * wl.d_latent
                     + B * T * H * wl.row_width) * e,
        "attend": (B * T * H * wl.row_width + B * wl.n_keys * wl.row_width
                   + B * T * H * wl.d_latent) * e + B * T * H * 4,
        "up_v": (B * T * H * wl.d_latent + H * wl.d_nope * wl.d_latent + B * T * H * wl.d_nope) * e,
    }


def materialised_flops(wl) -> int:
    """Flops of the non-absorbed alternative for the same attention: K and V materialised
    once per (key, head) from the latent, then attention over d_h + d_R and d_h."""
    mat = 2 * 2 * wl.batch * wl.n_keys * wl.n_heads * wl.d_latent * wl.d_nope
    att = visible_pairs(wl) * wl.n_heads * (2 * (wl.d_nope + wl.d_rope) + 2 * wl.d_nope)
    return mat + att


def kernel_rooflines(wl, kernels_ms, peaks) -> dict:
    """Per call of the step: achieved TFLOP/s and GB/s against the measured peaks, and the
    bound that binds (the larger of flops/peak and bytes/bandwidth)."""
    fl, by = step_flops(wl), step_bytes(wl)
    tf, bw = float(peaks["bf16_tflops"]), float(peaks["hbm_gbs"])
    out = {}
    for k, ms in kernels_ms.items():
        s = ms * 1e-3
        t_tensor, t_hbm = fl[k] / (tf * 1e12), by[k] / (bw * 1e9)
        out[k] = {"ms": ms, "flops": fl[k], "bytes": by[k],
                  "tflops": fl[k] / s / 1e12, "frac_tensor": fl[k] / s / 1e12 / tf,
                  "gbs": by[k] / s / 1e9, "frac_hbm": by[k] / s / 1e9 / bw,
                  "bound": "tensor" if t_tensor >= t_hbm else "hbm",
                  "frac_of_bound": max(t_tensor, t_hbm) / s}
    return out


def step_config(wl, world: int) -> dict:
    """The workload a step runs, as both arms report it."""
    return {"workload": wl.name, "batch": wl.batch, "n_heads": wl.n_heads,
            "d_nope": wl.d_nope, "d_latent": wl.d_latent, "d_rope": wl.d_rope,
            "frame": f"{wl.grid_h}x{wl.grid_w}", "window_frames": wl.window_frames,
            "chunk_frames": wl.chunk_frames, "keys": wl.n_keys, "queries": wl.n_queries,
            "d_model": wl.d_model, "step": "cache_write+absorb_q+attend+up_v",
            "flops_per_step": sum(step_flops(wl).values()),
            "l2": "flushed (256 MB write) before each step",
            "per_call_times": "from as many steps again, interleaved with the timed ones, that "
                              "record an event between the calls",
            "parallelism": f"replicas x{world} (independent sequences)"}


def percentiles(xs) -> list:
    q = sorted(xs)
    pick = lambda f: q[min(len(q) - 1, int(round(f * (len(q) - 1))))]
    return [pick(0.1), pick(0.5), pick(0.9)]


def decode_bytes(wl) -> int:
    """Algorithmic bytes of one decode attention call: every cached row read once,
    q_abs read, o_lat and the LSE written."""
    e = wl.elem_bytes
    rows = wl.batch * wl.n_keys * wl.row_width * e
    q = wl.batch * wl.n_heads * wl.row_width * e
    o = wl.batch * wl.n_heads * wl.d_latent * e + wl.batch * wl.n_heads * 4
    return rows + q + o


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# ------------------------------------------------------------------ clocks


class ClockSampler:
    """SM clock and clock-event (throttle) reasons of this rank's GPU, polled through
    NVML every 10 ms in a background thread while the timed region runs."""
    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown"}

    def __init__(self, torch_device: int):
        self.dev = torch_device
        self.samples = []
        self.max_mhz = None
        self._stop = threading.Event()
        self.h = None

    def _handle(self):
        import pynvml
        import torch
        pynvml.nvmlInit()
        props = torch.cuda.get_device_properties(self.dev)
        bus = getattr(props, "pci_bus_id", None)
        if bus is not None:
            dom = getattr(props, "pci_domain_id", 0)
            devid = getattr(props, "pci_device_id", 0)
            for fmt in ("%08X:%02X:%02X.0", "%04X:%02X:%02X.0"):
                try:
                    return pynvml.nvmlDeviceGetHandleByPciBusId((fmt % (dom, bus, devid)).encode())
                except pynvml.NVMLError:
                    pass
        return pynvml.nvmlDeviceGetHandleByIndex(self.dev)

    def __enter__(self):
        try:
            import pynvml
            self.h = self._handle()
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            getr = getattr(pynvml, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                pynvml.nvmlDeviceGetCurrentClocksThrottleReasons

            def loop():
                while not self._stop.is_set():
                    try:
                        self.samples.append((pynvml.nvmlDeviceGetClockInfo(self.h, pynvml.NVML_CLOCK_SM),
                                             getr(self.h)))
                    except pynvml.NVMLError:
                        pass
                    time.sleep(0.01)

            self.t = threading.Thread(target=loop, daemon=True)
            self.t.start()
        except Exception:  # noqa: BLE001  (no NVML: the line reports no samples)
            self.h = None
        return self

    def __exit__(self, *a):
        self._stop.set()
        if self.h is not None:
            self.t.join(timeout=2)

    def summary(self):
        sm = [c for c, _ in self.samples]
        reasons = set()
        for _, r in self.samples:
            for bit, name in self.REASONS.items():
                if r & bit:
                    reasons.add(name)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": self.max_mhz,
                "reasons": sorted(reasons), "samples": len(sm), "source": "nvml 10 ms"}


# ------------------------------------------------------------------ our arm


class Step:
    """Device-resident state of one sequence's video-chunk step."""

    def __init__(self, wl, seed, torch, mla):
        self.wl, self.torch, self.mla = wl, torch, mla
        dev = "cuda"
        self.shape = mla.make_shape(wl)

        def up(t):
            return torch.from_numpy(t.storage.view(np.int16)).to(dev).view(torch.bfloat16)

        w = G.weights(wl, seed)
        self.w = {k: up(v) for k, v in w.items()}
        F = wl.tokens_per_frame
        self.cache = torch.zeros((wl.batch, wl.ring_slots, wl.row_width), dtype=torch.bfloat16,
                                 device=dev)
        first = wl.first_chunk_frame
        for f in range(first):                       # the window, written before timing
            h = up(G.hidden_frame(wl, seed, f))
            mla.mla_cache_write(self.shape, h, wl.d_model, F, f * F, self.w["w_dkv"],
                                self.w["w_kr"], self.cache)
        hq = G.hidden_frames(wl, seed, first, wl.chunk_frames)
        q = G.queries(wl, seed)
        self.host = {"h": hq.storage.view(np.int16), "q_nope": q["q_nope"].storage.view(np.int16),
                     "q_rope": q["q_rope"].storage.view(np.int16)}
        self.dev_in = {k: torch.from_numpy(v).to(dev).view(torch.bfloat16)
                       for k, v in self.host.items()}
        self.pinned = {k: torch.from_numpy(v).pin_memory() for k, v in self.host.items()}
        T = wl.n_queries
        self.q_abs = torch.empty((wl.batch, T, wl.n_heads, wl.row_width), dtype=torch.bfloat16,
                                 device=dev)
        self.o_lat = torch.empty((wl.batch, T, wl.n_heads, wl.d_latent), dtype=torch.bfloat16,
                                 device=dev)
        self.lse = torch.empty((wl.batch, T, wl.n_heads), dtype=torch.float32, device=dev)
        self.out = torch.empty((wl.batch, T, wl.n_heads, wl.d_nope), dtype=torch.bfloat16,
                               device=dev)
        self.out_host = torch.empty(self.out.shape, dtype=torch.bfloat16).pin_memory()
        self.ws_bytes = mla.mla_attend_workspace_size(self.shape, T, wl.n_keys)
        self.ws = torch.empty(max(self.ws_bytes, 16), dtype=torch.uint8, device=dev)
    STAGES = ("cache_write", "absorb_q", "attend", "up_v")

    def run(self, inp=None, ev=None, out=None):
        """One step; with `ev` (5 CUDA events) the boundaries between its calls are
        recorded on the current stream, the one the library launches on."""
        wl, mla = self.wl, self.mla
        inp = inp or self.dev_in
        out = self.out if out is None else out
        T = wl.n_queries
        F = wl.tokens_per_frame
        mark = (lambda i: ev[i].record()) if ev is not None else (lambda i: None)
        mark(0)
        mla.mla_cache_write(self.shape, inp["h"], wl.d_model, T, wl.first_chunk_frame * F,
                            self.w["w_dkv"], self.w["w_kr"], self.cache)
        mark(1)
        mla.mla_absorb_q(self.shape, inp["q_nope"], inp["q_rope"], T, wl.q_first_tok,
                         self.w["w_uk"], self.q_abs)
        mark(2)
        mla.mla_attend(self.shape, self.q_abs, T, wl.q_first_tok, self.cache, wl.k_first_tok,
                       wl.n_keys, wl.softmax_scale, self.o_lat, self.lse, self.ws, self.ws_bytes)
        mark(3)
        mla.mla_up_v(self.shape, self.o_lat, T, self.w["w_uv"], out)
        mark(4)

    def run_e2e(self, steps):
        """`steps` steps end to end through the public calls, from pinned host inputs to
        the host copy of each step's output, as a serving loop would run them: an upload
        stream brings step i+1's inputs and a download stream takes step i-1's output
        while step i computes (two device input sets and two output buffers).  Every
        step's copies are inside the timed region.  Returns the elapsed ms (CUDA events:
        the first upload's start to the last download's end)."""
        torch = self.torch
        comp = torch.cuda.current_stream()
        up, down = torch.cuda.Stream(), torch.cuda.Stream()
        sets = [self.dev_in, {k: torch.empty_like(v) for k, v in self.dev_in.items()}]
        outs = [self.out, torch.empty_like(self.out)]
        hosts = [self.out_host, torch.empty_like(self.out_host).pin_memory()]
        ev = lambda: torch.cuda.Event()
        inp_ready, comp_done, d2h_done = [ev(), ev()], [ev(), ev()], [ev(), ev()]
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        up.record_event(t0)
        for i in range(steps):
            k = i & 1
            with torch.cuda.stream(up):
                if i >= 2:
                    up.wait_event(comp_done[k])            # set k no longer read
                for name, v in self.pinned.items():
                    sets[k][name].view(torch.int16).copy_(v, non_blocking=True)
                up.record_event(inp_ready[k])
            comp.wait_event(inp_ready[k])
            if i >= 2:
                comp.wait_event(d2h_done[k])              # output k downloaded
            self.run(inp=sets[k], out=outs[k])
            comp.record_event(comp_done[k])
            with torch.cuda.stream(down):
                down.wait_event(comp_done[k])
                hosts[k].copy_(outs[k], non_blocking=True)
                down.record_event(d2h_done[k])
        down.wait_event(d2h_done[(steps - 1) & 1])
        copy = down
        copy.record_event(t1)
        torch.cuda.synchronize()
        return t0.elapsed_time(t1)


def time_steps(torch, fn, steps, flush, n_marks=0):
    """Per step: flush L2 (untimed), then CUDA events around the step on the current
    stream.  Returns (step ms list, per-interval ms lists between the n_marks events
    the step records itself)."""
    st, parts = [], [[] for _ in range(max(0, n_marks - 1))]
    for _ in range(steps):
        flush.zero_()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        marks = [torch.cuda.Event(enable_timing=True) for _ in range(n_marks)] or None
        e0.record()
        fn(marks)
        e1.record()
        torch.cuda.synchronize()
        st.append(e0.elapsed_time(e1))
        for i in range(n_marks - 1):
            parts[i].append(marks[i].elapsed_time(marks[i + 1]))
    return st, parts


def time_steps_and_calls(torch, step, steps, flush):
    """`steps` timed steps for the step's rate, interleaved with as many steps that record
    an event between each of the step's calls for the per-call breakdown.  An event
    between two kernels keeps the second from starting while the first finishes, so the
    timed steps carry none; interleaving puts both under the same clocks.  Returns
    (step ms list, per-call ms lists)."""
    st, parts = [], [[] for _ in Step.STAGES]
    for i in range(2 * steps):
        marked = i % 2 == 1
        flush.zero_()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        marks = [torch.cuda.Event(enable_timing=True) for _ in range(5)] if marked else None
        e0.record()
        step.run(ev=marks)
        e1.record()
        torch.cuda.synchronize()
        if marked:
            for k in range(4):
                parts[k].append(marks[k].elapsed_time(marks[k + 1]))
        else:
            st.append(e0.elapsed_time(e1))
    return st, parts


def materialised_leg(torch, mla, step, steps, warmup, flush, absorbed_ms):
    """The non-absorbed form of the same chunk: mla_attend_materialised (the per-head keys
    and values rebuilt from the latent, then attention in head space, output up-projected)
    on the step's queries and cache; it replaces the absorption, the absorbed attention and
    the up-projection of the step."""
    wl = step.wl
    if mla.mla_attend_materialised_workspace_size(step.shape) == 0:
        return None
    T = wl.n_queries
    nws = mla.mla_attend_materialised_workspace_size(step.shape)
    ws = torch.empty(nws, dtype=torch.uint8, device="cuda")
    out = torch.empty_like(step.out)
    lse = torch.empty_like(step.lse)

    def call(_a=None):
        mla.mla_attend_materialised(step.shape, step.dev_in["q_nope"], step.dev_in["q_rope"], T,
                                    wl.q_first_tok, step.cache, wl.k_first_tok, wl.n_keys,
                                    wl.softmax_scale, step.w["w_uk"], step.w["w_uv"], out, lse,
                                    ws, nws)

    for _ in range(warmup):
        call()
    ms, _ = time_steps(torch, call, steps, flush)
    t = statistics.mean(ms)
    fl = materialised_flops(wl)
    return {"call": "mla_attend_materialised", "ms": t, "flops": fl,
            "tflops": fl / (t * 1e-3) / 1e12,
            "replaces_ms": absorbed_ms, "speedup_vs_absorbed": absorbed_ms / t,
            "note": "per-head K and V of every ring slot rebuilt, then attention in head "
                    "space; replaces absorb_q + attend + up_v of the step"}


def shift_leg(torch, mla, step, steps, warmup, flush):
    """Whole-frame re-indexing of the window's cached RoPE keys (mla_cache_shift_frames),
    forward and back by one frame per call pair so the ring stays valid."""
    wl = step.wl
    n = wl.n_keys

    def call(_a=None):
        mla.mla_cache_shift_frames(step.shape, step.cache, wl.k_first_tok, n, 1)
        mla.mla_cache_shift_frames(step.shape, step.cache, wl.k_first_tok, n, -1)

    for _ in range(warmup):
        call()
    ms, _ = time_steps(torch, call, steps, flush)
    t = statistics.mean(ms) / 2                       # per call
    moved = 2 * wl.batch * n * 2 * wl.rope_pairs[0] * wl.elem_bytes     # read + write
    return {"call": "mla_cache_shift_frames", "rows": wl.batch * n, "ms": t, "bytes": moved,
            "value": moved / (t * 1e-3) / 1e9, "unit": "GB/s",
            "note": "the window's t-axis RoPE pairs turned in place; a few hundred KB, so "
                    "launch-bound"}


def quant_token_bytes(wl, content_bits: int, rope_bits: int) -> int:
    """Bytes of one token in the low-bit ring: both packed paths and two float32 scales."""
    return wl.d_latent * content_bits // 8 + wl.d_rope * rope_bits // 8 + 8


def quant_leg(torch, mla, step, steps, warmup, flush, bits=(4, 4)):
    """The window's rows into the low-bit ring (mla_cache_quantise), and back into a second
    ring (mla_cache_dequantise); INT4 content and RoPE by default."""
    wl = step.wl
    cb, rb = bits
    B, S, n = wl.batch, wl.ring_slots, wl.n_keys
    qc = torch.empty((B, S, wl.d_latent * cb // 8), dtype=torch.uint8, device="cuda")
    qr = torch.empty((B, S, wl.d_rope * rb // 8), dtype=torch.uint8, device="cuda")
    sc = torch.empty((B, S), dtype=torch.float32, device="cuda")
    sr = torch.empty_like(sc)
    back = torch.empty_like(step.cache)

    def quant(_a=None):
        mla.mla_cache_quantise(step.shape, step.cache, wl.k_first_tok, n, cb, rb, qc, qr, sc,
                               sr)

    def dequant(_a=None):
        mla.mla_cache_dequantise(step.shape, qc, qr, sc, sr, cb, rb, wl.k_first_tok, n, back)

    for _ in range(warmup):
        quant()
        dequant()
    ms_q, _ = time_steps(torch, quant, steps, flush)
    ms_d, _ = time_steps(torch, dequant, steps, flush)
    row = wl.row_width * wl.elem_bytes
    packed = quant_token_bytes(wl, cb, rb)
    moved = B * n * (row + packed)                    # one side read, the other written
    tq, td = statistics.mean(ms_q), statistics.mean(ms_d)
    return {"calls": "mla_cache_quantise, mla_cache_dequantise",
            "bits": {"content": cb, "rope": rb}, "rows": B * n, "bytes_per_token": packed,
            "compression": row / packed, "bytes": moved,
            "quantise": {"ms": tq, "value": moved / (tq * 1e-3) / 1e9, "unit": "GB/s"},
            "dequantise": {"ms": td, "value": moved / (td * 1e-3) / 1e9, "unit": "GB/s"},
            "note": "the window's rows; ~9 MB each way, so launch- and latency-bound"}


def decode_leg(torch, mla, steps, warmup, flush, wl=C.DECODE):
    shape = mla.make_shape(wl)
    dev = "cuda"
    cache = torch.from_numpy(G.direct_cache(wl, 0).storage.view(np.int16)).to(dev).view(
        torch.bfloat16)
    q = G.queries(wl, 0)
    w = G.weights(wl, 0)
    up = lambda t: torch.from_numpy(t.storage.view(np.int16)).to(dev).view(torch.bfloat16)
    q_abs = torch.empty((wl.batch, 1, wl.n_heads, wl.row_width), dtype=torch.bfloat16, device=dev)
    mla.mla_absorb_q(shape, up(q["q_nope"]), up(q["q_rope"]), 1, wl.q_first_tok, up(w["w_uk"]),
                     q_abs)
    o_lat = torch.empty((wl.batch, 1, wl.n_heads, wl.d_latent), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((wl.batch, 1, wl.n_heads), dtype=torch.float32, device=dev)
    nws = mla.mla_attend_workspace_size(shape, 1, wl.n_keys)
    ws = torch.empty(max(nws, 16), dtype=torch.uint8, device=dev)

    def call(_a=None):
        mla.mla_attend(shape, q_abs, 1, wl.q_first_tok, cache, wl.k_first_tok, wl.n_keys,
                       wl.softmax_scale, o_lat, lse, ws, nws)

    for _ in range(warmup):
        call()
    ms, _ = time_steps(torch, call, steps, flush)
    t = statistics.mean(ms)
    return {"workload": wl.name, "value": decode_bytes(wl) / (t * 1e-3) / 1e9, "unit": "GB/s",
            "ms": t, "bytes": decode_bytes(wl),
            "tflops": step_flops(wl)["attend"] / (t * 1e-3) / 1e12}


def workload_leg(torch, mla, name, steps, warmup, flush, peaks, device):
    """The whole step (cache write of the chunk, absorption, attention, up-projection) of
    another workload, timed like the main step with the L2 flushed before each one; the
    attention's rate against the measured bf16 peak, with the clocks seen meanwhile."""
    wl = C.BY_NAME[name]
    step = Step(wl, seed=0, torch=torch, mla=mla)
    for _ in range(warmup):
        step.run()
    torch.cuda.synchronize()
    with ClockSampler(device) as clocks:
        ms, parts = time_steps_and_calls(torch, step, steps, flush)
    torch.cuda.synchronize()
    kms = {k: statistics.mean(v) for k, v in zip(Step.STAGES, parts)}
    fl = step_flops(wl)
    att = fl["attend"] / (kms["attend"] * 1e-3) / 1e12
    peak = float(peaks["bf16_tflops"])
    out = {"workload": wl.name, "config": step_config(wl, 1), "steps": steps,
           "ms_per_step": statistics.mean(ms),
           "tflops_per_step": sum(fl.values()) / (statistics.mean(ms) * 1e-3) / 1e12,
           "attend": {"ms": kms["attend"], "flops": fl["attend"], "tflops": att, "peak": peak,
                      "frac": att / peak, "p10_p50_p90": percentiles(dict(zip(Step.STAGES, parts))["attend"])},
           "kernels_ms": kms, "clocks": clocks.summary()}
    mat = materialised_leg(torch, mla, step, steps, warmup, flush,
                           kms["absorb_q"] + kms["attend"] + kms["up_v"])
    if mat:
        mat["frac"] = mat["tflops"] / peak
        out["materialised"] = mat
    del step
    torch.cuda.empty_cache()
    return out


def quant_attend_leg(torch, mla, steps, warmup, flush, peaks, chunk_step=None):
    """Attention with the dequantisation fused in (mla_attend_quantised): the decode
    workload over its ring quantised to INT4 / INT4 and INT2 / INT4, and the video chunk
    over an INT4 ring; bytes are those the call reads and writes (packed ring, q_abs, o_lat)."""
    out = {}
    wl = C.DECODE
    shape = mla.make_shape(wl)
    dev = "cuda"
    up = lambda t: torch.from_numpy(t.storage.view(np.int16)).to(dev).view(torch.bfloat16)
    cache = up(G.direct_cache(wl, 0))
    q = G.queries(wl, 0)
    w = G.weights(wl, 0)
    q_abs = torch.empty((wl.batch, 1, wl.n_heads, wl.row_width), dtype=torch.bfloat16, device=dev)
    mla.mla_absorb_q(shape, up(q["q_nope"]), up(q["q_rope"]), 1, wl.q_first_tok, up(w["w_uk"]),
                     q_abs)

    def run(shape, wl, q_abs, cache, T, cb, rb):
        B, S = wl.batch, wl.ring_slots
        qc = torch.empty((B, S, wl.d_latent * cb // 8), dtype=torch.uint8, device=dev)
        qr = torch.empty((B, S, wl.d_rope * rb // 8), dtype=torch.uint8, device=dev)
        sc = torch.empty((B, S), dtype=torch.float32, device=dev)
        sr = torch.empty_like(sc)
        mla.mla_cache_quantise(shape, cache, wl.k_first_tok, wl.n_keys, cb, rb, qc, qr, sc, sr)
        o = torch.empty((B, T, wl.n_heads, wl.d_latent), dtype=torch.bfloat16, device=dev)
        lse = torch.empty((B, T, wl.n_heads), dtype=torch.float32, device=dev)
        nws = mla.mla_attend_workspace_size(shape, T, wl.n_keys)
        ws = torch.empty(max(nws, 16), dtype=torch.uint8, device=dev)

        def call(_a=None):
            mla.mla_attend_quantised(shape, q_abs, T, wl.q_first_tok, qc, qr, sc, sr, cb, rb,
                                     wl.k_first_tok, wl.n_keys, wl.softmax_scale, o, lse, ws,
                                     nws)

        for _ in range(warmup):
            call()
        ms, _ = time_steps(torch, call, steps, flush)
        t = statistics.mean(ms)
        tok = quant_token_bytes(wl, cb, rb)
        moved = wl.batch * wl.n_keys * tok + q_abs.numel() * 2 + o.numel() * 2 + lse.numel() * 4
        return t, tok, moved

    for cb, rb in ((4, 4), (2, 4)):
        t, tok, moved = run(shape, wl, q_abs, cache, 1, cb, rb)
        out[f"decode_c{cb}r{rb}"] = {
            "workload": wl.name, "ms": t, "bytes": moved, "value": moved / (t * 1e-3) / 1e9,
            "unit": "GB/s", "frac_hbm": moved / (t * 1e-3) / 1e9 / float(peaks["hbm_gbs"]),
            "bytes_per_token": tok, "capacity_vs_bf16": wl.row_width * 2 / tok,
            "tflops": step_flops(wl)["attend"] / (t * 1e-3) / 1e12}
    if chunk_step is not None:
        st = chunk_step
        t, tok, moved = run(st.shape, st.wl, st.q_abs, st.cache, st.wl.n_queries, 4, 4)
        fl = step_flops(st.wl)["attend"]
        out["video_chunk_c4r4"] = {"workload": st.wl.name, "ms": t, "tflops": fl / (t * 1e-3) / 1e12,
                                   "frac": fl / (t * 1e-3) / 1e12 / float(peaks["bf16_tflops"]),
                                   "bytes_per_token": tok}
    out["note"] = ("mla_attend_quantised: two warps per CTA dequantise each block's packed rows "
                   "into the K/V stage; decode reads the packed ring once")
    return out


def fold_leg(torch, mla, steps, warmup, flush, chunk_step=None):
    """Whether to fold W_UV into the output projection ("Multi-Head Latent Attention" concept
    page, "Low-rank joint compression": the same trick folds W^UV into the output
    projection).  The pages give no output projection; W_O is taken as [n_h d_h, d] with the
    hidden width d = 4096.  Two forms of y = concat_h(W_UV[h] o_lat[h]) W_O, both timed with
    the L2 flushed: mla_up_v and then the W_O GEMM, against one GEMM with the folded weight
    [n_h d_c, d] (W_UV[h]^T W_O[h] stacked over heads).  Both W_O GEMMs are cuBLAS calls
    (torch.matmul), as a measurement: the projection is not part of the path."""
    res = {}
    d = 4096
    dev = "cuda"
    cases = []
    wl = C.DECODE
    shape = mla.make_shape(wl)
    g = torch.Generator(device=dev).manual_seed(0)
    o_lat = (torch.randn((wl.batch, 1, wl.n_heads, wl.d_latent), device=dev, generator=g)
             .to(torch.bfloat16))
    w_uv = (torch.randn((wl.n_heads, wl.d_nope, wl.d_latent), device=dev, generator=g)
            / wl.d_latent ** 0.5).to(torch.bfloat16)
    cases.append(("decode", wl, shape, o_lat, w_uv, 1))
    if chunk_step is not None:
        st = chunk_step
        cases.append(("video_chunk", st.wl, st.shape, st.o_lat, st.w["w_uv"], st.wl.n_queries))
    for name, wl, shape, o_lat, w_uv, T in cases:
        H, dh, dc = wl.n_heads, wl.d_nope, wl.d_latent
        w_o = (torch.randn((H * dh, d), device=dev, generator=g) / (H * dh) ** 0.5).to(torch.bfloat16)
        # folded weight: rows h*dc .. h*dc+dc-1 = W_UV[h]^T W_O[h*dh : (h+1)*dh]
        w_fold = torch.einsum("hkc,hkd->hcd", w_uv.float(), w_o.view(H, dh, d).float()) \
            .reshape(H * dc, d).to(torch.bfloat16)
        out = torch.empty((wl.batch, T, H, dh), dtype=torch.bfloat16, device=dev)
        rows = wl.batch * T

        def two_step(_a=None):
            mla.mla_up_v(shape, o_lat, T, w_uv, out)
            return out.view(rows, H * dh) @ w_o

        def folded(_a=None):
            return o_lat.view(rows, H * dc) @ w_fold

        y2, y1 = two_step(), folded()
        torch.cuda.synchronize()
        rel = float((y1.float() - y2.float()).norm() / y2.float().norm())
        for _ in range(warmup):
            two_step()
            folded()
        ms2, _ = time_steps(torch, two_step, steps, flush)
        ms1, _ = time_steps(torch, folded, steps, flush)
        res[name] = {"rows": rows, "two_step_ms": statistics.mean(ms2),
                     "folded_ms": statistics.mean(ms1),
                     "folded_over_two_step": statistics.mean(ms1) / statistics.mean(ms2),
                     "weight_bytes_two_step": int((w_uv.numel() + w_o.numel()) * 2),
                     "weight_bytes_folded": int(w_fold.numel() * 2),
                     "flops_two_step": 2 * rows * H * dc * dh + 2 * rows * H * dh * d,
                     "flops_folded": 2 * rows * H * dc * d,
                     "rel_diff": rel}
        del w_fold, w_o
    res["note"] = ("W_O [n_h d_h, 4096] assumed (the pages give none); both W_O GEMMs are "
                   "cuBLAS; the folded weight is d_c / d_h = 4x the size of W_O")
    return res


_CPU_STATE = {}


def _cpu_state(wl):
    """Weights, the window's rows from the oracle's own cache write, and the chunk's inputs
    (built once per workload, not timed)."""
    if wl.name not in _CPU_STATE:
        import oracle.mla_oracle as O
        w = {k: v.values for k, v in G.weights(wl, 0).items()}
        F = wl.tokens_per_frame
        cache = np.zeros((wl.batch, wl.ring_slots, wl.row_width))
        for f in range(wl.first_chunk_frame):
            h = G.hidden_frame(wl, 0, f).values
            cache, _ = O.cache_write(cache, h, w["w_dkv"], w["w_kr"], f * F, wl)
        q = G.queries(wl, 0)
        _CPU_STATE[wl.name] = (w, cache, G.hidden_frame(wl, 0, wl.first_chunk_frame).values,
                               q["q_nope"].values, q["q_rope"].values)
    return _CPU_STATE[wl.name]


def cpu_baseline(seconds: float = 12.0, wl=WORKLOAD):
    """The fp64 oracle, as it stands, on a bounded sample of the same step: the cache
    write, absorption, absorbed attention and up-projection of a prefix of the chunk's
    queries (all heads), repeated until ``seconds`` elapse."""
    import oracle.mla_oracle as O
    w, rng_cache, hq, qn, qr = _cpu_state(wl)
    n_q = 0
    flops = 0
    t0 = time.perf_counter()
    chunk = 8
    while time.perf_counter() - t0 < seconds and n_q < wl.n_queries:
        sl = slice(n_q, n_q + chunk)
        n = min(chunk, wl.n_queries - n_q)
        c2, _ = O.cache_write(rng_cache, hq[:, sl], w["w_dkv"], w["w_kr"], wl.q_first_tok + n_q, wl)
        qa = O.absorb_q(qn[:, sl], qr[:, sl], w["w_uk"], wl.q_first_tok + n_q, wl)
        lat, _ = O.attend_latent(qa, c2, wl.q_first_tok + n_q, wl.k_first_tok, wl.n_keys,
                                 wl.softmax_scale, wl)
        O.up_v(lat, w["w_uv"])
        n_q += n
        per_q = step_flops(wl)
        flops += n * sum(per_q.values()) / wl.n_queries
    dt = time.perf_counter() - t0
    try:
        import threadpoolctl
        info = threadpoolctl.threadpool_info()
        threads = max([i.get("num_threads", 1) for i in info] or [1])
    except Exception:  # noqa: BLE001
        threads = os.cpu_count()
    cpu_model = None
    try:
        with open("/proc/cpuinfo") as f:
            cpu_model = next((ln.split(":", 1)[1].strip() for ln in f if ln.startswith("model name")),
                             None)
    except OSError:
        pass
    return {"value": flops / dt / 1e12, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
            "cpu_model": cpu_model, "cpu_count": os.cpu_count(),
            "sample": f"first {n_q} of {wl.n_queries} chunk queries"
                      + (f" of each of {wl.batch} sequences" if wl.batch > 1 else "")
                      + f" (all {wl.n_heads} heads, {wl.n_keys} keys): cache write, absorption, "
                      f"latent attention, up-projection in fp64 NumPy; {dt:.1f} s",
            "seconds": dt}


# DRAM bytes (read + write) of one chunk mla_attend call, from one ncu capture of the
# attention kernel and one of its split-key merge.  Counters describe the kernel sources they
# were taken on (the two kernels and the headers they compile in): the value is reported
# only while those sources are unchanged.
ATTEND_TRAFFIC = {"workload": "video_chunk_bf16",
                  "bytes": (72_825_088 + 19_140_096) + (19_032_832 + 0),
                  "sources": {
                      "latent_kv_cache_write_b200/csrc/tc_attend.cu":
                          "d0c241022ed547e0bf770fb1ef23c7614fb7d20773ece53013be06c69422d3f6",
                      "latent_kv_cache_write_b200/csrc/attend_combine.cu":
                          "5e8fc3df4ef69be02af18fb893f2e454375ade78f18b76088e53fda914d78820",
                      "latent_kv_cache_write_b200/csrc/attend_common.cuh":
                          "d3ebc13662019fed51c1286a818a6dfbd805793934bf6b3a535157d562f02017",
                      "latent_kv_cache_write_b200/csrc/tc_ptx.cuh":
                          "c4c4bb68b95a3de94a535528d9ca5cbdbd8ccbcda5f068c8974e20d715cafac1"}}


def attend_traffic(wl=WORKLOAD):
    import hashlib
    if wl.name != ATTEND_TRAFFIC["workload"]:
        return None
    root = os.path.dirname(os.path.abspath(__file__))
    for rel, want in ATTEND_TRAFFIC["sources"].items():
        try:
            with open(os.path.join(root, rel), "rb") as f:
                if hashlib.sha256(f.read()).hexdigest() != want:
                    return None
        except OSError:
            return None
    return ATTEND_TRAFFIC["bytes"]


def ranks_max(value: float, dist, device) -> float:
    """The slowest rank's value (timings are max over ranks); the value itself when
    there is no process group."""
    if dist is None or not dist.is_initialized() or dist.get_world_size() == 1:
        return value
    import torch
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(world: int, units_per_step: float, steps: int, t_max_ms: float) -> float:
    """Whole-job rate: the units all ranks processed over the slowest rank's time."""
    return world * units_per_step * steps / (t_max_ms * 1e-3)


def run_ours(args):
    import torch
    import torch.distributed as dist
    import latent_kv_cache_write_b200 as mla
    from latent_kv_cache_write_b200 import build

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.gpus > 1 or world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    torch.cuda.set_device(local)
    if rank == 0:
        build.build()
    if world > 1:
        dist.barrier()
    wl = C.BY_NAME[args.workload]
    step = Step(wl, seed=rank, torch=torch, mla=mla)
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device="cuda")
    for _ in range(args.warmup):
        step.run()
    torch.cuda.synchronize()
    assert mla.mla_device_error() == 0
    n0 = mla.mla_kernel_launches()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(local) as clocks:
        ms, parts = time_steps_and_calls(torch, step, args.steps, flush)
    torch.cuda.synchronize()
    launches = (mla.mla_kernel_launches() - n0) // 2      # the timed steps' half
    if world > 1:
        dist.barrier()
    t_max = ranks_max(sum(ms), dist if world > 1 else None, "cuda")
    # end to end through host buffers (copies overlapped with compute across steps)
    step.run_e2e(max(2, args.warmup))
    e2e_total = ranks_max(step.run_e2e(args.steps), dist if world > 1 else None, "cuda")
    fl = step_flops(wl)
    flops_step = sum(fl.values())
    ms_step = t_max / args.steps
    value = job_throughput(world, flops_step, args.steps, t_max) / 1e12
    peaks, peak_src = load_peaks()
    kernels_ms = {k: statistics.mean(v) for k, v in zip(Step.STAGES, parts)}
    attend_ms_all = dict(zip(Step.STAGES, parts))["attend"]
    att_ms = kernels_ms["attend"]
    achieved = fl["attend"] / (att_ms * 1e-3) / 1e12
    peak = float(peaks["bf16_tflops"])
    legs = set(LEGS) if args.legs == "all" else \
        set() if args.legs == "none" else set(args.legs.split(","))
    unknown = legs - set(LEGS)
    if unknown:
        raise SystemExit(f"unknown legs: {sorted(unknown)}")
    leg = lambda name: rank == 0 and name in legs
    dec = decode_leg(torch, mla, max(3, args.steps), args.warmup, flush) if leg("decode") else None
    if dec:
        # small-batch decode: one sequence, its keys split over every cluster
        one = decode_leg(torch, mla, max(3, args.steps), args.warmup, flush,
                         C.DECODE.scaled(name="decode_one_sequence", batch=1))
        dec["one_sequence"] = {"ms": one["ms"], "value": one["value"], "unit": "GB/s",
                               "bytes": one["bytes"]}
    mat = materialised_leg(torch, mla, step, max(3, args.steps), args.warmup, flush,
                           kernels_ms["absorb_q"] + kernels_ms["attend"] + kernels_ms["up_v"]) \
        if leg("materialised") else None
    if mat:
        mat["frac"] = mat["tflops"] / float(peaks["bf16_tflops"])
    shift = shift_leg(torch, mla, step, max(3, args.steps), args.warmup, flush) \
        if leg("shift") else None
    quant = quant_leg(torch, mla, step, max(3, args.steps), args.warmup, flush) \
        if leg("quant") else None
    if dec:
        dec["peak_gbs"] = float(peaks["hbm_gbs"])
        dec["frac"] = dec["value"] / dec["peak_gbs"]
    fold = fold_leg(torch, mla, max(3, args.steps), args.warmup, flush, step) \
        if leg("fold") else None
    qatt = quant_attend_leg(torch, mla, max(3, args.steps), args.warmup, flush, peaks, step) \
        if leg("quant_attend") else None
    # the long-window and wide-positional-key steps, in the same run
    others = {n: workload_leg(torch, mla, n, max(3, min(args.steps, 10)), args.warmup, flush,
                              peaks, local)
              for n in ("long_window_bf16", "wide_key_bf16") if n != wl.name} \
        if leg("workloads") else None
    if rank == 0:
        line = {
            "metric": "absorbed MLA attention TFLOP/s (chunk) and latent-cache GB/s (decode) "
                      "vs B200 peak",
            "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": step_config(wl, world),
            "roofline": {"kernel": "mla_attend", "bound": "tensor", "achieved": achieved,
                         "peak": peak, "unit": "TFLOP/s", "frac": achieved / peak,
                         "peak_source": f"{peak_src} bf16_tflops (burst)",
                         "traffic": attend_traffic(wl), "traffic_unit": "B per launch (ncu)",
                         "ms_per_launch": att_ms,
                         "materialised_flops": materialised_flops(wl),
                         "materialised_note": "the non-absorbed alternative's flops for the "
                                              "same attention, for context; not what runs"},
            "ms_percentiles": {"step_p10_p50_p90": percentiles(ms),
                               "attend_p10_p50_p90": percentiles(attend_ms_all)},
            "kernel_rooflines": kernel_rooflines(wl, kernels_ms, peaks),
            "e2e": {"value": job_throughput(world, flops_step, args.steps, e2e_total) / 1e12,
                    "pipelining": "upload and download streams overlap step i+1's inputs and "
                                  "step i-1's output with step i's compute; no L2 flush (a "
                                  "step moves more bytes through HBM than L2 holds)",
                    "unit": "TFLOP/s",
                    "h2d_bytes_per_step": int(sum(v.nbytes for v in step.host.values())),
                    "d2h_bytes_per_step": int(step.out.numel() * 2),
                    "ms_per_step": e2e_total / args.steps},
            "gpu_launches": int(launches),
            "decode": dec,
            "materialised": mat,
            "k_rope_shift": shift,
            "quant_ring": quant,
            "quant_attend": qatt,
            "fold_w_uv_into_w_o": fold,
            "workloads": others,
            "clocks": clocks.summary(),
            "kernels_ms": kernels_ms,
        }
        if not args.no_cpu_baseline:
            line["cpu_baseline"] = cpu_baseline(wl=wl)
            # the same oracle on one thread (BLAS limited to one), a shorter sample
            try:
                from threadpoolctl import threadpool_limits
                with threadpool_limits(limits=1):
                    one = cpu_baseline(seconds=4.0, wl=wl)
                line["cpu_baseline"]["single_thread"] = {"value": one["value"],
                                                         "sample": one["sample"]}
            except ImportError:
                pass
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def run_reference(args):
    """The reference arm: the fp64 oracle on the host cores, on a bounded sample of
    the same workload per step."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    # each step's sample is sized so that the whole run stays near two minutes
    per_step_s = max(0.1, min(4.0, 120.0 / max(1, args.steps)))
    wl = C.BY_NAME[args.workload]
    for _ in range(args.warmup):
        cpu_baseline(seconds=0.5, wl=wl)
    vals, secs = [], 0.0
    last = None
    for _ in range(args.steps):
        last = cpu_baseline(seconds=per_step_s, wl=wl)
        vals.append(last["value"])
        secs += last["seconds"]
    v = statistics.mean(vals)
    line = {
        "impl": "reference",
        "metric": "absorbed MLA attention TFLOP/s (chunk) and latent-cache GB/s (decode) "
                  "vs B200 peak",
        "value": v, "unit": "TFLOP/s", "n_gpus": int(os.environ.get("WORLD_SIZE", "1")),
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * secs / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": step_config(wl, int(os.environ.get("WORLD_SIZE", "1"))),
        "cpu_baseline": {"value": v, "unit": "TFLOP/s", "kind": "oracle",
                         "cores": last["cores"], "sample": last["sample"]},
        "e2e": {"value": v, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--workload", default=WORKLOAD.name, choices=STEP_WORKLOADS,
                    help="the step's workload (default: the video chunk)")
    ap.add_argument("--legs", default="all",
                    help="comma-separated extra legs to run after the step (default all: "
                         + ",".join(LEGS) + "; or none); fewer legs make a shorter run to "
                         "profile")
    args = ap.parse_args()
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
