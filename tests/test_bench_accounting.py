"""The work accounting bench.py reports beside its timings (CPU only): algorithmic bytes per
call, the non-absorbed alternative's flops, which roofline bound binds, and the step
workloads the --workload option offers."""

import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402
from synth import configs as C  # noqa: E402

PEAKS = {"bf16_tflops": 1647.8, "hbm_gbs": 6537.3}


def test_chunk_bytes_per_call():
    wl = C.VIDEO_CHUNK
    by = bench.step_bytes(wl)
    # h [1560, 4096] + [W_DKV | W_KR] [4096, 576] read, 1560 cache rows of 576 written
    assert by["cache_write"] == (1560 * 4096 + 4096 * 576 + 1560 * 576) * 2
    # q_nope and q_R [1560, 32, 128 + 64] + W_UK [32, 128, 512] read, q_abs [1560, 32, 576] written
    assert by["absorb_q"] == (1560 * 32 * 192 + 32 * 128 * 512 + 1560 * 32 * 576) * 2
    # q_abs and the window's 6240 rows read, o_lat [1560, 32, 512] and the fp32 LSE written
    assert by["attend"] == (1560 * 32 * 576 + 6240 * 576 + 1560 * 32 * 512) * 2 + 1560 * 32 * 4
    assert by["up_v"] == (1560 * 32 * 512 + 32 * 128 * 512 + 1560 * 32 * 128) * 2


def test_materialised_alternative_flops():
    wl = C.VIDEO_CHUNK
    # every chunk query sees all 6240 window keys; K and V materialised once per (key, head)
    mat = 2 * 2 * 6240 * 32 * 512 * 128
    att = 1560 * 6240 * 32 * (2 * (128 + 64) + 2 * 128)
    assert bench.materialised_flops(wl) == mat + att
    assert bench.materialised_flops(wl) == pytest.approx(0.2517e12, rel=1e-3)
    # the absorbed form does more flops than the materialised one at the chunk
    assert bench.step_flops(wl)["attend"] > 2.5 * bench.materialised_flops(wl)


def test_binding_bound_per_call():
    wl = C.VIDEO_CHUNK
    ms = {"cache_write": 0.0273, "absorb_q": 0.0289, "attend": 0.6395, "up_v": 0.0226}
    r = bench.kernel_rooflines(wl, ms, PEAKS)
    # 7.36 GFLOP (4.5 us at peak) against 19.3 MB (3.0 us): the tensor bound binds
    assert r["cache_write"]["bound"] == "tensor"
    # 6.5 GFLOP against ~81 MB and ~68 MB: HBM binds
    assert r["absorb_q"]["bound"] == "hbm"
    assert r["up_v"]["bound"] == "hbm"
    assert r["attend"]["bound"] == "tensor"
    for k, v in r.items():
        assert v["frac_of_bound"] == pytest.approx(max(v["frac_tensor"], v["frac_hbm"]))
    # 677.8 GFLOP in 0.6395 ms
    assert r["attend"]["tflops"] == pytest.approx(677.8 / 0.6395, rel=1e-3)


def test_percentiles_nearest_rank():
    assert bench.percentiles([5.0]) == [5.0, 5.0, 5.0]
    assert bench.percentiles(list(range(1, 12))) == [2, 6, 10]


def test_step_workloads():
    assert bench.STEP_WORKLOADS == ("video_chunk_bf16", "long_window_bf16", "wide_key_bf16")
    assert bench.WORKLOAD.name == "video_chunk_bf16"


def test_quant_ring_bytes():
    wl = C.VIDEO_CHUNK
    # INT4 content (256 B) and RoPE (32 B) plus two float32 scales, against 1152 B in bf16
    assert bench.quant_token_bytes(wl, 4, 4) == 296
    assert bench.quant_token_bytes(wl, 2, 4) == 168
    assert bench.quant_token_bytes(C.WIDE_KEY, 4, 4) == 256 + 256 + 8


def test_both_arms_report_one_config():
    wl = C.VIDEO_CHUNK
    cfg = bench.step_config(wl, 2)
    assert cfg["workload"] == wl.name and cfg["keys"] == 6240 and cfg["queries"] == 1560
    assert cfg["flops_per_step"] == sum(bench.step_flops(wl).values())
    assert cfg["parallelism"] == "replicas x2 (independent sequences)"


class _FakeEvent:
    """A CUDA event stand-in whose record() takes the next tick of a shared clock."""
    clock = [0.0]

    def __init__(self, enable_timing=False):
        self.t = None

    def record(self):
        _FakeEvent.clock[0] += 1.0
        self.t = _FakeEvent.clock[0]

    def elapsed_time(self, other):
        return other.t - self.t


class _FakeTorch:
    class cuda:
        Event = _FakeEvent

        @staticmethod
        def synchronize():
            pass


class _FakeStep:
    """Records which steps carried events between their calls."""
    def __init__(self):
        self.calls = []

    def run(self, ev=None):
        self.calls.append(ev is not None)
        if ev is not None:
            for e in ev:
                e.record()


class _FakeFlush:
    def zero_(self):
        pass


def test_timed_steps_carry_no_events_between_calls():
    """The rate comes from steps with no event between their calls (an event there would
    keep a kernel from starting while the previous one finishes); the per-call breakdown
    comes from as many steps interleaved with them."""
    step = _FakeStep()
    ms, parts = bench.time_steps_and_calls(_FakeTorch, step, 5, _FakeFlush())
    assert step.calls == [False, True] * 5
    assert len(ms) == 5 and all(m == 1.0 for m in ms)     # e0 then e1 around a bare step
    assert len(parts) == len(bench.Step.STAGES) == 4
    assert all(len(p) == 5 and all(x == 1.0 for x in p) for p in parts)
