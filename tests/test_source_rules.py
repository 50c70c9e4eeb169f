"""Rules the CUDA sources keep, checked on the text (CPU only).

- Every kernel launched with launch_dependent (programmatic dependent launch) calls
  grid_dep_wait, and that call comes before the kernel's role branches, where the
  first global accesses are.  A dependent launch without the wait could read a buffer
  before the previous kernel has written it.
- No such kernel is also launched with the plain <<<...>>> syntax.
- No TMA or bulk load uses cluster multicast: the library's kernels may be given memory of
  another GPU, and multicast loads of such memory are not used here."""

import glob
import os
import re

CSRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                    "latent_kv_cache_write_b200", "csrc")


# TMA operations and the global buffers the dependent kernels take in their arguments
ACCESS = ("tma_load_", "tma_store_", "tma_prefetch_", "mapa(", ".ws_o", ".ws_lse", ".q_abs",
          ".o_lat", ".q_rope", ".q_nope", ".out", ".lse", ".slots", ".err")


def _sources():
    out = {}
    for p in sorted(glob.glob(os.path.join(CSRC, "*.cu")) + glob.glob(os.path.join(CSRC, "*.cuh"))
                    + glob.glob(os.path.join(CSRC, "*.h"))):
        with open(p) as f:
            out[os.path.basename(p)] = f.read()
    return out


def _kernel_body(src, name):
    """Text of the __global__ function `name`, from its definition to the next one."""
    m = re.search(r"__global__[^;{]*?\b" + name + r"\s*\(", src, re.S)
    if m is None:
        return None
    nxt = src.find("__global__", m.end())
    return src[m.start(): nxt if nxt >= 0 else len(src)]


def test_dependent_launches_wait_before_touching_memory():
    srcs = _sources()
    launched = set()
    for text in srcs.values():
        launched |= set(re.findall(r"launch_dependent\(\s*(\w+)", text))
    launched.discard("void")                         # the helper's own definition
    assert {"tc_gemm_kernel", "attend_kernel", "combine_kernel", "attend_mat_kernel"} <= launched
    for name in launched:
        bodies = [b for b in (_kernel_body(t, name) for t in srcs.values()) if b]
        assert len(bodies) == 1, name
        body = bodies[0]
        assert "grid_dep_wait()" in body, f"{name} is launched dependent but never waits"
        # the wait precedes the first TMA operation and the first use of a global buffer
        # argument
        code = re.sub(r"//[^\n]*", "", body)
        access = [code.find(tok) for tok in ACCESS if code.find(tok) >= 0]
        assert access and code.find("grid_dep_wait()") < min(access), name
        for text in srcs.values():
            assert not re.search(r"\b" + name + r"\s*(<[^>]*>)?\s*<<<", text), \
                f"{name} also has a plain launch"


def test_no_multicast_loads():
    for fname, text in _sources().items():
        for line in text.splitlines():
            if "cp.async.bulk" in line and "multicast::cluster" in line:
                raise AssertionError(f"{fname}: multicast bulk load: {line.strip()}")
