"""The C ABI from a plain C11 program (gcc, no C++ and no Python in between): the header
compiles as C, the library links, and host-side validation answers as documented.  Runs
without a GPU."""

import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
LIB_DIR = os.path.join(ROOT, "latent_kv_cache_write_b200")


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
def test_plain_c_host(tmp_path):
    from latent_kv_cache_write_b200 import build
    build.build()                       # incremental: a no-op when libmla.so is current
    exe = tmp_path / "validate"
    subprocess.run(["gcc", "-std=c11", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"),
                    os.path.join(ROOT, "tests", "c_host", "validate.c"), "-o", str(exe),
                    "-L" + LIB_DIR, "-lmla", "-Wl,-rpath," + LIB_DIR],
                   check=True, capture_output=True, text=True)
    out = subprocess.run([str(exe)], check=True, capture_output=True, text=True,
                         timeout=120).stdout.split("\n")
    assert out[:11] == [
        "status MLA_ERR_RANGE",
        f"materialised_ws {2 * 6240 * 32 * 128 * 2}",
        "attend_range MLA_ERR_RANGE",
        "shape_arg MLA_ERR_ARG",
        "empty_up_v MLA_OK",
        "empty_shift MLA_OK",
        "quant_bits MLA_ERR_ARG",
        "empty_dequant MLA_OK",
        "fixed_range MLA_ERR_RANGE",
        "fixed_align MLA_ERR_ALIGN",
        "fixed_empty MLA_OK",
    ]
