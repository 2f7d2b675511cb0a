"""The C ABI from plain C: tests/c/abi_host.c includes only include/dllm_qgemm.h,
compiles as C99 with warnings as errors, links only the library, and calls the entry
points that need no device.  This checks that the header is valid C (no C++ in the
declarations) and that the symbols resolve at link time, not only through ctypes."""
import shutil
import subprocess
from pathlib import Path

import pytest

from quantized_int8_gemm_q4_b200 import build as nbuild

ROOT = Path(__file__).resolve().parent.parent
SRC = ROOT / "tests" / "c" / "abi_host.c"


@pytest.fixture(scope="module")
def results(tmp_path_factory):
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("gcc not available")
    lib = nbuild.build()
    exe = tmp_path_factory.mktemp("cabi") / "abi_host"
    cmd = [gcc, "-std=c99", "-Wall", "-Wextra", "-Werror", "-pedantic", "-I", str(ROOT / "include"), str(SRC),
           "-o", str(exe), "-L", str(lib.parent), "-ldllm_qgemm", f"-Wl,-rpath,{lib.parent}"]
    subprocess.run(cmd, check=True)
    out = subprocess.run([str(exe)], check=True, capture_output=True, text=True).stdout
    return {k: int(v) for k, v in (line.split() for line in out.splitlines())}


def test_sizes(results):
    assert results["repacked_q4k_rc"] == 0 and results["repacked_q4k_bytes"] == 4096 * 16 * 144
    assert results["repacked_q6k_rc"] == 0 and results["repacked_q6k_bytes"] == 4096 * 48 * 210
    assert results["act_rc"] == 0
    assert results["act_q"] == 160 * 4096 and results["act_scale"] == 160 * 16 * 4
    assert results["act_sums"] == 160 * 16 * 64


def test_rejections(results):
    assert results["act_bad_k"] == -1 and results["repacked_bad_n"] == -1
    assert results["quantize_null"] == -1 and results["rmsnorm_eps0"] == -1
    assert results["plan_bad"] == -1
    assert results["status_row_range_nonempty"] == 1


def test_plan_from_c(results):
    assert results["plan_rc"] == 0
    assert (results["plan_kc"], results["plan_full_tiles"], results["plan_tail_k"], results["plan_tail_big"]) == \
        (1, 148, 3, 16)


def test_attention_rejections(results):
    assert results["attn_dh64"] == -1 and results["attn_group"] == -1 and results["attn_no_keys"] == -1
    assert results["attn_null"] == -1 and results["attn_align"] == -2
    assert results["attn_empty"] == 0  # no queries: nothing to do, nothing launched
