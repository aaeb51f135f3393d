"""The C ABI from plain C: tests/c_abi_check.c is compiled as C99 with
-Wall -Wextra -Werror -pedantic against include/ttcd.h alone, linked to
libttcd.so and run (host-side calls only, no GPU).  Its results must match the
Python binding's, which reaches the same library through ctypes."""
import os
import shutil
import subprocess

import pytest

import dual_window_attention_b200 as ttcd
from dual_window_attention_b200 import build
from ttcd_workloads import QWEN3_0P6B_64K

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def c_results(tmp_path_factory):
    if shutil.which("gcc") is None:
        pytest.skip("gcc not found")
    lib = build.build()
    libdir = os.path.dirname(lib)
    exe = str(tmp_path_factory.mktemp("cabi") / "c_abi_check")
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-pedantic",
                    "-I", os.path.join(ROOT, "include"), os.path.join(ROOT, "tests", "c_abi_check.c"),
                    "-L", libdir, "-lttcd", f"-Wl,-rpath,{libdir}", "-o", exe], check=True)
    out = subprocess.run([exe], check=True, capture_output=True, text=True).stdout
    return {ln.split(" ", 1)[0]: ln.split(" ", 1)[1] for ln in out.splitlines()}


def test_c_program_agrees_with_the_binding(c_results):
    ttcd.load_library()
    p = ttcd.BlockParams.from_shape(QWEN3_0P6B_64K)
    r = c_results
    assert r["version"].startswith("ttcd")
    assert int(r["block_ws"]) == ttcd.block_forward_workspace_size(p) > 0
    assert int(r["mlp_ws"]) == ttcd.fastweight_mlp_workspace_size(p) > 0
    assert int(r["decode_state"]) > 0 and int(r["decode_ws"]) > 0
    assert int(r["noalloc_capacity"]) == 32 << 20
    status, off = map(int, r["offset_Wall"].split())
    assert status == ttcd.OK and off == ttcd.workspace_offset(p, "Wall")
    assert int(r["offset_unknown"]) == ttcd.ERR_INVALID_ARG
    assert int(r["bad_windows_ws"]) == 0
    status, text = r["null_block"].split(" ", 1)
    assert int(status) == ttcd.ERR_INVALID_ARG and text == ttcd.status_string(ttcd.ERR_INVALID_ARG)
    assert r["status_timeout"] == ttcd.status_string(ttcd.ERR_TIMEOUT)
