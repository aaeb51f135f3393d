"""Build libttcd.so in-tree for sm_100a with nvcc (no GPU needed to build).

    python -m dual_window_attention_b200.build [--verbose-ptxas]
    python -m dual_window_attention_b200.build --attn-timeline

The second form builds libttcd_timeline.so, the same library with the attention
kernel's clock64 timeline compiled in (TTCD_ATTN_TIMELINE=1), for
`python -m dual_window_attention_b200.timeline`.
"""
from __future__ import annotations

import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
LIB = os.path.join(PKG, "libttcd.so")
TIMELINE_LIB = os.path.join(PKG, "libttcd_timeline.so")
SOURCES = [os.path.join(CSRC, "ttcd.cu")]
DEPS = SOURCES + [os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith(".cuh")] + [
    os.path.join(ROOT, "include", "ttcd.h")]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", shutil.which("nvcc")):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def needs_build() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    return any(os.path.getmtime(p) > t for p in DEPS)


def build(force: bool = False, ptxas_verbose: bool = False, attn_timeline: bool = False,
          out: str = None) -> str:
    """Builds the library (or, attn_timeline, the instrumented one) at `out`
    (default: in the package) and returns its path."""
    if out is None:
        out = TIMELINE_LIB if attn_timeline else LIB
    if not force and not attn_timeline and out == LIB and not needs_build():
        return LIB
    cmd = [nvcc(), "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo",
           "-std=c++17", "--expt-relaxed-constexpr", "-Xcompiler", "-fPIC,-O2", "-shared",
           "-I" + os.path.join(ROOT, "include"), "-o", out + ".tmp", *SOURCES]
    if attn_timeline:
        cmd.insert(1, "-DTTCD_ATTN_TIMELINE=1")
    if ptxas_verbose:
        cmd.insert(1, "-Xptxas=-v")
    subprocess.run(cmd, check=True)
    os.replace(out + ".tmp", out)
    return out


if __name__ == "__main__":
    print(build(force=True, ptxas_verbose="--verbose-ptxas" in sys.argv,
                attn_timeline="--attn-timeline" in sys.argv))
