"""The attention kernel's compile-time timeline (diagnostic build).

The library built with TTCD_ATTN_TIMELINE=1 records clock64 marks at the
softmax phase boundaries of every visit of one CTA; the timeline tool reads
them.  This checks that the instrumented build runs, that the marks of each
visit are in order and that the tool prints its summary.  The kernel's
arithmetic is the same as the library's (the marks only read the clock).
"""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def timeline_lib(tmp_path_factory):
    """A fresh instrumented build of the current sources (never a stale copy)."""
    from dual_window_attention_b200 import build
    return build.build(attn_timeline=True,
                       out=str(tmp_path_factory.mktemp("timeline") / "libttcd_timeline.so"))


def test_timeline_marks_are_ordered(timeline_lib):
    code = r"""
import sys, torch, dual_window_attention_b200 as m
m.load_library(sys.argv[1])
T = 4096
g = torch.Generator(device="cuda").manual_seed(0)
q = torch.randn(1, T, 16, 128, device="cuda", generator=g).to(torch.bfloat16)
k = torch.randn(1, T, 8, 128, device="cuda", generator=g).to(torch.bfloat16)
v = torch.randn(1, T, 8, 128, device="cuda", generator=g).to(torch.bfloat16)
m.dual_window_attn(q, k, v, 512, 2048)
torch.cuda.synchronize()
tl = m.attn_timeline_read()
# the longest query tile (31) visits key tiles 0-4 for the student window
# and 4-16 for the teacher-only band: 5 + 13 visits
nv = int((tl[0, :, 0] != 0).sum())
assert nv == 18, nv
for h in range(2):
    for vv in range(nv):
        r = tl[h, vv].tolist()
        assert 0 < r[0] <= r[1] <= r[2] <= r[3] <= r[4], (h, vv, r)
        assert r[5] > 0 and r[6] >= r[5], (h, vv, r)
    assert all(tl[h, vv, 0] < tl[h, vv + 1, 0] for vv in range(nv - 1))
assert m.attn_timeline_read().abs().sum() == 0  # cleared by the read
print("ok")
"""
    r = subprocess.run([sys.executable, "-c", code, timeline_lib], cwd=ROOT, capture_output=True,
                       text=True, timeout=600)
    assert r.returncode == 0 and r.stdout.strip().endswith("ok"), r.stdout + r.stderr


def test_timeline_tool_prints_the_phases(timeline_lib):
    r = subprocess.run([sys.executable, "-m", "dual_window_attention_b200.timeline", "--T", "8192",
                        "--lib", timeline_lib], cwd=ROOT, capture_output=True, text=True,
                       timeout=600)
    assert r.returncode == 0, r.stdout + r.stderr
    assert "visit period" in r.stdout and "head 1" in r.stdout, r.stdout
