"""Per-visit timeline of the fused dual-window attention kernel (diagnostic).

    python -m dual_window_attention_b200.build --attn-timeline
    python -m dual_window_attention_b200.timeline [--T 16384] [--windows 512/8192]

Runs ttcd_dual_window_attn once on seeded bf16 inputs with the Qwen3-0.6B head
layout (16 query heads, 8 KV heads, head dim 128) through libttcd_timeline.so,
the library built with the kernel's clock64 marks compiled in, and prints for
the CTA of the longest query tile (two query heads of one KV group):

  - the median cycles between consecutive marks of a visit, per head:
    S ready -> S in registers -> row maximum -> rescale check -> P published;
  - the median visit period (S ready of visit v to S ready of visit v + 1);
  - the median gap from P published to the issue of the next QK product.

Visits 2 .. n-3 are the steady state; the first and last are excluded.  The
marks are read in a separate library so the normal build carries none of them.
"""
from __future__ import annotations

import argparse
import os
import sys

import torch

MARKS = ["S ready", "S in registers", "row maximum", "rescale check", "P published",
         "PV issued", "next QK issued"]


def _median(xs):
    xs = sorted(xs)
    return xs[len(xs) // 2] if xs else float("nan")


def summarise(tl: torch.Tensor, visits: int) -> dict:
    """Per-head medians from the [2, 128, 8] mark tensor."""
    out = {}
    for h in range(2):
        rows = [tl[h, v].tolist() for v in range(2, max(2, visits - 2))]
        rows = [r for r in rows if r[0] and r[4]]
        if not rows:
            continue
        phases = {f"{MARKS[k]} -> {MARKS[k + 1]}": _median([r[k + 1] - r[k] for r in rows])
                  for k in range(4)}
        period = _median([tl[h, v + 1, 0].item() - tl[h, v, 0].item()
                          for v in range(2, max(2, visits - 3)) if tl[h, v + 1, 0] and tl[h, v, 0]])
        to_qk = _median([r[6] - r[4] for r in rows if r[6]])
        out[f"head {h}"] = {"phases": phases, "softmax": _median([r[4] - r[0] for r in rows]),
                            "visit period": period, "P published -> next QK issued": to_qk,
                            "visits": len(rows)}
    return out


def main(argv=None) -> int:
    ap = argparse.ArgumentParser(description=__doc__.split("\n\n")[0])
    ap.add_argument("--T", type=int, default=16384)
    ap.add_argument("--windows", default="512/8192", help="w_S/w_T")
    ap.add_argument("--lib", default=None, help="the instrumented library (default: the package's)")
    args = ap.parse_args(argv)
    import dual_window_attention_b200 as m
    from dual_window_attention_b200 import build

    lib = args.lib or build.TIMELINE_LIB
    if not os.path.exists(lib):
        raise SystemExit(f"{lib} is missing: run "
                         "`python -m dual_window_attention_b200.build --attn-timeline`")
    m.load_library(lib)
    w_S, w_T = (int(x) for x in args.windows.split("/"))
    g = torch.Generator(device="cuda").manual_seed(0)
    q = torch.randn(1, args.T, 16, 128, device="cuda", generator=g).to(torch.bfloat16)
    k = torch.randn(1, args.T, 8, 128, device="cuda", generator=g).to(torch.bfloat16)
    v = torch.randn(1, args.T, 8, 128, device="cuda", generator=g).to(torch.bfloat16)
    m.dual_window_attn(q, k, v, w_S, w_T)  # warm-up
    torch.cuda.synchronize()
    m.attn_timeline_read()
    m.dual_window_attn(q, k, v, w_S, w_T)
    torch.cuda.synchronize()
    tl = m.attn_timeline_read()
    visits = int((tl[0, :, 0] != 0).sum())
    print(f"T {args.T}, w_S {w_S}, w_T {w_T}: {visits} visits in the CTA of the longest query tile")
    for head, d in summarise(tl, visits).items():
        print(f"{head} ({d['visits']} steady visits; cycles, median)")
        for name, c in d["phases"].items():
            print(f"  {name:40s} {c:8.0f}")
        print(f"  {'softmax (S ready -> P published)':40s} {d['softmax']:8.0f}")
        print(f"  {'visit period':40s} {d['visit period']:8.0f}")
        print(f"  {'P published -> next QK issued':40s} {d['P published -> next QK issued']:8.0f}")
    return 0


if __name__ == "__main__":
    sys.exit(main())
