#!/usr/bin/env python
"""Benchmark of the IP-TTCD block forward (prefill) on B200.

One step = one ttcd_block_forward over one batch of the Qwen3-0.6B-shaped
block at T = 65536 (d 1024, 16/8 heads, hd 128, d_ff 3072, w_S 512, w_T 8192,
C 1024, conv width 4), with synthetic seeded inputs already resident in HBM.
Prints one JSON line (rank 0).  Multi-GPU runs are independent replicas
(weak scaling, no collective on the data path); launch with torchrun.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

from ttcd_workloads import (ATTN_SWEEP_W_S, ATTN_SWEEP_W_T, QWEN3_0P6B_64K,  # noqa: E402
                            make_block_inputs)

METRIC = "IP-TTCD block prefill tokens/s @64K (Qwen3-0.6B shape); dual-attn % BF16 peak"
UNIT = "tokens/s"
STAGES = ["rope+rms_rowscale_in", "qkv_gemm_rope", "dual_window_attn", "o_proj_residual_rmsstats",
          "gate_up_swiglu_conv_keys", "key_scales", "M_wdown_wproj", "R_gemm",
          "chunk_scan_dW", "out_gemm"]
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return FALLBACK_PEAKS, "fallback"


TRAFFIC_JSON = os.path.join(ROOT, "profiles", "ncu_traffic.json")
CSRC = os.path.join(ROOT, "dual_window_attention_b200", "csrc")


def sources_digest(names) -> str:
    """sha256 (16 hex digits) over the named kernel sources, in order."""
    h = hashlib.sha256()
    for n in names:
        with open(os.path.join(CSRC, n), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def recorded_traffic(kernel: str, T: int):
    """DRAM bytes (read + write) per launch of `kernel` at T tokens, from the ncu
    capture recorded in profiles/ncu_traffic.json (scaled by T when the capture
    ran at another length).  None when there is no record, or once the kernel's
    sources differ from the ones that were profiled."""
    try:
        with open(TRAFFIC_JSON) as f:
            rec = json.load(f)[kernel]
        if sources_digest(rec["sources"]) != rec["sources_sha256_16"]:
            return None
        return float(rec["bytes_per_launch"]) * T / int(rec["T"])
    except (OSError, KeyError, ValueError):
        return None


def record_traffic(csv_path: str, kernel: str, T: int, sources, workload: str, command: str,
                   algorithmic: float, note: str = "") -> dict:
    """Writes the DRAM bytes of one ncu capture (a --csv log of
    gpu__time_duration.sum, dram__bytes_read.sum and dram__bytes_write.sum for
    one launch) into profiles/ncu_traffic.json under `kernel`, with the digest of
    the kernel's sources at the time of the capture."""
    import csv
    vals = {}
    with open(csv_path) as f:
        lines = [l for l in f if l.startswith('"')]
    for row in csv.DictReader(lines):
        vals[row["Metric Name"]] = float(row["Metric Value"].replace(",", ""))
    rec = {"workload": workload, "T": T,
           "dram_bytes_read": int(vals["dram__bytes_read.sum"]),
           "dram_bytes_write": int(vals["dram__bytes_write.sum"]),
           "bytes_per_launch": int(vals["dram__bytes_read.sum"] + vals["dram__bytes_write.sum"]),
           "algorithmic_bytes": int(algorithmic),
           "gpu_time_duration_ns_under_ncu": int(vals.get("gpu__time_duration.sum", 0)),
           "sources": list(sources), "sources_sha256_16": sources_digest(sources),
           "command": command, "note": note}
    try:
        with open(TRAFFIC_JSON) as f:
            table = json.load(f)
    except OSError:
        table = {}
    table[kernel] = rec
    with open(TRAFFIC_JSON, "w") as f:
        json.dump(table, f, indent=1)
        f.write("\n")
    return rec


ATTN_SWEEP_PAIRS = [(wS, wT) for wT in ATTN_SWEEP_W_T for wS in ATTN_SWEEP_W_S]


def attention_bytes(shape) -> float:
    """Compulsory DRAM bytes of one attention launch: q, k, v read once, o_T and
    o_S written once (bf16)."""
    BT, hd = shape.B * shape.T, shape.head_dim
    return 2.0 * BT * hd * ((shape.n_q_heads + 2 * shape.n_kv_heads) + 2 * shape.n_q_heads)


def attention_flops(shape) -> float:
    """4 * hd * Hq FLOPs per (query, key) pair inside the teacher window."""
    T, w = shape.T, shape.w_T
    pairs = w * (w + 1) // 2 + (T - w) * w if T >= w else T * (T + 1) // 2
    return 4.0 * shape.head_dim * shape.n_q_heads * shape.B * pairs


def stage_costs(s):
    """(bound, algorithmic amount) per stage: FLOPs for tensor stages, bytes for HBM ones."""
    BT, d, f, hd = s.B * s.T, s.d_model, s.d_ff, s.head_dim
    Hq, Hkv = s.n_q_heads, s.n_kv_heads
    dqkv = (Hq + 2 * Hkv) * hd
    Cp = (s.chunk + 63) // 64 * 64
    P = s.B * s.n_chunks * Cp
    return [
        # x read for the row scales (+ rstd out), W_qkv read and W_qkv diag(g) written,
        # half2 cos/sin table written
        ("hbm", BT * d * 2 + BT * 4 + 2 * dqkv * d * 2 + s.T * hd // 2 * 4),
        ("tensor", 2.0 * BT * d * dqkv),
        ("tensor", attention_flops(s)),
        ("tensor", 2.0 * 2 * BT * Hq * hd * d),
        # gate/up for both paths; the epilogue also writes D, K' and Z_S (bf16)
        ("tensor", 2.0 * 2 * BT * d * 2 * f),
        # key scales: the per-column-tile partial sums of squares in, one scale out
        ("hbm", (f // 128 + 2) * P * 4 + BT * 4),
        ("tensor", 2.0 * d * f * f),
        ("tensor", 2.0 * d * f * P),
        ("tensor", 2.0 * d * f * P),
        ("tensor", 2.0 * BT * f * d),
    ]


class ClockSampler:
    """Samples SM clock and clock-event reasons with NVML during the timed region."""

    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown"}

    def __init__(self, index: int, period_s: float = 0.01):
        self.samples, self.reasons, self.max_mhz = [], 0, None
        self.period = period_s
        self._stop = threading.Event()
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception:
            self.nv = None

    def _run(self):
        while not self._stop.is_set():
            try:
                self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
                self.reasons |= self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.nv:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *a):
        if self.nv:
            self._stop.set()
            self.t.join()

    def summary(self):
        if not self.nv:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvml unavailable"]}
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "samples": len(self.samples),
                "reasons": [n for b, n in self.REASONS.items() if self.reasons & b]}


def dist_setup(backend=None, timeout_s: float = 300.0):
    """One process per GPU from the torchrun environment.  NCCL when CUDA is
    present (the bench), gloo otherwise (host-side tests of the same code)."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if backend is None:
        backend = "nccl" if torch.cuda.is_available() else "gloo"
    if world > 1:
        import torch.distributed as dist
        if backend == "nccl":
            torch.cuda.set_device(local)
            dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=timeout_s),
                                    device_id=torch.device("cuda", local))
        else:
            dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=timeout_s))
    elif torch.cuda.is_available():
        torch.cuda.set_device(local)
    return world, rank, local


def _nccl() -> bool:
    import torch.distributed as dist
    return dist.get_backend() == "nccl"


def barrier(world, local):
    if world > 1:
        import torch.distributed as dist
        if _nccl():
            dist.barrier(device_ids=[local])
        else:
            dist.barrier()


def max_over_ranks(world, v: float) -> float:
    if world == 1:
        return v
    import torch.distributed as dist
    t = torch.tensor([v], dtype=torch.float64, device="cuda" if _nccl() else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(world, units_per_rank: float, ms_local: float):
    """Replicas: every rank processes its own units.  The job's time per step is
    the slowest rank's; the job's rate counts the units of all ranks."""
    ms = max_over_ranks(world, ms_local)
    return ms, units_per_rank * world / (ms / 1e3)


def oracle_throughput(shape, sample_tokens: int, repeats: int = 1):
    """Time the float64 oracle on the first `sample_tokens` tokens (tokens/s, seconds)."""
    from oracle import ttcd_oracle as orc
    inp = make_block_inputs(shape.with_(T=sample_tokens, n_layers=1), seed=0)
    w = {k: v.double().numpy() for k, v in inp["layers"][0].items()}
    x = inp["x"].double().numpy()
    times = []
    for _ in range(repeats):
        t0 = time.perf_counter()
        orc.block_forward(x, w["beta"], w, n_q_heads=shape.n_q_heads, n_kv_heads=shape.n_kv_heads,
                          head_dim=shape.head_dim, w_S=shape.w_S, w_T=shape.w_T,
                          chunk=shape.chunk, rms_eps=shape.rms_eps, l2_eps=shape.l2_eps,
                          rope_theta=shape.rope_theta)
        times.append(time.perf_counter() - t0)
    return shape.B * sample_tokens / statistics.median(times), times


def cpu_cores() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except Exception:
        return os.cpu_count() or 1


def workload_config(shape, extra=None):
    cfg = {"workload": shape.name, "B": shape.B, "T": shape.T, "d_model": shape.d_model,
           "n_q_heads": shape.n_q_heads, "n_kv_heads": shape.n_kv_heads,
           "head_dim": shape.head_dim, "d_ff": shape.d_ff, "w_S": shape.w_S, "w_T": shape.w_T,
           "chunk": shape.chunk, "conv_k": shape.conv_k,
           "l2": "no flush: one step reads and writes ~10 GB, far above the 126 MB L2"}
    if extra:
        cfg.update(extra)
    return cfg


def run_reference(args, world, rank):
    """Reference arm: the float64 CPU oracle, timed on the host's cores (rank 0 only)."""
    if rank != 0:
        return
    shape = QWEN3_0P6B_64K
    sample = args.ref_sample_tokens
    for _ in range(args.warmup):
        oracle_throughput(shape, sample)
    _, times = oracle_throughput(shape, sample, repeats=args.steps)
    total = sum(times)
    value = shape.B * sample * args.steps / total
    desc = (f"first {sample} tokens of the workload per step (attention windows truncated by "
            f"position), float64 NumPy oracle")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1000 * total / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": workload_config(shape, {"sample_tokens": sample}),
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": cpu_cores(),
                             "kind": "oracle", "sample": desc},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def run_ours(args, world, rank, local):
    import dual_window_attention_b200 as ttcd
    ttcd.load_library()
    shape = QWEN3_0P6B_64K if args.T == QWEN3_0P6B_64K.T else QWEN3_0P6B_64K.with_(
        name=f"qwen3_0.6b_block_T{args.T}", T=args.T)
    peaks, peak_kind = load_peaks()
    dev = torch.device("cuda", local)
    inp = make_block_inputs(shape, seed=0)
    x = inp["x"].to(dev)
    w = {k: v.to(dev) for k, v in inp["layers"][0].items()}
    beta = w["beta"]
    p = ttcd.BlockParams.from_shape(shape)
    ws = ttcd.alloc_workspace(ttcd.block_forward_workspace_size(p), dev)
    out = torch.empty_like(x)
    stream = torch.cuda.current_stream()

    def step(events=None):
        ttcd.block_forward(x, beta, w, p, out=out, workspace=ws, stream=stream, events=events)

    for _ in range(args.warmup):
        step()
    if ttcd.check_device_status(ws, stream) != ttcd.OK:
        raise RuntimeError("a device wait timed out during warm-up")

    # ---- device-timed region: K steps, each call recording its own stage events
    n_ev = len(STAGES) + 1
    events = [[torch.cuda.Event(enable_timing=True) for _ in range(n_ev)]
              for _ in range(args.steps)]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world, local)
    torch.cuda.synchronize()
    launches0 = ttcd.kernel_launch_count()
    with ClockSampler(local) as clk:
        start.record(stream)
        for i in range(args.steps):
            step(events[i])
        end.record(stream)
        torch.cuda.synchronize()
    launches = ttcd.kernel_launch_count() - launches0
    barrier(world, local)
    ms, value = job_throughput(world, shape.B * shape.T, start.elapsed_time(end) / args.steps)
    if ttcd.check_device_status(ws, stream) != ttcd.OK:
        raise RuntimeError("a device wait timed out in the timed region")
    tokens = shape.B * shape.T * world

    # per-stage times (mean over steps) and roofline fractions.  The timed region
    # is well under a second, so tensor stages are held to the burst GEMM peak.
    costs = stage_costs(shape)
    stage_ms = [statistics.mean(events[i][k].elapsed_time(events[i][k + 1])
                                for i in range(args.steps)) for k in range(len(STAGES))]
    stages = {}
    for name, (bound, amt), t in zip(STAGES, costs, stage_ms):
        if bound == "tensor":
            ach, peak, unit = amt / (t / 1e3) / 1e12, peaks["bf16_tflops"], "TFLOP/s"
        else:
            ach, peak, unit = amt / (t / 1e3) / 1e9, peaks["hbm_gbs"], "GB/s"
        stages[name] = {"ms": round(t, 4), "bound": bound, "achieved": round(ach, 2),
                        "unit": unit, "frac": round(ach / peak, 4)}
    att = stages["dual_window_attn"]
    total_flops = sum(a for b, a in costs if b == "tensor")

    # ---- end to end through the public API with host buffers.  Every step copies
    # its inputs in from pinned host memory and its result back out; as a serving
    # loop would, the upload of the next step and the read-back of the previous
    # one run on two copy streams while this step computes (double-buffered
    # device tensors, ordered by events).
    x_h = inp["x"].pin_memory()
    b_h = inp["layers"][0]["beta"].pin_memory()
    out_h = [torch.empty(out.shape, dtype=out.dtype).pin_memory() for _ in range(2)]
    x_d = [torch.empty_like(x) for _ in range(2)]
    b_d = [torch.empty_like(beta) for _ in range(2)]
    o_d = [torch.empty_like(out) for _ in range(2)]
    h2d, d2h = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_done = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]

    def e2e_steps(n):
        for i in range(n):
            k = i % 2
            with torch.cuda.stream(h2d):
                if i >= 2:
                    h2d.wait_event(ev_done[k])  # x_d[k], b_d[k] were read by step i-2
                x_d[k].copy_(x_h, non_blocking=True)
                b_d[k].copy_(b_h, non_blocking=True)
                ev_in[k].record(h2d)
            stream.wait_event(ev_in[k])
            if i >= 2:
                stream.wait_event(ev_out[k])  # o_d[k] was read back by step i-2
            ttcd.block_forward(x_d[k], b_d[k], w, p, out=o_d[k], workspace=ws, stream=stream)
            ev_done[k].record(stream)
            with torch.cuda.stream(d2h):
                d2h.wait_event(ev_done[k])
                out_h[k].copy_(o_d[k], non_blocking=True)
                ev_out[k].record(d2h)

    e2e_steps(2)
    torch.cuda.synchronize()
    barrier(world, local)
    s2, e2 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s2.record(h2d)
    e2e_steps(args.steps)
    d2h.wait_event(ev_done[(args.steps - 1) % 2])
    e2.record(d2h)
    torch.cuda.synchronize()
    barrier(world, local)
    ms_e2e, _ = job_throughput(world, shape.B * shape.T, s2.elapsed_time(e2) / args.steps)
    assert torch.equal(out_h[(args.steps - 1) % 2], out.cpu())
    if ttcd.check_device_status(ws, stream) != ttcd.OK:
        raise RuntimeError("a device wait timed out in the end-to-end steps")

    traffic = (args.attn_traffic_bytes if args.attn_traffic_bytes is not None
               else recorded_traffic("dual_window_attn_kernel<128>", shape.T))
    att_flops = attention_flops(shape)
    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": workload_config(shape, {"parallelism": f"replicas{world}"}),
            "tflops_per_s": total_flops / (ms / 1e3) / 1e12,
            "roofline": {"kernel": "dual_window_attn_kernel<128>", "bound": "tensor",
                         "achieved": att["achieved"], "peak": peaks["bf16_tflops"],
                         "unit": "TFLOP/s", "frac": att["frac"],
                         "frac_of_sustained": round(att["achieved"] /
                                                    peaks["bf16_tflops_sustained"], 4),
                         "traffic": traffic,
                         "algorithmic_bytes": attention_bytes(shape),
                         "traffic_over_algorithmic": (round(traffic / attention_bytes(shape), 3)
                                                      if traffic else None),
                         "peak_source": f"{peak_kind} bf16_tflops (burst: the timed region "
                                        f"lasts well under a second)",
                         "flops_per_launch": att_flops},
            "stages": stages,
            "e2e": {"value": tokens / (ms_e2e / 1000.0), "unit": UNIT,
                    "h2d_bytes_per_step": x_h.numel() * x_h.element_size() +
                    b_h.numel() * b_h.element_size(),
                    "d2h_bytes_per_step": out_h[0].numel() * out_h[0].element_size(),
                    "copies": "two copy streams; the next step's upload and the previous "
                              "step's read-back overlap this step's compute"},
            "gpu_launches": launches,
            "clocks": clk.summary()}
    del x, w, beta, ws, out, x_d, b_d, o_d, inp
    torch.cuda.empty_cache()
    if not args.no_extras:
        # The other two workloads of the benchmark set, measured in the same run:
        # the attention sweep (fused form at every window pair, LSE form at
        # 512/8192) and the 28-layer stack at both batch shapes.
        line["attention_sweep"] = [
            measure_attention(args, world, local, wS, wT, "fused", steps=args.extra_steps,
                              warmup=args.extra_warmup)
            for wS, wT in ATTN_SWEEP_PAIRS] + [
            measure_attention(args, world, local, 512, 8192, "lse", steps=args.extra_steps,
                              warmup=args.extra_warmup)]
        line["stack"] = [measure_stack(args, world, local, B, T, steps=max(2, args.extra_steps // 2),
                                       warmup=args.extra_warmup)
                         for B, T in ((1, 65536), (4, 16384))]
        # the plain sliding-window block of layers outside the TTT layer set
        line["swa_block"] = measure_swa_block(args, world, local, steps=args.extra_steps,
                                              warmup=args.extra_warmup)
        # the backward kernels at the same block shape (B 1, T 65536)
        line["backward"] = measure_backward(args, local, 1, shape.T, steps=3, warmup=1)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        v, times = oracle_throughput(shape, args.cpu_sample_tokens)
        line["cpu_baseline"] = {
            "value": v, "unit": UNIT, "cores": cpu_cores(), "kind": "oracle",
            "sample": f"first {args.cpu_sample_tokens} tokens of the workload (attention windows "
                      f"truncated by position), float64 NumPy oracle, {times[0]:.1f} s"}
    if rank == 0:
        print(json.dumps(line), flush=True)


_ATTN_INPUTS = {}


def measure_attention(args, world, local, wS, wT, form, steps, warmup):
    """Dual-window attention alone at the Qwen3-0.6B head layout (16 / 8 heads,
    hd 128), B x T from the arguments: device time per call (CUDA events on the
    launch stream, max over ranks) and the fraction of the burst GEMM peak."""
    import dual_window_attention_b200 as ttcd
    from ttcd_workloads import make_attention_inputs
    ttcd.load_library()
    peaks, peak_kind = load_peaks()
    s0 = QWEN3_0P6B_64K.with_(T=args.T, B=args.B)
    key = (s0.B, s0.T, local)
    if key not in _ATTN_INPUTS:
        _ATTN_INPUTS.clear()
        q, k, v = make_attention_inputs(s0.B, s0.T, s0.n_q_heads, s0.n_kv_heads, s0.head_dim,
                                        seed=0)
        dev = torch.device("cuda", local)
        _ATTN_INPUTS[key] = (q.to(dev), k.to(dev), v.to(dev))
    q, k, v = _ATTN_INPUTS[key]
    o_T, o_S = torch.empty_like(q), torch.empty_like(q)
    stream = torch.cuda.current_stream()

    def call():
        if form == "lse":
            ttcd.dual_window_attn_lse(q, k, v, wS, wT)
        else:
            ttcd.dual_window_attn(q, k, v, wS, wT, o_T=o_T, o_S=o_S)

    shape = s0.with_(w_S=wS, w_T=wT)
    for _ in range(warmup):
        call()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world, local)
    with ClockSampler(local, period_s=0.002) as clk:
        e0.record(stream)
        for _ in range(steps):
            call()
        e1.record(stream)
        torch.cuda.synchronize()
    ms = max_over_ranks(world, e0.elapsed_time(e1)) / steps
    if ttcd.get_device_error()[0] != ttcd.OK:
        raise RuntimeError("a device wait timed out in the attention benchmark")
    fl = attention_flops(shape)
    ach = fl / (ms / 1e3) / 1e12
    return {"form": form, "w_S": wS, "w_T": wT, "B": shape.B, "T": shape.T, "ms": ms,
            "tokens_per_s": shape.B * shape.T * world / (ms / 1e3), "tflops_per_s": ach,
            "frac": ach / peaks["bf16_tflops"],
            "peak_source": f"{peak_kind} bf16_tflops (burst: kernel timed alone)",
            "steps": steps, "warmup": warmup, "clocks": clk.summary()}


def run_attention(args, world, rank, local):
    """Dual-window attention alone (Qwen3-0.6B head layout) for each window pair."""
    pairs = [(int(a), int(b)) for a, b in (w.split("/") for w in args.windows.split(","))]
    for wS, wT in pairs:
        r = measure_attention(args, world, local, wS, wT, args.form, args.steps, args.warmup)
        if rank == 0:
            print(json.dumps({
                "metric": ("LSE-combination" if args.form == "lse" else "fused") +
                          " dual-window attention tokens/s (Qwen3-0.6B heads)",
                "value": r["tokens_per_s"], "unit": UNIT, "n_gpus": world,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": r["ms"],
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
                "dtype": "bf16", "data": "synthetic",
                "config": {"workload": "dual_window_attention", "B": r["B"], "T": r["T"],
                           "n_q_heads": 16, "n_kv_heads": 8, "head_dim": 128, "w_S": wS,
                           "w_T": wT},
                "roofline": {"kernel": "dual_window_attn_kernel<128>" +
                                       (" + lse_merge_kernel" if args.form == "lse" else ""),
                             "bound": "tensor", "achieved": r["tflops_per_s"],
                             "peak": load_peaks()[0]["bf16_tflops"], "unit": "TFLOP/s",
                             "frac": r["frac"], "peak_source": r["peak_source"],
                             "flops_per_launch": attention_flops(
                                 QWEN3_0P6B_64K.with_(T=r["T"], B=r["B"], w_S=wS, w_T=wT))}}),
                  flush=True)


def run_decode_bench(args, world, rank, local):
    """Token-by-token decode of the Qwen3-0.6B-shaped block (B sequences in
    lockstep).  Times --steps consecutive tokens from a position past the teacher
    window (the cache is full; chunk commits fall inside the timed tokens at their
    natural rate).  The HBM floor of one token step is the weights it must read:
    the shared slow weights plus each sequence's W_down + S and K/V window."""
    import dual_window_attention_b200 as ttcd
    ttcd.load_library()
    peaks, peak_kind = load_peaks()
    shape = QWEN3_0P6B_64K.with_(name="qwen3_0.6b_block_decode", B=args.B, T=1)
    dev = torch.device("cuda", local)
    inp = make_block_inputs(shape, seed=0)
    w = {k: v.to(dev) for k, v in inp["layers"][0].items()}
    p = ttcd.BlockParams.from_shape(shape)
    dec = ttcd.Decoder(w, p, graph=args.graph)
    g = torch.Generator().manual_seed(0)
    x = torch.randn(args.B, shape.d_model, generator=g).to(torch.bfloat16).to(dev)
    beta = (0.1 * torch.sigmoid(torch.randn(args.B, generator=g))).to(dev)
    y = torch.empty_like(x)
    if args.graph:  # the decoder's own fixed buffers: no copies around the replays
        dec.x_buf.copy_(x)
        dec.b_buf.copy_(beta)
        x, beta, y = dec.x_buf, dec.b_buf, dec.y_buf
    dec.seek(4 * shape.w_T + 7)  # past the window: full K/V reads every step
    stream = torch.cuda.current_stream()
    for _ in range(max(args.warmup, 3 if args.graph else 0)):
        dec.step(x, beta, y)
    torch.cuda.synchronize()
    barrier(world, local)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    launches0 = ttcd.kernel_launch_count()
    replayed0 = dec.replayed_launches
    with ClockSampler(local) as clk:
        e0.record(stream)
        for _ in range(args.steps):
            dec.step(x, beta, y)
        e1.record(stream)
        torch.cuda.synchronize()
    launches = ttcd.kernel_launch_count() - launches0
    if args.graph:  # replays launch the captured kernels without the host counter
        launches += dec.replayed_launches - replayed0
    ms, value = job_throughput(world, args.B * args.steps, e0.elapsed_time(e1))
    if dec.check_status() != ttcd.OK:
        raise RuntimeError("a device wait timed out in the decode benchmark")
    s_ = shape
    dqkv = (s_.n_q_heads + 2 * s_.n_kv_heads) * s_.head_dim
    shared = 2 * (dqkv * s_.d_model + s_.d_model * s_.n_q_heads * s_.head_dim +
                  2 * s_.d_ff * s_.d_model + s_.d_model * s_.d_ff)
    per_seq = 2 * s_.d_model * s_.d_ff + 2 * 2 * s_.w_T * s_.n_kv_heads * s_.head_dim
    bytes_per_step = shared + args.B * per_seq
    step_ms = ms / args.steps
    ach = bytes_per_step / (step_ms / 1e3) / 1e9
    if rank == 0:
        print(json.dumps({
            "metric": "IP-TTCD block decode tokens/s (Qwen3-0.6B shape, w_S 512, w_T 8192)",
            "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": step_ms, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": workload_config(shape, {"sequences": args.B, "position": "past w_T",
                                              "launch": "cuda graph" if args.graph else "eager",
                                              "parallelism": f"replicas{world}"}),
            "roofline": {"kernel": "decode step (all kernels)", "bound": "hbm", "achieved": ach,
                         "peak": peaks["hbm_gbs"], "unit": "GB/s", "frac": ach / peaks["hbm_gbs"],
                         "bytes_per_step": bytes_per_step, "peak_source": f"{peak_kind} hbm_gbs"},
            "gpu_launches": launches, "clocks": clk.summary()}), flush=True)


def window_pairs(T: int, w: int) -> int:
    """(query, key) pairs of one sequence and head inside a causal window of w keys."""
    return w * (w + 1) // 2 + (T - w) * w if T >= w else T * (T + 1) // 2


def run_backward(args, world, rank, local):
    """`--mode backward`: one JSON line per backward kernel."""
    lines = measure_backward(args, local, args.B, args.T, args.steps, args.warmup)
    if rank == 0:
        for l in lines:
            print(json.dumps(l), flush=True)


def measure_backward(args, local, B_, T_, steps, warmup):
    """The backward kernels at the Qwen3-0.6B block shape (B_ x T_):
    ttcd_fastweight_mlp_backward (the forward's front half and chunk scan
    recomputed inside) and ttcd_dual_window_attn_backward, each timed alone with
    CUDA events.  FLOPs are the algorithmic contractions of each call."""
    import dual_window_attention_b200 as ttcd
    from ttcd_workloads import make_mlp_inputs
    ttcd.load_library()
    peaks, peak_kind = load_peaks()
    shape = QWEN3_0P6B_64K.with_(name=f"qwen3_0.6b_backward_T{T_}", B=B_, T=T_)
    dev = torch.device("cuda", local)
    stream = torch.cuda.current_stream()
    B, T, d, f = shape.B, shape.T, shape.d_model, shape.d_ff
    Hq, Hkv, hd = shape.n_q_heads, shape.n_kv_heads, shape.head_dim
    BT = B * T
    Cp = (shape.chunk + 63) // 64 * 64
    P = B * shape.n_chunks * Cp
    g = torch.Generator().manual_seed(0)

    def timed(fn, steps, warmup):
        for _ in range(warmup):
            fn()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(steps):
            fn()
        e1.record(stream)
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / steps

    lines = []
    # fast-weight MLP backward
    inp = make_mlp_inputs(shape, seed=0)
    w = {k: v.to(dev) for k, v in inp.items()}
    d_y = torch.randn(B, T, d, generator=g).to(torch.bfloat16).to(dev)
    p = ttcd.BlockParams.from_shape(shape)
    _, ws = ttcd.fastweight_mlp_backward(w["u_T"], w["u_S"], w["beta"], w, p, d_y)
    ms = timed(lambda: ttcd.fastweight_mlp_backward(w["u_T"], w["u_S"], w["beta"], w, p, d_y,
                                                    workspace=ws), steps, warmup)
    if ttcd.check_device_status(ws) != ttcd.OK:
        raise RuntimeError("a device wait timed out in the MLP backward")
    recompute = 2 * 2 * BT * 2 * f * d + 2 * d * f * f + 2 * 2 * P * f * d
    backward = (2 * BT * d * f + 5 * 2 * P * d * f + 2 * 2 * d * f * f + 2 * 2 * 2 * BT * 2 * f * d
                + 2 * 2 * 2 * BT * f * d)
    flops = recompute + backward
    lines.append({"kernel": "ttcd_fastweight_mlp_backward", "ms": ms, "flops": flops,
                  "tflops_per_s": flops / ms / 1e9})
    del w, ws, inp
    # dual-window attention backward
    q = torch.randn(B, T, Hq, hd, generator=g).to(torch.bfloat16).to(dev)
    k = torch.randn(B, T, Hkv, hd, generator=g).to(torch.bfloat16).to(dev)
    v = torch.randn(B, T, Hkv, hd, generator=g).to(torch.bfloat16).to(dev)
    o_T, o_S, lse_T, lse_S = ttcd.dual_window_attn(q, k, v, shape.w_S, shape.w_T, lse=True)
    do_T = torch.randn(B, T, Hq, hd, generator=g).to(torch.bfloat16).to(dev)
    do_S = torch.randn(B, T, Hq, hd, generator=g).to(torch.bfloat16).to(dev)
    _, _, _, aws = ttcd.dual_window_attn_backward(q, k, v, o_T, o_S, lse_T, lse_S, do_T, do_S,
                                                  shape.w_S, shape.w_T)
    ms = timed(lambda: ttcd.dual_window_attn_backward(q, k, v, o_T, o_S, lse_T, lse_S, do_T, do_S,
                                                      shape.w_S, shape.w_T, workspace=aws),
               steps, warmup)
    if ttcd.check_device_status(aws) != ttcd.OK:
        raise RuntimeError("a device wait timed out in the attention backward")
    # per visible pair and head: S recomputed, dP, dV, dK, dQ (2 hd FLOPs each)
    pairs = B * Hq * (window_pairs(T, shape.w_T) + window_pairs(T, shape.w_S))
    flops = 10.0 * hd * pairs
    lines.append({"kernel": "ttcd_dual_window_attn_backward", "ms": ms, "flops": flops,
                  "tflops_per_s": flops / ms / 1e9})
    for l in lines:
        l.update({"metric": "backward kernel time (Qwen3-0.6B block shape)",
                  "config": workload_config(shape), "steps": steps, "warmup": warmup,
                  "peak_tflops": peaks["bf16_tflops"],
                  "frac": l["tflops_per_s"] / peaks["bf16_tflops"],
                  "peak_source": f"{peak_kind} bf16_tflops"})
    del q, k, v, o_T, o_S, lse_T, lse_S, do_T, do_S, aws
    torch.cuda.empty_cache()
    return lines


def measure_stack(args, world, local, B, T, steps, warmup):
    """The 28-layer stack of Qwen3-0.6B-shaped blocks end to end (B x T): every
    layer one ttcd_block_forward on its own weights, one shared workspace."""
    import dual_window_attention_b200 as ttcd
    from ttcd_workloads import QWEN3_STACK_B1, QWEN3_STACK_B4
    ttcd.load_library()
    base = QWEN3_STACK_B4 if (B, T) == (4, 16384) else QWEN3_STACK_B1
    shape = base if (B, T) == (base.B, base.T) else base.with_(
        name=f"qwen3_0.6b_stack28_B{B}_T{T}", B=B, T=T)
    dev = torch.device("cuda", local)
    inp = make_block_inputs(shape, seed=0)
    x = inp["x"].to(dev)
    layers = [{k: v.to(dev) for k, v in lw.items()} for lw in inp["layers"]]
    del inp
    p = ttcd.BlockParams.from_shape(shape)
    ws = ttcd.alloc_workspace(ttcd.block_forward_workspace_size(p), dev)
    stream = torch.cuda.current_stream()

    def step():
        return ttcd.block_stack_forward(x, layers, p, workspace=ws, stream=stream)

    for _ in range(warmup):
        step()
    if ttcd.check_device_status(ws, stream) != ttcd.OK:
        raise RuntimeError("a device wait timed out during the stack warm-up")
    barrier(world, local)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    launches0 = ttcd.kernel_launch_count()
    with ClockSampler(local) as clk:
        e0.record(stream)
        for _ in range(steps):
            step()
        e1.record(stream)
        torch.cuda.synchronize()
    launches = ttcd.kernel_launch_count() - launches0
    barrier(world, local)
    ms = max_over_ranks(world, e0.elapsed_time(e1)) / steps
    if ttcd.check_device_status(ws, stream) != ttcd.OK:
        raise RuntimeError("a device wait timed out in the stack benchmark")
    flops = shape.n_layers * sum(a for b, a in stage_costs(shape) if b == "tensor")
    del x, layers, ws
    torch.cuda.empty_cache()
    return {"workload": shape.name, "B": shape.B, "T": shape.T, "n_layers": shape.n_layers,
            "ms_per_pass": ms, "tokens_per_s": shape.B * shape.T * world / (ms / 1e3),
            "tflops_per_s": flops / (ms / 1e3) / 1e12, "steps": steps, "warmup": warmup,
            "gpu_launches": launches, "clocks": clk.summary()}


def measure_swa_block(args, world, local, steps, warmup):
    """The plain sliding-window block of the layers outside the TTT layer set
    (ttcd_swa_block_forward: one w_T = 8192 window, static MLP) at the Qwen3
    block shape, B 1, T 65536."""
    import dual_window_attention_b200 as ttcd
    ttcd.load_library()
    shape = QWEN3_0P6B_64K
    dev = torch.device("cuda", local)
    inp = make_block_inputs(shape, seed=0)
    x = inp["x"].to(dev)
    w = {k: v.to(dev) for k, v in inp["layers"][0].items()
         if k not in ("beta", "w_proj", "conv_T", "conv_S")}
    del inp
    p = ttcd.BlockParams.from_shape(shape)
    ws = ttcd.alloc_workspace(ttcd.swa_block_forward_workspace_size(p), dev)
    out = torch.empty_like(x)
    stream = torch.cuda.current_stream()
    for _ in range(warmup):
        ttcd.swa_block_forward(x, w, p, out=out, workspace=ws, stream=stream)
    barrier(world, local)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        ttcd.swa_block_forward(x, w, p, out=out, workspace=ws, stream=stream)
    e1.record(stream)
    torch.cuda.synchronize()
    barrier(world, local)
    ms = max_over_ranks(world, e0.elapsed_time(e1)) / steps
    if ttcd.check_device_status(ws, stream) != ttcd.OK:
        raise RuntimeError("a device wait timed out in the plain-block benchmark")
    BT, d, f = shape.B * shape.T, shape.d_model, shape.d_ff
    hq, hkv, hd = shape.n_q_heads, shape.n_kv_heads, shape.head_dim
    attn = 4.0 * hd * hq * sum(min(t + 1, shape.w_T) for t in range(shape.T)) * shape.B
    gemm = 2.0 * BT * d * (hq + 2 * hkv) * hd + 2.0 * BT * hq * hd * d + 2.0 * BT * d * 2 * f \
        + 2.0 * BT * f * d
    del x, w, ws, out
    torch.cuda.empty_cache()
    return {"workload": "qwen3_0.6b_plain_swa_block_T65536", "window": shape.w_T, "ms": ms,
            "tokens_per_s": BT * world / (ms / 1e3),
            "tflops_per_s": (attn + gemm) / (ms / 1e3) / 1e12, "steps": steps, "warmup": warmup}


def run_stack(args, world, rank, local):
    """The 28-layer stack of Qwen3-0.6B-shaped blocks, end-to-end prefill tokens/s
    (B 1 x T 65536 by default, or --B 4 --T 16384)."""
    r = measure_stack(args, world, local, args.B, args.T, args.steps, args.warmup)
    if rank == 0:
        print(json.dumps({
            "metric": "IP-TTCD 28-layer stack prefill tokens/s (Qwen3-0.6B shape)",
            "value": r["tokens_per_s"], "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": r["ms_per_pass"],
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic",
            "config": {"workload": r["workload"], "B": r["B"], "T": r["T"],
                       "n_layers": r["n_layers"], "parallelism": f"replicas{world}"},
            "tflops_per_s": r["tflops_per_s"], "gpu_launches": r["gpu_launches"],
            "clocks": r["clocks"]}), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-sample-tokens", type=int, default=16384)
    ap.add_argument("--ref-sample-tokens", type=int, default=512)
    ap.add_argument("--mode", choices=["block", "attn", "stack", "decode", "backward"],
                    default="block",
                    help="block: the whole IP-TTCD block (default); attn: attention alone; "
                         "stack: 28 blocks end to end; decode: one token at a time")
    ap.add_argument("--T", type=int, default=65536,
                    help="tokens per sequence (65536 is the benchmark workload; smaller values "
                         "are for profiling)")
    ap.add_argument("--B", type=int, default=1, help="--mode attn / stack / decode: sequences")
    ap.add_argument("--graph", action="store_true",
                    help="--mode decode: replay each token step from one CUDA graph")
    ap.add_argument("--windows", default="512/8192",
                    help="--mode attn: comma-separated w_S/w_T pairs")
    ap.add_argument("--form", choices=["fused", "lse"], default="fused",
                    help="--mode attn: fused kernel, or student window + far band merged by LSE")
    ap.add_argument("--attn-traffic-bytes", type=float, default=None,
                    help="DRAM bytes per attention launch from an ncu capture")
    ap.add_argument("--no-extras", action="store_true",
                    help="block mode: skip the attention sweep, the 28-layer stack and the backward kernels")
    ap.add_argument("--extra-steps", type=int, default=5,
                    help="timed calls per attention window pair / stack shape")
    ap.add_argument("--extra-warmup", type=int, default=3)
    ap.add_argument("--record-traffic", metavar="CSV", default=None,
                    help="write the DRAM bytes of an ncu capture of the attention kernel at "
                         "--T into profiles/ncu_traffic.json (no GPU work)")
    ap.add_argument("--record-command", default="", help="with --record-traffic: the capture's command")
    args = ap.parse_args()
    if args.record_traffic:
        shape = QWEN3_0P6B_64K.with_(T=args.T)
        rec = record_traffic(args.record_traffic, "dual_window_attn_kernel<128>", args.T,
                             ["attention.cuh", "gemm.cuh", "ptx.cuh"],
                             f"Qwen3-0.6B head layout, B 1, T {args.T}, 16/8 heads, hd 128, "
                             "w_S 512, w_T 8192", args.record_command, attention_bytes(shape),
                             "one launch at the full workload (one-pass metrics)")
        print(json.dumps(rec))
        return
    world, rank, local = dist_setup()
    try:
        if args.impl == "reference":
            run_reference(args, world, rank)
        elif args.mode == "attn":
            run_attention(args, world, rank, local)
        elif args.mode == "stack":
            run_stack(args, world, rank, local)
        elif args.mode == "decode":
            run_decode_bench(args, world, rank, local)
        elif args.mode == "backward":
            run_backward(args, world, rank, local)
        else:
            run_ours(args, world, rank, local)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
