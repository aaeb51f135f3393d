"""Host-side multi-rank logic of bench.py, run as world-size-2 gloo process
groups on the CPU (no GPU): process-group setup from the torchrun
environment, the barrier, the max-over-ranks step time, the whole-job
throughput of independent replicas, and the reference arm's rank-0-only rule.

The block forward has no exchange step (batch elements are independent), so
N GPUs run N replicas; these are the only collectives on the path.
"""
import importlib.util
import json
import os
import socket

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    spec = importlib.util.spec_from_file_location("ttcd_bench", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir):
    os.environ.update({"MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port),
                       "WORLD_SIZE": str(world), "RANK": str(rank), "LOCAL_RANK": str(rank)})
    bench = _bench()
    import torch.distributed as dist
    w, r, local = bench.dist_setup(backend="gloo", timeout_s=60)
    res = {"world": w, "rank": r, "local": local, "backend": dist.get_backend()}
    bench.barrier(w, local)
    res["max"] = bench.max_over_ranks(w, float(10 * (r + 1)))
    # replicas: rank r took (r + 1) * 5 ms for 1000 tokens
    res["ms"], res["value"] = bench.job_throughput(w, 1000.0, 5.0 * (r + 1))

    class Args:
        steps, warmup, ref_sample_tokens = 1, 0, 64

    # the reference arm: rank 0 alone runs the oracle and prints; the others return at once
    if r != 0:
        bench.run_reference(Args, w, r)
        res["ref_returned"] = True
    bench.barrier(w, local)
    dist.destroy_process_group()
    with open(os.path.join(out_dir, f"rank{r}.json"), "w") as f:
        json.dump(res, f)


def test_two_rank_replicas_gloo(tmp_path):
    world, port = 2, _free_port()
    mp.start_processes(_rank_main, args=(world, port, str(tmp_path)), nprocs=world,
                       start_method="spawn", join=True)
    res = [json.load(open(tmp_path / f"rank{r}.json")) for r in range(world)]
    for r, d in enumerate(res):
        assert (d["world"], d["rank"], d["local"], d["backend"]) == (2, r, r, "gloo")
        assert d["max"] == 20.0                      # max over ranks, seen by every rank
        assert d["ms"] == pytest.approx(10.0)        # the slowest replica's step time
        assert d["value"] == pytest.approx(2 * 1000.0 / 0.010)  # tokens of both ranks
    assert res[1]["ref_returned"]


def test_single_rank_needs_no_process_group(monkeypatch):
    for k in ("WORLD_SIZE", "RANK", "LOCAL_RANK"):
        monkeypatch.delenv(k, raising=False)
    bench = _bench()
    w, r, local = bench.dist_setup(backend="gloo")
    assert (w, r, local) == (1, 0, 0)
    assert bench.max_over_ranks(1, 3.5) == 3.5
    assert bench.job_throughput(1, 100.0, 2.0) == (2.0, pytest.approx(50000.0))
