"""Shared test utilities: error measures and oracle invocation on seeded inputs."""
import numpy as np
import torch

# Tolerances of the block forward: bf16 (and fp32-interface) outputs
# max|d|/max|ref| <= 1e-2; the fp32 fast-weight state relative Frobenius <= 5e-3.
TOL_OUT = 1e-2
TOL_STATE = 5e-3


def np64(t):
    if isinstance(t, torch.Tensor):
        return t.detach().float().cpu().double().numpy() if t.dtype == torch.bfloat16 else \
            t.detach().cpu().double().numpy()
    return np.asarray(t, np.float64)


def rel_max(got, ref) -> float:
    got, ref = np64(got), np64(ref)
    return float(np.max(np.abs(got - ref)) / max(np.max(np.abs(ref)), 1e-30))


def rel_fro(got, ref) -> float:
    got, ref = np64(got), np64(ref)
    return float(np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-30))


def oracle_block(shape, inp, layer=0, T=None):
    """Run the oracle block forward on the seeded inputs (optionally a prefix of T tokens)."""
    from oracle import ttcd_oracle as orc
    w = {k: np64(v) for k, v in inp["layers"][layer].items()}
    x = np64(inp["x"])
    beta = w["beta"]
    if T is not None:
        x, beta = x[:, :T], beta[:, :T]
    return orc.block_forward(x, beta, w, n_q_heads=shape.n_q_heads, n_kv_heads=shape.n_kv_heads,
                             head_dim=shape.head_dim, w_S=shape.w_S, w_T=shape.w_T,
                             chunk=shape.chunk, rms_eps=shape.rms_eps, l2_eps=shape.l2_eps,
                             rope_theta=shape.rope_theta)


def to_device(inp, layer=0, device="cuda"):
    w = {k: v.to(device) for k, v in inp["layers"][layer].items()}
    return inp["x"].to(device), w


# ---------------------------------------------------------------------------
# Oracle runs in worker processes.  The processes are started with "spawn":
# a process forked from one that has used CUDA can hang.


def _oracle_block_job(job):
    """The oracle block forward of one job; weights may come in their storage
    type (bf16 tensors pickle at a quarter of the float64 size)."""
    shape, w, x, beta, threads = job
    from threadpoolctl import threadpool_limits
    from oracle import ttcd_oracle as orc
    w = {k: np64(v) for k, v in w.items()}
    with threadpool_limits(threads):
        return orc.block_forward(np64(x), np64(beta), w, n_q_heads=shape.n_q_heads,
                                 n_kv_heads=shape.n_kv_heads, head_dim=shape.head_dim,
                                 w_S=shape.w_S, w_T=shape.w_T, chunk=shape.chunk,
                                 rms_eps=shape.rms_eps, l2_eps=shape.l2_eps,
                                 rope_theta=shape.rope_theta)["out"]


def _oracle_chain_job(job):
    """Layers applied in sequence from x; each output optionally rounded to bf16.
    Returns the last output and the per-layer relative Frobenius size of that
    rounding."""
    shape, layers, x, betas, round_bf16, threads = job
    e = []
    for w, beta in zip(layers, betas):
        z = _oracle_block_job((shape, w, x, beta, threads))
        if round_bf16:
            x = torch.from_numpy(z).to(torch.bfloat16).double().numpy()
            e.append(rel_fro(x, z))
        else:
            x = z
    return x, e


def pool_size(n_jobs: int, gb_per_job: float):
    """(workers, BLAS threads per worker) from the host's cores and free memory."""
    import os
    try:
        cores = len(os.sched_getaffinity(0))
    except Exception:
        cores = os.cpu_count() or 1
    try:
        import psutil
        avail_gb = psutil.virtual_memory().available / 2 ** 30
    except Exception:
        avail_gb = 16.0
    workers = max(1, min(n_jobs, cores, int(0.7 * avail_gb // gb_per_job)))
    return workers, max(1, cores // workers)


def oracle_map(fn, jobs, gb_per_job: float):
    """fn(job + (threads,)) for every job, in spawn-started worker processes."""
    import multiprocessing as mp
    workers, threads = pool_size(len(jobs), gb_per_job)
    with mp.get_context("spawn").Pool(workers) as pool:
        return pool.map(fn, [tuple(j) + (threads,) for j in jobs], chunksize=1)
