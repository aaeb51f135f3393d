"""GPU parity of a 28-layer stack of Qwen3-0.6B-shaped IP-TTCD blocks.

Each block is the one of papernotes.org review "Learning What to Remember",
方法详解 (flowchart A-F); the stack applies them in sequence (layer l's output is
layer l+1's input), with random-init bf16 weights N(0, 1/fan_in) and token
embeddings N(0, 1).  Two batch shapes: B = 1, T = 65536 and B = 4, T = 16384.

Every block is causal, so the first T' outputs of each layer depend only on the
first T' tokens of its input.  The stack runs at full length on the GPU; the
oracle runs on a prefix of T' tokens that spans ten chunks and a ragged tail,
past the 8192-key teacher window.

* The parity check, every layer: layer l of the oracle, fed the GPU's (bf16)
  output of layer l-1, against the GPU's output of layer l (bf16 outputs,
  max|d|/max|ref| <= 1e-2).  This is the stack's parity evidence: each layer of
  the stack is held to the block tolerance.
* A diagnostic, printed and not asserted: the last layer against the oracle
  chained in float64 from the embeddings, beside the same float64 chain with
  every layer's output rounded to bf16 as the library stores it.  A random-init
  stack amplifies any perturbation of its residual stream layer after layer, so
  neither ends within 1e-2 of the float64 chain; the printout shows how far the
  GPU ends next to how far bf16 storage alone takes the chain.
"""
import numpy as np
import pytest
import torch

from tests.helpers import (TOL_OUT, _oracle_block_job, _oracle_chain_job, np64, oracle_map,
                           rel_max)
from ttcd_workloads import QWEN3_STACK_B1, QWEN3_STACK_B4, make_block_inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ttcd():
    import dual_window_attention_b200 as m
    m.load_library()
    return m


@pytest.mark.parametrize("shape,Tp,seqs,chain_Tp", [
    (QWEN3_STACK_B1, 10 * 1024 + 300, [0], 1024 + 300),
    (QWEN3_STACK_B4, 10 * 1024 + 200, [0, 3], None),
], ids=["B1_T65536", "B4_T16384"])
def test_stack_parity(ttcd, shape, Tp, seqs, chain_Tp):
    assert shape.n_layers == 28 and Tp >= 10 * shape.chunk
    inp = make_block_inputs(shape, seed=0)
    p = ttcd.BlockParams.from_shape(shape)
    x = inp["x"].cuda()
    layers = [{k: v.cuda() for k, v in lw.items()} for lw in inp["layers"]]
    prefixes = []
    ws = ttcd.alloc_workspace(ttcd.block_forward_workspace_size(p))
    out = ttcd.block_stack_forward(
        x, layers, p, workspace=ws, on_layer=lambda l, o: prefixes.append(o[seqs, :Tp].cpu()))
    assert ttcd.check_device_status(ws) == ttcd.OK
    assert len(prefixes) == 28 and torch.isfinite(out).all()
    assert torch.equal(out[seqs, :Tp].cpu(), prefixes[-1])
    del layers, x, out, ws
    torch.cuda.empty_cache()

    weights = inp["layers"]  # bf16 on the CPU; the workers widen them to float64
    betas = [np64(w["beta"])[seqs, :Tp] for w in weights]
    x0 = np64(inp["x"])[seqs, :Tp]
    jobs = [(shape, weights[l], x0 if l == 0 else np64(prefixes[l - 1]), betas[l])
            for l in range(28)]
    refs = oracle_map(_oracle_block_job, jobs, gb_per_job=2.5 * len(seqs) * Tp / 5000)
    errs = [rel_max(prefixes[l], refs[l]) for l in range(28)]
    print(f"\n{shape.name}: per-layer max|d|/max|ref| on {Tp} rows x {len(seqs)} seqs: "
          f"max {max(errs):.2e}, mean {np.mean(errs):.2e}")
    assert max(errs) <= TOL_OUT, errs

    if chain_Tp:
        # Diagnostic only (see the module docstring): how far the GPU's last layer
        # ends from the float64 chain, next to the bf16-storage chain.
        x0c = x0[:, :chain_Tp]
        bc = [b[:, :chain_Tp] for b in betas]
        (y64, _), (y16, e_s) = oracle_map(
            _oracle_chain_job, [(shape, weights, x0c, bc, False), (shape, weights, x0c, bc, True)],
            gb_per_job=1.0)
        gpu_last = np64(prefixes[-1])[:, :chain_Tp]
        print(f"{shape.name} diagnostic, last layer vs the float64 chain on {chain_Tp} rows: "
              f"GPU {rel_max(gpu_last, y64):.2e}, bf16-storage chain {rel_max(y16, y64):.2e} "
              f"(bf16 storage perturbs each layer by {np.mean(e_s):.2e} rel. Frobenius)")
        assert np.isfinite(y64).all() and np.isfinite(gpu_last).all()
