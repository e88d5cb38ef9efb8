"""GPU parity of the 24-layer GDN stack sweep: B in {1, 8, 32, 128, 512} x
C in {1, 2, 4, 8, 16}, 512 decode steps per layer.

The stack's layers are independent decode problems (each has its own state
and inputs; one decode step per layer in sequence), so the check samples
(layer, slot, head) triples: the first and the last layer, decoded together
as a two-layer graph-captured merge cycle (the stack's execution path, with
each kernel streaming its base during the previous layer's kernel), every
head when a layer has at most 128 of them, else 24 heads (the first, the
last and 22 drawn at random).  Every output of every one of the 512 steps
and the final state of those heads are compared with the oracle's eager
recurrence (which does not depend on C), at 2e-2 (bf16 outputs) and 1e-4
(fp32 state).  The final log length is 512 mod C = 0 for every C, so the
base itself is the materialised state.
"""
import numpy as np
import pytest
import torch

import oracle
from oracle import rel_err
from recurrent_state_head_b200 import device as D
from recurrent_state_head_b200 import synth

from test_gpu_cycle import run_cycles
from test_gpu_parity import TOL_STATE, oracle_inputs, to_np, tol_out

pytestmark = pytest.mark.gpu

LAYERS = (0, 23)
CS = (1, 2, 4, 8, 16)
BLOCK = 64                      # tokens generated per host batch


def _inputs(w, layer, heads):
    """All 512 tokens of one layer on the device, and the sampled heads'
    stored inputs on the host as a [T, len(heads), 1, ...] batch of one-head
    slots (generated in blocks to bound host memory)."""
    T, NH = w.T, w.heads
    x = None
    keep = {k: [] for k in ("q", "k", "v", "beta", "g")}
    for t0 in range(0, T, BLOCK):
        ti = synth.tokens(w, t0, min(BLOCK, T - t0), layer=layer, want64=False)
        xb = D.to_device(ti, w)
        if x is None:
            x = {k: torch.empty((T,) + tuple(v.shape[1:]), dtype=v.dtype, device=v.device)
                 for k, v in xb.items()}
        for k, v in xb.items():
            x[k][t0:t0 + v.shape[0]].copy_(v)
        n = ti.q.shape[0]
        for k in keep:
            a = getattr(ti, k)
            keep[k].append(np.expand_dims(a.reshape((n, NH) + a.shape[3:])[:, heads], 2))
    host = synth.TokenInputs(*(np.concatenate(keep[k]) for k in ("q", "k", "v", "beta", "g")),
                             np.zeros(0), np.zeros(0), np.zeros(0))
    return x, host


@pytest.mark.parametrize("Bsz", [1, 8, 32, 128, 512])
def test_stack_sweep(Bsz):
    w1 = synth.WORKLOADS[f"gdn-stack24-b{Bsz}-h16-d128-c1"]
    T, NH = w1.T, w1.heads
    assert T == 512
    rng = np.random.default_rng(500 + Bsz)
    heads = np.arange(NH) if NH <= 128 else np.unique(
        np.concatenate([[0, NH - 1], rng.choice(np.arange(1, NH - 1), 22, replace=False)]))
    xs, refs, S0s = [], [], []
    for l in LAYERS:
        x, host = _inputs(w1, l, heads)
        S0 = synth.initial_state(w1, layer=l)
        # the sampled heads' inputs, as the oracle sees them (a one-slot view)
        hw = w1.with_(B=len(heads), H=1)
        Sr, q, k, v, beta, g, _ = oracle_inputs(hw, host, S0=S0.reshape(NH, w1.dk, w1.dv)[heads])
        refs.append(oracle.eager_run(w1.op, Sr, q, k, v, beta, g, None, w1.scale))
        xs.append(x)
        S0s.append(S0)
    for C in CS:
        w = synth.WORKLOADS[f"gdn-stack24-b{Bsz}-h16-d128-c{C}"]
        layers = [D.DecodeLayer(w, S0s[i], None) for i in range(len(LAYERS))]
        outs, _ = run_cycles(layers, xs, w, 0, T, C)
        for i, l in enumerate(LAYERS):
            S_ref, o_ref = refs[i]
            o = to_np(outs[i][:, torch.from_numpy(heads).to(outs[i].device)])
            worst = max(rel_err(o[t], o_ref[t]) for t in range(T))
            assert worst <= tol_out(w), (C, l, worst)
            assert layers[i].L == 0
            base = to_np(layers[i].base[torch.from_numpy(heads).to(layers[i].base.device)])
            assert rel_err(base, S_ref) <= TOL_STATE, (C, l)
        del layers, outs
        torch.cuda.empty_cache()
