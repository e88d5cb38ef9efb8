"""GPU parity of the graph-captured merge cycle (dl_cycle_*) against the oracle.

A cycle is C tokens through every layer, token-major, as one CUDA graph; the
graph reads its inputs from fixed buffers, so to decode T tokens the caller
copies each cycle's C tokens into those buffers before the launch.  With two
or more layers that have heads, each kernel may stream its base while the
previous layer's kernel finishes (programmatic dependent launch): the tests
below cover that path against the fp64 oracle -- every layer's outputs for
every token and the materialised state after every cycle -- and a cycle in
which a layer without heads sits between the steps of one layer, where that
overlap must not happen.  Tolerances as in test_gpu_parity.
"""
import numpy as np
import pytest
import torch

import oracle
from oracle import rel_err
from recurrent_state_head_b200 import binding as B
from recurrent_state_head_b200 import device as D
from recurrent_state_head_b200 import synth

from test_gpu_parity import (MODES, OPS, TOL_STATE, oracle_inputs, run_oracle_eager, small, to_np,
                              tol_out)
from test_gpu_slots import _oracle_materialize_slots, _oracle_slots

pytestmark = pytest.mark.gpu


def run_cycles(layers, xs, w, t0, T, C, after_cycle=None):
    """Decode tokens [t0, t0 + T) of every layer (T a multiple of C) through
    one graph-captured merge cycle launched T / C times, the next cycle's
    inputs copied into the graph's buffers before each launch.  Returns the
    outputs [T, NH, dv] of every layer and the kernels per launch;
    after_cycle() (if given) runs after each launch has been queued."""
    R = len(layers)
    rw = w.op == synth.RWKV6
    stage = [None if xs[l] is None else {k: v[t0:t0 + C].clone() for k, v in xs[l].items()}
             for l in range(R)]
    souts = [layers[l].new_out(C) for l in range(R)]

    def io(l, t):
        if stage[l] is None:                       # a layer without heads
            return (None,) * 6
        s = stage[l]
        return (s["q"][t], s["k"][t], s["v"][t], None if rw else s["beta"][t], s["g"][t],
                souts[l][t])

    cyc = B.Cycle([L_.handle for L_ in layers], [[io(l, t) for l in range(R)] for t in range(C)])
    outs = [layers[l].new_out(T) for l in range(R)]
    for c0 in range(t0, t0 + T, C):
        for l in range(R):
            if stage[l] is not None:
                for k in stage[l]:
                    stage[l][k].copy_(xs[l][k][c0:c0 + C])
        cyc.launch()
        for l in range(R):
            if stage[l] is not None:
                outs[l][c0 - t0:c0 - t0 + C].copy_(souts[l])
        if after_cycle is not None:
            after_cycle()
    torch.cuda.synchronize()
    kernels = cyc.kernels
    cyc.close()
    return outs, kernels


@pytest.mark.parametrize("op", OPS)
@pytest.mark.parametrize("mode", MODES)
@pytest.mark.parametrize("R", [2, 4])
def test_cycle_matches_oracle(op, mode, R):
    """R layers, two cycles and the second cycle's inputs copied in between:
    outputs of every layer and token, and the state after each cycle."""
    C = 4
    T = 2 * C
    w = small(op, 128, 128, C=C, T=T, in_dt="bf16", out_dt="bf16", seed=60 + op)
    layers, xs, tis, S0s, bons = [], [], [], [], []
    for l in range(R):
        S0s.append(synth.initial_state(w, layer=l))
        bons.append(synth.bonus(w, layer=l))
        tis.append(synth.tokens(w, 0, T, layer=l))
        xs.append(D.to_device(tis[l], w))
        layers.append(D.DecodeLayer(w, S0s[l], bons[l], auto_merge=mode))
    snaps = []
    outs, kernels = run_cycles(layers, xs, w, 0, T, C,
                               after_cycle=lambda: snaps.append([L_.base.clone() for L_ in layers]))
    assert all(L_.L == 0 for L_ in layers)
    states = [[to_np(x) for x in snap] for snap in snaps]
    assert kernels == R * (C + 1 if mode == B.DL_MERGE_SEPARATE else C)
    for l in range(R):
        Sr, q, k, v, beta, g, bon = oracle_inputs(w, tis[l], S0=S0s[l], bonus=bons[l])
        S = Sr
        o = to_np(outs[l])
        for c in range(2):
            sl = slice(c * C, (c + 1) * C)
            S, o_ref = oracle.eager_run(w.op, S, q[sl], k[sl], v[sl],
                                        None if op == synth.RWKV6 else beta[sl], g[sl], bon,
                                        w.scale)
            for i, t in enumerate(range(c * C, (c + 1) * C)):
                assert rel_err(o[t], o_ref[i]) <= tol_out(w), (l, t)
            assert rel_err(states[c][l], S) <= TOL_STATE, (l, c)


@pytest.mark.parametrize("op", OPS)
@pytest.mark.parametrize("mode", MODES)
@pytest.mark.parametrize("layout", ["heads-empty", "heads-empty-heads"])
def test_cycle_staggered_with_empty_layer(op, mode, layout):
    """Slots at staggered log lengths, with a layer without heads (B = 0)
    between the layers that have them.  With one such layer the cycle's
    consecutive kernels are that layer's own steps (no early base stream);
    with two they alternate.  Against the oracle's per-slot run."""
    C = 4
    T0 = C - 1                                   # staggering tokens, issued one by one
    T = T0 + 2 * C
    w = small(op, 128, 64, C=C, T=T, Bsz=5, H=2, in_dt="bf16", out_dt="f32", seed=33 + op)
    w0 = small(op, 128, 64, C=C, T=T, Bsz=0, H=2, in_dt="bf16", out_dt="f32")
    kinds = layout.split("-")
    layers, xs, refs = [], [], []
    act = np.ones((T, w.B), bool)
    for t in range(T0):
        act[t] = [(b % C) > t for b in range(w.B)]
    for l, kind in enumerate(kinds):
        if kind == "empty":
            layers.append(D.DecodeLayer(w0, np.zeros((0, w.H, w.dk, w.dv), np.float32),
                                        synth.bonus(w0), auto_merge=mode))
            xs.append(None)
            refs.append(None)
            continue
        S0 = synth.initial_state(w, layer=l)
        bonus = synth.bonus(w, layer=l)
        ti = synth.tokens(w, 0, T, layer=l)
        x = D.to_device(ti, w)
        lay = D.DecodeLayer(w, S0, bonus, auto_merge=mode)
        pre = lay.new_out(T0)
        for t in range(T0):
            lay.step(x, t, pre[t], active=act[t].tolist())
        layers.append(lay)
        xs.append(x)
        refs.append((ti, S0, bonus, pre))
    start = [[L_.slot_len(b) for b in range(L_.w.B)] for L_ in layers]
    outs, kernels = run_cycles(layers, xs, w, T0, 2 * C, C)
    for l, L_ in enumerate(layers):
        assert [L_.slot_len(b) for b in range(L_.w.B)] == start[l]
        if refs[l] is None:
            continue
        ti, S0, bonus, pre = refs[l]
        st, Ls_ref, o_ref, Ltr = _oracle_slots(w, ti, S0, bonus, C, act, {}, {})
        o = np.concatenate([to_np(pre), to_np(outs[l])])
        H = w.H
        for t in range(T):
            rows = np.repeat(act[t], H)
            assert rel_err(o[t][rows], o_ref[t][rows]) <= tol_out(w), (l, t)
        mat_ref = _oracle_materialize_slots(w, st, Ls_ref, C)
        assert rel_err(to_np(L_.materialize()), mat_ref) <= TOL_STATE, l
        assert [L_.slot_len(b) for b in range(w.B)] == Ltr[-1].tolist()


@pytest.mark.parametrize("name", ["gdn-b128-h16-d128-c8", "kda-b128-h32-d128-c8",
                                  "kda-b128-h32-d128-c4", "rwkv6-b128-h32-d64-c8",
                                  "rwkv6-b128-h32-d64-c4"])
@pytest.mark.parametrize("mode", MODES)
def test_cycle_full_size(mode, name):
    """The bench's workloads as four-layer cycles (the bench's step), two
    cycles: byte-for-byte equal to the same steps issued one by one, and
    every head of every layer against the oracle (outputs of every token,
    state after each cycle)."""
    w = synth.WORKLOADS[name]
    C, R = w.C, 4
    T = 2 * C
    a, b, xs, tis, S0s, bons = [], [], [], [], [], []
    for l in range(R):
        S0s.append(synth.initial_state(w, layer=l))
        bons.append(synth.bonus(w, layer=l))
        tis.append(synth.tokens(w, 0, T, layer=l, want64=False))
        xs.append(D.to_device(tis[l], w))
        a.append(D.DecodeLayer(w, S0s[l], bons[l], auto_merge=mode))
        b.append(D.DecodeLayer(w, S0s[l], bons[l], auto_merge=mode))
    outs_a = [L_.new_out(T) for L_ in a]
    states_a, states_b = [], []
    for c in range(2):
        for t in range(c * C, (c + 1) * C):
            for l in range(R):
                a[l].step(xs[l], t, outs_a[l][t])
        states_a.append([L_.base.clone() for L_ in a])
    outs_b, _ = run_cycles(b, xs, w, 0, T, C,
                           after_cycle=lambda: states_b.append([L_.base.clone() for L_ in b]))
    for l in range(R):
        assert torch.equal(outs_a[l], outs_b[l]), l
        for c in range(2):
            assert torch.equal(states_a[c][l], states_b[c][l]), (l, c)
    del a, outs_a, states_a
    for l in range(R):
        Sr, q, k, v, beta, g, bon = oracle_inputs(w, tis[l], S0=S0s[l], bonus=bons[l])
        S = Sr
        o = to_np(outs_b[l])
        for c in range(2):
            sl = slice(c * C, (c + 1) * C)
            S, o_ref = run_oracle_eager(w, S, q[sl], k[sl], v[sl], beta[sl], g[sl], bon)
            for i, t in enumerate(range(c * C, (c + 1) * C)):
                assert rel_err(o[t], o_ref[i]) <= tol_out(w), (l, t)
            assert rel_err(to_np(states_b[c][l]), S) <= TOL_STATE, (l, c)
