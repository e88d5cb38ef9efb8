"""GPU parity of per-slot log lengths (continuous batching) through the C ABI.

Slots decode only when active, start new sequences (their base rows
rewritten, their log dropped) at random tokens, and so fill their logs at
different tokens; the kernels then run over slot lists, each slot at its own
log length.  Reference: the oracle's per-slot base+log run on the same
seeded inputs (itself pinned to the eager recurrence on each slot's tokens).
Tolerances as in test_gpu_parity: outputs 1e-4 (fp32) / 2e-2 (bf16), state
1e-4; per-slot log lengths exact; idle slots' output rows untouched.
"""
import numpy as np
import pytest
import torch

import oracle
from oracle import rel_err
from recurrent_state_head_b200 import binding as B
from recurrent_state_head_b200 import device as D
from recurrent_state_head_b200 import synth

from test_gpu_parity import MODES, OPS, TOL_STATE, oracle_inputs, small, to_np, tol_out

pytestmark = pytest.mark.gpu


def _schedule(rng, T, nslots, p_active=0.7, p_reset=0.08):
    act = rng.random((T, nslots)) < p_active
    resets = {}
    for t in range(1, T):
        r = [s for s in range(nslots) if rng.random() < p_reset]
        if r:
            resets[t] = r
    return act, resets


def _oracle_slots(w, ti, S0, bonus, C, act, resets, new_states):
    """Per-slot oracle run split at the reset tokens."""
    Sr, q, k, v, beta, g, bon = oracle_inputs(w, ti, S0=S0, bonus=bonus)
    T, nslots, H = q.shape[0], w.B, w.H
    st = oracle.LogState(w.op, Sr, C)
    Ls = np.zeros(nslots, dtype=np.int32)
    out = np.full((T, w.heads, w.dv), np.nan)
    Ltr = np.zeros((T, nslots), dtype=np.int32)
    cuts = sorted(resets) + [T]
    t0 = 0
    b_ = None if w.op == synth.RWKV6 else beta
    for t1 in cuts:
        if t1 > t0:
            sl = slice(t0, t1)
            o, tr = oracle.deltalog_slots_run(st, H, Ls, act[sl], q[sl], k[sl], v[sl],
                                              None if b_ is None else b_[sl], g[sl], bon,
                                              w.scale)
            out[sl] = o
            Ltr[sl] = tr
        if t1 < T:
            for s in resets[t1]:
                st.base[s * H:(s + 1) * H] = new_states[(t1, s)].astype(np.float64)
                Ls[s] = 0
        t0 = t1
    return st, Ls, out, Ltr


def _oracle_materialize_slots(w, st, Ls, C):
    H = w.H
    mats = []
    for s in range(w.B):
        hs = slice(s * H, (s + 1) * H)
        mats.append(oracle.materialize(oracle.LogState(w.op, st.base[hs], C, int(Ls[s]),
                                                       st.K[hs], st.U[hs], st.Lam[hs])))
    return np.concatenate(mats) if mats else st.base.copy()


def _run_gpu(w, x, S0, bonus, C, mode, act, resets, new_states):
    layer = D.DecodeLayer(w, S0, bonus, C=C, auto_merge=mode)
    T = act.shape[0]
    outs = layer.new_out(T)
    outs.fill_(float("nan"))
    Ls = []
    for t in range(T):
        for s in resets.get(t, []):
            layer.slot_reset(s, torch.from_numpy(new_states[(t, s)]).cuda())
        layer.step(x, t, outs[t], active=act[t].tolist())
        Ls.append([layer.slot_len(b) for b in range(w.B)])
    torch.cuda.synchronize()
    return layer, outs, np.array(Ls)


def _compare(w, outs, o_ref, act):
    o = to_np(outs)
    H = w.H
    for t in range(o.shape[0]):
        rows = np.repeat(act[t], H)
        assert np.all(np.isnan(o[t][~rows])), t           # idle slots untouched
        if rows.any():
            assert rel_err(o[t][rows], o_ref[t][rows]) <= tol_out(w), t


@pytest.mark.parametrize("op", OPS)
@pytest.mark.parametrize("dims", [(64, 64), (128, 128), (128, 64)])
@pytest.mark.parametrize("C", [1, 3, 4, 8, 16])
@pytest.mark.parametrize("mode", MODES)
def test_slots_match_oracle(op, dims, C, mode):
    T = 3 * C + 5
    w = small(op, *dims, C=C, T=T, Bsz=6, H=3, in_dt="bf16", out_dt="f32",
              seed=11 + C + 3 * op)
    rng = np.random.default_rng(1000 + 7 * C + op + dims[0])
    act, resets = _schedule(rng, T, w.B)
    new_states = {(t, s): (0.5 * rng.standard_normal((w.H, w.dk, w.dv))).astype(np.float32)
                  for t, ss in resets.items() for s in ss}
    S0 = synth.initial_state(w)
    bonus = synth.bonus(w)
    ti = synth.tokens(w, 0, T)
    x = D.to_device(ti, w)
    layer, outs, Ls = _run_gpu(w, x, S0, bonus, C, mode, act, resets, new_states)
    st, Ls_ref, o_ref, Ltr = _oracle_slots(w, ti, S0, bonus, C, act, resets, new_states)
    assert np.array_equal(Ls, Ltr)
    _compare(w, outs, o_ref, act)
    mat_ref = _oracle_materialize_slots(w, st, Ls_ref, C)
    assert rel_err(to_np(layer.materialize()), mat_ref) <= TOL_STATE
    # dl_merge folds every slot at its own length
    layer.merge()
    torch.cuda.synchronize()
    assert layer.L == 0
    assert rel_err(to_np(layer.base), mat_ref) <= TOL_STATE


@pytest.mark.parametrize("mode", MODES)
def test_slot_lists_longer_than_one_launch(mode):
    """600 slots (more than one launch's 512-slot list) at mixed lengths."""
    C, T = 3, 8
    w = small(synth.GDN, 64, 64, C=C, T=T, Bsz=600, H=1, in_dt="bf16", out_dt="bf16", seed=5)
    rng = np.random.default_rng(600)
    act, resets = _schedule(rng, T, w.B, p_active=0.8, p_reset=0.02)
    new_states = {(t, s): (0.5 * rng.standard_normal((w.H, w.dk, w.dv))).astype(np.float32)
                  for t, ss in resets.items() for s in ss}
    S0 = synth.initial_state(w)
    ti = synth.tokens(w, 0, T)
    x = D.to_device(ti, w)
    layer, outs, Ls = _run_gpu(w, x, S0, None, C, mode, act, resets, new_states)
    st, Ls_ref, o_ref, Ltr = _oracle_slots(w, ti, S0, None, C, act, resets, new_states)
    assert np.array_equal(Ls, Ltr)
    _compare(w, outs, o_ref, act)
    mat_ref = _oracle_materialize_slots(w, st, Ls_ref, C)
    assert rel_err(to_np(layer.materialize()), mat_ref) <= TOL_STATE


def _stagger(layer, w, x, C, outs):
    """Slot b takes part in the first (b mod C) tokens only: afterwards slot
    b's log holds b mod C entries."""
    for t in range(C - 1):
        layer.step(x, t, outs[t], active=[(b % C) > t for b in range(w.B)])


@pytest.mark.parametrize("op", OPS)
@pytest.mark.parametrize("mode", MODES)
def test_cycle_from_staggered_lengths(op, mode):
    """A merge cycle captured with the slots at different lengths replays the
    same bytes as the steps issued one by one, and leaves every slot's length
    where it started; a launch from other lengths is refused."""
    C = 4
    T = 2 * C - 1
    w = small(op, 128, 64, C=C, T=T, Bsz=5, H=2, in_dt="bf16", out_dt="bf16", seed=21)
    layers_a, layers_b, xs, outs_a, outs_b = [], [], [], [], []
    for l in range(2):
        S0 = synth.initial_state(w, layer=l)
        bonus = synth.bonus(w, layer=l)
        xs.append(D.to_device(synth.tokens(w, 0, T, layer=l), w))
        for lst, outl in ((layers_a, outs_a), (layers_b, outs_b)):
            lay = D.DecodeLayer(w, S0, bonus, auto_merge=mode)
            o = lay.new_out(T)
            o.zero_()                          # idle slots leave their rows as they are
            _stagger(lay, w, xs[l], C, o)
            lst.append(lay)
            outl.append(o)
    start = [[layers_b[l].slot_len(b) for b in range(w.B)] for l in range(2)]
    assert start[0] == [b % C for b in range(w.B)]
    for t in range(C - 1, T):
        for l in range(2):
            layers_a[l].step(xs[l], t, outs_a[l][t])
    ios = [[(xs[l]["q"][t], xs[l]["k"][t], xs[l]["v"][t],
             None if op == synth.RWKV6 else xs[l]["beta"][t], xs[l]["g"][t], outs_b[l][t])
            for l in range(2)] for t in range(C - 1, T)]
    cyc = B.Cycle([lb.handle for lb in layers_b], ios)
    cyc.launch()
    torch.cuda.synchronize()
    for l in range(2):
        assert [layers_b[l].slot_len(b) for b in range(w.B)] == start[l]
        assert [layers_a[l].slot_len(b) for b in range(w.B)] == start[l]
        assert torch.equal(outs_a[l], outs_b[l])
        assert torch.equal(layers_a[l].base, layers_b[l].base)
        assert torch.equal(layers_a[l].log, layers_b[l].log)
    layers_b[0].step(xs[0], 0, outs_b[0][0])
    with pytest.raises(B.DeltaLogError) as e:
        cyc.launch()
    assert e.value.status == B.DL_ESTATE
    cyc.close()


@pytest.mark.parametrize("mode", MODES)
def test_staggered_full_size(mode):
    """The GDN B128 H16 d128 C8 workload with its slots at staggered lengths
    (slot b joins b mod C tokens late), two more cycles and a ragged tail;
    sampled slots (all their heads) against the eager oracle on each slot's
    own tokens."""
    w = synth.WORKLOADS["gdn-b128-h16-d128-c8"]
    C = w.C
    T = 3 * C + 3
    S0 = synth.initial_state(w)
    ti = synth.tokens(w, 0, T, want64=False)
    x = D.to_device(ti, w)
    layer = D.DecodeLayer(w, S0, None, auto_merge=mode)
    outs = layer.new_out(T)
    outs.fill_(float("nan"))
    act = np.ones((T, w.B), bool)
    for t in range(C - 1):
        act[t] = [(b % C) > t for b in range(w.B)]
    for t in range(T):
        layer.step(x, t, outs[t], active=act[t].tolist())
    mat = layer.materialize()
    torch.cuda.synchronize()
    rng = np.random.default_rng(77)
    slots = np.unique(np.concatenate([[0, C - 1, w.B - 1], rng.choice(w.B, 5, replace=False)]))
    for s in slots:
        heads = np.arange(s * w.H, (s + 1) * w.H)
        ts = np.nonzero(act[:, s])[0]
        Sr, q, k, v, beta, g, _ = oracle_inputs(w, ti, heads=heads, S0=S0)
        S_ref, o_ref = oracle.eager_run(w.op, Sr, q[ts], k[ts], v[ts], beta[ts], g[ts], None,
                                        w.scale)
        o = to_np(outs[:, heads])
        for i, t in enumerate(ts):
            assert rel_err(o[t], o_ref[i]) <= tol_out(w), (s, t)
        assert np.all(np.isnan(o[~act[:, s]]))
        assert rel_err(to_np(mat[heads]), S_ref) <= TOL_STATE, s
        assert layer.slot_len(int(s)) == len(ts) % C
