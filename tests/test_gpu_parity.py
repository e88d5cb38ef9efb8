"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle.

Tolerances (normwise-max relative error, max|x - ref| / max|ref|, per step):
  outputs stored in fp32   1e-4
  outputs stored in bf16   2e-2
  fp32 state (materialised / eager S)   1e-4
Log-length schedule and merge points: exact.  Logged keys: bit-exact copies.
Inputs come from the seeded generator only; the oracle sees the very same
rounded values, widened to float64.
"""
import numpy as np
import pytest
import torch

import oracle
from oracle import rel_err
from recurrent_state_head_b200 import binding as B
from recurrent_state_head_b200 import device as D
from recurrent_state_head_b200 import synth

pytestmark = pytest.mark.gpu

TOL_STATE = 1e-4
OPS = (synth.GDN, synth.KDA, synth.RWKV6)
SHAPES = ((64, 64), (128, 128), (64, 128), (128, 64))


def tol_out(w):
    return 2e-2 if w.out_dtype == "bf16" else 1e-4


def small(op, dk, dv, C=4, T=12, Bsz=3, H=5, in_dt="f32", out_dt="f32", seed=7,
          init_std=0.5):
    scale = 1.0 if op == synth.RWKV6 else dk ** -0.5
    return synth.Workload(f"test-{op}-{dk}x{dv}", op, Bsz, H, dk, dv, C, T, in_dt, out_dt,
                          scale, seed, init_std)


def oracle_inputs(w, ti, heads=None, S0=None, bonus=None):
    """Float64 oracle views of the stored inputs, optionally for some heads."""
    T = ti.q.shape[0]
    NH = w.heads
    sel = (lambda a: a.reshape((T, NH) + a.shape[3:])) if heads is None else \
        (lambda a: a.reshape((T, NH) + a.shape[3:])[:, heads])
    q = synth.exact64(sel(ti.q), w.in_dtype)
    k = synth.exact64(sel(ti.k), w.in_dtype)
    v = synth.exact64(sel(ti.v), w.in_dtype)
    beta = sel(ti.beta).astype(np.float64)
    g = sel(ti.g).astype(np.float64)
    if g.ndim == 2:
        g = g[:, :, None]
    hsel = np.arange(NH) if heads is None else np.asarray(heads)
    S = S0.reshape(NH, w.dk, w.dv)[hsel].astype(np.float64)
    bon = None if bonus is None else bonus[hsel % w.H].astype(np.float64)
    return S, q, k, v, beta, g, bon


def to_np(t):
    return t.float().cpu().numpy().astype(np.float64)


def run_oracle_eager(w, S, q, k, v, beta, g, bon):
    return oracle.eager_run(w.op, S, q, k, v, None if w.op == synth.RWKV6 else beta, g, bon,
                            w.scale)


# --------------------------------------------------------------- eager ----

@pytest.mark.parametrize("op", OPS)
@pytest.mark.parametrize("dims", SHAPES)
@pytest.mark.parametrize("dts", [("f32", "f32"), ("bf16", "bf16")])
def test_eager_matches_oracle(op, dims, dts):
    w = small(op, *dims, in_dt=dts[0], out_dt=dts[1])
    S0 = synth.initial_state(w)
    bonus = synth.bonus(w)
    ti = synth.tokens(w, 0, w.T)
    x = D.to_device(ti, w)
    S = torch.from_numpy(S0).reshape(w.heads, w.dk, w.dv).cuda()
    bon_d = None if bonus is None else torch.from_numpy(bonus).cuda()
    outs = torch.empty(w.T, w.heads, w.dv, dtype=D.TORCH_DTYPE[w.out_dtype], device="cuda")
    for t in range(w.T):
        D.eager_step(w, S, x, t, bon_d, outs[t])
    torch.cuda.synchronize()
    Sr, q, k, v, beta, g, bon = oracle_inputs(w, ti, S0=S0, bonus=bonus)
    S_ref, o_ref = run_oracle_eager(w, Sr, q, k, v, beta, g, bon)
    o = to_np(outs)
    for t in range(w.T):
        assert rel_err(o[t], o_ref[t]) <= tol_out(w), t
    assert rel_err(to_np(S), S_ref) <= TOL_STATE


# ------------------------------------------------------------ DeltaLog ----

def run_deltalog(w, x, S0, bonus, C, check_every_step=None, auto_merge=1):
    layer = D.DecodeLayer(w, S0, bonus, C=C, auto_merge=auto_merge)
    outs = layer.new_out(w.T)
    Ls, mats = [], []
    for t in range(w.T):
        layer.step(x, t, outs[t])
        Ls.append(layer.L)
        if check_every_step:
            mats.append(to_np(layer.materialize()))
    torch.cuda.synchronize()
    return layer, outs, Ls, mats


MODES = (B.DL_MERGE_FOLD, B.DL_MERGE_SEPARATE)


@pytest.mark.parametrize("op", OPS)
@pytest.mark.parametrize("dims", SHAPES)
@pytest.mark.parametrize("C", [1, 2, 3, 4, 8, 16])
@pytest.mark.parametrize("mode", MODES)
def test_deltalog_matches_eager_oracle(op, dims, C, mode):
    """Outputs every token, the logical (materialised) state after every
    token and the log-length schedule, over two full cycles and a ragged
    third, with the merge folded into the C-th token or run separately."""
    w = small(op, *dims, C=C, T=2 * C + 3, seed=11 + C)
    S0 = synth.initial_state(w)
    bonus = synth.bonus(w)
    ti = synth.tokens(w, 0, w.T)
    x = D.to_device(ti, w)
    layer, outs, Ls, mats = run_deltalog(w, x, S0, bonus, C, check_every_step=True,
                                         auto_merge=mode)
    Sr, q, k, v, beta, g, bon = oracle_inputs(w, ti, S0=S0, bonus=bonus)
    st = oracle.LogState(w.op, Sr, C)
    _, L_ref, _ = oracle.deltalog_run(st, q, k, v, None if op == synth.RWKV6 else beta, g, bon,
                                      w.scale)
    assert Ls == L_ref.tolist()
    o = to_np(outs)
    S = Sr
    for t in range(w.T):
        S, o_ref = run_oracle_eager(w, S, q[t:t + 1], k[t:t + 1], v[t:t + 1], beta[t:t + 1],
                                    g[t:t + 1], bon)
        assert rel_err(o[t], o_ref[0]) <= tol_out(w), t
        assert rel_err(mats[t], S) <= TOL_STATE, t
    if layer.L == 0:
        assert rel_err(to_np(layer.base), S) <= TOL_STATE


@pytest.mark.parametrize("op", OPS)
@pytest.mark.parametrize("dims", SHAPES)
@pytest.mark.parametrize("nh", [300, 600])
@pytest.mark.parametrize("mode", MODES)
def test_deltalog_tile_widths(op, dims, nh, mode):
    """Head counts that select each value-tile width (a whole head per CTA
    while that gives four CTAs per SM, halved tiles below; on a 148-SM B200:
    600 heads -> whole heads, 300 -> 64 columns for d_v = 128, 15 heads in
    the other tests -> 32 columns).  Every head, every token, and the logical
    state after each token."""
    C = 4
    w = small(op, *dims, C=C, T=2 * C + 3, Bsz=nh // 4, H=4, seed=40 + nh)
    S0 = synth.initial_state(w)
    bonus = synth.bonus(w)
    ti = synth.tokens(w, 0, w.T)
    x = D.to_device(ti, w)
    layer, outs, Ls, mats = run_deltalog(w, x, S0, bonus, C, check_every_step=True,
                                         auto_merge=mode)
    Sr, q, k, v, beta, g, bon = oracle_inputs(w, ti, S0=S0, bonus=bonus)
    o = to_np(outs)
    S = Sr
    for t in range(w.T):
        S, o_ref = run_oracle_eager(w, S, q[t:t + 1], k[t:t + 1], v[t:t + 1], beta[t:t + 1],
                                    g[t:t + 1], bon)
        assert rel_err(o[t], o_ref[0]) <= tol_out(w), t
        assert rel_err(mats[t], S) <= TOL_STATE, t
    assert Ls == [(t + 1) % C for t in range(w.T)]


@pytest.mark.parametrize("op", OPS)
@pytest.mark.parametrize("dts", [("bf16", "bf16"), ("bf16", "f32"), ("f32", "bf16")])
def test_deltalog_mixed_dtypes(op, dts):
    w = small(op, 128, 128, C=4, T=11, in_dt=dts[0], out_dt=dts[1])
    S0 = synth.initial_state(w)
    bonus = synth.bonus(w)
    ti = synth.tokens(w, 0, w.T)
    x = D.to_device(ti, w)
    layer, outs, Ls, _ = run_deltalog(w, x, S0, bonus, w.C)
    Sr, q, k, v, beta, g, bon = oracle_inputs(w, ti, S0=S0, bonus=bonus)
    S_ref, o_ref = run_oracle_eager(w, Sr, q, k, v, beta, g, bon)
    o = to_np(outs)
    for t in range(w.T):
        assert rel_err(o[t], o_ref[t]) <= tol_out(w), t
    assert rel_err(to_np(layer.materialize()), S_ref) <= TOL_STATE


@pytest.mark.parametrize("op", OPS)
@pytest.mark.parametrize("in_dt", ["f32", "bf16"])
def test_log_contents(op, in_dt):
    """Slot j: k_j bit for bit, the step's value factor (delta-rule u, or v
    itself for RWKV6), and the cumulative log-decay since the merge."""
    C = 6
    w = small(op, 64, 128, C=C, T=C - 1, in_dt=in_dt, out_dt="f32")
    S0 = synth.initial_state(w)
    bonus = synth.bonus(w)
    ti = synth.tokens(w, 0, w.T)
    x = D.to_device(ti, w)
    layer, outs, Ls, _ = run_deltalog(w, x, S0, bonus, C)
    assert layer.L == C - 1
    K, U, Lam = layer.log_views()
    Sr, q, k, v, beta, g, bon = oracle_inputs(w, ti, S0=S0, bonus=bonus)
    _, _, u_ref = oracle.eager_run(w.op, Sr, q, k, v, None if op == synth.RWKV6 else beta, g,
                                   bon, w.scale, want_u=True)
    Kd = K.cpu()
    kin = x["k"].cpu()
    for j in range(C - 1):
        if in_dt == "bf16":
            assert torch.equal(Kd[:, j].view(torch.int16), kin[j].view(torch.int16))
        else:
            assert torch.equal(Kd[:, j].view(torch.int32), kin[j].view(torch.int32))
        assert rel_err(to_np(U[:, j]), u_ref[j]) <= TOL_STATE
        assert rel_err(to_np(Lam[:, j]), np.sum(g[:j + 1], axis=0)) <= 1e-6
    # the base is never written by an append
    assert torch.equal(layer.base.cpu(), torch.from_numpy(S0).reshape(w.heads, w.dk, w.dv))


@pytest.mark.parametrize("op", OPS)
@pytest.mark.parametrize("mode", MODES)
def test_capacity_one_equals_gpu_eager(op, mode):
    w = small(op, 128, 128, C=1, T=9)
    S0 = synth.initial_state(w)
    bonus = synth.bonus(w)
    ti = synth.tokens(w, 0, w.T)
    x = D.to_device(ti, w)
    layer, outs, Ls, _ = run_deltalog(w, x, S0, bonus, 1, auto_merge=mode)
    assert Ls == [0] * w.T
    S = torch.from_numpy(S0).reshape(w.heads, w.dk, w.dv).cuda()
    bon_d = None if bonus is None else torch.from_numpy(bonus).cuda()
    oe = torch.empty_like(outs)
    for t in range(w.T):
        D.eager_step(w, S, x, t, bon_d, oe[t])
    torch.cuda.synchronize()
    assert rel_err(to_np(outs), to_np(oe)) <= 1e-5
    assert rel_err(to_np(layer.base), to_np(S)) <= 1e-5


@pytest.mark.parametrize("op", OPS)
def test_explicit_merge_and_materialize(op):
    """auto_merge = 0: the log fills, a further step is refused (nothing
    launched), dl_merge folds a partial or full log; materialise leaves base
    and log untouched."""
    C = 5
    w = small(op, 128, 64, C=C, T=C + 2)
    S0 = synth.initial_state(w)
    bonus = synth.bonus(w)
    ti = synth.tokens(w, 0, w.T)
    x = D.to_device(ti, w)
    layer = D.DecodeLayer(w, S0, bonus, C=C, auto_merge=0)
    outs = layer.new_out(w.T)
    for t in range(C):
        layer.step(x, t, outs[t])
    assert layer.L == C
    sentinel = torch.full_like(outs[C], 7.0)
    with pytest.raises(B.DeltaLogError) as e:
        layer.step(x, C, sentinel)
    assert e.value.status == B.DL_ESTATE
    torch.cuda.synchronize()
    assert torch.all(sentinel == 7.0)
    base_before = layer.base.clone()
    log_before = layer.log.clone()
    mat = layer.materialize()
    torch.cuda.synchronize()
    assert torch.equal(layer.base, base_before) and torch.equal(layer.log, log_before)
    layer.merge()
    assert layer.L == 0
    torch.cuda.synchronize()
    assert torch.equal(layer.base, mat)
    # a partial log: two more tokens, then merge
    layer.step(x, C, outs[C])
    layer.step(x, C + 1, outs[C + 1])
    layer.merge()
    torch.cuda.synchronize()
    Sr, q, k, v, beta, g, bon = oracle_inputs(w, ti, S0=S0, bonus=bonus)
    S_ref, o_ref = run_oracle_eager(w, Sr, q, k, v, beta, g, bon)
    assert rel_err(to_np(layer.base), S_ref) <= TOL_STATE
    for t in range(w.T):
        assert rel_err(to_np(outs[t]), o_ref[t]) <= tol_out(w)


@pytest.mark.parametrize("op", OPS)
@pytest.mark.parametrize("mode", MODES)
def test_cycle_graph_equals_steps(op, mode):
    """One graph-captured merge cycle over two layers gives the same bytes as
    the same steps issued one by one."""
    C = 4
    w = small(op, 128, 128, C=C, T=C, in_dt="bf16", out_dt="bf16")
    layers_a, layers_b, xs = [], [], []
    for l in range(2):
        S0 = synth.initial_state(w, layer=l)
        bonus = synth.bonus(w, layer=l)
        xs.append(D.to_device(synth.tokens(w, 0, C, layer=l), w))
        layers_a.append(D.DecodeLayer(w, S0, bonus, auto_merge=mode))
        layers_b.append(D.DecodeLayer(w, S0, bonus, auto_merge=mode))
    outs_a = [layers_a[l].new_out(C) for l in range(2)]
    outs_b = [layers_b[l].new_out(C) for l in range(2)]
    for t in range(C):
        for l in range(2):
            layers_a[l].step(xs[l], t, outs_a[l][t])
    ios = [[(xs[l]["q"][t], xs[l]["k"][t], xs[l]["v"][t],
             None if op == synth.RWKV6 else xs[l]["beta"][t], xs[l]["g"][t], outs_b[l][t])
            for l in range(2)] for t in range(C)]
    cyc = B.Cycle([lb.handle for lb in layers_b], ios)
    assert cyc.kernels == 2 * (C + 1 if mode == B.DL_MERGE_SEPARATE else C)
    cyc.launch()
    torch.cuda.synchronize()
    for l in range(2):
        assert layers_b[l].L == 0
        assert torch.equal(outs_a[l], outs_b[l])
        assert torch.equal(layers_a[l].base, layers_b[l].base)
    cyc.close()


def test_no_heads_on_gpu():
    w = small(synth.GDN, 128, 128, C=2, T=3, Bsz=0)
    layer = D.DecodeLayer(w, np.zeros((0, 1, 128, 128), np.float32))
    for t in range(3):
        B.dl_decode_step(layer.handle.h, None, None, None, None, None, None)
    assert layer.L == 1


# ------------------------------------------------ full-size workloads ----

def _every_head(w, T=None, chunk=1024):
    """Both merge modes over T tokens of a full-size workload, then every
    head's outputs (every token) and final materialised state against the
    oracle's eager recurrence; the oracle runs once, over head chunks, and
    the per-token error is the normwise-max over all heads."""
    T = w.T if T is None else T
    S0 = synth.initial_state(w)
    bonus = synth.bonus(w)
    ti = synth.tokens(w, 0, T, want64=False)
    x = D.to_device(ti, w)
    runs = []
    for mode in MODES:
        layer = D.DecodeLayer(w, S0, bonus, auto_merge=mode)
        outs = layer.new_out(T)
        for t in range(T):
            layer.step(x, t, outs[t])
        runs.append((outs, layer.materialize(), layer.L))
        del layer
    torch.cuda.synchronize()
    del x
    for outs, _, L in runs:
        assert torch.isfinite(outs.float()).all()
        assert L == T % w.C
    num_o = np.zeros((len(runs), T))
    den_o = np.zeros(T)
    num_s = np.zeros(len(runs))
    den_s = 0.0
    for h0 in range(0, w.heads, chunk):
        heads = np.arange(h0, min(w.heads, h0 + chunk))
        Sr, q, k, v, beta, g, bon = oracle_inputs(w, ti, heads=heads, S0=S0, bonus=bonus)
        S_ref, o_ref = run_oracle_eager(w, Sr, q, k, v, beta, g, bon)
        den_o = np.maximum(den_o, np.abs(o_ref).reshape(T, -1).max(axis=1))
        den_s = max(den_s, float(np.abs(S_ref).max()))
        for i, (outs, mat, _) in enumerate(runs):
            o = to_np(outs[:, h0:h0 + len(heads)])
            num_o[i] = np.maximum(num_o[i], np.abs(o - o_ref).reshape(T, -1).max(axis=1))
            num_s[i] = max(num_s[i], float(np.abs(to_np(mat[h0:h0 + len(heads)]) - S_ref).max()))
    for i, mode in enumerate(MODES):
        worst = float((num_o[i] / den_o).max())
        assert worst <= tol_out(w), (mode, worst)
        assert num_s[i] / den_s <= TOL_STATE, (mode, num_s[i] / den_s)


def test_full_gdn_fp32_small():
    """The fp32 GDN case (B=1, H=2, d=64, C=4, 32 tokens from zero): every head."""
    w = synth.WORKLOADS["gdn-b1-h2-d64-c4-fp32"]
    S0 = synth.initial_state(w)
    ti = synth.tokens(w, 0, w.T)
    x = D.to_device(ti, w)
    layer, outs, Ls, mats = run_deltalog(w, x, S0, None, w.C, check_every_step=True)
    Sr, q, k, v, beta, g, bon = oracle_inputs(w, ti, S0=S0)
    S = Sr
    for t in range(w.T):
        S, o_ref = run_oracle_eager(w, S, q[t:t + 1], k[t:t + 1], v[t:t + 1], beta[t:t + 1],
                                    g[t:t + 1], None)
        assert rel_err(to_np(outs[t]), o_ref[0]) <= 1e-4
        assert rel_err(mats[t], S) <= TOL_STATE
    assert Ls == [(t + 1) % w.C for t in range(w.T)]


@pytest.mark.parametrize("name", ["gdn-b128-h16-d128-c8", "kda-b128-h32-d128-c4",
                                  "kda-b128-h32-d128-c8", "rwkv6-b128-h32-d64-c4",
                                  "rwkv6-b128-h32-d64-c8"])
def test_full_size_every_head(name):
    """The full-size workloads, 256 tokens, both merge modes: every head."""
    _every_head(synth.WORKLOADS[name])


@pytest.mark.parametrize("op", OPS)
@pytest.mark.parametrize("mode", MODES)
def test_checkpoint_resume(op, mode):
    """Checkpoint = materialise the logical state mid-cycle; resume = a new
    handle over that dense state with an empty log.  The resumed run's
    outputs and final state match the uninterrupted run's."""
    C = 5
    w = small(op, 128, 64, C=C, T=2 * C + 2, in_dt="bf16", out_dt="f32")
    S0 = synth.initial_state(w)
    bonus = synth.bonus(w)
    ti = synth.tokens(w, 0, w.T)
    x = D.to_device(ti, w)
    ref, outs_ref, _, _ = run_deltalog(w, x, S0, bonus, C, auto_merge=mode)
    cut = C + 2                                   # mid-cycle: L = 2
    first = D.DecodeLayer(w, S0, bonus, C=C, auto_merge=mode)
    outs = first.new_out(w.T)
    for t in range(cut):
        first.step(x, t, outs[t])
    assert first.L == 2
    ckpt = first.materialize().cpu().numpy()
    second = D.DecodeLayer(w, ckpt.reshape(w.B, w.H, w.dk, w.dv), bonus, C=C, auto_merge=mode)
    for t in range(cut, w.T):
        second.step(x, t, outs[t])
    torch.cuda.synchronize()
    assert rel_err(to_np(outs), to_np(outs_ref)) <= 1e-5
    assert rel_err(to_np(second.materialize()), to_np(ref.materialize())) <= 1e-5


@pytest.mark.parametrize("op", OPS)
@pytest.mark.parametrize("mode", MODES)
def test_strong_decay_long_log(op, mode):
    """C = 16 with log-decays eight times the usual scale (the cumulative
    decay over a cycle reaches e^-100): outputs and states against the
    eager oracle, no overflow or NaN in the replay factors."""
    C = 16
    w = small(op, 128, 64, C=C, T=2 * C + 5, in_dt="bf16", out_dt="f32", seed=91)
    S0 = synth.initial_state(w)
    bonus = synth.bonus(w)
    ti = synth.tokens(w, 0, w.T)
    ti.g[...] = (ti.g.astype(np.float64) * 8.0).astype(np.float32)
    x = D.to_device(ti, w)
    layer, outs, Ls, mats = run_deltalog(w, x, S0, bonus, C, check_every_step=True,
                                         auto_merge=mode)
    Sr, q, k, v, beta, g, bon = oracle_inputs(w, ti, S0=S0, bonus=bonus)
    S = Sr
    o = to_np(outs)
    assert np.all(np.isfinite(o))
    for t in range(w.T):
        S, o_ref = run_oracle_eager(w, S, q[t:t + 1], k[t:t + 1], v[t:t + 1], beta[t:t + 1],
                                    g[t:t + 1], bon)
        assert rel_err(o[t], o_ref[0]) <= tol_out(w), t
        assert rel_err(mats[t], S) <= TOL_STATE, t
