"""Pins of the fp64 oracle against facts that do not come from the oracle.

Each test fixes the oracle to something other than its own code: values
worked by hand (tests/golden), closed forms of special cases, published
alternative forms of the same recurrences (the generalised-Householder
transition of Gated DeltaNet / KDA, the parallel attention form of RWKV6),
library matrix products, and brute force of the base + log formulation
against the eager recurrence on tiny inputs.  Shapes are kept non-square
(d_k != d_v) so that a transposed operand cannot pass.
"""
import math
import os

import numpy as np
import pytest

import oracle
from oracle import GDN, KDA, RWKV6, LogState, rel_err

OPS = (GDN, KDA, RWKV6)
GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
TIGHT = 1e-12


def rand_inputs(rng, op, nh, dk, dv, T, *, unit_k=True, g_scale=1.0):
    q = rng.standard_normal((T, nh, dk))
    k = rng.standard_normal((T, nh, dk))
    if unit_k and op != RWKV6:
        q /= np.linalg.norm(q, axis=-1, keepdims=True)
        k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.standard_normal((T, nh, dv))
    beta = 1.0 / (1.0 + np.exp(-rng.standard_normal((T, nh))))
    m = oracle.decay_width(op, dk)
    g = -np.log1p(np.exp(rng.standard_normal((T, nh, m)))) * g_scale
    bonus = rng.standard_normal((nh, dk)) * 0.1 if op == RWKV6 else None
    return q, k, v, beta, g, bonus


# ------------------------------------------------------------------ golden --

def _read_golden(name):
    rec = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            key, *vals = line.split()
            rec[key] = vals
    return rec


@pytest.mark.parametrize("fname", ["gdn_worked_2x2.txt", "kda_worked_2x2.txt",
                                   "rwkv6_worked_2x2.txt"])
def test_golden_worked_examples(oracle_lib, fname):
    rec = _read_golden(fname)
    op = {"gdn": GDN, "kda": KDA, "rwkv6": RWKV6}[rec["op"][0]]
    dk, dv = int(rec["dk"][0]), int(rec["dv"][0])
    scale = float(rec["scale"][0])
    f = lambda key: np.array([float(x) for x in rec[key]])  # noqa: E731
    S0 = f("S0").reshape(1, dk, dv)
    bonus = f("bonus").reshape(1, dk) if "bonus" in rec else None
    T = 2
    q = np.stack([f(f"t{t}.q") for t in (1, 2)]).reshape(T, 1, dk)
    k = np.stack([f(f"t{t}.k") for t in (1, 2)]).reshape(T, 1, dk)
    v = np.stack([f(f"t{t}.v") for t in (1, 2)]).reshape(T, 1, dv)
    beta = (np.array([f(f"t{t}.beta")[0] for t in (1, 2)]).reshape(T, 1)
            if op != RWKV6 else None)
    g = np.stack([np.log(f(f"t{t}.alpha")) for t in (1, 2)]).reshape(T, 1, -1)
    # step by step, so that the state after each step is checked
    S = S0
    for t in range(T):
        S, out, u = oracle.eager_run(op, S, q[t:t + 1], k[t:t + 1], v[t:t + 1],
                                     None if beta is None else beta[t:t + 1],
                                     g[t:t + 1], bonus, scale, want_u=True)
        np.testing.assert_allclose(S.reshape(-1), f(f"t{t + 1}.S"), rtol=0, atol=1e-13)
        np.testing.assert_allclose(out.reshape(-1), f(f"t{t + 1}.o"), rtol=0, atol=1e-13)
        np.testing.assert_allclose(u.reshape(-1), f(f"t{t + 1}.u"), rtol=0, atol=1e-13)
    # the base + log formulation reaches the same outputs at every capacity
    for C in (1, 2, 3):
        st = LogState(op, S0, C)
        out, _, _ = oracle.deltalog_run(st, q, k, v, beta, g, bonus, scale)
        for t in range(T):
            np.testing.assert_allclose(out[t].reshape(-1), f(f"t{t + 1}.o"),
                                       rtol=0, atol=1e-13)
        np.testing.assert_allclose(oracle.materialize(st).reshape(-1), f("t2.S"),
                                   rtol=0, atol=1e-13)


# ------------------------------------------------------- closed-form cases --

@pytest.mark.parametrize("op", [GDN, KDA])
def test_no_decay_no_write_keeps_state(oracle_lib, op):
    """alpha = 1 (g = 0) and beta = 0: the state is unchanged, o = scale S^T q."""
    rng = np.random.default_rng(1)
    nh, dk, dv, T = 3, 5, 7, 6
    S0 = rng.standard_normal((nh, dk, dv))
    q, k, v, beta, g, _ = rand_inputs(rng, op, nh, dk, dv, T)
    S, out = oracle.eager_run(op, S0, q, k, v, np.zeros_like(beta), np.zeros_like(g),
                              scale=0.5)
    assert np.array_equal(S, S0)
    ref = 0.5 * np.einsum("hij,thi->thj", S0, q)
    assert rel_err(out, ref) < TIGHT


@pytest.mark.parametrize("op", [GDN, KDA])
def test_delta_rule_writes_value_exactly(oracle_lib, op):
    """beta = 1, |k| = 1: after the step S_t^T k_t = v_t, whatever the decay."""
    rng = np.random.default_rng(2)
    nh, dk, dv, T = 2, 6, 4, 9
    S0 = rng.standard_normal((nh, dk, dv))
    q, k, v, beta, g, _ = rand_inputs(rng, op, nh, dk, dv, T)
    S = S0
    for t in range(T):
        S, _ = oracle.eager_run(op, S, q[t:t + 1], k[t:t + 1], v[t:t + 1],
                                np.ones((1, nh)), g[t:t + 1])
        recall = np.einsum("hij,hi->hj", S, k[t])
        assert rel_err(recall, v[t]) < TIGHT


@pytest.mark.parametrize("op", OPS)
def test_zero_state_single_step(oracle_lib, op):
    """From S = 0 one step gives the rank-one write and its readout."""
    rng = np.random.default_rng(3)
    nh, dk, dv = 4, 3, 5
    q, k, v, beta, g, bonus = rand_inputs(rng, op, nh, dk, dv, 1)
    S, out = oracle.eager_run(op, np.zeros((nh, dk, dv)), q, k, v, beta, g, bonus,
                              scale=0.25)
    if op == RWKV6:
        S_ref = np.einsum("hi,hj->hij", k[0], v[0])
        o_ref = 0.25 * np.einsum("hi,hi->h", q[0], bonus * k[0])[:, None] * v[0]
    else:
        S_ref = beta[0][:, None, None] * np.einsum("hi,hj->hij", k[0], v[0])
        o_ref = 0.25 * (beta[0] * np.einsum("hi,hi->h", k[0], q[0]))[:, None] * v[0]
    assert rel_err(S, S_ref) < TIGHT
    assert rel_err(out[0], o_ref) < TIGHT


@pytest.mark.parametrize("op", OPS)
def test_decay_only(oracle_lib, op):
    """beta = 0 (GDN/KDA) or k = 0 (RWKV6): only the decay acts on the state."""
    rng = np.random.default_rng(4)
    nh, dk, dv, T = 2, 4, 6, 7
    S0 = rng.standard_normal((nh, dk, dv))
    q, k, v, beta, g, bonus = rand_inputs(rng, op, nh, dk, dv, T)
    if op == RWKV6:
        k = np.zeros_like(k)
    S, out = oracle.eager_run(op, S0, q, k, v, np.zeros_like(beta), g, bonus)
    cum = np.cumsum(g, axis=0)                       # [T, nh, m]
    dec = np.exp(cum[-1])                            # [nh, m]
    assert rel_err(S, dec[:, :, None] * S0) < TIGHT
    for t in range(T):
        # GDN/KDA read the state after the step's decay, RWKV6 before it
        c = cum[t] if op != RWKV6 else (cum[t - 1] if t else np.zeros_like(cum[0]))
        St = np.exp(c)[:, :, None] * S0
        assert rel_err(out[t], np.einsum("hij,hi->hj", St, q[t])) < TIGHT


def test_associative_recall_orthonormal_keys(oracle_lib):
    """alpha = 1, beta = 1, orthonormal keys written in turn: each is recalled."""
    rng = np.random.default_rng(5)
    nh, dk, dv = 2, 6, 3
    Q, _ = np.linalg.qr(rng.standard_normal((dk, dk)))
    keys = Q.T                                        # rows orthonormal
    S0 = rng.standard_normal((nh, dk, dv))
    T = dk
    k = np.broadcast_to(keys[:, None, :], (T, nh, dk)).copy()
    v = rng.standard_normal((T, nh, dv))
    q = k.copy()
    for op in (GDN, KDA):
        m = oracle.decay_width(op, dk)
        S, _ = oracle.eager_run(op, S0, q, k, v, np.ones((T, nh)), np.zeros((T, nh, m)))
        for i in range(T):
            assert rel_err(np.einsum("hij,i->hj", S, keys[i]), v[i]) < 1e-11


@pytest.mark.parametrize("op", [GDN, KDA])
def test_householder_transition_form(oracle_lib, op):
    """Published transition form of the gated delta rule, in d_k x d_v layout:
    GDN  S_t = alpha_t (I - beta_t k k^T) S_{t-1} + beta_t k v^T
    KDA  S_t = (I - beta_t k k^T) D(a_t) S_{t-1} + beta_t k v^T
    evaluated with dense matrix products, o_t = scale S_t^T q_t."""
    rng = np.random.default_rng(6)
    nh, dk, dv, T = 3, 5, 4, 8
    S0 = rng.standard_normal((nh, dk, dv))
    q, k, v, beta, g, _ = rand_inputs(rng, op, nh, dk, dv, T)
    S_or, out_or = oracle.eager_run(op, S0, q, k, v, beta, g, scale=0.3)
    I = np.eye(dk)
    for h in range(nh):
        S = S0[h].copy()
        for t in range(T):
            kk = k[t, h][:, None]
            P = I - beta[t, h] * (kk @ kk.T)
            D = np.diag(np.exp(np.broadcast_to(g[t, h], (dk,))))
            S = P @ D @ S + beta[t, h] * (kk @ v[t, h][None, :])
            assert rel_err(out_or[t, h], 0.3 * S.T @ q[t, h]) < 1e-11
        assert rel_err(S_or[h], S) < 1e-11


def test_rwkv6_no_decay_is_sum_of_outer_products(oracle_lib):
    """w = 1: S_T = S_0 + K^T V (a single matrix product)."""
    rng = np.random.default_rng(7)
    nh, dk, dv, T = 2, 5, 3, 10
    S0 = rng.standard_normal((nh, dk, dv))
    q, k, v, _, g, bonus = rand_inputs(rng, RWKV6, nh, dk, dv, T)
    S, _ = oracle.eager_run(RWKV6, S0, q, k, v, None, np.zeros_like(g), bonus)
    for h in range(nh):
        assert rel_err(S[h], S0[h] + k[:, h].T @ v[:, h]) < TIGHT


def test_rwkv6_parallel_attention_form(oracle_lib):
    """RWKV6 output in its parallel form: o_t = scale (sum_{s<t} (r_t * k_s *
    prod_{s<tau<t} w_tau) . 1 v_s + (r_t . (u * k_t)) v_t + (prod_{tau<t} w_tau * r_t)^T S_0)."""
    rng = np.random.default_rng(8)
    nh, dk, dv, T = 2, 4, 3, 7
    S0 = rng.standard_normal((nh, dk, dv))
    q, k, v, _, g, bonus = rand_inputs(rng, RWKV6, nh, dk, dv, T)
    _, out = oracle.eager_run(RWKV6, S0, q, k, v, None, g, bonus, scale=1.5)
    cum = np.concatenate([np.zeros((1, nh, dk)), np.cumsum(g, axis=0)])  # cum[t] = sum_{tau<t}
    for h in range(nh):
        for t in range(T):
            acc = (np.exp(cum[t, h]) * q[t, h]) @ S0[h]
            for s in range(t):
                wdec = np.exp(cum[t, h] - cum[s + 1, h])     # decays of steps s+1..t-1
                acc = acc + np.sum(q[t, h] * k[s, h] * wdec) * v[s, h]
            acc = acc + np.sum(q[t, h] * bonus[h] * k[t, h]) * v[t, h]
            assert rel_err(out[t, h], 1.5 * acc) < 1e-11


# -------------------------------------------------- base + log vs eager -----

@pytest.mark.parametrize("op", OPS)
@pytest.mark.parametrize("dims", [(2, 3), (3, 2), (4, 4)])
def test_base_log_matches_eager_bruteforce(oracle_lib, op, dims):
    """Every capacity C = 1..5, T = 3C tokens: outputs and the materialised
    logical state equal the eager recurrence after every token."""
    dk, dv = dims
    nh = 2
    for C in range(1, 6):
        rng = np.random.default_rng(100 * C + dk)
        T = 3 * C
        S0 = rng.standard_normal((nh, dk, dv))
        q, k, v, beta, g, bonus = rand_inputs(rng, op, nh, dk, dv, T)
        st = LogState(op, S0, C)
        S = S0
        for t in range(T):
            sl = slice(t, t + 1)
            S, o_e = oracle.eager_run(op, S, q[sl], k[sl], v[sl],
                                      None if op == RWKV6 else beta[sl], g[sl], bonus, 0.7)
            o_l, Ltr, mg = oracle.deltalog_run(st, q[sl], k[sl], v[sl],
                                               None if op == RWKV6 else beta[sl], g[sl],
                                               bonus, 0.7)
            assert rel_err(o_l, o_e) < TIGHT, (C, t)
            assert rel_err(oracle.materialize(st), S) < TIGHT, (C, t)
            assert st.L == (t + 1) % C


@pytest.mark.parametrize("op", OPS)
def test_base_log_with_strong_decay_over_a_long_log(oracle_lib, op):
    """C = 16 with log-decays eight times the usual scale: the cumulative
    decay over a cycle reaches e^-100 and below.  The replay factors
    e^(Lambda_t - Lambda_j) stay bounded by 1, so the base + log formulation
    still equals the eager recurrence (a formulation that divided the keys
    by the decay would overflow here)."""
    rng = np.random.default_rng(41 + op)
    nh, dk, dv, C, T = 2, 4, 3, 16, 40
    S0 = rng.standard_normal((nh, dk, dv))
    q, k, v, beta, g, bonus = rand_inputs(rng, op, nh, dk, dv, T, g_scale=8.0)
    b_ = None if op == RWKV6 else beta
    S_e, o_e = oracle.eager_run(op, S0, q, k, v, b_, g, bonus, 0.5)
    st = LogState(op, S0, C)
    o_l, _, _ = oracle.deltalog_run(st, q, k, v, b_, g, bonus, 0.5)
    assert np.all(np.isfinite(o_l)) and np.all(np.isfinite(st.base))
    assert rel_err(o_l, o_e) < 1e-11
    assert rel_err(oracle.materialize(st), S_e) < 1e-11


@pytest.mark.parametrize("op", OPS)
def test_capacity_one_is_eager(oracle_lib, op):
    rng = np.random.default_rng(9)
    nh, dk, dv, T = 3, 8, 5, 20
    S0 = rng.standard_normal((nh, dk, dv))
    q, k, v, beta, g, bonus = rand_inputs(rng, op, nh, dk, dv, T)
    S_e, o_e = oracle.eager_run(op, S0, q, k, v, beta, g, bonus, 0.5)
    st = LogState(op, S0, 1)
    o_l, Ltr, mg = oracle.deltalog_run(st, q, k, v, beta, g, bonus, 0.5)
    assert rel_err(o_l, o_e) < TIGHT
    assert rel_err(st.base, S_e) < TIGHT
    assert np.all(Ltr == 0) and np.all(mg == 1)


@pytest.mark.parametrize("op", OPS)
def test_log_contents(oracle_lib, op):
    """Slot j holds k_j, the eager step's value factor u_j, and the cumulative
    log-decay since the last merge (inclusive of step j)."""
    rng = np.random.default_rng(10)
    nh, dk, dv, C = 2, 4, 3, 5
    T = C - 1
    S0 = rng.standard_normal((nh, dk, dv))
    q, k, v, beta, g, bonus = rand_inputs(rng, op, nh, dk, dv, T)
    _, _, u = oracle.eager_run(op, S0, q, k, v, beta, g, bonus, want_u=True)
    st = LogState(op, S0, C)
    oracle.deltalog_run(st, q, k, v, beta, g, bonus)
    assert st.L == T
    assert np.array_equal(st.base, S0)                  # append never touches the base
    for j in range(T):
        assert np.array_equal(st.K[:, j], k[j])
        assert rel_err(st.U[:, j], u[j]) < TIGHT
        assert rel_err(st.Lam[:, j], np.sum(g[:j + 1], axis=0)) < TIGHT


@pytest.mark.parametrize("op", OPS)
def test_merge_properties(oracle_lib, op):
    rng = np.random.default_rng(11)
    nh, dk, dv, C = 2, 3, 4, 6
    S0 = rng.standard_normal((nh, dk, dv))
    q, k, v, beta, g, bonus = rand_inputs(rng, op, nh, dk, dv, 4)
    st = LogState(op, S0, C)
    before = st.base.copy()
    oracle.merge(st)                                    # L = 0: identity
    assert np.array_equal(st.base, before) and st.L == 0
    oracle.deltalog_run(st, q, k, v, beta, g, bonus)
    mat = oracle.materialize(st)
    oracle.merge(st)
    assert st.L == 0
    assert np.array_equal(st.base, mat)
    # after the merge the decode continues from the materialised state
    S_e, _ = oracle.eager_run(op, S0, q, k, v, beta, g, bonus)
    assert rel_err(st.base, S_e) < TIGHT


@pytest.mark.parametrize("C", [1, 2, 3, 4, 8, 16])
@pytest.mark.parametrize("L0", [0, 1])
def test_schedule(oracle_lib, C, L0):
    if L0 >= C:
        pytest.skip("start length must be below capacity")
    T = 3 * C + 2
    st = LogState(GDN, np.zeros((0, 2, 2)), C, L=L0)
    z = np.zeros((T, 0, 2))
    _, Ltr, mg = oracle.deltalog_run(st, z, z, z, np.zeros((T, 0)), np.zeros((T, 0, 1)))
    exp_L = [(L0 + t + 1) % C for t in range(T)]
    exp_m = [int((L0 + t + 1) % C == 0) for t in range(T)]
    assert Ltr.tolist() == exp_L and mg.tolist() == exp_m
    assert st.L == exp_L[-1]


# ---------------------------------------------------- per-slot log lengths --

def _slot_mask(rng, T, nslots, p=0.6):
    act = rng.random((T, nslots)) < p
    act[0, :] = True
    return act


@pytest.mark.parametrize("op", OPS)
@pytest.mark.parametrize("C", [1, 2, 3, 5])
def test_slots_match_eager_on_each_slots_tokens(oracle_lib, op, C):
    """Continuous batching: every slot, on its own, is the eager recurrence
    over the tokens it took part in (from the state it had on entry), and its
    log length counts those tokens modulo C.  Entry lengths differ (a common
    prefix of 1 or 2 tokens is decoded first), idle slots are not touched."""
    rng = np.random.default_rng(300 + 10 * op + C)
    nslots, H, dk, dv, T = 3, 2, 3, 2, 4 * C + 3
    nh = nslots * H
    S0 = rng.standard_normal((nh, dk, dv))
    q, k, v, beta, g, bonus = rand_inputs(rng, op, nh, dk, dv, T + 2)
    b_ = None if op == RWKV6 else beta
    st = LogState(op, S0, C)
    pre = 1 + (C > 2)                                     # common prefix
    o_pre, _, _ = oracle.deltalog_run(st, q[:pre], k[:pre], v[:pre],
                                      None if b_ is None else b_[:pre], g[:pre], bonus, 0.6)
    Ls = np.full(nslots, st.L, dtype=np.int32)
    act = _slot_mask(rng, T, nslots)
    sl = slice(pre, pre + T)
    out, Ltr = oracle.deltalog_slots_run(st, H, Ls, act, q[sl], k[sl], v[sl],
                                         None if b_ is None else b_[sl], g[sl], bonus, 0.6)
    for s in range(nslots):
        hs = slice(s * H, (s + 1) * H)
        ts = [pre + t for t in range(T) if act[t, s]]
        idx = list(range(pre)) + ts
        S_e, o_e = oracle.eager_run(op, S0[hs], q[idx][:, hs], k[idx][:, hs], v[idx][:, hs],
                                    None if b_ is None else b_[idx][:, hs], g[idx][:, hs],
                                    None if bonus is None else bonus[hs], 0.6)
        got = out[[t - pre for t in ts]][:, hs]
        assert rel_err(got, o_e[pre:]) < TIGHT, s
        assert np.all(np.isnan(out[~act[:, s]][:, hs])), s
        mat = oracle.materialize(LogState(op, st.base[hs], C, int(Ls[s]), st.K[hs], st.U[hs],
                                          st.Lam[hs]))
        assert rel_err(mat, S_e) < TIGHT, s
        count = pre + np.cumsum(act[:, s])
        assert Ltr[:, s].tolist() == (count % C).tolist()
        assert Ls[s] == count[-1] % C


@pytest.mark.parametrize("op", OPS)
def test_slots_all_active_is_the_shared_schedule(oracle_lib, op):
    """With every slot active every token the per-slot run is the shared-length
    run, to the last bit."""
    rng = np.random.default_rng(77 + op)
    nslots, H, dk, dv, C, T = 2, 3, 4, 3, 3, 8
    nh = nslots * H
    S0 = rng.standard_normal((nh, dk, dv))
    q, k, v, beta, g, bonus = rand_inputs(rng, op, nh, dk, dv, T)
    b_ = None if op == RWKV6 else beta
    a = LogState(op, S0, C, L=1)
    b = LogState(op, S0, C, L=1)
    o_a, Ltr, _ = oracle.deltalog_run(a, q, k, v, b_, g, bonus, 0.5)
    Ls = np.ones(nslots, dtype=np.int32)
    o_b, Ltr_b = oracle.deltalog_slots_run(b, H, Ls, np.ones((T, nslots), bool), q, k, v, b_, g,
                                           bonus, 0.5)
    assert np.array_equal(o_a, o_b)
    assert np.array_equal(a.base, b.base) and np.array_equal(a.U, b.U)
    assert np.all(Ltr_b == Ltr[:, None]) and np.all(Ls == a.L)


def test_rel_err_definition():
    assert rel_err([1.0, -2.0], [1.0, -2.0]) == 0.0
    assert math.isclose(rel_err([1.1, -2.0], [1.0, -2.0]), 0.05)
    assert rel_err([0.0], [0.0]) == 0.0
