"""The oracle's pins have teeth: a copy of the oracle with one plausible
mistake planted (a dropped term, a wrong sign, a wrong index, a decay applied
at the wrong time) must fail at least one pin.  Mistakes are planted only in
temporary copies of the C source, compiled on the CPU."""
import os
import subprocess

import pytest

import oracle
from oracle import oracle as oracle_mod

import test_oracle_pins as pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "deltalog_oracle.c")

MUTANTS = {
    "eager decay dropped":
        ("S[(size_t)i * dv + c] *= a;", "S[(size_t)i * dv + c] *= 1.0 + 0.0 * a;"),
    "delta rule sign":
        ("double u = beta * (v[c] - pred);", "double u = beta * (v[c] + pred);"),
    "delta rule without beta":
        ("double u = beta * (v[c] - pred);", "double u = (v[c] - pred);"),
    "rwkv6 bonus dropped":
        ("out[c] = scale * (acc + rb * v[c]);", "out[c] = scale * acc;"),
    "rwkv6 decay after write":
        ("S[(size_t)i * dv + c] = w * S[(size_t)i * dv + c] + k[i] * v[c];",
         "S[(size_t)i * dv + c] = w * (S[(size_t)i * dv + c] + k[i] * v[c]);"),
    "kda decay as scalar":
        ("double a = exp(g[didx(op, i)]);", "double a = exp(g[0]);"),
    "log snapshot excludes own decay":
        ("lam_t[x] = lam_prev[x] + g[x];", "lam_t[x] = lam_prev[x];"),
    "replay decay dropped":
        ("double e = exp(lam_t[x] - Lam[(size_t)j * m + x]) * K[(size_t)j * dk + i];",
         "double e = K[(size_t)j * dk + i];"),
    "merge base decay dropped":
        ("double gam = exp(lamL);", "double gam = 1.0;"),
    "self term dropped":
        ("out[c] = scale * (xq + rq + kq * u[c]);", "out[c] = scale * (xq + rq);"),
    "rwkv6 readout uses current decay":
        ("xr += base[(size_t)i * dv + c] * exp(lam_prev[i]) * q[i];",
         "xr += base[(size_t)i * dv + c] * exp(lam_t[i]) * q[i];"),
    "value replay uses key coefficient":
        ("rq += dj[j] * U[(size_t)j * dv + c];", "rq += cj[j] * U[(size_t)j * dv + c];"),
    "idle slot still decodes":
        ("if (!active[(size_t)t * nslots + s]) continue;",
         "if (0 && !active[(size_t)t * nslots + s]) continue;"),
    "merge replays one entry too few":
        ("for (int j = 0; j < L; ++j) s += coef[j] * U[(size_t)j * dv + c];",
         "for (int j = 0; j + 1 < L; ++j) s += coef[j] * U[(size_t)j * dv + c];"),
    "output scale dropped":
        ("out[c] = scale * acc;", "out[c] = acc;"),
    "replay reads the next snapshot":
        ("Lam[(size_t)j * m + x]) * K[(size_t)j * dk + i]",
         "Lam[(size_t)(j + 1 < L ? j + 1 : j) * m + x]) * K[(size_t)j * dk + i]"),
    "base read-out decays to the previous snapshot":
        ("double gam = exp(lam_t[didx(op, i)]);", "double gam = exp(lam_prev[didx(op, i)]);"),
    "merge decays to the first snapshot":
        ("double lamL = L > 0 ? Lam[(size_t)(L - 1) * m + x] : 0.0;",
         "double lamL = L > 0 ? Lam[x] : 0.0;"),
    "self term uses k.k":
        ("kq += k[i] * q[i];", "kq += k[i] * k[i];"),
    "rwkv6 bonus without the key":
        ("rb += q[i] * bonus[i] * k[i];", "rb += q[i] * bonus[i];"),
    "read-out with the key":
        ("acc += S[(size_t)i * dv + c] * q[i];", "acc += S[(size_t)i * dv + c] * k[i];"),
    "log stores the previous snapshot":
        ("Lam[(size_t)L * m + x] = lam_t[x];", "Lam[(size_t)L * m + x] = lam_prev[x];"),
    "log stores the query as key":
        ("K[(size_t)L * dk + i] = k[i];", "K[(size_t)L * dk + i] = q[i];"),
    "merge one token early":
        ("if (L == C) {", "if (L == C - 1 || L == C) {"),
    "rwkv6 read-out from the base without decay":
        ("xr += base[(size_t)i * dv + c] * exp(lam_prev[i]) * q[i];",
         "xr += base[(size_t)i * dv + c] * q[i];"),
}

PIN_CALLS = [
    lambda: [pins.test_golden_worked_examples(None, f) for f in
             ("gdn_worked_2x2.txt", "kda_worked_2x2.txt", "rwkv6_worked_2x2.txt")],
    lambda: [pins.test_no_decay_no_write_keeps_state(None, op) for op in (0, 1)],
    lambda: [pins.test_delta_rule_writes_value_exactly(None, op) for op in (0, 1)],
    lambda: [pins.test_zero_state_single_step(None, op) for op in (0, 1, 2)],
    lambda: [pins.test_decay_only(None, op) for op in (0, 1, 2)],
    lambda: [pins.test_householder_transition_form(None, op) for op in (0, 1)],
    lambda: pins.test_rwkv6_parallel_attention_form(None),
    lambda: [pins.test_base_log_matches_eager_bruteforce(None, op, d)
             for op in (0, 1, 2) for d in ((2, 3), (3, 2))],
    lambda: [pins.test_log_contents(None, op) for op in (0, 1, 2)],
    lambda: [pins.test_merge_properties(None, op) for op in (0, 1, 2)],
    lambda: [pins.test_slots_match_eager_on_each_slots_tokens(None, op, C)
             for op in (0, 1, 2) for C in (1, 3)],
]


def _failures():
    n = 0
    for call in PIN_CALLS:
        try:
            call()
        except AssertionError:
            n += 1
    return n


def test_unmutated_copy_passes(tmp_path):
    oracle.build()
    assert _failures() == 0


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_mistake_is_caught(tmp_path, name):
    old, new = MUTANTS[name]
    src = open(SRC).read()
    assert src.count(old) >= 1, f"mutation site not found: {old}"
    mutated = src.replace(old, new)
    c = tmp_path / "mutant.c"
    so = tmp_path / "mutant.so"
    c.write_text(mutated)
    subprocess.run(["gcc", "-O2", "-fopenmp", "-std=c11", "-shared", "-fPIC", str(c),
                    "-o", str(so), "-lm"], check=True)
    prev = oracle_mod._use_library(str(so))
    try:
        caught = _failures()
    finally:
        oracle_mod._restore_library(prev)
    assert caught >= 1, f"no pin caught the planted mistake: {name}"
