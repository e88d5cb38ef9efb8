"""ctypes front end of the fp64 C oracle (deltalog_oracle.c).

TEST INFRASTRUCTURE ONLY: the test suite, the package smoke check and the
benchmark's CPU-baseline leg may call it; the CUDA path never does.

Follows "DeltaLog: Deferred Materialization of Recurrent States for Linear
Attention Decoding" (arXiv 2608.15533): the eager recurrences of the three
operators named in its technical summary (GDN, KDA, RWKV6) and the base +
bounded log formulation with its append / merge schedule (Fig. 4 caption;
technical summary, "Meccanismo Core: Base + Log").  Every array crossing
into C is float64 and C-contiguous; inputs in narrower types are widened
exactly before the call.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

GDN, KDA, RWKV6 = 0, 1, 2
OP_NAMES = {GDN: "gdn", KDA: "kda", RWKV6: "rwkv6"}

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "deltalog_oracle.c")
_LIB = os.path.join(_HERE, "_liboracle.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (fp64, -O2, OpenMP). Returns the .so path."""
    if (not force and os.path.exists(_LIB)
            and os.path.getmtime(_LIB) >= os.path.getmtime(_SRC)):
        return _LIB
    tmp = _LIB + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-fopenmp", "-std=c11", "-Wall", "-shared", "-fPIC",
           _SRC, "-o", tmp, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            P = ctypes.c_void_p
            i, d = ctypes.c_int, ctypes.c_double
            lib.oracle_eager_run.argtypes = [i, i, i, i, i, d, P, P, P, P, P, P, P, P, P, i]
            lib.oracle_deltalog_run.argtypes = [i, i, i, i, i, i, d, P, P, P, P, P,
                                                P, P, P, P, P, P, P, P, P, i]
            lib.oracle_deltalog_slots_run.argtypes = [i, i, i, i, i, i, i, d, P, P, P, P, P, P,
                                                      P, P, P, P, P, P, P, P, i]
            lib.oracle_materialize.argtypes = [i, i, i, i, i, i, P, P, P, P, P]
            lib.oracle_merge.argtypes = [i, i, i, i, i, i, P, P, P, P]
            lib.oracle_max_threads.argtypes = []
            for f in ("oracle_eager_run", "oracle_deltalog_run", "oracle_deltalog_slots_run",
                      "oracle_materialize", "oracle_merge", "oracle_max_threads"):
                getattr(lib, f).restype = ctypes.c_int
            _lib = lib
    return _lib


def _use_library(path):
    """Swap the loaded oracle library for another build of the same source
    (used by the tests that plant mistakes in a copy of it). Returns the
    previous library so that it can be put back."""
    global _lib
    prev = _load()
    if path is None:
        return prev
    lib = ctypes.CDLL(path)
    for f in ("oracle_eager_run", "oracle_deltalog_run", "oracle_deltalog_slots_run",
              "oracle_materialize", "oracle_merge", "oracle_max_threads"):
        getattr(lib, f).argtypes = getattr(prev, f).argtypes
        getattr(lib, f).restype = ctypes.c_int
    with _lock:
        _lib = lib
    return prev


def _restore_library(lib):
    global _lib
    with _lock:
        _lib = lib


def decay_width(op: int, dk: int) -> int:
    """Width of the per-step log-decay g: 1 for GDN (scalar), d_k otherwise."""
    return 1 if op == GDN else dk


def max_threads() -> int:
    return int(_load().oracle_max_threads())


def _f64(a, shape=None):
    if a is None:
        return None
    a = np.ascontiguousarray(np.asarray(a, dtype=np.float64))
    if shape is not None and a.shape != tuple(shape):
        a = a.reshape(shape)
    return a


def _p(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _threads(n):
    if n is None or n <= 0:
        return max(1, len(os.sched_getaffinity(0)))
    return int(n)


def eager_run(op, S0, q, k, v, beta, g, bonus=None, scale=1.0, n_threads=None,
              want_u=False):
    """Eager recurrence over T tokens (the plain definition).

    S0 [nh, dk, dv]; q, k [T, nh, dk]; v [T, nh, dv]; beta [T, nh] (ignored
    for RWKV6); g [T, nh, m] log-decay; bonus [nh, dk] (RWKV6 only).
    Returns (S_T, out [T, nh, dv]) and, with want_u, the value factor of each
    step u [T, nh, dv] (the delta-rule u; v itself for RWKV6).
    """
    S = _f64(S0).copy()
    nh, dk, dv = S.shape
    q = _f64(q); T = q.shape[0]
    m = decay_width(op, dk)
    k = _f64(k); v = _f64(v)
    g = _f64(g, (T, nh, m))
    beta = _f64(beta, (T, nh)) if beta is not None else np.zeros((T, nh))
    bonus = _f64(bonus, (nh, dk)) if bonus is not None else (
        np.zeros((nh, dk)) if op == RWKV6 else None)
    assert q.shape == (T, nh, dk) and k.shape == (T, nh, dk) and v.shape == (T, nh, dv)
    out = np.zeros((T, nh, dv))
    u = np.zeros((T, nh, dv)) if want_u else None
    rc = _load().oracle_eager_run(op, nh, dk, dv, T, float(scale), _p(S), _p(q), _p(k),
                                  _p(v), _p(beta), _p(g), _p(bonus), _p(out), _p(u),
                                  _threads(n_threads))
    if rc:
        raise ValueError("oracle_eager_run rejected its arguments")
    return (S, out, u) if want_u else (S, out)


class LogState:
    """Base + bounded log of one layer (all heads share the log length L)."""

    def __init__(self, op, base, C, L=0, K=None, U=None, Lam=None):
        self.op, self.C = op, int(C)
        self.base = _f64(base).copy()
        nh, dk, dv = self.base.shape
        m = decay_width(op, dk)
        self.K = np.zeros((nh, C, dk)) if K is None else _f64(K).copy()
        self.U = np.zeros((nh, C, dv)) if U is None else _f64(U).copy()
        self.Lam = np.zeros((nh, C, m)) if Lam is None else _f64(Lam, (nh, C, m)).copy()
        self.L = int(L)


def deltalog_run(state: LogState, q, k, v, beta, g, bonus=None, scale=1.0,
                 n_threads=None):
    """Base+log decode of T tokens, advancing `state` in place.

    Returns (out [T, nh, dv], L_trace [T], merged [T]): the log length after
    each token and whether the merge ran after it.
    """
    op, C = state.op, state.C
    nh, dk, dv = state.base.shape
    q = _f64(q); T = q.shape[0]
    m = decay_width(op, dk)
    k = _f64(k); v = _f64(v)
    g = _f64(g, (T, nh, m))
    beta = _f64(beta, (T, nh)) if beta is not None else np.zeros((T, nh))
    bonus = _f64(bonus, (nh, dk)) if bonus is not None else (
        np.zeros((nh, dk)) if op == RWKV6 else None)
    out = np.zeros((T, nh, dv))
    L_trace = np.zeros(T, dtype=np.int32)
    merged = np.zeros(T, dtype=np.int32)
    L_io = ctypes.c_int(state.L)
    rc = _load().oracle_deltalog_run(
        op, nh, dk, dv, C, T, float(scale), _p(state.base), _p(state.K), _p(state.U),
        _p(state.Lam), ctypes.cast(ctypes.pointer(L_io), ctypes.c_void_p), _p(q), _p(k),
        _p(v), _p(beta), _p(g), _p(bonus), _p(out), _p(L_trace), _p(merged),
        _threads(n_threads))
    if rc:
        raise ValueError("oracle_deltalog_run rejected its arguments")
    state.L = int(L_io.value)
    return out, L_trace, merged


def deltalog_slots_run(state: LogState, H, Ls, active, q, k, v, beta, g, bonus=None,
                       scale=1.0, n_threads=None):
    """Base+log decode with a log length per slot: the state's heads are
    grouped into slots of H heads (head = slot * H + h), slot s takes part in
    token t only where active[t, s], and each slot appends and merges on its
    own schedule.  `Ls` (int array, one entry per slot) is advanced in place;
    state.L is not used.

    Returns (out [T, nh, dv] with NaN rows for idle slots, L_trace [T, nslots]).
    """
    op, C = state.op, state.C
    nh, dk, dv = state.base.shape
    if nh % H:
        raise ValueError("heads are not a whole number of slots")
    nslots = nh // H
    q = _f64(q); T = q.shape[0]
    m = decay_width(op, dk)
    k = _f64(k); v = _f64(v)
    g = _f64(g, (T, nh, m))
    beta = _f64(beta, (T, nh)) if beta is not None else np.zeros((T, nh))
    bonus = _f64(bonus, (nh, dk)) if bonus is not None else (
        np.zeros((nh, dk)) if op == RWKV6 else None)
    act = np.ascontiguousarray(np.asarray(active, dtype=bool).reshape(T, nslots), dtype=np.uint8)
    Ls_c = np.ascontiguousarray(np.asarray(Ls).reshape(nslots), dtype=np.int32).copy()
    out = np.full((T, nh, dv), np.nan)
    L_trace = np.zeros((T, nslots), dtype=np.int32)
    rc = _load().oracle_deltalog_slots_run(
        op, nslots, H, dk, dv, C, T, float(scale), _p(state.base), _p(state.K), _p(state.U),
        _p(state.Lam), _p(Ls_c), _p(act), _p(q), _p(k), _p(v), _p(beta), _p(g), _p(bonus),
        _p(out), _p(L_trace), _threads(n_threads))
    if rc:
        raise ValueError("oracle_deltalog_slots_run rejected its arguments")
    Ls[...] = Ls_c.reshape(np.shape(Ls))
    return out, L_trace


def materialize(state: LogState):
    """Logical dense state (base + replayed log); the state is left as is."""
    S = np.empty_like(state.base)
    nh, dk, dv = state.base.shape
    rc = _load().oracle_materialize(state.op, nh, dk, dv, state.C, state.L,
                                    _p(state.base), _p(state.K), _p(state.U),
                                    _p(state.Lam), _p(S))
    if rc:
        raise ValueError("oracle_materialize rejected its arguments")
    return S


def merge(state: LogState):
    """Fold the log into the base in place and reset L to 0."""
    nh, dk, dv = state.base.shape
    rc = _load().oracle_merge(state.op, nh, dk, dv, state.C, state.L, _p(state.base),
                              _p(state.K), _p(state.U), _p(state.Lam))
    if rc:
        raise ValueError("oracle_merge rejected its arguments")
    state.L = 0


def rel_err(x, ref) -> float:
    """Normwise-max relative error max|x - ref| / max|ref| (0 when both are 0)."""
    x = np.asarray(x, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    den = float(np.max(np.abs(ref))) if ref.size else 0.0
    num = float(np.max(np.abs(x - ref))) if ref.size else 0.0
    if den == 0.0:
        return num
    return num / den
