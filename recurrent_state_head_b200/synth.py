"""Seeded synthetic decode inputs for DeltaLog (GDN, KDA, RWKV6).

This module only draws random numbers and rounds them to the storage types;
it holds none of the recurrence arithmetic, so both the CUDA path and the
fp64 checker consume the very same bytes from it.

Recipe (all draws in float64 from NumPy's PCG64, then rounded):
  * every (layer, stream) pair has its own Generator(PCG64([seed, layer, s])):
    s = 0 for the initial state, 1 for the bonus, 2 + t for token t.
  * initial state S0 [B, H, dk, dv]: zero, or N(0, 0.02) (standard deviation)
    rounded to fp32.
  * RWKV6 bonus u [H, dk]: N(0, 0.1) rounded to fp32.
  * token t draws, in this order:
      q (r for RWKV6) [B, H, dk], k [B, H, dk], v [B, H, dv]   ~ N(0, 1)
      beta [B, H]      = sigmoid(N(0, 1))                      (GDN, KDA)
      g (log-decay)    GDN  [B, H]     = -softplus(N(0, 1))     (alpha = exp(g))
                       KDA  [B, H, dk] = -softplus(N(0, 1))     (a = exp(g))
                       RWKV6[B, H, dk] = -exp(N(-0.5, 0.5))     (w = exp(g))
    q and k are L2-normalised per head in float64 for GDN and KDA, not for
    RWKV6.  q, k, v are then rounded to the input dtype (fp32, or bf16 by
    round-to-nearest-even), beta and g to fp32.
A per-token generator lets any token be drawn on its own, in any order.
"""
from __future__ import annotations

import concurrent.futures as cf
import dataclasses
import math
import os
from typing import Optional

import numpy as np

GDN, KDA, RWKV6 = 0, 1, 2
OP_BY_NAME = {"gdn": GDN, "kda": KDA, "rwkv6": RWKV6}


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    op: int
    B: int
    H: int
    dk: int
    dv: int
    C: int
    T: int
    in_dtype: str          # "f32" | "bf16"
    out_dtype: str         # "f32" | "bf16"
    scale: float
    seed: int
    init_std: float        # 0.0 -> zero initial state
    layers: int = 1

    @property
    def heads(self) -> int:
        return self.B * self.H

    @property
    def m(self) -> int:
        return 1 if self.op == GDN else self.dk

    def state_bytes(self) -> int:
        return 4 * self.layers * self.heads * self.dk * self.dv

    def with_(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


def _w(name, op, B, H, d, C, T, in_dt, out_dt, seed, init_std, layers=1):
    scale = 1.0 if op == RWKV6 else 1.0 / math.sqrt(d)
    return Workload(name, op, B, H, d, d, C, T, in_dt, out_dt, scale, seed,
                    init_std, layers)


# The decode workloads the method is evaluated on (single-layer unless stated).
WORKLOADS = {
    "gdn-b1-h2-d64-c4-fp32": _w("gdn-b1-h2-d64-c4-fp32", GDN, 1, 2, 64, 4, 32,
                                "f32", "f32", 0, 0.0),
    "gdn-b128-h16-d128-c8": _w("gdn-b128-h16-d128-c8", GDN, 128, 16, 128, 8, 256,
                               "bf16", "bf16", 1, 0.02),
    "kda-b128-h32-d128-c4": _w("kda-b128-h32-d128-c4", KDA, 128, 32, 128, 4, 256,
                               "bf16", "bf16", 2, 0.02),
    "kda-b128-h32-d128-c8": _w("kda-b128-h32-d128-c8", KDA, 128, 32, 128, 8, 256,
                               "bf16", "bf16", 2, 0.02),
    "rwkv6-b128-h32-d64-c4": _w("rwkv6-b128-h32-d64-c4", RWKV6, 128, 32, 64, 4, 256,
                                "bf16", "bf16", 3, 0.02),
    "rwkv6-b128-h32-d64-c8": _w("rwkv6-b128-h32-d64-c8", RWKV6, 128, 32, 64, 8, 256,
                                "bf16", "bf16", 3, 0.02),
}
for _B in (1, 8, 32, 128, 512):
    for _C in (1, 2, 4, 8, 16):
        _n = f"gdn-stack24-b{_B}-h16-d128-c{_C}"
        WORKLOADS[_n] = _w(_n, GDN, _B, 16, 128, _C, 512, "bf16", "bf16", 4, 0.02,
                           layers=24)


# ----------------------------------------------------------- dtype helpers --

def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bfloat16 (nearest, ties to even); raw uint16 bits."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    r = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return r.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def round_to(x64: np.ndarray, dtype: str):
    """Round float64 draws to storage: returns (stored array, exact float64 value)."""
    f32 = x64.astype(np.float32)
    if dtype == "f32":
        return f32, f32.astype(np.float64)
    if dtype == "bf16":
        bits = f32_to_bf16_bits(f32)
        return bits, bf16_bits_to_f32(bits).astype(np.float64)
    raise ValueError(dtype)


# ------------------------------------------------------------- generation --

def _softplus(x):
    return np.maximum(x, 0.0) + np.log1p(np.exp(-np.abs(x)))


def _l2n(x):
    return x / np.linalg.norm(x, axis=-1, keepdims=True)


@dataclasses.dataclass
class TokenInputs:
    """Inputs of a run of tokens, stacked [T, ...]; stored and float64 views."""
    q: np.ndarray       # [T, B, H, dk]  stored (float32 or bf16 bits as uint16)
    k: np.ndarray
    v: np.ndarray       # [T, B, H, dv]
    beta: np.ndarray    # [T, B, H] float32 (zeros for RWKV6)
    g: np.ndarray       # [T, B, H] or [T, B, H, dk] float32
    q64: np.ndarray     # exact float64 values of the stored q, k, v
    k64: np.ndarray
    v64: np.ndarray


def initial_state(w: Workload, layer: int = 0) -> np.ndarray:
    """S0 [B, H, dk, dv] float32 for one layer."""
    shape = (w.B, w.H, w.dk, w.dv)
    if w.init_std == 0.0:
        return np.zeros(shape, dtype=np.float32)
    rng = np.random.Generator(np.random.PCG64([w.seed, layer, 0]))
    return (rng.standard_normal(shape) * w.init_std).astype(np.float32)


def bonus(w: Workload, layer: int = 0) -> Optional[np.ndarray]:
    """RWKV6 bonus u [H, dk] float32 (None for the delta-rule operators)."""
    if w.op != RWKV6:
        return None
    rng = np.random.Generator(np.random.PCG64([w.seed, layer, 1]))
    return (rng.standard_normal((w.H, w.dk)) * 0.1).astype(np.float32)


def tokens(w: Workload, t0: int, n: int, layer: int = 0,
           heads: Optional[np.ndarray] = None, want64: bool = True) -> TokenInputs:
    """Inputs of tokens t0 .. t0+n-1 of one layer.

    `heads` (flat b*H + h indices) keeps only those heads; the draws are the
    same as in the full tensors.  With want64=False the float64 views are
    left empty (see `exact64` to widen a selection later).
    """
    B, H, dk, dv = w.B, w.H, w.dk, w.dv

    def one(t):
        rng = np.random.Generator(np.random.PCG64([w.seed, layer, 2 + t]))
        q = rng.standard_normal((B, H, dk))
        k = rng.standard_normal((B, H, dk))
        v = rng.standard_normal((B, H, dv))
        if w.op == RWKV6:
            beta = np.zeros((B, H))
            g = -np.exp(rng.standard_normal((B, H, dk)) * 0.5 - 0.5)
        else:
            beta = 1.0 / (1.0 + np.exp(-rng.standard_normal((B, H))))
            if w.op == GDN:
                g = -_softplus(rng.standard_normal((B, H)))
            else:
                g = -_softplus(rng.standard_normal((B, H, dk)))
            q, k = _l2n(q), _l2n(k)
        if heads is not None:
            sel = lambda a: a.reshape((B * H,) + a.shape[2:])[heads]  # noqa: E731
            q, k, v, beta, g = sel(q), sel(k), sel(v), sel(beta), sel(g)
        qs_, q64 = round_to(q, w.in_dtype)
        ks_, k64 = round_to(k, w.in_dtype)
        vs_, v64 = round_to(v, w.in_dtype)
        if not want64:
            q64 = k64 = v64 = None
        return qs_, ks_, vs_, beta.astype(np.float32), g.astype(np.float32), q64, k64, v64

    # tokens are independent streams: draw them in parallel, keep their order
    n_workers = max(1, min(n, len(os.sched_getaffinity(0)), 16))
    if n_workers > 1:
        with cf.ThreadPoolExecutor(max_workers=n_workers) as ex:
            rows = list(ex.map(one, range(t0, t0 + n)))
    else:
        rows = [one(t) for t in range(t0, t0 + n)]
    qs, ks, vs, bs, gs, q6, k6, v6 = (list(c) for c in zip(*rows)) if rows else ([],) * 8
    st = np.stack
    e = np.zeros(0)
    return TokenInputs(st(qs), st(ks), st(vs), st(bs), st(gs),
                       st(q6) if want64 else e, st(k6) if want64 else e,
                       st(v6) if want64 else e)


def exact64(stored: np.ndarray, dtype: str) -> np.ndarray:
    """Exact float64 values of stored inputs (float32, or bf16 bits)."""
    if dtype == "bf16":
        return bf16_bits_to_f32(stored).astype(np.float64)
    return np.asarray(stored, dtype=np.float32).astype(np.float64)
