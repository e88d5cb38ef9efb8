"""Device memory for DeltaLog decode: PyTorch allocates, the library computes.

``DecodeLayer`` owns one layer's base state, log workspace and (RWKV6)
bonus as torch tensors and a ``binding.Handle`` over them;
``to_device`` moves seeded host inputs (``synth.TokenInputs``) to the GPU
in the library's dtypes.  Nothing here computes any part of the recurrence.
"""
from __future__ import annotations

import numpy as np
import torch

from . import binding as B
from .synth import RWKV6, TokenInputs, Workload

DTYPE_CODE = {"f32": B.DL_F32, "bf16": B.DL_BF16}
TORCH_DTYPE = {"f32": torch.float32, "bf16": torch.bfloat16}


def host_tensor(a: np.ndarray, dtype: str) -> torch.Tensor:
    """Wrap a host array stored as `dtype` (bf16 arrives as raw uint16 bits)."""
    if dtype == "bf16":
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16)
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32))


def to_device(ti: TokenInputs, w: Workload, device="cuda", pin: bool = False):
    """Stacked token inputs as tensors: q, k [T, NH, dk]; v [T, NH, dv];
    beta [T, NH]; g [T, NH, m].  With device=None the tensors stay on the host
    (pinned if `pin`)."""
    T = ti.q.shape[0]
    NH = w.heads
    out = {
        "q": host_tensor(ti.q, w.in_dtype).reshape(T, NH, w.dk),
        "k": host_tensor(ti.k, w.in_dtype).reshape(T, NH, w.dk),
        "v": host_tensor(ti.v, w.in_dtype).reshape(T, NH, w.dv),
        "beta": torch.from_numpy(np.ascontiguousarray(ti.beta, dtype=np.float32)).reshape(T, NH),
        "g": torch.from_numpy(np.ascontiguousarray(ti.g, dtype=np.float32)).reshape(T, NH, w.m),
    }
    if device is None:
        if pin:
            out = {k: v.pin_memory() for k, v in out.items()}
        return out
    return {k: v.to(device, non_blocking=True) for k, v in out.items()}


def config_of(w: Workload, C=None, auto_merge=1) -> B.dl_config:
    return B.make_config(w.op, w.B, w.H, w.dk, w.dv, w.C if C is None else C,
                         DTYPE_CODE[w.in_dtype], DTYPE_CODE[w.out_dtype], w.scale, auto_merge)


class DecodeLayer:
    """One layer of DeltaLog decode state on the GPU.  S0 is the starting
    dense state: a host array (copied to the device), or a float32 device
    tensor of NH * dk * dv elements, used as the base itself (not copied)."""

    def __init__(self, w: Workload, S0, bonus=None, device="cuda", C=None,
                 auto_merge=1):
        self.w = w
        self.cfg = config_of(w, C, auto_merge)
        if isinstance(S0, torch.Tensor):
            if S0.dtype != torch.float32 or S0.numel() != w.heads * w.dk * w.dv:
                raise ValueError("device base must be float32 with NH * dk * dv elements")
            self.base = S0.reshape(w.heads, w.dk, w.dv)
            device = S0.device
        else:
            self.base = torch.from_numpy(np.ascontiguousarray(S0, dtype=np.float32)).reshape(
                w.heads, w.dk, w.dv).to(device)
        self.log = torch.zeros(max(B.dl_log_bytes(self.cfg), 16), dtype=torch.uint8,
                               device=device)
        self.bonus = (torch.from_numpy(np.ascontiguousarray(bonus, dtype=np.float32)).to(device)
                      if w.op == RWKV6 else None)
        self.handle = B.Handle(self.cfg, self.base, self.log, self.bonus)
        self.out_dtype = TORCH_DTYPE[w.out_dtype]
        self.device = device

    @property
    def L(self) -> int:
        return self.handle.L

    def new_out(self, T=None):
        shape = (self.w.heads, self.w.dv) if T is None else (T, self.w.heads, self.w.dv)
        return torch.empty(shape, dtype=self.out_dtype, device=self.device)

    def step(self, x: dict, t: int, out: torch.Tensor, stream=None, active=None):
        """Decode token t of the stacked inputs `x` into `out` [NH, dv]; with
        `active` (B truth values) only those slots decode."""
        beta = None if self.w.op == RWKV6 else x["beta"][t]
        self.handle.decode_step(x["q"][t], x["k"][t], x["v"][t], beta, x["g"][t], out, stream,
                                active)

    def slot_len(self, slot: int) -> int:
        return self.handle.slot_len(slot)

    def slot_reset(self, slot: int, S_new: torch.Tensor):
        """Slot `slot` starts a new sequence from the dense state S_new
        [H, dk, dv] (its log is dropped)."""
        H = self.w.H
        self.base[slot * H:(slot + 1) * H].copy_(S_new.reshape(H, self.w.dk, self.w.dv))
        self.handle.slot_reset(slot)

    def materialize(self, stream=None) -> torch.Tensor:
        S = torch.empty_like(self.base)
        self.handle.materialize(S, stream)
        return S

    def merge(self, stream=None):
        self.handle.merge(stream)

    def log_views(self):
        """(K, U, Lambda) views of the log workspace for inspection."""
        oK, oU, oL = B.dl_log_layout(self.cfg)
        NH, C, dk, dv, m = self.w.heads, self.cfg.C, self.w.dk, self.w.dv, self.w.m
        in_t = TORCH_DTYPE[self.w.in_dtype]
        u_t = in_t if self.w.op == RWKV6 else torch.float32
        esz = lambda t: torch.tensor([], dtype=t).element_size()  # noqa: E731
        K = self.log[oK:oK + NH * C * dk * esz(in_t)].view(in_t).view(NH, C, dk)
        U = self.log[oU:oU + NH * C * dv * esz(u_t)].view(u_t).view(NH, C, dv)
        Lam = self.log[oL:oL + NH * C * m * 4].view(torch.float32).view(NH, C, m)
        return K, U, Lam


def eager_step(w: Workload, S: torch.Tensor, x: dict, t: int, bonus, out, stream=None):
    cfg = config_of(w)
    beta = None if w.op == RWKV6 else x["beta"][t]
    B.dl_eager_step(cfg, S, x["q"][t], x["k"][t], x["v"][t], beta, x["g"][t], bonus, out,
                    stream)


# ---------------------------------------------- device-drawn timing inputs --

def draw_state(w: Workload, layer: int, device, generator: torch.Generator) -> torch.Tensor:
    """A starting state [NH, dk, dv] drawn on the device with the workload's
    distribution (N(0, init_std), or zero), for timing runs too large to draw
    on the host.  Torch's device generator, not synth's: these values never
    meet the checker."""
    shape = (w.heads, w.dk, w.dv)
    if w.init_std == 0.0:
        return torch.zeros(shape, dtype=torch.float32, device=device)
    S = torch.empty(shape, dtype=torch.float32, device=device)
    S.normal_(0.0, w.init_std, generator=generator)
    return S


def draw_tokens(w: Workload, n: int, device, generator: torch.Generator) -> dict:
    """n tokens of inputs drawn on the device with synth's distributions
    (q, k, v ~ N(0, 1), q and k L2-normalised for GDN/KDA; beta =
    sigmoid(N(0, 1)); g = -softplus(N(0, 1)) for GDN/KDA, -exp(N(-0.5, 0.5))
    for RWKV6), rounded to the workload's dtypes; laid out as to_device's."""
    NH = w.heads
    f = dict(dtype=torch.float32, device=device)
    q = torch.randn((n, NH, w.dk), generator=generator, **f)
    k = torch.randn((n, NH, w.dk), generator=generator, **f)
    v = torch.randn((n, NH, w.dv), generator=generator, **f)
    x = torch.randn((n, NH, w.m), generator=generator, **f)
    if w.op == RWKV6:
        beta = torch.zeros((n, NH), **f)
        g = -torch.exp(x * 0.5 - 0.5)
    else:
        beta = torch.sigmoid(torch.randn((n, NH), generator=generator, **f))
        g = -torch.nn.functional.softplus(x)
        q = q / q.norm(dim=-1, keepdim=True)
        k = k / k.norm(dim=-1, keepdim=True)
    t = TORCH_DTYPE[w.in_dtype]
    return {"q": q.to(t), "k": k.to(t), "v": v.to(t), "beta": beta, "g": g}
