"""Thin ctypes binding of libdeltalog.so (include/deltalog.h).

Argument marshalling only: tensors (anything with ``data_ptr()``) or raw
integer addresses go in as device pointers, a torch stream (or raw
``cudaStream_t`` integer) as the stream; every step of the computation runs
in the library's CUDA kernels.  The functions carry the C names; ``Handle``
and ``Cycle`` are small owners of the opaque C objects.

The library is opened on first use; if it is missing or cannot be loaded
this raises (there is no other implementation to fall back on).
"""
from __future__ import annotations

import ctypes
import os
import threading

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libdeltalog.so")

DL_OK, DL_EINVAL, DL_ESTATE, DL_ECUDA, DL_ENOMEM = 0, 1, 2, 3, 4
DL_GDN, DL_KDA, DL_RWKV6 = 0, 1, 2
DL_F32, DL_BF16 = 0, 1
DL_MERGE_OFF, DL_MERGE_FOLD, DL_MERGE_SEPARATE = 0, 1, 2

# Every symbol include/deltalog.h declares.
EXPORTS = (
    "dl_log_bytes", "dl_log_layout", "dl_create", "dl_decode_step", "dl_merge",
    "dl_materialize", "dl_eager_step", "dl_log_len", "dl_destroy",
    "dl_decode_step_masked", "dl_slot_reset", "dl_slot_len",
    "dl_cycle_create", "dl_cycle_launch", "dl_cycle_kernels", "dl_cycle_destroy",
    "dl_strerror", "dl_last_error", "dl_debug_fake_launches",
)


class dl_config(ctypes.Structure):
    _fields_ = [("op", ctypes.c_int), ("B", ctypes.c_int), ("H", ctypes.c_int),
                ("dk", ctypes.c_int), ("dv", ctypes.c_int), ("C", ctypes.c_int),
                ("in_dtype", ctypes.c_int), ("out_dtype", ctypes.c_int),
                ("scale", ctypes.c_float), ("auto_merge", ctypes.c_int)]


class dl_step_io(ctypes.Structure):
    _fields_ = [("q", ctypes.c_void_p), ("k", ctypes.c_void_p), ("v", ctypes.c_void_p),
                ("beta", ctypes.c_void_p), ("g", ctypes.c_void_p), ("out", ctypes.c_void_p)]


class DeltaLogError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"[{status}] {message}")
        self.status = status


_lock = threading.Lock()
_lib = None


def lib() -> ctypes.CDLL:
    """The loaded library (raises if it is missing or unloadable)."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise RuntimeError(
                    f"{LIB_PATH} is missing: build it with "
                    "`python -m recurrent_state_head_b200.build`")
            L = ctypes.CDLL(LIB_PATH)
            P, I, S = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
            CP = ctypes.POINTER(dl_config)
            L.dl_log_bytes.argtypes, L.dl_log_bytes.restype = [CP], S
            L.dl_log_layout.argtypes = [CP, ctypes.POINTER(S), ctypes.POINTER(S),
                                        ctypes.POINTER(S)]
            L.dl_create.argtypes = [CP, P, P, P, ctypes.POINTER(P)]
            L.dl_decode_step.argtypes = [P, P, P, P, P, P, P, P]
            L.dl_merge.argtypes = [P, P]
            L.dl_materialize.argtypes = [P, P, P]
            L.dl_eager_step.argtypes = [CP, P, P, P, P, P, P, P, P, P]
            L.dl_log_len.argtypes, L.dl_log_len.restype = [P], I
            L.dl_decode_step_masked.argtypes = [P, P, P, P, P, P, P, P, P]
            L.dl_slot_reset.argtypes = [P, I]
            L.dl_slot_len.argtypes, L.dl_slot_len.restype = [P, I], I
            L.dl_destroy.argtypes, L.dl_destroy.restype = [P], None
            L.dl_cycle_create.argtypes = [ctypes.POINTER(P), I, ctypes.POINTER(dl_step_io),
                                          ctypes.POINTER(P)]
            L.dl_cycle_launch.argtypes = [P, P]
            L.dl_cycle_kernels.argtypes, L.dl_cycle_kernels.restype = [P], I
            L.dl_cycle_destroy.argtypes, L.dl_cycle_destroy.restype = [P], None
            L.dl_strerror.argtypes, L.dl_strerror.restype = [I], ctypes.c_char_p
            L.dl_last_error.argtypes, L.dl_last_error.restype = [], ctypes.c_char_p
            L.dl_debug_fake_launches.argtypes = [ctypes.c_longlong]
            L.dl_debug_fake_launches.restype = None
            for f in ("dl_log_layout", "dl_create", "dl_decode_step", "dl_merge",
                      "dl_materialize", "dl_eager_step", "dl_cycle_create",
                      "dl_cycle_launch"):
                getattr(L, f).restype = I
            _lib = L
    return _lib


def _check(status: int):
    if status != DL_OK:
        L = lib()
        raise DeltaLogError(status, f"{L.dl_strerror(status).decode()}: "
                                    f"{L.dl_last_error().decode()}")


def _ptr(x):
    if x is None:
        return None
    if isinstance(x, int):
        return x
    return x.data_ptr()


def _stream(s):
    if s is None:
        import torch
        return torch.cuda.current_stream().cuda_stream if torch.cuda.is_available() else None
    if isinstance(s, int):
        return s
    return s.cuda_stream


def make_config(op, B, H, dk, dv, C=1, in_dtype=DL_F32, out_dtype=DL_F32, scale=1.0,
                auto_merge=1) -> dl_config:
    return dl_config(int(op), int(B), int(H), int(dk), int(dv), int(C), int(in_dtype),
                     int(out_dtype), float(scale), int(auto_merge))


# ------------------------------------------------------ C-named functions --

def dl_log_bytes(cfg: dl_config) -> int:
    return int(lib().dl_log_bytes(ctypes.byref(cfg)))


def dl_log_layout(cfg: dl_config):
    a, b, c = ctypes.c_size_t(), ctypes.c_size_t(), ctypes.c_size_t()
    _check(lib().dl_log_layout(ctypes.byref(cfg), ctypes.byref(a), ctypes.byref(b),
                               ctypes.byref(c)))
    return a.value, b.value, c.value


def dl_create(cfg: dl_config, base, log_ws, bonus=None) -> int:
    h = ctypes.c_void_p()
    _check(lib().dl_create(ctypes.byref(cfg), _ptr(base), _ptr(log_ws), _ptr(bonus),
                           ctypes.byref(h)))
    return h.value


def dl_decode_step(h: int, q, k, v, beta, g, out, stream=None):
    _check(lib().dl_decode_step(h, _ptr(q), _ptr(k), _ptr(v), _ptr(beta), _ptr(g),
                                _ptr(out), _stream(stream)))


def dl_decode_step_masked(h: int, active, q, k, v, beta, g, out, stream=None):
    """`active`: None (every slot) or a sequence of B truth values (host)."""
    act = None
    if active is not None:
        flags = bytes(1 if a else 0 for a in active)
        act = ctypes.create_string_buffer(flags, len(flags))
    _check(lib().dl_decode_step_masked(h, act, _ptr(q), _ptr(k), _ptr(v), _ptr(beta), _ptr(g),
                                       _ptr(out), _stream(stream)))


def dl_slot_reset(h: int, slot: int):
    _check(lib().dl_slot_reset(h, int(slot)))


def dl_slot_len(h: int, slot: int) -> int:
    return int(lib().dl_slot_len(h, int(slot)))


def dl_merge(h: int, stream=None):
    _check(lib().dl_merge(h, _stream(stream)))


def dl_materialize(h: int, S_out, stream=None):
    _check(lib().dl_materialize(h, _ptr(S_out), _stream(stream)))


def dl_eager_step(cfg: dl_config, S, q, k, v, beta, g, bonus, out, stream=None):
    _check(lib().dl_eager_step(ctypes.byref(cfg), _ptr(S), _ptr(q), _ptr(k), _ptr(v),
                               _ptr(beta), _ptr(g), _ptr(bonus), _ptr(out),
                               _stream(stream)))


def dl_log_len(h: int) -> int:
    return int(lib().dl_log_len(h))


def dl_destroy(h: int):
    lib().dl_destroy(h)


def dl_cycle_create(handles, ios) -> int:
    """handles: [n_layers] handle addresses; ios: [C][n_layers] of
    (q, k, v, beta, g, out) tuples."""
    n = len(handles)
    harr = (ctypes.c_void_p * n)(*handles)
    flat = [x for row in ios for x in row]
    iarr = (dl_step_io * len(flat))(*[dl_step_io(*[_ptr(a) for a in io]) for io in flat])
    cy = ctypes.c_void_p()
    _check(lib().dl_cycle_create(harr, n, iarr, ctypes.byref(cy)))
    return cy.value


def dl_cycle_launch(cy: int, stream=None):
    _check(lib().dl_cycle_launch(cy, _stream(stream)))


def dl_cycle_kernels(cy: int) -> int:
    return int(lib().dl_cycle_kernels(cy))


def dl_cycle_destroy(cy: int):
    lib().dl_cycle_destroy(cy)


def dl_strerror(status: int) -> str:
    return lib().dl_strerror(status).decode()


def dl_last_error() -> str:
    return lib().dl_last_error().decode()


def dl_debug_fake_launches(n_ok: int):
    """Test hook: with n_ok >= 0 no kernel is issued; the next n_ok launches
    report success, later ones fail.  n_ok < 0 restores real launches."""
    lib().dl_debug_fake_launches(int(n_ok))


# ------------------------------------------------------------- owners ----

class Handle:
    """Owner of a dl_handle; keeps the tensors it points to alive."""

    def __init__(self, cfg: dl_config, base, log_ws, bonus=None):
        self.cfg = cfg
        self._keep = (base, log_ws, bonus)
        self.h = dl_create(cfg, base, log_ws, bonus)

    @property
    def L(self) -> int:
        return dl_log_len(self.h)

    def decode_step(self, q, k, v, beta, g, out, stream=None, active=None):
        if active is None:
            dl_decode_step(self.h, q, k, v, beta, g, out, stream)
        else:
            dl_decode_step_masked(self.h, active, q, k, v, beta, g, out, stream)

    def slot_len(self, slot: int) -> int:
        return dl_slot_len(self.h, slot)

    def slot_reset(self, slot: int):
        dl_slot_reset(self.h, slot)

    def merge(self, stream=None):
        dl_merge(self.h, stream)

    def materialize(self, S_out, stream=None):
        dl_materialize(self.h, S_out, stream)

    def close(self):
        if self.h:
            dl_destroy(self.h)
            self.h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


class Cycle:
    """Owner of a dl_cycle (one graph-captured merge cycle over layers)."""

    def __init__(self, handles, ios):
        self._keep = (list(handles), ios)
        self.cy = dl_cycle_create([h.h for h in handles], ios)

    @property
    def kernels(self) -> int:
        return dl_cycle_kernels(self.cy)

    def launch(self, stream=None):
        dl_cycle_launch(self.cy, stream)

    def close(self):
        if self.cy:
            dl_cycle_destroy(self.cy)
            self.cy = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass
