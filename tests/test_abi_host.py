"""C-ABI checks that need no GPU: the library builds for sm_100a, loads, and
exports every symbol include/deltalog.h declares; arguments are validated on
the host before any launch; the log-length schedule matches the oracle's;
a failing launch maps to DL_ECUDA and leaves the handle as it was."""
import ctypes
import os
import re

import numpy as np
import pytest

from recurrent_state_head_b200 import binding as B
from recurrent_state_head_b200 import build as libbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "deltalog.h")


@pytest.fixture(scope="module")
def lib():
    libbuild.build()
    return B.lib()


def header_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(dl_[a-z_]+)\s*\(", text)))


def test_header_and_binding_agree():
    assert header_functions() == sorted(B.EXPORTS)


def test_library_exports_every_declared_symbol(lib):
    raw = ctypes.CDLL(libbuild.LIB)
    for name in header_functions():
        assert hasattr(raw, name), name


def cfg(**kw):
    base = dict(op=B.DL_GDN, B=2, H=3, dk=64, dv=128, C=4, in_dtype=B.DL_BF16,
                out_dtype=B.DL_BF16, scale=0.125, auto_merge=1)
    base.update(kw)
    return B.make_config(**base)


@pytest.mark.parametrize("bad", [
    dict(op=3), dict(op=-1), dict(B=-1), dict(H=0), dict(dk=32), dict(dv=96),
    dict(dk=256), dict(C=0), dict(C=17), dict(in_dtype=2), dict(out_dtype=-1),
    dict(scale=float("nan")), dict(scale=float("inf")), dict(auto_merge=3),
    dict(auto_merge=-1),
])
def test_invalid_configs_rejected(lib, bad):
    c = cfg(**bad)
    assert B.dl_log_bytes(c) == 0
    h = ctypes.c_void_p()
    st = lib.dl_create(ctypes.byref(c), 4096, 8192, None, ctypes.byref(h))
    assert st == B.DL_EINVAL and h.value is None
    assert B.dl_last_error() != ""


@pytest.mark.parametrize("op", [B.DL_GDN, B.DL_KDA, B.DL_RWKV6])
@pytest.mark.parametrize("dt", [B.DL_F32, B.DL_BF16])
def test_log_layout(lib, op, dt):
    c = cfg(op=op, in_dtype=dt, dk=128, dv=64, C=5)
    NH = 6
    oK, oU, oL = B.dl_log_layout(c)
    esz = 2 if dt == B.DL_BF16 else 4
    m = 1 if op == B.DL_GDN else 128
    uesz = esz if op == B.DL_RWKV6 else 4
    up = lambda x: (x + 255) // 256 * 256  # noqa: E731
    assert oK == 0
    assert oU == up(NH * 5 * 128 * esz)
    assert oL == up(oU + NH * 5 * 64 * uesz)
    assert B.dl_log_bytes(c) == up(oL + NH * 5 * m * 4)
    assert oU % 256 == 0 and oL % 256 == 0


def test_create_checks_pointers(lib):
    c = cfg()
    h = ctypes.c_void_p()
    assert lib.dl_create(ctypes.byref(c), None, 4096, None, ctypes.byref(h)) == B.DL_EINVAL
    assert lib.dl_create(ctypes.byref(c), 4096 + 8, 4096, None, ctypes.byref(h)) == B.DL_EINVAL
    assert lib.dl_create(ctypes.byref(c), 4096, 4096 + 4, None, ctypes.byref(h)) == B.DL_EINVAL
    r = cfg(op=B.DL_RWKV6)
    assert lib.dl_create(ctypes.byref(r), 4096, 8192, None, ctypes.byref(h)) == B.DL_EINVAL
    assert lib.dl_create(ctypes.byref(c), 4096, 8192, None, None) == B.DL_EINVAL
    # creation touches no device memory: fake aligned addresses are accepted
    hh = B.dl_create(c, 4096, 8192, None)
    assert B.dl_log_len(hh) == 0
    B.dl_destroy(hh)
    assert B.dl_log_len(0) == -1


def test_decode_step_checks_pointers_before_launch(lib):
    hh = B.dl_create(cfg(), 4096, 8192, None)
    try:
        a = 1 << 20
        with pytest.raises(B.DeltaLogError) as e:
            B.dl_decode_step(hh, None, a, a, a, a, a)
        assert e.value.status == B.DL_EINVAL
        with pytest.raises(B.DeltaLogError) as e:           # beta needed for GDN
            B.dl_decode_step(hh, a, a, a, None, a, a)
        assert e.value.status == B.DL_EINVAL
        with pytest.raises(B.DeltaLogError) as e:           # bf16 q must be 2-byte aligned
            B.dl_decode_step(hh, a + 1, a, a, a, a, a)
        assert e.value.status == B.DL_EINVAL
        assert B.dl_log_len(hh) == 0
    finally:
        B.dl_destroy(hh)


def _has_gpu():
    try:
        import torch
        return torch.cuda.is_available()
    except Exception:
        return False


@pytest.mark.skipif(_has_gpu(), reason="checks the no-device failure path")
def test_failed_launch_is_reported_and_leaves_handle(lib):
    hh = B.dl_create(cfg(), 4096, 8192, None)
    try:
        a = 1 << 20
        with pytest.raises(B.DeltaLogError) as e:
            B.dl_decode_step(hh, a, a, a, a, a, a, stream=0)
        assert e.value.status == B.DL_ECUDA
        assert B.dl_log_len(hh) == 0
        with pytest.raises(B.DeltaLogError) as e:
            B.dl_eager_step(cfg(), a, a, a, a, a, a, None, a, stream=0)
        assert e.value.status == B.DL_ECUDA
    finally:
        B.dl_destroy(hh)


@pytest.mark.parametrize("C", [1, 2, 3, 5, 16])
@pytest.mark.parametrize("mode", [B.DL_MERGE_FOLD, B.DL_MERGE_SEPARATE])
def test_schedule_matches_oracle_without_heads(lib, C, mode, oracle_lib):
    """B = 0: nothing is launched, but L advances exactly as the oracle's
    schedule (append; merge when L reaches C)."""
    import oracle
    T = 3 * C + 1
    st = oracle.LogState(oracle.GDN, np.zeros((0, 2, 2)), C)
    z = np.zeros((T, 0, 2))
    _, Ltr, merged = oracle.deltalog_run(st, z, z, z, np.zeros((T, 0)), np.zeros((T, 0, 1)))
    hh = B.dl_create(cfg(B=0, C=C, auto_merge=mode), None, None, None)
    try:
        got = []
        for t in range(T):
            B.dl_decode_step(hh, None, None, None, None, None, None, stream=0)
            got.append(B.dl_log_len(hh))
        assert got == Ltr.tolist()
    finally:
        B.dl_destroy(hh)


def test_full_log_without_auto_merge(lib):
    C = 3
    hh = B.dl_create(cfg(B=0, C=C, auto_merge=0), None, None, None)
    try:
        for t in range(C):
            B.dl_decode_step(hh, None, None, None, None, None, None, stream=0)
        assert B.dl_log_len(hh) == C
        with pytest.raises(B.DeltaLogError) as e:
            B.dl_decode_step(hh, None, None, None, None, None, None, stream=0)
        assert e.value.status == B.DL_ESTATE
        assert B.dl_log_len(hh) == C
        B.dl_merge(hh, stream=0)
        assert B.dl_log_len(hh) == 0
        B.dl_merge(hh, stream=0)                 # merge of an empty log is a no-op
        assert B.dl_log_len(hh) == 0
    finally:
        B.dl_destroy(hh)


def test_eager_without_heads_is_noop(lib):
    B.dl_eager_step(cfg(B=0), None, None, None, None, None, None, None, None, stream=0)


def test_cycle_rejects_bad_layers(lib):
    h1 = B.dl_create(cfg(B=0, C=2), None, None, None)
    h2 = B.dl_create(cfg(B=0, C=3), None, None, None)
    h3 = B.dl_create(cfg(B=0, C=2, auto_merge=0), None, None, None)
    try:
        io = [[(None,) * 6] * 2] * 3
        for pair in ((h1, h2), (h1, h3)):
            with pytest.raises(B.DeltaLogError) as e:
                B.dl_cycle_create(list(pair), io)
            assert e.value.status == B.DL_EINVAL
    finally:
        for h in (h1, h2, h3):
            B.dl_destroy(h)


def test_slot_calls_check_arguments(lib):
    hh = B.dl_create(cfg(B=3), 4096, 8192, None)
    try:
        for bad in (-1, 3):
            with pytest.raises(B.DeltaLogError) as e:
                B.dl_slot_reset(hh, bad)
            assert e.value.status == B.DL_EINVAL
            assert B.dl_slot_len(hh, bad) == -1
        assert [B.dl_slot_len(hh, b) for b in range(3)] == [0, 0, 0]
        B.dl_slot_reset(hh, 1)                      # already empty: nothing changes
        assert B.dl_log_len(hh) == 0
    finally:
        B.dl_destroy(hh)
    assert B.dl_slot_len(0, 0) == -1


def test_idle_slots_launch_nothing(lib):
    """A step in which no slot is active launches nothing and moves no length
    (the fake device addresses are never touched)."""
    hh = B.dl_create(cfg(B=3, C=2), 4096, 8192, None)
    try:
        a = 1 << 20
        for _ in range(3):
            B.dl_decode_step_masked(hh, [0, 0, 0], a, a, a, a, a, a, stream=0)
        assert B.dl_log_len(hh) == 0
    finally:
        B.dl_destroy(hh)


@pytest.mark.skipif(_has_gpu(), reason="checks the no-device failure path")
def test_failed_slot_step_leaves_lengths(lib):
    hh = B.dl_create(cfg(B=3, C=3), 4096, 8192, None)
    try:
        a = 1 << 20
        with pytest.raises(B.DeltaLogError) as e:
            B.dl_decode_step_masked(hh, [1, 0, 1], a, a, a, a, a, a, stream=0)
        assert e.value.status == B.DL_ECUDA
        assert [B.dl_slot_len(hh, b) for b in range(3)] == [0, 0, 0]
    finally:
        B.dl_destroy(hh)


def test_per_slot_lengths_need_16_bit_slot_ids(lib):
    """Slot lists carry 16-bit ids: with more slots, steps that need per-slot
    lengths are refused before any launch (shared-length steps still run)."""
    hh = B.dl_create(cfg(B=70000, H=1), 4096, 8192, None)
    try:
        a = 1 << 20
        with pytest.raises(B.DeltaLogError) as e:
            B.dl_decode_step_masked(hh, [1] + [0] * 69999, a, a, a, a, a, a, stream=0)
        assert e.value.status == B.DL_EINVAL
        assert B.dl_log_len(hh) == 0
    finally:
        B.dl_destroy(hh)


def test_strerror(lib):
    for s in range(5):
        assert B.dl_strerror(s)
    assert B.dl_strerror(99) == "unknown status"
