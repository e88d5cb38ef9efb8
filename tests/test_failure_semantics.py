"""Log-length bookkeeping when a launch fails partway through a call.

The failures are injected on the host (dl_debug_fake_launches: no kernel is
issued, the first n launches report success and later ones fail), so these
run without a GPU and touch no device memory; the pointers are fake aligned
addresses.  After a failed call every slot's length must say what happened
to it: a slot whose kernel launched has taken the step, the others have not.
"""
import pytest

from recurrent_state_head_b200 import binding as B
from recurrent_state_head_b200 import build as libbuild

A = 1 << 20          # a fake, aligned device address (never dereferenced)


@pytest.fixture(scope="module")
def lib():
    libbuild.build()
    return B.lib()


@pytest.fixture
def fake():
    yield B.dl_debug_fake_launches
    B.dl_debug_fake_launches(-1)


def cfg(**kw):
    base = dict(op=B.DL_GDN, B=2, H=1, dk=64, dv=64, C=4, in_dtype=B.DL_BF16,
                out_dtype=B.DL_BF16, scale=0.125, auto_merge=B.DL_MERGE_FOLD)
    base.update(kw)
    return B.make_config(**base)


def step(h, active=None):
    if active is None:
        B.dl_decode_step(h, A, A, A, A, A, A, stream=0)
    else:
        B.dl_decode_step_masked(h, active, A, A, A, A, A, A, stream=0)


def lens(h, n):
    return [B.dl_slot_len(h, b) for b in range(n)]


def test_hook_off_by_default_and_restorable(lib, fake):
    fake(2)
    h = B.dl_create(cfg(), A, A, None)
    try:
        step(h)
        step(h)
        assert B.dl_log_len(h) == 2
        with pytest.raises(B.DeltaLogError) as e:
            step(h)
        assert e.value.status == B.DL_ECUDA
        assert B.dl_log_len(h) == 2
    finally:
        B.dl_destroy(h)


def test_shared_merge_token_failure_keeps_length(lib, fake):
    C = 3
    fake(1 << 30)
    h = B.dl_create(cfg(C=C), A, A, None)
    try:
        for _ in range(C - 1):
            step(h)
        assert B.dl_log_len(h) == C - 1
        fake(0)
        with pytest.raises(B.DeltaLogError) as e:
            step(h)
        assert e.value.status == B.DL_ECUDA
        assert B.dl_log_len(h) == C - 1          # the merge-token did not launch
        fake(1)
        step(h)                                  # the retry takes it
        assert B.dl_log_len(h) == 0
    finally:
        B.dl_destroy(h)


def test_shared_separate_merge_failure_leaves_full_log(lib, fake):
    """The C-th append launched, its merge did not: L = C, the next step is
    refused until dl_merge has folded the log."""
    C = 4
    fake(1 << 30)
    h = B.dl_create(cfg(C=C, auto_merge=B.DL_MERGE_SEPARATE), A, A, None)
    try:
        for _ in range(C - 1):
            step(h)
        fake(1)                                  # the append launches, the merge fails
        with pytest.raises(B.DeltaLogError) as e:
            step(h)
        assert e.value.status == B.DL_ECUDA
        assert B.dl_log_len(h) == C
        fake(1 << 30)
        with pytest.raises(B.DeltaLogError) as e:
            step(h)
        assert e.value.status == B.DL_ESTATE
        assert "dl_merge" in B.dl_last_error()
        assert B.dl_log_len(h) == C
        B.dl_merge(h, stream=0)
        assert B.dl_log_len(h) == 0
        step(h)
        assert B.dl_log_len(h) == 1
    finally:
        B.dl_destroy(h)


def _stagger(h, nslots, C):
    """Slot b takes the first (b mod C) tokens only: L_b = b mod C."""
    for t in range(C - 1):
        step(h, [(b % C) > t for b in range(nslots)])
    assert lens(h, nslots) == [b % C for b in range(nslots)]


@pytest.mark.parametrize("ok_chunks", [0, 1])
def test_slot_step_commits_each_launched_chunk(lib, fake, ok_chunks):
    """600 slots need two slot-list launches; the merge-token slots (at
    L = C-1) come first.  When only the first launch succeeds, exactly its
    slots move."""
    C, n = 4, 600
    fake(1 << 30)
    h = B.dl_create(cfg(B=n, C=C), A, A, None)
    try:
        _stagger(h, n, C)
        fake(ok_chunks)
        with pytest.raises(B.DeltaLogError) as e:
            step(h)
        assert e.value.status == B.DL_ECUDA
        order = [b for b in range(n) if b % C == C - 1] + [b for b in range(n) if b % C != C - 1]
        launched = set(order[:512 * ok_chunks])
        want = [((b % C) + 1) % C if b in launched else b % C for b in range(n)]
        assert lens(h, n) == want
    finally:
        B.dl_destroy(h)


def test_slot_separate_merge_failure(lib, fake):
    """DL_MERGE_SEPARATE: the appends launch, the merge of the slots whose
    log filled does not.  Those slots sit at C, a step that includes them is
    refused, dl_merge folds them."""
    C, n = 3, 7
    fake(1 << 30)
    h = B.dl_create(cfg(B=n, C=C, auto_merge=B.DL_MERGE_SEPARATE), A, A, None)
    try:
        _stagger(h, n, C)
        fake(1)                                  # the append list launches, the merge fails
        with pytest.raises(B.DeltaLogError) as e:
            step(h)
        assert e.value.status == B.DL_ECUDA
        assert lens(h, n) == [C if b % C == C - 1 else b % C + 1 for b in range(n)]
        fake(1 << 30)
        with pytest.raises(B.DeltaLogError) as e:
            step(h)
        assert e.value.status == B.DL_ESTATE
        # a step that leaves the full slots idle is allowed
        step(h, [b % C != C - 1 for b in range(n)])
        B.dl_merge(h, stream=0)
        assert lens(h, n) == [0] * n
    finally:
        B.dl_destroy(h)


def test_slot_merge_commits_each_launched_chunk(lib, fake):
    C, n = 5, 700
    fake(1 << 30)
    h = B.dl_create(cfg(B=n, C=C, auto_merge=B.DL_MERGE_OFF), A, A, None)
    try:
        _stagger(h, n, C)
        nonzero = [b for b in range(n) if b % C]
        fake(1)
        with pytest.raises(B.DeltaLogError) as e:
            B.dl_merge(h, stream=0)
        assert e.value.status == B.DL_ECUDA
        first = set(nonzero[:512])
        assert lens(h, n) == [0 if (b in first or b % C == 0) else b % C for b in range(n)]
        fake(1 << 30)
        B.dl_merge(h, stream=0)
        assert B.dl_log_len(h) == 0
    finally:
        B.dl_destroy(h)


def test_cycle_create_leaves_lengths(lib, fake):
    """dl_cycle_create works on copies of the lengths: a failed capture
    leaves every layer as it was (on a machine without a GPU the capture
    itself fails)."""
    fake(1 << 30)
    h = B.dl_create(cfg(B=3, C=2), A, A, None)
    try:
        step(h, [1, 0, 1])
        before = lens(h, 3)
        io = [[(A, A, A, A, A, A)] for _ in range(2)]
        try:
            cy = B.dl_cycle_create([h], io)
            B.dl_cycle_destroy(cy)
        except B.DeltaLogError:
            pass
        assert lens(h, 3) == before
    finally:
        B.dl_destroy(h)
