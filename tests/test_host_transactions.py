"""A call whose launch fails leaves the pool's host state unchanged (CPU, no device fault).

The library's test hook makes the k-th device operation of a call fail on the host (on a
host-only pool, the operations it would issue are counted the same way).  For every call that
changes state -- append, prefill, demotion, copy, reset -- and every k, the failed call must leave
the tables, lengths and footprint as they were, and repeating the call without the failure must
then give exactly the tables of a twin pool that never failed (so the free-slot lists were
restored too)."""
import numpy as np
import pytest

from mixed_format_paged_mkv_b200 import MkvError, Pool

HKV, D, SEQS, MAXP = 2, 64, 8, 4096


def new_pool(fp8=12000, tq3=12000):
    p = Pool(HKV, D, SEQS, MAXP, fp8, tq3, host_only=True)
    rng = np.random.default_rng(3)
    for fmt, n in ((0, fp8), (1, tq3)):
        p.set_slot_order(fmt, rng.permutation(n).astype(np.int32))
    return p


def state(p):
    tables = [p.block_table(s) for s in range(SEQS)]
    return tables, p.stats()


def build(p):
    p.append([0, 1, 2], [700, 33, 1600])
    p.set_protected(2, 5)
    p.demote([0, 2], 64)
    p.append([1], [3000])
    p.append([3], [16 * 2700])


CALLS = {
    # name -> (call on a pool, device operations it issues)
    "append": (lambda p: p.append([0, 1, 3], [20, 16 * 1600, 5]), None),
    "append_one": (lambda p: p.append([2], [7]), None),
    "demote": (lambda p: p.demote([1, 0, 2, 3], 16), None),
    "prefill": (lambda p: p.prefill([4, 5], [16 * 2600 + 3, 900], window=48), None),
    "copy": (lambda p: p.copy(1, 6), None),
    "reset": (lambda p: p.reset(2), None),
}




@pytest.mark.parametrize("name", list(CALLS))
def test_failed_launch_leaves_host_state_unchanged(name):
    call = CALLS[name][0]
    twin = new_pool()
    build(twin)
    before = state(twin)
    call(twin)
    after = state(twin)
    assert after != before or name == "reset"
    failures = 0
    for k in range(0, 64):
        p = new_pool()
        build(p)
        assert state(p) == before
        p.test_fail_launch(k)
        try:
            call(p)
        except MkvError as e:
            assert e.name == "CUDA"
            assert "injected" in str(e)
            assert state(p) == before, f"{name}: failure at operation {k} changed the pool"
            failures += 1
            call(p)                       # the same call, now without the failure
            assert state(p) == after, f"{name}: retry after failure {k} differs from the twin"
            continue
        # k is past the call's last operation: it succeeded; disarm and compare
        p.test_fail_launch(-1)
        assert state(p) == after
        break
    assert failures >= 1
    if name in ("append", "demote", "prefill"):
        assert failures >= 2, f"{name}: expected a call split over several launches"


def test_hook_arguments():
    p = new_pool(16, 16)
    with pytest.raises(MkvError) as e:
        p.test_fail_launch(-2)
    assert e.value.name == "INVALID_ARG"
    p.test_fail_launch(0)
    p.test_fail_launch(-1)      # switched off again: the next call succeeds
    p.append([0], [3])
    assert p.block_table(0)[1] == 3
