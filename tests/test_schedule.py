"""Host logic of the split-KV schedule (CPU only): the host planner produces
valid plans (every page covered exactly once, items contiguous per part and
per request, split bookkeeping consistent) across lengths and part counts."""

import numpy as np
import pytest

from mla_paged_kv_04_b200 import schedule


@pytest.mark.parametrize("parts", [1, 2, 3, 7, 74, 148, 500])
def test_plan_is_valid_random(parts):
    rng = np.random.default_rng(parts)
    for batch in (1, 2, 17, 128, 1000):
        L = rng.integers(0, 9000, batch)
        sched, ns = schedule.plan(L, parts)
        schedule.validate(sched, ns, L, parts)


def test_plan_edge_lengths():
    for L in ([0], [1], [63, 64, 65], [0, 0, 0], [131072] * 8, [1] * 300):
        for parts in (1, 5, 74):
            sched, ns = schedule.plan(L, parts)
            schedule.validate(sched, ns, L, parts)


def test_long_context_is_split_across_parts():
    # 8 requests of 2048 pages on 74 CTA pairs: every request is split ~9 ways
    sched, ns = schedule.plan([131072] * 8, 74)
    splits = np.diff(ns)
    assert splits.min() >= 9 and int(sched[5]) == 8
    loads = [sum(p1 - p0 for _, p0, p1, _ in part) for part in schedule.parse(sched, 74)]
    assert max(loads) <= -(-8 * 2048 // 74) + 4  # within the per-request overhead of a perfect split
    assert min(loads) >= 8 * 2048 // 74 - 16


def test_single_part_never_splits():
    L = np.arange(0, 5000, 37)
    sched, ns = schedule.plan(L, 1)
    assert np.all(np.diff(ns) == 1) and int(sched[5]) == 0


def test_validate_rejects_a_broken_plan():
    L = [300, 500]
    sched, ns = schedule.plan(L, 4)
    bad = sched.copy()
    io = schedule.items_offset(4)
    bad[io + 2] += 1  # first item's end page overlaps the next item
    with pytest.raises(AssertionError):
        schedule.validate(bad, ns, L, 4)


def test_whole_requests_when_the_batch_fits():
    # 64 equal requests on 74 CTA pairs: one request per pair, nothing split
    L = [4096] * 64
    sched, ns = schedule.plan(L, 74)
    schedule.validate(sched, ns, L, 74)
    assert int(sched[6]) == 1 and int(sched[5]) == 0
    assert np.array_equal(np.diff(ns), np.ones(64, dtype=np.int32))
    parts = schedule.parse(sched, 74)
    assert [len(x) for x in parts] == [1] * 64 + [0] * 10
    assert all(parts[b][0] == (b, 0, 64, -1) for b in range(64))


def test_equal_requests_above_the_parts_stay_whole():
    # 128 equal requests of 32 pages (the sparse decode's 2048-entry lists) on
    # 74 CTA pairs: two whole requests per pair (72 units against a balanced
    # cut of 63) instead of splitting nearly every request
    L = [2048] * 128
    sched, ns = schedule.plan(L, 74)
    schedule.validate(sched, ns, L, 74)
    assert int(sched[6]) == 1 and int(sched[5]) == 0 and int(sched[2]) == 72
    parts = schedule.parse(sched, 74)
    assert [len(x) for x in parts] == [2] * 64 + [0] * 10
    assert all(parts[k] == [(2 * k, 0, 32, -1), (2 * k + 1, 0, 32, -1)] for k in range(64))


def test_imbalanced_batch_is_still_split():
    # one request far above the balanced cut: splitting wins over the penalty
    L = [4096] * 63 + [65536]
    sched, ns = schedule.plan(L, 74)
    schedule.validate(sched, ns, L, 74)
    assert int(sched[6]) == 0 and int(sched[5]) >= 1


def test_batch_above_parts_uses_the_balanced_cut():
    L = [4096] * 128
    sched, ns = schedule.plan(L, 74)
    schedule.validate(sched, ns, L, 74)
    assert int(sched[6]) == 0


@pytest.mark.parametrize("rtiles", [2, 3, 8])
def test_row_tiles_are_planned_as_virtual_requests(rtiles):
    rng = np.random.default_rng(rtiles)
    for parts in (1, 5, 74):
        L = rng.integers(0, 6000, 23)
        sched, ns = schedule.plan(L, parts, rtiles=rtiles)
        schedule.validate(sched, ns, L, parts, rtiles=rtiles)
        assert int(sched[3]) == 23 * rtiles and int(sched[7]) == rtiles and ns.size == 23 * rtiles + 1
        # every row tile of request b has request b's pages
        items = [it for part in schedule.parse(sched, parts) for it in part]
        for v in range(23 * rtiles):
            pages = sum(p1 - p0 for vb, p0, p1, _ in items if vb == v)
            assert pages == -(-int(L[v // rtiles]) // 64)
