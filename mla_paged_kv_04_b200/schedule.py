"""Host-side view of the split-KV schedule written by mla_get_metadata.

`plan` computes the same schedule on the host (numpy) — for callers whose
sequence lengths already live in host memory, and as an independent second
implementation the device kernel is tested against.  `validate` checks the
invariants every schedule must satisfy; `parse` turns the int32 buffer into
per-part work lists.

Requests with M = s_q * h_q > 128 query rows are planned as ceil(M / 128)
row tiles, each a "virtual request" v = b * row_tiles + tile with request b's
length; everything below (items, splits, num_splits) is over virtual requests.

Buffer layout (int32):
  [0] parts [1] items [2] units per part [3] virtual batch [4] per-request
  overhead [5] split (virtual) requests [6] 1 in whole-request mode
  [7] row tiles
  [8, 8 + parts + 1)      first item of each part
  then `parts` ints       ids of split requests (first [5] valid)
  then, 16-byte aligned,  4 ints per item: request, first page, end page, slot
"""

from __future__ import annotations

import numpy as np

PAGE = 64
HEADER = 8
DEFAULT_OVERHEAD = 4
# Whole-request mode (ceil(batch / parts) consecutive requests per part,
# nothing split) is taken when the costliest part exceeds the balanced cut by
# at most this many pages: splitting costs a round trip of fp32 partials, the
# combine pass and a pipeline drain per extra item.
SPLIT_PENALTY = 16


def split_list_offset(parts: int) -> int:
    return HEADER + parts + 1


def items_offset(parts: int) -> int:
    return (split_list_offset(parts) + parts + 3) & ~3


def sched_ints(batch: int, parts: int) -> int:
    return items_offset(parts) + 4 * (batch + parts)


def row_tiles(s_q: int, h_q: int) -> int:
    return -(-(s_q * h_q) // 128)


def plan(seqlens, parts: int, overhead: int = DEFAULT_OVERHEAD, rtiles: int = 1):
    """Host computation of the schedule -> (sched int32[sched_ints], num_splits
    int32[batch * rtiles + 1]), over the virtual requests of `rtiles` row tiles."""
    L = np.repeat(np.maximum(np.asarray(seqlens, dtype=np.int64), 0), rtiles)
    B = L.size
    n = (L + PAGE - 1) // PAGE
    cost = n + overhead
    C = np.concatenate([[0], np.cumsum(cost)])
    T = int(C[-1])
    t = max(1, -(-T // parts))
    m = max(1, -(-B // parts))  # requests per part in whole-request mode
    firsts = np.minimum(np.arange(parts + 1) * m, B)
    span = int((C[firsts[1:]] - C[firsts[:-1]]).max(initial=0))
    if span <= t + SPLIT_PENALTY:
        sched = np.zeros(sched_ints(B, parts), dtype=np.int32)
        sched[:8] = (parts, B, span, B, overhead, 0, 1, rtiles)
        sched[HEADER:HEADER + parts + 1] = firsts
        io = items_offset(parts)
        items = np.stack([np.arange(B), np.zeros(B, dtype=np.int64), n, np.full(B, -1)], axis=1)
        sched[io:io + 4 * B] = items.reshape(-1)
        return sched, np.arange(B + 1, dtype=np.int32)
    k0 = C[:-1] // t
    k1 = (C[1:] - 1) // t
    K = k1 - k0 + 1
    S = np.concatenate([[0], np.cumsum(K)])
    I = int(S[-1])
    sched = np.zeros(sched_ints(B, parts), dtype=np.int32)
    items = np.zeros((I, 4), dtype=np.int64)
    split_reqs = []
    for b in range(B):
        for s in range(int(K[b])):
            k = int(k0[b]) + s
            v0 = max(int(C[b]), k * t) - int(C[b])
            v1 = min(int(C[b + 1]), (k + 1) * t) - int(C[b])
            p0 = min(max(v0 - overhead, 0), int(n[b]))
            p1 = min(max(v1 - overhead, 0), int(n[b]))
            idx = int(S[b]) + s
            items[idx] = (b, p0, p1, idx if K[b] > 1 else -1)
        if K[b] > 1:
            split_reqs.append(b)
    sched[:8] = (parts, I, t, B, overhead, len(split_reqs), 0, rtiles)
    for k in range(parts + 1):
        pos = k * t
        if k == parts or pos >= T:
            first = I
        else:
            b = int(np.searchsorted(C[:-1], pos, side="right") - 1)
            first = int(S[b]) + (k - int(C[b]) // t)
        sched[HEADER + k] = first
    off = split_list_offset(parts)
    sched[off:off + len(split_reqs)] = split_reqs
    io = items_offset(parts)
    sched[io:io + 4 * I] = items.reshape(-1)
    return sched, S.astype(np.int32)


def parse(sched, parts: int):
    """-> list over parts of lists of (request, first page, end page, slot)."""
    sched = np.asarray(sched)
    I = int(sched[1])
    first = sched[HEADER:HEADER + parts + 1]
    items = sched[items_offset(parts):items_offset(parts) + 4 * I].reshape(I, 4)
    return [[tuple(int(x) for x in items[i]) for i in range(first[k], first[k + 1])] for k in range(parts)]


def validate(sched, num_splits, seqlens, parts: int, rtiles: int = 1):
    """Raise AssertionError unless the schedule is a valid split-KV plan for
    `seqlens` with `rtiles` row tiles per request (every page of every row
    tile covered exactly once)."""
    sched = np.asarray(sched)
    L = np.repeat(np.maximum(np.asarray(seqlens, dtype=np.int64), 0), rtiles)
    B = L.size
    n = (L + PAGE - 1) // PAGE
    assert int(sched[0]) == parts and int(sched[3]) == B and int(sched[7]) == rtiles
    I = int(sched[1])
    assert 0 < I <= B + parts
    first = sched[HEADER:HEADER + parts + 1]
    assert first[0] == 0 and first[-1] == I and np.all(np.diff(first) >= 0)
    items = sched[items_offset(parts):items_offset(parts) + 4 * I].reshape(I, 4)
    ns = np.asarray(num_splits)
    assert ns[0] == 0 and ns[-1] == I and np.all(np.diff(ns) >= 1)
    covered = [np.zeros(int(x), dtype=np.int64) for x in n]
    split_reqs = set()
    for idx, (b, p0, p1, slot) in enumerate(items):
        assert 0 <= b < B and 0 <= p0 <= p1 <= n[b]
        assert ns[b] <= idx < ns[b + 1]
        k_b = ns[b + 1] - ns[b]
        assert slot == (idx if k_b > 1 else -1)
        covered[b][p0:p1] += 1
        if k_b > 1:
            split_reqs.add(int(b))
    for b in range(B):
        assert np.all(covered[b] == 1), f"request {b}: pages not covered exactly once"
        # items of a request are contiguous in page order
        its = items[ns[b]:ns[b + 1]]
        assert its[0][1] == 0 and its[-1][2] == n[b]
        assert np.all(its[1:, 1] == its[:-1, 2])
    nsr = int(sched[5])
    off = split_list_offset(parts)
    assert set(int(x) for x in sched[off:off + nsr]) == split_reqs and nsr == len(split_reqs)
    return True
