"""Per-tile timestamps of the decode kernel, from the trace build.

`build.build(trace=True)` compiles libmla_b200_trace.so with MLA_TRACE: the
decode kernel then records the SM clock (clock64) at fixed points of every
warp role, for the first CTAs of the grid and their first tiles, into a
caller-owned device buffer (layout below, and in csrc/common.cuh).  This
module records one call and reduces the timestamps to the median length of
each phase of the pipeline, in SM cycles.  The product library records
nothing and pays nothing for it.

Layout: uint64 [CTAS, ROLES, TILES, SLOTS], zero where nothing was recorded.
"""

from __future__ import annotations

import numpy as np
import torch

CTAS, ROLES, TILES, SLOTS = 4, 7, 128, 16
PRODUCER, QK, PV, SOFTMAX, DEQUANT, ITEM, CTA = range(7)

# (name, role, from slot, to slot): the phase between two points of one role
# on the same tile.
PHASES = [
    ("producer: wait for a free stage", PRODUCER, 0, 1),
    ("qk: wait for the page", QK, 0, 1),
    ("qk: wait for S to be free", QK, 1, 2),
    ("qk: issue", QK, 2, 3),
    ("pv: wait for P", PV, 0, 1),
    ("pv: issue", PV, 1, 2),
    ("softmax: wait for S", SOFTMAX, 0, 1),
    ("softmax: load S", SOFTMAX, 1, 2),
    ("softmax: row max", SOFTMAX, 2, 3),
    ("softmax: exchange-buffer credit", SOFTMAX, 3, 4),
    ("softmax: exponentiate + send", SOFTMAX, 4, 5),
    ("softmax: wait for the peer's first half", SOFTMAX, 5, 6),
    ("softmax: form P (second half)", SOFTMAX, 6, 7),
    ("softmax: reference chain", SOFTMAX, 7, 8),
    ("softmax: P buffer free", SOFTMAX, 8, 9),
    ("softmax: rescale O", SOFTMAX, 9, 10),
    ("softmax: store P", SOFTMAX, 10, 11),
    ("softmax: S ready -> P stored", SOFTMAX, 1, 11),
    ("dequant: wait for raw bytes", DEQUANT, 0, 1),
    ("dequant: wait for a free stage", DEQUANT, 1, 2),
    ("dequant: convert a page half", DEQUANT, 2, 3),
]

# (name, role, slot, role, slot): between points of two roles on the same tile
CROSS = [
    ("page copies issued -> qk sees the page (bf16)", PRODUCER, 1, QK, 1),
    ("dequant done -> qk sees the page", DEQUANT, 3, QK, 1),
    ("qk issued -> softmax sees S", QK, 3, SOFTMAX, 1),
    ("P stored -> pv sees P", SOFTMAX, 11, PV, 1),
]


def record(run, lib=None) -> np.ndarray:
    """Run `run()` (which enqueues decode calls on the current device) with the
    trace buffer set; returns the timestamps as uint64 [CTAS, ROLES, TILES, SLOTS]."""
    import mla_paged_kv_04_b200 as mla
    lib = lib or mla.load_library(trace=True)
    nbytes = int(lib.mla_debug_trace_bytes())
    assert nbytes == CTAS * ROLES * TILES * SLOTS * 8
    buf = torch.zeros(nbytes // 8, dtype=torch.int64, device="cuda")
    st = lib.mla_debug_set_trace_buffer(buf.data_ptr(), nbytes)
    if st != 0:
        raise RuntimeError(f"mla_debug_set_trace_buffer: status {st} (is this the trace build?)")
    try:
        run()
        torch.cuda.synchronize()
    finally:
        lib.mla_debug_set_trace_buffer(None, 0)
    return buf.cpu().numpy().view(np.uint64).reshape(CTAS, ROLES, TILES, SLOTS)


def _diffs(ts, r0, s0, r1, s1, skip):
    a = ts[:, r0, :, s0].astype(np.int64)
    b = ts[:, r1, :, s1].astype(np.int64)
    ok = (a > 0) & (b > 0)
    ok[:, :skip] = False
    d = (b - a)[ok]
    return d


def summarize(ts: np.ndarray, skip: int = 4) -> dict:
    """Median cycles of each phase over the recorded tiles (the first `skip`
    tiles of a CTA, the pipeline's fill, left out), the period between
    consecutive QK^T issues, and the CTA-level start-up points."""
    out = {}
    for name, role, s0, s1 in PHASES:
        d = _diffs(ts, role, s0, role, s1, skip)
        if d.size:
            out[name] = float(np.median(d))
    for name, r0, s0, r1, s1 in CROSS:
        d = _diffs(ts, r0, s0, r1, s1, skip)
        if d.size:
            out[name] = float(np.median(d))
    per = []
    for c in range(ts.shape[0]):
        t = ts[c, QK, :, 3].astype(np.int64)
        t = t[t > 0]
        if t.size > skip + 1:
            per.append(np.diff(t[skip:]))
    if per:
        out["period: qk issue to qk issue"] = float(np.median(np.concatenate(per)))
    starts = []
    for c in range(ts.shape[0]):
        e = ts[c, CTA, 0].astype(np.int64)
        first_qk = ts[c, QK, 0, 3].astype(np.int64)
        if e[0] > 0:
            starts.append((e[1] - e[0], e[2] - e[0], first_qk - e[0] if first_qk > 0 else -1,
                           e[3] - e[0], e[4] - e[0]))
    if starts:
        s = np.median(np.array(starts, dtype=np.float64), axis=0)
        out["cta: entry -> set up"] = float(s[0])
        out["cta: entry -> schedule readable"] = float(s[1])
        out["cta: entry -> first qk issued"] = float(s[2])
        out["cta: entry -> roles done"] = float(s[3])
        out["cta: entry -> exit"] = float(s[4])
    items = []
    for c in range(ts.shape[0]):
        for it in range(TILES):
            e = ts[c, ITEM, it].astype(np.int64)
            if e[0] > 0 and e[3] > 0 and e[6] > 0:
                items.append((e[1] - e[0], e[3] - e[2], e[4] - e[2], e[5] - e[4], e[6] - e[5], e[3] - e[6]))
    if items:
        s = np.median(np.array(items, dtype=np.float64), axis=0)
        out["item: Q load"] = float(s[0])
        out["item: epilogue"] = float(s[1])
        out["item: epilogue, final reference"] = float(s[2])
        out["item: epilogue, row sums joined"] = float(s[3])
        out["item: epilogue, last PV done"] = float(s[4])
        out["item: epilogue, O out"] = float(s[5])
    return out


def format_summary(summary: dict) -> str:
    w = max(len(k) for k in summary) if summary else 0
    return "\n".join(f"{k:<{w}}  {v:10.0f}" for k, v in summary.items())
