"""Failure detection on the GPU without a fault: a wait that runs out.

Every wait inside the decode kernel is bounded (mla_set_wait_timeout_ns).
mla_debug_hold_at_tile makes the thread that issues the P*V tensor-core work
wait, at a chosen tile, for a device flag; these tests give it a flag that
nothing sets and a short limit, so the wait runs out while pages, MMAs and
pair messages are in flight.  The call must end through the abort path with
MLA_ERR_TIMEOUT in the status word and the context usable, and the next call
on the same workspace must match the oracle again.
"""

import time

import numpy as np
import pytest
import torch

import workloads as W
from _gpu_helpers import check, oracle_for

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from mla_paged_kv_04_b200 import build
    build.build()
    import mla_paged_kv_04_b200 as mla
    mla.load_library()


# Few CTA pairs, so that the pairs run past the held tile (with the default 74
# pairs these requests would be cut into items of one or two pages).
@pytest.mark.parametrize("fmt,parts", [("bf16", 2), ("fp8_656", 2), ("bf16", 4)])
def test_wait_that_runs_out_is_reported_and_the_next_call_is_correct(fmt, parts):
    import mla_paged_kv_04_b200 as mla
    from mla_paged_kv_04_b200 import schedule
    dev = torch.device("cuda")
    w = W.Workload("timeout", 3, 1, 128, (1, 1), fmt=fmt, seed=31)
    c = W.make_case(w, seqlens=[2000, 1500, 700])  # 32, 24 and 11 pages
    q, kv, bt, L = (c[k].to(dev) for k in ("q", "kv_cache", "block_table", "cache_seqlens"))
    B = 3
    sched, ns = mla.mla_get_metadata(L, 1, 128, parts)
    per_pair = [sum(p1 - p0 for _, p0, p1, _ in part) for part in schedule.parse(sched.cpu().numpy(), parts)]
    assert max(per_pair) > 5, per_pair  # some pair reaches the held tile (one is enough to time out)
    ws = mla.alloc_workspace(B, 1, 128, parts, dev)
    out = torch.empty((B, 1, 128, 512), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((B, 1, 128), dtype=torch.float32, device=dev)
    flag = torch.zeros(1, dtype=torch.int32, device=dev)  # nothing ever sets it

    def call():
        mla.mla_decode_fwd(q, kv, fmt, bt, L, c["softmax_scale"], False, sched, ns, parts, out, lse, ws)

    call()  # warm: the first launch pays for module loading, not the waits
    assert mla.mla_last_device_status(ws) == 0
    prev = mla.mla_set_wait_timeout_ns(2_000_000)  # 2 ms per wait
    mla.mla_debug_hold_at_tile(flag, 5)
    try:
        t0 = time.perf_counter()
        call()
        status = mla.mla_last_device_status(ws)
        elapsed = time.perf_counter() - t0
    finally:
        mla.mla_debug_hold_at_tile(None)
        assert mla.mla_set_wait_timeout_ns(prev) == 2_000_000
    assert mla.STATUS[status] == "MLA_ERR_TIMEOUT"
    assert elapsed < 5.0, f"the abort path took {elapsed:.2f} s"
    # The context is usable and the workspace reusable once the status is cleared.
    mla.mla_clear_device_status(ws)
    call()
    assert mla.mla_last_device_status(ws) == 0
    ro, rl = oracle_for(c, dequant_bf16=(fmt == "fp8_656"))
    check(out.float().cpu().double().numpy(), lse.cpu().double().numpy(), ro, rl, f"{fmt} after a timeout")


def test_hold_released_by_the_flag_is_not_an_error():
    """The same hold with the flag already set passes straight through."""
    import mla_paged_kv_04_b200 as mla
    dev = torch.device("cuda")
    w = W.Workload("hold", 2, 1, 64, (1, 1), seed=32)
    c = W.make_case(w, seqlens=[900, 400])
    q, kv, bt, L = (c[k].to(dev) for k in ("q", "kv_cache", "block_table", "cache_seqlens"))
    flag = torch.ones(1, dtype=torch.int32, device=dev)
    mla.mla_debug_hold_at_tile(flag, 3)
    try:
        out, lse = mla.decode(q, kv, bt, L, c["softmax_scale"], False)
        torch.cuda.synchronize()
    finally:
        mla.mla_debug_hold_at_tile(None)
    ro, rl = oracle_for(c)
    check(out.float().cpu().double().numpy(), lse.cpu().double().numpy(), ro, rl, "released hold")
    assert np.all(np.isfinite(out.float().cpu().numpy()))
