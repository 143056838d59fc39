"""GPU parity: the CUDA path (through the C ABI) against the float64 oracle.

Small cases run the oracle on every output element; the five configured
workloads run at full size in the launch configuration the bench times, with
the oracle evaluated on every request.
"""

import numpy as np
import pytest
import torch

import workloads as W
from _gpu_helpers import check, oracle_chunked, oracle_for, run_gpu

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from mla_paged_kv_04_b200 import build
    build.build()
    import mla_paged_kv_04_b200 as mla
    mla.load_library()


def _case(batch, s_q, h_q, seqlens, fmt="bf16", causal=False, seed=0, poison=True):
    w = W.Workload("t", batch, s_q, h_q, (1, 1), fmt=fmt, causal=causal, seed=seed)
    return W.make_case(w, seqlens=list(seqlens), poison=poison)


def test_tiny_config_full():
    c = W.make_case(W.WORKLOADS["tiny"])
    out, lse, st = run_gpu(c)
    assert st == 0
    ro, rl = oracle_for(c)
    check(out, lse, ro, rl, "tiny")


SMALL = [
    # batch, s_q, h_q, seqlens, causal
    (4, 1, 128, (300, 1000, 64, 130), False),
    (3, 2, 64, (700, 1, 65), True),
    (5, 1, 16, (63, 64, 65, 128, 1), False),
    (2, 2, 32, (129, 2), True),
    (2, 1, 100, (257, 190), False),   # M not a power of two
    (2, 4, 32, (333, 4), True),       # s_q = 4
]

# M = s_q * h_q above 128: row tiles of 128 rows scheduled as separate units
WIDE = [
    # batch, s_q, h_q, seqlens, causal, parts
    (2, 2, 128, (700, 1500), True, None),     # M = 256, speculative pair with 128 heads
    (3, 4, 64, (65, 2000, 3), True, None),    # M = 256
    (1, 3, 128, (2500,), True, None),         # M = 384, three row tiles
    (2, 2, 100, (900, 64), False, None),      # M = 200: a full and a partial row tile
    (2, 8, 128, (1200, 130), True, None),     # M = 1024, the largest
    (3, 2, 128, (3000, 100, 1777), True, 7),  # row tiles and split-KV together
]


@pytest.mark.parametrize("batch,s_q,h_q,seqlens,causal", SMALL)
def test_small_bf16(batch, s_q, h_q, seqlens, causal):
    c = _case(batch, s_q, h_q, seqlens, causal=causal, seed=batch + s_q)
    out, lse, st = run_gpu(c)
    assert st == 0
    ro, rl = oracle_for(c)
    check(out, lse, ro, rl, f"bf16 {seqlens}")


@pytest.mark.parametrize("batch,s_q,h_q,seqlens,causal,parts", WIDE)
def test_wide_rows_bf16(batch, s_q, h_q, seqlens, causal, parts):
    c = _case(batch, s_q, h_q, seqlens, causal=causal, seed=40 + s_q * h_q)
    out, lse, st = run_gpu(c, num_sm_parts=parts)
    assert st == 0
    ro, rl = oracle_for(c)
    check(out, lse, ro, rl, f"bf16 M={s_q * h_q} {seqlens}")


def test_wide_rows_fp8():
    c = _case(2, 2, 128, (1500, 333), fmt="fp8_656", causal=True, seed=44)
    out, lse, st = run_gpu(c)
    assert st == 0
    ro, rl = oracle_for(c, dequant_bf16=True)
    check(out, lse, ro, rl, "fp8 M=256")


@pytest.mark.parametrize("batch,s_q,h_q,seqlens,causal", SMALL[:4])
def test_small_fp8(batch, s_q, h_q, seqlens, causal):
    c = _case(batch, s_q, h_q, seqlens, fmt="fp8_656", causal=causal, seed=7 + batch)
    out, lse, st = run_gpu(c)
    assert st == 0
    ro, rl = oracle_for(c, dequant_bf16=True)
    check(out, lse, ro, rl, f"fp8 {seqlens}")


def test_fp8_against_exact_dequant_oracle():
    # The exact e4m3*scale products (no bf16 rounding) stay within the same
    # tolerances once requests hold more than a handful of tokens.
    c = _case(3, 1, 128, (2000, 700, 4000), fmt="fp8_656", seed=3)
    out, lse, st = run_gpu(c)
    assert st == 0
    ro, rl = oracle_for(c)
    check(out, lse, ro, rl, "fp8 exact")


@pytest.mark.parametrize("parts", [1, 2, 3, 7, 74, 200])
def test_forced_splits_agree(parts):
    c = _case(3, 2, 64, (1500, 100, 777), causal=True, seed=11)
    out, lse, st = run_gpu(c, num_sm_parts=parts)
    assert st == 0
    ro, rl = oracle_for(c)
    check(out, lse, ro, rl, f"parts={parts}")


def test_zero_length_and_empty_causal_row():
    c = _case(3, 2, 16, (0, 1, 70), causal=True, seed=2)
    out, lse, st = run_gpu(c)
    assert st == 0
    ro, rl = oracle_for(c)
    check(out, lse, ro, rl, "empty rows")
    assert np.all(out[0] == 0) and np.all(np.isneginf(lse[0]))
    assert np.all(out[1, 0] == 0) and np.all(np.isneginf(lse[1, 0]))


def test_poison_does_not_change_results():
    seqlens = (65, 200, 7)
    clean = _case(3, 1, 64, seqlens, poison=False, seed=4)
    dirty = _case(3, 1, 64, seqlens, poison=True, seed=4)
    o1, l1, s1 = run_gpu(clean)
    o2, l2, s2 = run_gpu(dirty)
    assert s1 == 0 and s2 == 0
    np.testing.assert_array_equal(o1, o2)
    np.testing.assert_array_equal(l1, l2)


def test_deterministic():
    c = _case(2, 1, 128, (900, 300), seed=5)
    o1, l1, _ = run_gpu(c, num_sm_parts=8)
    o2, l2, _ = run_gpu(c, num_sm_parts=8)
    np.testing.assert_array_equal(o1, o2)
    np.testing.assert_array_equal(l1, l2)


def test_bad_block_index_reported():
    import mla_paged_kv_04_b200 as mla
    c = _case(2, 1, 16, (130, 64), seed=6)
    c["block_table"][0, 1] = c["num_blocks"] + 5
    out, lse, st = run_gpu(c)
    assert mla.STATUS[st] == "MLA_ERR_BAD_BLOCK_INDEX"


def test_metadata_covers_every_page_once():
    import mla_paged_kv_04_b200 as mla
    from mla_paged_kv_04_b200 import schedule
    g = torch.Generator().manual_seed(9)
    for parts in (1, 5, 74, 300):
        L = torch.randint(0, 5000, (97,), generator=g, dtype=torch.int32)
        L[3] = 0
        sched, ns = mla.mla_get_metadata(L.cuda(), 1, 128, parts)
        torch.cuda.synchronize()
        dev_sched, dev_ns = sched.cpu().numpy(), ns.cpu().numpy()
        schedule.validate(dev_sched, dev_ns, L.numpy(), parts)
        host_sched, host_ns = schedule.plan(L.numpy(), parts)
        np.testing.assert_array_equal(dev_ns, host_ns)
        used = schedule.items_offset(parts) + 4 * int(host_sched[1])
        np.testing.assert_array_equal(dev_sched[:8], host_sched[:8])
        np.testing.assert_array_equal(dev_sched[8:8 + parts + 1], host_sched[8:8 + parts + 1])
        io = schedule.items_offset(parts)
        np.testing.assert_array_equal(dev_sched[io:used], host_sched[io:used])
    # two and three row tiles per request (M = 256, 384)
    for s_q, rt in ((2, 2), (3, 3)):
        L = torch.randint(0, 5000, (41,), generator=g, dtype=torch.int32)
        sched, ns = mla.mla_get_metadata(L.cuda(), s_q, 128, 74)
        torch.cuda.synchronize()
        dev_sched, dev_ns = sched.cpu().numpy(), ns.cpu().numpy()
        schedule.validate(dev_sched, dev_ns, L.numpy(), 74, rtiles=rt)
        host_sched, host_ns = schedule.plan(L.numpy(), 74, rtiles=rt)
        np.testing.assert_array_equal(dev_ns, host_ns)
        np.testing.assert_array_equal(dev_sched[:8 + 74 + 1], host_sched[:8 + 74 + 1])
        off, nsr = schedule.split_list_offset(74), int(host_sched[5])
        np.testing.assert_array_equal(dev_sched[off:off + nsr], host_sched[off:off + nsr])
        io = schedule.items_offset(74)
        used = io + 4 * int(host_sched[1])
        np.testing.assert_array_equal(dev_sched[io:used], host_sched[io:used])


def _same_schedule(dev_sched, dev_ns, host_sched, host_ns, parts):
    np.testing.assert_array_equal(dev_ns, host_ns)
    np.testing.assert_array_equal(dev_sched[:8 + parts + 1], host_sched[:8 + parts + 1])
    off, nsr = schedule_mod().split_list_offset(parts), int(host_sched[5])
    np.testing.assert_array_equal(dev_sched[off:off + nsr], host_sched[off:off + nsr])
    io = schedule_mod().items_offset(parts)
    used = io + 4 * int(host_sched[1])
    np.testing.assert_array_equal(dev_sched[io:used], host_sched[io:used])


def schedule_mod():
    from mla_paged_kv_04_b200 import schedule
    return schedule


@pytest.mark.parametrize("lengths,parts", [([2048] * 128, 74), ([640] * 300, 74), ([100, 90, 80, 70, 60], 2)])
def test_metadata_whole_requests_several_per_pair(lengths, parts):
    """Equal requests above the CTA-pair count: the device schedule takes the
    whole-request mode with ceil(batch / parts) requests per pair, exactly as
    the host planner does."""
    import mla_paged_kv_04_b200 as mla
    schedule = schedule_mod()
    L = torch.tensor(lengths, dtype=torch.int32)
    sched, ns = mla.mla_get_metadata(L.cuda(), 1, 128, parts)
    torch.cuda.synchronize()
    dev_sched, dev_ns = sched.cpu().numpy(), ns.cpu().numpy()
    schedule.validate(dev_sched, dev_ns, L.numpy(), parts)
    host_sched, host_ns = schedule.plan(L.numpy(), parts)
    assert int(host_sched[6]) == 1
    _same_schedule(dev_sched, dev_ns, host_sched, host_ns, parts)


@pytest.mark.parametrize("batch,s_q,h_q,topk,parts", [(128, 1, 128, 2048, 74), (3, 2, 200, 300, 5), (40, 4, 64, 64, 74)])
def test_sparse_metadata_matches_the_host_planner(batch, s_q, h_q, topk, parts):
    """The sparse schedule plans batch * s_q units of h_q rows (row tiles of
    128), each of length topk, like the dense planner with equal lengths."""
    import mla_paged_kv_04_b200 as mla
    schedule = schedule_mod()
    sched, ns = mla.mla_get_sparse_metadata(batch, s_q, h_q, topk, parts, device="cuda")
    torch.cuda.synchronize()
    rt = schedule.row_tiles(1, h_q)
    lengths = np.full(batch * s_q, topk)
    dev_sched, dev_ns = sched.cpu().numpy(), ns.cpu().numpy()
    schedule.validate(dev_sched, dev_ns, lengths, parts, rtiles=rt)
    host_sched, host_ns = schedule.plan(lengths, parts, rtiles=rt)
    _same_schedule(dev_sched, dev_ns, host_sched, host_ns, parts)


@pytest.mark.parametrize("name", W.ORDER)
def test_full_size_every_request(name):
    """Each configured workload at full size, in the launch configuration the
    bench times (default CTA-pair count), compared with the oracle on every
    request, element by element.  FP8: against the oracle fed the dequantised
    cache the kernel computes on (reading R8) and against the exact products."""
    w = W.WORKLOADS[name]
    c = W.make_case(w, device="cuda")
    out, lse, st = run_gpu(c)
    assert st == 0
    variants = [True, False] if w.fmt == "fp8_656" else [False]
    for dequant_bf16 in variants:
        ro, rl = oracle_chunked(c, dequant_bf16=dequant_bf16)
        for b in range(w.batch):
            check(out[b], lse[b], ro[b], rl[b], f"{name} request {b} (bf16 dequant oracle: {dequant_bf16})")


def test_schedule_of_another_batch_is_rejected_on_the_device():
    """A schedule made for a larger batch (same CTA-pair count) must not be
    followed: its request ids and slots lie outside this call's tensors.  The
    kernels report MLA_ERR_INVALID_ARG and write nothing."""
    import mla_paged_kv_04_b200 as mla
    dev = torch.device("cuda")
    c = _case(3, 1, 64, (300, 70, 1000), seed=12)
    q, kv, bt, L = (c[k].to(dev) for k in ("q", "kv_cache", "block_table", "cache_seqlens"))
    parts = mla.mla_default_num_sm_parts()
    big_L = torch.full((97,), 2000, dtype=torch.int32, device=dev)
    sched, ns = mla.mla_get_metadata(big_L, 1, 64, parts)
    ws = mla.alloc_workspace(3, 1, 64, parts, dev)
    out = torch.full((3, 1, 64, 512), 7.0, dtype=torch.bfloat16, device=dev)
    lse = torch.full((3, 1, 64), 7.0, dtype=torch.float32, device=dev)
    mla.mla_decode_fwd(q, kv, "bf16", bt, L, c["softmax_scale"], False, sched, ns, parts, out, lse, ws)
    assert mla.STATUS[mla.mla_last_device_status(ws)] == "MLA_ERR_INVALID_ARG"
    assert torch.all(out == 7.0) and torch.all(lse == 7.0)
    # the right schedule on the same workspace, once the status is cleared
    mla.mla_clear_device_status(ws)
    sched, ns = mla.mla_get_metadata(L, 1, 64, parts)
    mla.mla_decode_fwd(q, kv, "bf16", bt, L, c["softmax_scale"], False, sched, ns, parts, out, lse, ws)
    assert mla.mla_last_device_status(ws) == 0
    ro, rl = oracle_for(c)
    check(out.float().cpu().double().numpy(), lse.cpu().double().numpy(), ro, rl, "after a rejected schedule")
