"""The allocation-free decode entry point (mla_decode_fwd_noalloc).

Callers that cannot allocate device memory (graph capture, engine plugins,
servers that pre-reserve all memory) use this variant: its split-KV scratch is
a fixed array inside the library.  These tests call it through the C ABI and
compare it with the regular entry point, which gets a caller-allocated
workspace, on two calls in a row with different inputs.  The second call
sees the first call's leftovers in the shared array, so it also checks that
no stale state leaks between calls.  This file is named to be collected last.
"""

import ctypes

import numpy as np
import pytest
import torch

import workloads as W

pytestmark = pytest.mark.gpu

OUT_MAX_TOL = 2e-2
OUT_MEAN_TOL = 2e-3
LSE_TOL = 1e-3


@pytest.fixture(scope="module")
def lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from mla_paged_kv_04_b200 import build
    build.build()
    import mla_paged_kv_04_b200 as mla
    lib = mla.load_library()
    vp, c_int = ctypes.c_void_p, ctypes.c_int
    lib.mla_decode_fwd_noalloc.restype = c_int
    lib.mla_decode_fwd_noalloc.argtypes = [vp, vp, c_int, ctypes.c_int64, vp, c_int, vp, c_int, c_int, c_int,
                                           ctypes.c_float, c_int, vp, vp, c_int, vp, vp, vp]
    lib.mla_noalloc_last_device_status.restype = c_int
    lib.mla_noalloc_last_device_status.argtypes = [vp]
    return lib


def _inputs(seqlens, s_q, h_q, causal, fmt, seed):
    w = W.Workload("noalloc", len(seqlens), s_q, h_q, (1, 1), fmt=fmt, causal=causal, seed=seed)
    c = W.make_case(w, seqlens=list(seqlens), device="cuda")
    return c


def _call_noalloc(lib, c, parts, sched, ns, out, lse):
    import mla_paged_kv_04_b200 as mla
    q, kv, bt, L = c["q"], c["kv_cache"], c["block_table"], c["cache_seqlens"]
    B, s_q, h_q, _ = q.shape
    stream = torch.cuda.current_stream().cuda_stream
    return lib.mla_decode_fwd_noalloc(q.data_ptr(), kv.data_ptr(), mla.FORMATS[c["fmt"]], kv.shape[0],
                                      bt.data_ptr(), bt.shape[1], L.data_ptr(), B, s_q, h_q,
                                      float(c["softmax_scale"]), 1 if c["causal"] else 0, sched.data_ptr(),
                                      ns.data_ptr(), parts, out.data_ptr(), lse.data_ptr(), stream)


def _run_both(lib, c, parts):
    import mla_paged_kv_04_b200 as mla
    q, kv, bt, L = c["q"], c["kv_cache"], c["block_table"], c["cache_seqlens"]
    B, s_q, h_q, _ = q.shape
    sched, ns = mla.mla_get_metadata(L, s_q, h_q, parts)
    # regular entry point with a caller-allocated workspace
    ws = mla.alloc_workspace(B, s_q, h_q, parts, q.device)
    out_ref = torch.empty((B, s_q, h_q, 512), dtype=torch.bfloat16, device=q.device)
    lse_ref = torch.empty((B, s_q, h_q), dtype=torch.float32, device=q.device)
    mla.mla_decode_fwd(q, kv, c["fmt"], bt, L, c["softmax_scale"], c["causal"], sched, ns, parts, out_ref,
                       lse_ref, ws)
    # allocation-free entry point
    out = torch.full((B, s_q, h_q, 512), float("nan"), dtype=torch.bfloat16, device=q.device)
    lse = torch.full((B, s_q, h_q), float("nan"), dtype=torch.float32, device=q.device)
    st = _call_noalloc(lib, c, parts, sched, ns, out, lse)
    assert st == 0, mla.STATUS.get(st, st)
    torch.cuda.synchronize()
    assert mla.mla_last_device_status(ws) == 0
    # the status word of the allocation-free call lives in the library's array
    assert lib.mla_noalloc_last_device_status(torch.cuda.current_stream().cuda_stream) == 0
    split_requests = int((ns[1:] - ns[:-1] > 1).sum())
    return out_ref, lse_ref, out, lse, split_requests


def _compare(out_ref, lse_ref, out, lse):
    a = out.float().cpu().numpy()
    b = out_ref.float().cpu().numpy()
    assert np.all(np.isfinite(a))
    err = np.abs(a - b)
    assert err.max() <= OUT_MAX_TOL and err.mean() <= OUT_MEAN_TOL
    la, lb = lse.cpu().numpy(), lse_ref.cpu().numpy()
    assert np.array_equal(np.isneginf(la), np.isneginf(lb))
    ok = np.isfinite(lb)
    assert np.all(np.abs(la[ok] - lb[ok]) <= LSE_TOL)


def test_noalloc_matches_regular_entry_point_twice_in_a_row(lib):
    # call 1: split requests (partials go through the static scratch)
    c1 = _inputs((3000, 100, 1777, 64), 2, 64, True, "bf16", seed=21)
    r1 = _run_both(lib, c1, parts=74)
    assert r1[4] > 0, "the first case must exercise split-KV partials"
    _compare(*r1[:4])
    # call 2: different shapes, FP8 cache, fewer parts; the scratch still holds call 1's data
    c2 = _inputs((5000, 1, 700), 1, 128, False, "fp8_656", seed=22)
    r2 = _run_both(lib, c2, parts=16)
    assert r2[4] > 0
    _compare(*r2[:4])


def test_noalloc_reports_device_errors_through_its_own_status(lib):
    # a block index outside the cache: the kernel records it in the static
    # array's status word, which mla_noalloc_last_device_status reads
    import mla_paged_kv_04_b200 as mla
    c = _inputs((130, 64), 1, 16, False, "bf16", seed=23)
    c["block_table"][0, 1] = c["num_blocks"] + 5
    B = 2
    sched, ns = mla.mla_get_metadata(c["cache_seqlens"], 1, 16, 74)
    out = torch.empty((B, 1, 16, 512), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((B, 1, 16), dtype=torch.float32, device="cuda")
    assert _call_noalloc(lib, c, 74, sched, ns, out, lse) == 0
    stream = torch.cuda.current_stream().cuda_stream
    assert mla.STATUS[lib.mla_noalloc_last_device_status(stream)] == "MLA_ERR_BAD_BLOCK_INDEX"
    # the next call starts from a cleared status word
    c["block_table"][0, 1] = c["block_table"][0, 0]
    assert _call_noalloc(lib, c, 74, sched, ns, out, lse) == 0
    assert lib.mla_noalloc_last_device_status(stream) == 0


def test_noalloc_rejects_shapes_beyond_its_scratch_before_enqueuing(lib):
    # (16384 + 74) requests x 128 rows of partials need far more than 64 MiB;
    # the call must refuse before enqueuing anything.  Real (small) device
    # tensors stand behind every pointer, so even a regression that launched
    # would read and write valid memory and report a status, not fault.
    import mla_paged_kv_04_b200 as mla
    WORKSPACE, INVALID = 3, 1
    dev = torch.device("cuda")
    q = torch.zeros((1, 1, 128, 576), dtype=torch.bfloat16, device=dev)
    kv = torch.zeros((1, 64, 576), dtype=torch.bfloat16, device=dev)
    bt = torch.zeros((1, 1), dtype=torch.int32, device=dev)
    L = torch.zeros(1, dtype=torch.int32, device=dev)
    sched = torch.zeros(mla.mla_metadata_size(1, 1, 128, 74) // 4, dtype=torch.int32, device=dev)
    ns = torch.zeros(2, dtype=torch.int32, device=dev)
    out = torch.zeros((1, 1, 128, 512), dtype=torch.bfloat16, device=dev)
    lse = torch.zeros((1, 1, 128), dtype=torch.float32, device=dev)
    f = lib.mla_decode_fwd_noalloc
    args = [q.data_ptr(), kv.data_ptr(), 0, 1, bt.data_ptr(), 1, L.data_ptr(), 16384, 1, 128, 0.04, 0,
            sched.data_ptr(), ns.data_ptr(), 74, out.data_ptr(), lse.data_ptr(), None]
    assert f(*args) == WORKSPACE
    bad_parts = list(args)
    bad_parts[14] = 0
    assert f(*bad_parts) == INVALID  # the same code mla_decode_fwd returns
    torch.cuda.synchronize()
