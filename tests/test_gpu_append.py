"""Parity of the cache-append kernel (mla_kv_append) with the oracle.

The append writes bytes, so the bar is bit-exactness: the whole cache after
the GPU append (every block, poisoned slots and spare blocks included) must
equal the oracle's cache after oracle.append_tokens, for both formats.  The
FP8 codes come from a binary32 division and a round-to-nearest-even
conversion on both sides (the same precision decides the integer).
"""

import numpy as np
import pytest
import torch

import oracle
import workloads as W
from _gpu_helpers import check, oracle_for

pytestmark = pytest.mark.gpu


def _rand_bf16(shape, seed, scale=1.0):
    g = torch.Generator().manual_seed(seed)
    return (torch.randn(shape, generator=g, dtype=torch.float32) * scale).to(torch.bfloat16)


def _new_tokens(batch, s_new, seed):
    x = _rand_bf16((batch, s_new, 576), seed)
    flat = x.view(-1, 576)
    n = flat.shape[0]
    # special groups: all zero, all -0.0, tiny values (E4M3 subnormals), one outlier
    flat[0 % n, 128:256] = 0
    flat[1 % n, 0:128] = -0.0
    flat[2 % n, 256:384] = _rand_bf16((128,), seed + 1, scale=1e-6)
    flat[3 % n, 384] = 300.0
    return x


def _bits(t):
    return t.view(torch.int16).numpy().view(np.uint16)


def _run_append(case, new, fmt):
    import mla_paged_kv_04_b200 as mla
    dev = torch.device("cuda")
    kv = case["kv_cache"].to(dev)
    ws = torch.zeros(256, dtype=torch.uint8, device=dev)
    mla.mla_kv_append(new.to(dev), kv, fmt, case["block_table"].to(dev), case["cache_seqlens"].to(dev), ws)
    return kv.cpu(), mla.mla_last_device_status(ws)


def _oracle_cache(case, new, fmt):
    a = W.oracle_arrays(case)
    return oracle.append_tokens(a["kv_cache"], fmt, _bits(new), a["block_table"], a["cache_seqlens"])


def _as_oracle_layout(kv, fmt):
    return kv.view(torch.int16).numpy().view(np.uint16) if fmt == "bf16" else kv.numpy()


@pytest.mark.parametrize("fmt", ["bf16", "fp8_656"])
@pytest.mark.parametrize("seqlens,s_new", [((70, 3, 128, 1), 1), ((70, 3, 128, 64), 2), ((200, 300, 130, 1000), 130)])
def test_append_bit_exact(fmt, seqlens, s_new):
    w = W.Workload("append", len(seqlens), 1, 1, (1, 1), fmt=fmt, seed=3)
    case = W.make_case(w, seqlens=list(seqlens), poison=True)
    new = _new_tokens(len(seqlens), s_new, 40 + s_new)
    kv, status = _run_append(case, new, fmt)
    assert status == 0
    np.testing.assert_array_equal(_as_oracle_layout(kv, fmt), _oracle_cache(case, new, fmt))


def test_append_reports_bad_rows_and_writes_the_rest():
    w = W.Workload("append", 3, 1, 1, (1, 1), fmt="fp8_656", seed=4)
    case = W.make_case(w, seqlens=[2, 70, 130], poison=True)
    bt = case["block_table"].clone()
    bt[2, 2] = case["kv_cache"].shape[0] + 7   # request 2's new tokens 128..129 sit on page 2
    case = dict(case, block_table=bt)
    new = _new_tokens(3, 3, 9)
    kv, status = _run_append(case, new, "fp8_656")
    # both kinds of bad row are present; the status keeps the first one recorded
    assert status in (1, 6)
    a = W.oracle_arrays(case)
    ref = oracle.append_tokens(a["kv_cache"], "fp8_656", _bits(new), a["block_table"], a["cache_seqlens"])
    np.testing.assert_array_equal(kv.numpy(), ref)
    # each kind alone gives its own status: a bad block index only ...
    case1 = dict(case, cache_seqlens=torch.tensor([5, 70, 130], dtype=torch.int32))
    assert _run_append(case1, new, "fp8_656")[1] == 6  # MLA_ERR_BAD_BLOCK_INDEX
    # ... and a request shorter than its new tokens only
    case2 = dict(case, block_table=W.make_case(w, seqlens=[2, 70, 130])["block_table"])
    assert _run_append(case2, new, "fp8_656")[1] == 1  # MLA_ERR_INVALID_ARG


def test_append_then_decode_matches_the_oracle():
    """FP8 append of each request's newest token, then the decode on the result."""
    from _gpu_helpers import run_gpu
    w = W.Workload("append", 4, 2, 64, (1, 1), fmt="fp8_656", causal=True, seed=6)
    seqlens = [700, 64, 129, 1]
    case = W.make_case(w, seqlens=seqlens, poison=True)
    new = _new_tokens(4, 1, 11)
    kv, status = _run_append(case, new, "fp8_656")
    assert status == 0
    case = dict(case, kv_cache=kv)
    out, lse, st = run_gpu(case)
    assert st == 0
    ref_out, ref_lse = oracle_for(case, dequant_bf16=True)
    check(out, lse, ref_out, ref_lse, "append+decode")
