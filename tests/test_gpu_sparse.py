"""GPU parity of the sparse decode (mla_sparse_decode_fwd) with the oracle.

Each query token attends to the positions its index list names (reading
R11): padding (-1), positions past the request's length, repeats, lists
shorter than a tile and longer than many, several query tokens and several
row tiles per request, and split-KV schedules.  FP8 cache: compared with the
oracle fed the dequantised cache the kernel computes on (reading R8), and,
on long lists, with the exact products.
"""

import numpy as np
import pytest
import torch

import workloads as W
from _gpu_helpers import check, oracle_sparse, run_gpu_sparse

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from mla_paged_kv_04_b200 import build
    build.build()
    import mla_paged_kv_04_b200 as mla
    mla.load_library()


def _case(batch, s_q, h_q, seqlens, seed):
    w = W.Workload("sparse", batch, s_q, h_q, (1, 1), fmt="fp8_656", seed=seed)
    return W.make_case(w, seqlens=list(seqlens))


CASES = [
    # batch, s_q, h_q, seqlens, topk, dup, pad, oob, parts
    (2, 1, 128, (300, 1500), 256, 0, 0, 0, None),
    (3, 2, 64, (5000, 40, 700), 200, 7, 9, 5, None),     # repeats, padding, past-the-end
    (2, 1, 16, (64, 900), 100, 2, 3, 1, None),           # topk not a multiple of 64
    (1, 1, 128, (3000,), 2048, 0, 0, 0, 3),              # long list, split over 3 pairs
    (2, 1, 200, (700, 1300), 128, 1, 1, 1, None),        # two row tiles (h_q = 200)
    (3, 1, 128, (2000, 333, 1500), 512, 0, 4, 0, 74),    # split-KV across the default pairs
    (2, 3, 32, (4, 777), 300, 5, 0, 2, 1),               # a list mostly padding; one pair
]


@pytest.mark.parametrize("batch,s_q,h_q,seqlens,topk,dup,pad,oob,parts", CASES)
def test_sparse_matches_oracle(batch, s_q, h_q, seqlens, topk, dup, pad, oob, parts):
    c = _case(batch, s_q, h_q, seqlens, seed=50 + topk)
    idx = W.make_sparse_indices(c["cache_seqlens"], s_q, topk, seed=topk, dup=dup, pad=pad, oob=oob)
    out, lse, st = run_gpu_sparse(c, idx, num_sm_parts=parts)
    assert st == 0
    ro, rl = oracle_sparse(c, idx, dequant_bf16=True)
    check(out, lse, ro, rl, f"sparse {seqlens} topk={topk}")


def test_sparse_against_exact_dequant_oracle():
    # The exact e4m3 * scale products (no bf16 rounding of the keys) stay
    # within the same tolerances once the lists hold enough keys for the
    # rounding to average out (as for the dense FP8 decode).
    c = _case(2, 1, 128, (6000, 3000), seed=58)
    idx = W.make_sparse_indices(c["cache_seqlens"], 1, 2048, seed=3)
    out, lse, st = run_gpu_sparse(c, idx)
    assert st == 0
    ro, rl = oracle_sparse(c, idx, dequant_bf16=False)
    check(out, lse, ro, rl, "sparse, exact dequant")


def test_lists_with_no_key_give_zero_and_minus_infinity():
    c = _case(2, 1, 64, (100, 0), seed=61)
    idx = torch.full((2, 1, 128), -1, dtype=torch.int32)
    idx[0, 0, :64] = 100 + torch.arange(64, dtype=torch.int32)   # all past the end
    idx[1, 0, :10] = torch.arange(10, dtype=torch.int32)          # request of length 0
    out, lse, st = run_gpu_sparse(c, idx)
    assert st == 0
    assert np.all(out == 0) and np.all(np.isneginf(lse))


def test_full_list_equals_the_dense_decode_oracle():
    import oracle
    c = _case(2, 1, 128, (700, 130), seed=62)
    idx = torch.full((2, 1, 704), -1, dtype=torch.int32)
    for b, Lb in enumerate((700, 130)):
        idx[b, 0, :Lb] = torch.arange(Lb, dtype=torch.int32)
    out, lse, st = run_gpu_sparse(c, idx)
    assert st == 0
    from _gpu_helpers import oracle_for
    ro, rl = oracle_for(c, dequant_bf16=True)
    check(out, lse, ro, rl, "full list vs dense oracle")


def test_position_on_a_page_outside_the_cache_is_reported():
    import mla_paged_kv_04_b200 as mla
    c = _case(1, 1, 16, (200,), seed=63)
    c["block_table"][0, 1] = c["num_blocks"] + 3
    idx = torch.arange(200, dtype=torch.int32).view(1, 1, 200)
    out, lse, st = run_gpu_sparse(c, idx)
    assert mla.STATUS[st] == "MLA_ERR_BAD_BLOCK_INDEX"


def test_full_size_sparse_every_unit():
    """The sparse workload at full size (b=128, h_q=128, topk=2048 over
    L ~ U[16384, 32768]), default pairs, compared with the oracle on every
    (request, query token)."""
    w = W.WORKLOADS["sparse_fp8"]
    c = W.make_case(w, device="cuda")
    out, lse, st = run_gpu_sparse(c, c["indices"])
    assert st == 0
    ro, rl = oracle_sparse(c, c["indices"], dequant_bf16=True)
    for b in range(w.batch):
        check(out[b], lse[b], ro[b], rl[b], f"sparse_fp8 request {b}")
