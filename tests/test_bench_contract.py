"""bench.py on the CPU: the algorithmic work it divides by, counted here a
second way (token by token, pair by pair), and the keys of the reference
arm's JSON line."""

import contextlib
import io
import json
import types

import numpy as np

import bench
import workloads as W


def _count(w, seqlens):
    """Bytes and flops by explicit enumeration of tokens, pages and visible pairs."""
    T = 1152 if w.fmt == "bf16" else 656
    nbytes, pairs = 0, 0
    for L in seqlens:
        nbytes += L * T                                  # every valid cached token once
        nbytes += 4 * len(range(0, L, 64))               # one block-table entry per page
        nbytes += 4                                      # its length
        for i in range(w.s_q):
            nbytes += w.h_q * (576 * 2 + 512 * 2 + 4)    # q rows in, out rows and lse out
            for j in range(L):
                if not w.causal or j <= L - w.s_q + i:
                    pairs += 1
    return nbytes, 2 * (576 + 512) * w.h_q * pairs


def test_algorithmic_work_matches_an_explicit_count():
    for w, seqlens in [(W.Workload("a", 3, 1, 16, (1, 1)), [256, 1, 130]),
                       (W.Workload("b", 4, 2, 64, (1, 1), causal=True), [1, 2, 65, 300]),
                       (W.Workload("c", 2, 1, 128, (1, 1), fmt="fp8_656"), [64, 1000])]:
        work = bench.algorithmic_work(w, np.array(seqlens))
        assert (work["bytes"], work["flops"]) == _count(w, seqlens)


def test_append_work_matches_an_explicit_count():
    for fmt, out in [("bf16", 1152), ("fp8_656", 656)]:
        assert bench.append_work(fmt, 3, 5) == 15 * (1152 + out + 4) + 3 * 4


def test_reference_line_keys():
    args = types.SimpleNamespace(workload="tiny", steps=1, warmup=0, gpus=1)
    buf = io.StringIO()
    with contextlib.redirect_stdout(buf):
        bench.run_reference(args, 1, 0)
    line = json.loads(buf.getvalue().strip().splitlines()[-1])
    for key in ("metric", "value", "unit", "impl", "n_gpus", "steps", "warmup", "higher_is_better", "scaling",
                "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in line, key
    assert line["impl"] == "reference" and line["metric"] == bench.METRIC and line["value"] > 0
    assert line["config"]["workload"].startswith("tiny")
    cpu = line["cpu_baseline"]
    assert cpu["kind"] == "oracle" and cpu["value"] == line["value"] and cpu["cores"] >= 1 and cpu["sample"]
    assert line["e2e"] == {"value": line["value"], "unit": line["unit"], "h2d_bytes_per_step": 0,
                           "d2h_bytes_per_step": 0}


def test_sparse_work_counts_valid_entries_only():
    w = W.Workload("s", 2, 1, 16, (1, 1), fmt="fp8_656", topk=4)
    L = np.array([10, 3])
    idx = np.array([[[0, 9, -1, 10]], [[2, 2, 5, -7]]])  # valid: 2 + 2
    work = bench.sparse_work(w, L, idx)
    assert work["flops"] == 2 * (576 + 512) * 16 * 4
    assert work["bytes"] == 656 * 4 + 2 * 16 * (1152 + 1024 + 4) + 4 * idx.size + 4 * 4 + 4 * 2
