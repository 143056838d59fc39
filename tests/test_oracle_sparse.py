"""Pins of the sparse decode oracle (oracle.mla_sparse_decode, reading R11).

Each query token attends to the positions its index list names; entries
outside [0, L) are padding; every valid entry is one softmax term.  The pins
come from outside the function: the dense decode (the list of every position
must reproduce it), invariances (order and padding of the list), closed forms
(one key, one key listed twice, no key) and brute-force Python loops that
decode keys with torch's own bf16 / float8 conversions.  Planted mistakes
(duplicates dropped, a causal mask added, positions taken as physical cache
slots, padding read as keys) each fail one of them.
"""

import math

import numpy as np
import pytest
import torch

import oracle
from oracle import mla as om
import workloads as W


def _case(batch=2, s_q=1, h_q=3, seqlens=(150, 7), fmt="bf16", seed=3):
    w = W.Workload("sparse", batch, s_q, h_q, (1, 1), fmt=fmt, seed=seed)
    return W.oracle_arrays(W.make_case(w, seqlens=list(seqlens)))


def _sparse(a, idx, fn=None):
    fn = fn or oracle.mla_sparse_decode
    return fn(a["q_bits"], a["kv_cache"], a["fmt"], a["block_table"], a["cache_seqlens"], idx, a["softmax_scale"])


def _random_indices(L, s_q, topk, rng, pad_frac=0.2, dup=True):
    """[b, s_q, topk] positions: random valid ones (with repeats if dup), some
    padding entries (-1 or >= L)."""
    B = len(L)
    idx = np.full((B, s_q, topk), -1, dtype=np.int32)
    for b in range(B):
        for i in range(s_q):
            if L[b] == 0:
                continue
            n = topk if dup else min(topk, int(L[b]))
            vals = rng.integers(0, int(L[b]), n) if dup else rng.permutation(int(L[b]))[:n]
            idx[b, i, :n] = vals
            pad = rng.random(topk) < pad_frac
            idx[b, i][pad] = np.where(rng.random(int(pad.sum())) < 0.5, -1, int(L[b]) + 3)
    return idx


def _brute(a, idx):
    """Pure-Python loops; keys decoded with torch's bf16 / float8 conversions."""
    q = torch.from_numpy(a["q_bits"].view(np.int16)).view(torch.bfloat16).double()
    B, s_q, h_q, _ = q.shape
    kv = a["kv_cache"]
    out = np.zeros((B, s_q, h_q, 512))
    lse = np.full((B, s_q, h_q), -np.inf)

    def key(b, j):
        row = kv[int(a["block_table"][b][j // 64]), j % 64]
        if a["fmt"] == "bf16":
            return torch.from_numpy(row.view(np.int16).copy()).view(torch.bfloat16).double().tolist()
        codes = torch.from_numpy(row[:512].copy()).view(torch.float8_e4m3fn).double()
        sc = torch.from_numpy(row[512:528].copy()).view(torch.float32).double()
        rope = torch.from_numpy(row[528:].copy()).view(torch.bfloat16).double().tolist()
        return [float(codes[d]) * float(sc[d // 128]) for d in range(512)] + rope

    for b in range(B):
        L = int(a["cache_seqlens"][b])
        for i in range(s_q):
            keys = [key(b, int(j)) for j in idx[b, i] if 0 <= int(j) < L]
            if not keys:
                continue
            for h in range(h_q):
                qv = q[b, i, h].tolist()
                xs = [a["softmax_scale"] * sum(qv[d] * k[d] for d in range(576)) for k in keys]
                m = max(xs)
                tot = sum(math.exp(x - m) for x in xs)
                lse[b, i, h] = m + math.log(tot)
                for d in range(512):
                    out[b, i, h, d] = sum(math.exp(x - m) / tot * k[d] for x, k in zip(xs, keys))
    return out, lse


@pytest.mark.parametrize("fmt", ["bf16", "fp8_656"])
def test_brute_force_with_repeats_and_padding(fmt):
    a = _case(batch=2, s_q=2, h_q=2, seqlens=(90, 5), fmt=fmt)
    idx = _random_indices([90, 5], 2, 12, np.random.default_rng(1))
    o, l = _sparse(a, idx)
    bo, bl = _brute(a, idx)
    np.testing.assert_allclose(o, bo, rtol=0, atol=1e-12)
    np.testing.assert_allclose(l, bl, rtol=0, atol=1e-12)


@pytest.mark.parametrize("fmt", ["bf16", "fp8_656"])
def test_every_position_listed_equals_the_dense_decode(fmt):
    L = [150, 7, 64]
    a = _case(batch=3, s_q=2, h_q=4, seqlens=L, fmt=fmt)
    topk = 160
    idx = np.full((3, 2, topk), -1, dtype=np.int32)
    for b in range(3):
        idx[b, :, :L[b]] = np.arange(L[b])
    o, l = _sparse(a, idx)
    do, dl = oracle.mla_decode(a["q_bits"], a["kv_cache"], a["fmt"], a["block_table"], a["cache_seqlens"],
                               a["softmax_scale"], False)
    np.testing.assert_allclose(o, do, rtol=0, atol=1e-12)
    np.testing.assert_allclose(l, dl, rtol=0, atol=1e-12)


def test_order_and_padding_of_the_list_do_not_matter():
    a = _case(batch=2, s_q=1, h_q=3, seqlens=(200, 40))
    rng = np.random.default_rng(2)
    idx = _random_indices([200, 40], 1, 32, rng, pad_frac=0.0)
    o, l = _sparse(a, idx)
    perm = idx[:, :, rng.permutation(32)]
    o2, l2 = _sparse(a, perm)
    np.testing.assert_allclose(o2, o, rtol=0, atol=1e-12)
    np.testing.assert_allclose(l2, l, rtol=0, atol=1e-12)
    padded = np.concatenate([idx, np.full((2, 1, 9), -1, np.int32), np.full((2, 1, 3), 10 ** 6, np.int32)], axis=2)
    o3, l3 = _sparse(a, padded)
    np.testing.assert_array_equal(o3, o)
    np.testing.assert_array_equal(l3, l)


def test_one_key_and_one_key_listed_twice():
    a = _case(batch=1, s_q=1, h_q=4, seqlens=(100,))
    j = 77
    k = om.gather_keys(a["kv_cache"], a["fmt"], a["block_table"][0], 100)[j]
    q = om.decode_bf16_bits(a["q_bits"][0, 0])
    x = a["softmax_scale"] * (q @ k)
    o, l = _sparse(a, np.array([[[j, -1, -1]]], dtype=np.int32))
    np.testing.assert_array_equal(o[0, 0], np.broadcast_to(k[:512], (4, 512)))
    np.testing.assert_allclose(l[0, 0], x, rtol=0, atol=1e-12)
    o, l = _sparse(a, np.array([[[j, 500, j]]], dtype=np.int32))
    np.testing.assert_allclose(o[0, 0], np.broadcast_to(k[:512], (4, 512)), rtol=0, atol=1e-12)
    np.testing.assert_allclose(l[0, 0], x + math.log(2.0), rtol=0, atol=1e-12)


def test_no_valid_entry_gives_zero_and_minus_infinity():
    a = _case(batch=2, s_q=1, h_q=2, seqlens=(10, 0))
    idx = np.array([[[-1, 10, 11]], [[0, 1, 2]]], dtype=np.int32)  # request 1 has no tokens
    o, l = _sparse(a, idx)
    assert np.all(o == 0) and np.all(np.isneginf(l))


def _mutant(kind):
    def fn(q_bits, kv_cache, fmt, block_table, cache_seqlens, indices, softmax_scale):
        B, s_q, h_q, _ = q_bits.shape
        out = np.zeros((B, s_q, h_q, 512))
        lse = np.full((B, s_q, h_q), -np.inf)
        for b in range(B):
            L = int(cache_seqlens[b])
            if kind == "physical_slots":
                flat = om.gather_keys(kv_cache, fmt, np.arange(kv_cache.shape[0]), kv_cache.shape[0] * 64)
                keys = flat
            else:
                keys = om.gather_keys(kv_cache, fmt, block_table[b], L)
            q = om.decode_bf16_bits(q_bits[b])
            for i in range(s_q):
                sel = np.asarray(indices[b, i], dtype=np.int64)
                if kind == "padding_read":
                    sel = sel[sel < L] % max(L, 1)
                else:
                    sel = sel[(sel >= 0) & (sel < L)]
                if kind == "dedup":
                    sel = np.unique(sel)
                if kind == "causal":
                    sel = sel[sel <= L - s_q + i]
                if sel.size == 0:
                    continue
                k = keys[sel]
                x = softmax_scale * (q[i] @ k.T)
                m = x.max(1)
                l_ = m + np.log(np.exp(x - m[:, None]).sum(1))
                out[b, i] = np.exp(x - l_[:, None]) @ k[:, :512]
                lse[b, i] = l_
        return out, lse
    return fn


@pytest.mark.parametrize("kind", ["dedup", "causal", "physical_slots", "padding_read"])
def test_planted_mistakes_are_caught(kind):
    bad = _mutant(kind)
    caught = []
    a = _case(batch=2, s_q=2, h_q=2, seqlens=(90, 5))
    idx = _random_indices([90, 5], 2, 12, np.random.default_rng(1))
    o, l = _sparse(a, idx, bad)
    bo, bl = _brute(a, idx)
    caught.append(not (np.allclose(o, bo, atol=1e-12) and np.allclose(l, bl, atol=1e-12, equal_nan=True)))
    assert any(caught), f"mutant {kind} passed every pin"
