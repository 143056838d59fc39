"""Pins for the float64 oracle (CPU only).

Each test checks the oracle against something other than itself: a closed
form, an invariant of the method, a library routine (torch's float8 / bf16
conversions, torch's float64 scaled_dot_product_attention), brute force on
tiny inputs, or the byte counts printed on the menfem.com DeepSeek page.  The
mutation tests at the end plant plausible mistakes in copies of the oracle and
check that at least one pin catches each of them.
"""

import math
import os

import numpy as np
import pytest
import torch

import oracle
from oracle import mla as om
import workloads as W

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _case(batch=2, s_q=1, h_q=4, seqlens=(70, 5), fmt="bf16", causal=False, seed=1, poison=True):
    w = W.Workload("t", batch, s_q, h_q, (1, 1), fmt=fmt, causal=causal, seed=seed)
    return W.make_case(w, seqlens=list(seqlens), poison=poison)


def _run(a, **over):
    kw = dict(a)
    kw.update(over)
    return oracle.mla_decode(kw["q_bits"], kw["kv_cache"], kw["fmt"], kw["block_table"],
                             kw["cache_seqlens"], kw["softmax_scale"], kw["causal"])


# ---------------------------------------------------------------------------
# number formats
# ---------------------------------------------------------------------------

def test_e4m3_known_values():
    # OCP FP8 E4M3: bias 7, max normal 448 = 1.75 * 2^8, min subnormal 2^-9.
    table = {0x00: 0.0, 0x01: 2.0 ** -9, 0x07: 7 / 8 * 2.0 ** -6, 0x08: 2.0 ** -6,
             0x38: 1.0, 0x40: 2.0, 0x3C: 1.5, 0x7E: 448.0, 0xFE: -448.0, 0xB8: -1.0}
    codes = np.array(list(table), dtype=np.uint8)
    got = oracle.decode_e4m3(codes)
    np.testing.assert_array_equal(got, np.array(list(table.values())))
    assert np.isnan(oracle.decode_e4m3(np.array([0x7F, 0xFF], dtype=np.uint8))).all()
    assert math.copysign(1.0, oracle.decode_e4m3(np.array([0x80], dtype=np.uint8))[0]) == -1.0


def test_e4m3_all_codes_match_torch():
    codes = np.arange(256, dtype=np.uint8)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = oracle.decode_e4m3(codes)
    np.testing.assert_array_equal(np.isnan(got), np.isnan(ref))
    ok = ~np.isnan(ref)
    np.testing.assert_array_equal(got[ok], ref[ok])
    # strictly increasing magnitude over the positive non-NaN codes
    assert np.all(np.diff(got[:0x7F]) > 0)


def test_bf16_decode_matches_torch():
    rng = np.random.default_rng(0)
    bits = np.concatenate([rng.integers(0, 1 << 16, 5000).astype(np.uint16),
                           np.array([0x3F80, 0xC000, 0x7F80, 0xFF80, 0x0001, 0x8000], np.uint16)])
    ref = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()
    got = oracle.decode_bf16_bits(bits)
    np.testing.assert_array_equal(np.isnan(got), np.isnan(ref))
    ok = ~np.isnan(ref)
    np.testing.assert_array_equal(got[ok], ref[ok])
    assert got[-6] == 1.0 and got[-5] == -2.0 and got[-4] == np.inf


def test_fp8_656_layout_golden():
    vals = {}
    with open(os.path.join(GOLDEN, "fp8_656_layout.txt")) as f:
        for line in f:
            if line.strip() and not line.startswith("#"):
                k, v = line.split()
                vals[k] = int(v)
    assert om.FP8_TOKEN_BYTES == vals["fp8_token_bytes"] == 656
    assert om.BF16_TOKEN_BYTES == vals["bf16_token_bytes"] == 1152
    assert om.D_LATENT == vals["latent_dims"] and om.D_ROPE == vals["rope_dims"]
    assert vals["fp8_latent_code_bytes"] + vals["fp8_scale_bytes"] + vals["fp8_rope_bytes"] == 656
    assert om.PAGE_SIZE == vals["page_tokens"]
    assert W.FP8_BYTES == 656 and W.PAGE == 64


def test_fp8_unpack_hand_built_token():
    tok = np.zeros(656, dtype=np.uint8)
    scales = np.array([0.5, 2.0, -1.0, 0.125], dtype="<f4")
    tok[512:528] = scales.view(np.uint8)
    tok[0] = 0x38      # 1.0 in group 0  -> 0.5
    tok[130] = 0x40    # 2.0 in group 1  -> 4.0
    tok[300] = 0xB8    # -1.0 in group 2 -> 1.0
    tok[511] = 0x7E    # 448 in group 3  -> 56
    rope = np.zeros(64, dtype="<u2")
    rope[0] = 0x3F80   # 1.0
    rope[63] = 0xC040  # -3.0
    tok[528:] = rope.view(np.uint8)
    k = oracle.unpack_fp8_656(tok)
    assert k.shape == (576,)
    assert k[0] == 0.5 and k[130] == 4.0 and k[300] == 1.0 and k[511] == 56.0
    assert k[512] == 1.0 and k[575] == -3.0
    assert np.count_nonzero(k) == 6


def test_fp8_roundtrip_through_generator():
    g = torch.Generator().manual_seed(3)
    lat = (torch.randn(257, 512, generator=g) * torch.tensor([0.01, 1.0, 30.0, 1e-3]).repeat_interleave(128)).to(torch.bfloat16)
    lat[5, 128:256] = 0  # an all-zero group: scale 0, codes 0
    rope = torch.randn(257, 64, generator=g).to(torch.bfloat16)
    packed = W.quantize_fp8_656(lat, rope).numpy()
    k = oracle.unpack_fp8_656(packed)
    x = lat.to(torch.float64).numpy()
    scale = np.ascontiguousarray(packed[:, 512:528]).view("<f4").astype(np.float64)
    bound = np.abs(x) * 2.0 ** -4 + np.repeat(scale, 128, axis=1) * 2.0 ** -10
    assert np.all(np.abs(k[:, :512] - x) <= bound * (1 + 1e-6))
    assert np.all(k[5, 128:256] == 0)
    np.testing.assert_array_equal(k[:, 512:], rope.to(torch.float64).numpy())
    # the group maximum lands on the e4m3 maximum code (448)
    codes = packed[:, :512].reshape(257, 4, 128)
    mags = codes & 0x7F
    assert np.all((mags.max(axis=2) == 0x7E) | (scale == 0))


def test_bf16_dequant_mirror_is_one_rounding_of_the_exact_keys():
    """The FP8 parity tests feed the oracle the cache the CUDA path computes on
    (reading R8): latent dims bf16(fp32(e4m3) * fp32(scale)), RoPE as stored.
    Pinned against the exact products: within one bf16 rounding (2^-8
    relative, plus the fp32 product's 2^-24) of them; equal to them when the scale is a power of two (an
    e4m3 code times a power of two is a bf16 number); the RoPE dims untouched."""
    from _gpu_helpers import fp8_cache_as_bf16
    g = torch.Generator().manual_seed(8)
    n = 640
    lat = (torch.randn(n, 512, generator=g) * torch.tensor([0.3, 1.0, 7.0, 50.0]).repeat_interleave(128))
    rope = torch.randn(n, 64, generator=g).to(torch.bfloat16)
    packed = W.quantize_fp8_656(lat.to(torch.bfloat16), rope)
    pk = packed.clone()
    pk[:64, 512:528] = torch.full((64, 4), 0.0625).view(torch.uint8).reshape(64, 16)  # tokens 0-63: scale 2^-4
    mirror = fp8_cache_as_bf16(pk.view(n // 64, 64, 656)).reshape(n, 576).double().numpy()
    exact = oracle.unpack_fp8_656(pk.numpy())
    np.testing.assert_array_equal(mirror[:64], exact[:64])
    err = np.abs(mirror[64:, :512] - exact[64:, :512])
    assert np.all(err <= np.abs(exact[64:, :512]) * (2.0 ** -8 + 2.0 ** -23))
    assert np.all(mirror[64:, :512][exact[64:, :512] == 0] == 0)
    assert err.max() > 0  # the rounding is really there
    np.testing.assert_array_equal(mirror[:, 512:], rope.double().numpy())


# ---------------------------------------------------------------------------
# attention pins
# ---------------------------------------------------------------------------

def _brute(a):
    """Pure-Python loops; keys decoded with torch's bf16/float8 conversions."""
    q = torch.from_numpy(a["q_bits"].view(np.int16)).view(torch.bfloat16).double()
    B, s_q, h_q, _ = q.shape
    kv = a["kv_cache"]
    out = np.zeros((B, s_q, h_q, 512))
    lse = np.full((B, s_q, h_q), -np.inf)
    for b in range(B):
        L = int(a["cache_seqlens"][b])
        keys = []
        for j in range(L):
            blk = int(a["block_table"][b][j // 64])
            row = kv[blk, j % 64]
            if a["fmt"] == "bf16":
                keys.append(torch.from_numpy(row.view(np.int16).copy()).view(torch.bfloat16).double().tolist())
            else:
                codes = torch.from_numpy(row[:512].copy()).view(torch.float8_e4m3fn).double()
                sc = torch.from_numpy(row[512:528].copy()).view(torch.float32).double()
                lat = [float(codes[d]) * float(sc[d // 128]) for d in range(512)]
                rope = torch.from_numpy(row[528:].copy()).view(torch.bfloat16).double().tolist()
                keys.append(lat + rope)
        for i in range(s_q):
            n = L if not a["causal"] else max(0, min(L, L - s_q + i + 1))
            for h in range(h_q):
                qv = q[b, i, h].tolist()
                xs = [a["softmax_scale"] * sum(qv[d] * keys[j][d] for d in range(576)) for j in range(n)]
                if not xs:
                    continue
                m = max(xs)
                tot = sum(math.exp(x - m) for x in xs)
                lse[b, i, h] = m + math.log(tot)
                for d in range(512):
                    out[b, i, h, d] = sum(math.exp(xs[j] - m) / tot * keys[j][d] for j in range(n))
    return out, lse


@pytest.mark.parametrize("fmt", ["bf16", "fp8_656"])
@pytest.mark.parametrize("causal,s_q", [(False, 1), (True, 2)])
def test_brute_force_tiny(fmt, causal, s_q):
    c = _case(batch=2, s_q=s_q, h_q=2, seqlens=(67, 3), fmt=fmt, causal=causal)
    a = W.oracle_arrays(c)
    o, l = _run(a)
    bo, bl = _brute(a)
    np.testing.assert_allclose(o, bo, rtol=0, atol=1e-12)
    np.testing.assert_allclose(l, bl, rtol=0, atol=1e-12)


@pytest.mark.parametrize("causal,s_q", [(False, 1), (True, 2), (True, 3)])
def test_matches_torch_sdpa_float64(causal, s_q):
    c = _case(batch=3, s_q=s_q, h_q=8, seqlens=(130, 64, 9), causal=causal, seed=5)
    a = W.oracle_arrays(c)
    o, _ = _run(a)
    for b in range(3):
        L = int(a["cache_seqlens"][b])
        blocks = a["block_table"][b][: (L + 63) // 64]
        K = torch.from_numpy(a["kv_cache"][blocks].reshape(-1, 576)[:L].view(np.int16).copy()).view(torch.bfloat16).double()
        q = torch.from_numpy(a["q_bits"][b].view(np.int16).copy()).view(torch.bfloat16).double()  # [s_q,h,576]
        qh = q.permute(1, 0, 2)[None]  # [1,h,s_q,576]
        kh = K[None, None].expand(1, 8, L, 576)
        vh = K[None, None, :, :512].expand(1, 8, L, 512)
        mask = torch.ones(s_q, L, dtype=torch.bool)
        if causal:
            mask = torch.arange(L)[None, :] <= (L - s_q + torch.arange(s_q))[:, None]
        ref = torch.nn.functional.scaled_dot_product_attention(qh, kh, vh, attn_mask=mask, scale=a["softmax_scale"])
        np.testing.assert_allclose(o[b], ref[0].permute(1, 0, 2).numpy(), rtol=0, atol=1e-12)


def test_single_token_returns_its_value():
    c = _case(batch=2, s_q=1, h_q=5, seqlens=(1, 1))
    a = W.oracle_arrays(c)
    o, l = _run(a)
    for b in range(2):
        k = oracle.decode_bf16_bits(a["kv_cache"][a["block_table"][b][0], 0])
        q = oracle.decode_bf16_bits(a["q_bits"][b, 0])
        np.testing.assert_array_equal(o[b, 0], np.broadcast_to(k[:512], (5, 512)))
        np.testing.assert_allclose(l[b, 0], a["softmax_scale"] * (q @ k), rtol=0, atol=1e-12)


@pytest.mark.parametrize("how", ["q_zero", "scale_zero"])
def test_equal_logits_give_mean_of_values(how):
    c = _case(batch=2, s_q=1, h_q=3, seqlens=(100, 37))
    a = W.oracle_arrays(c)
    if how == "q_zero":
        a["q_bits"] = np.zeros_like(a["q_bits"])
    else:
        a["softmax_scale"] = 0.0
    o, l = _run(a)
    for b in range(2):
        L = int(a["cache_seqlens"][b])
        K = oracle.gather_keys(a["kv_cache"], "bf16", a["block_table"][b], L)
        np.testing.assert_allclose(o[b, 0], np.broadcast_to(K[:, :512].mean(0), (3, 512)), rtol=0, atol=1e-12)
        np.testing.assert_allclose(l[b, 0], math.log(L), rtol=0, atol=1e-12)


def test_two_tokens_closed_form():
    c = _case(batch=1, s_q=1, h_q=2, seqlens=(2,))
    a = W.oracle_arrays(c)
    o, l = _run(a)
    blk = a["block_table"][0][0]
    k0 = oracle.decode_bf16_bits(a["kv_cache"][blk, 0])
    k1 = oracle.decode_bf16_bits(a["kv_cache"][blk, 1])
    for h in range(2):
        q = oracle.decode_bf16_bits(a["q_bits"][0, 0, h])
        x0, x1 = a["softmax_scale"] * (q @ k0), a["softmax_scale"] * (q @ k1)
        w0 = 1.0 / (1.0 + math.exp(x1 - x0))
        np.testing.assert_allclose(o[0, 0, h], w0 * k0[:512] + (1 - w0) * k1[:512], rtol=0, atol=1e-12)
        np.testing.assert_allclose(l[0, 0, h], max(x0, x1) + math.log1p(math.exp(-abs(x0 - x1))), atol=1e-12)


@pytest.mark.parametrize("fmt", ["bf16", "fp8_656"])
def test_block_permutation_invariance(fmt):
    c = _case(batch=3, s_q=1, h_q=4, seqlens=(200, 64, 1), fmt=fmt)
    a = W.oracle_arrays(c)
    o, l = _run(a)
    nb = a["kv_cache"].shape[0]
    perm = np.random.default_rng(7).permutation(nb)  # new position of old block i is perm[i]
    kv2 = np.empty_like(a["kv_cache"])
    kv2[perm] = a["kv_cache"]
    bt2 = a["block_table"].copy()
    valid = bt2 >= 0
    bt2[valid] = perm[bt2[valid]]
    o2, l2 = _run(a, kv_cache=kv2, block_table=bt2)
    np.testing.assert_array_equal(o, o2)
    np.testing.assert_array_equal(l, l2)


@pytest.mark.parametrize("fmt", ["bf16", "fp8_656"])
def test_poison_is_never_read(fmt):
    seqlens = (65, 130, 7)
    clean = W.oracle_arrays(_case(batch=3, h_q=4, seqlens=seqlens, fmt=fmt, poison=False))
    dirty = W.oracle_arrays(_case(batch=3, h_q=4, seqlens=seqlens, fmt=fmt, poison=True))
    assert not np.array_equal(clean["kv_cache"], dirty["kv_cache"])  # poison was planted
    o1, l1 = _run(clean)
    o2, l2 = _run(dirty)
    assert np.all(np.isfinite(o2))
    np.testing.assert_array_equal(o1, o2)
    np.testing.assert_array_equal(l1, l2)


@pytest.mark.parametrize("causal,s_q", [(False, 1), (True, 2)])
def test_split_combine_equals_unsplit(causal, s_q):
    c = _case(batch=2, s_q=s_q, h_q=4, seqlens=(300, 129), causal=causal)
    a = W.oracle_arrays(c)
    o, l = _run(a)
    rng = np.random.default_rng(11)
    for b in range(2):
        L = int(a["cache_seqlens"][b])
        q = oracle.decode_bf16_bits(a["q_bits"][b])
        K = oracle.gather_keys(a["kv_cache"], "bf16", a["block_table"][b], L)
        for nsplit in (2, 3, 7):
            cuts = np.sort(rng.choice(np.arange(1, L), nsplit - 1, replace=False))
            bounds = [0, *cuts.tolist(), L]
            parts = [oracle.mla_decode_partial(q, K, L, a["softmax_scale"], causal, bounds[k], bounds[k + 1])
                     for k in range(nsplit)]
            oc, lc = oracle.combine_splits(np.stack([p[1] for p in parts]), np.stack([p[0] for p in parts]))
            np.testing.assert_allclose(oc, o[b], rtol=0, atol=1e-12)
            np.testing.assert_allclose(lc, l[b], rtol=0, atol=1e-12)


def test_combine_with_empty_splits():
    lse = np.array([[-np.inf, 0.3], [-np.inf, -np.inf]])
    o = np.array([[[0.0], [2.0]], [[0.0], [5.0]]])
    out, l = oracle.combine_splits(lse, o)
    assert l[0] == -np.inf and out[0, 0] == 0.0
    assert l[1] == pytest.approx(0.3) and out[1, 0] == pytest.approx(2.0)


def test_causal_two_queries_equal_two_single_queries():
    c = _case(batch=2, s_q=2, h_q=3, seqlens=(77, 64), causal=True)
    a = W.oracle_arrays(c)
    o, l = _run(a)
    for i in range(2):
        single = dict(a)
        single["q_bits"] = a["q_bits"][:, i:i + 1].copy()
        single["cache_seqlens"] = a["cache_seqlens"] - (1 - i)
        single["causal"] = False
        o1, l1 = _run(single)
        np.testing.assert_allclose(o[:, i], o1[:, 0], rtol=0, atol=1e-12)
        np.testing.assert_allclose(l[:, i], l1[:, 0], rtol=0, atol=1e-12)


def test_empty_causal_row_and_zero_length():
    c = _case(batch=2, s_q=2, h_q=2, seqlens=(1, 0), causal=True)
    a = W.oracle_arrays(c)
    o, l = _run(a)
    assert np.all(o[0, 0] == 0) and np.all(l[0, 0] == -np.inf)
    k = oracle.decode_bf16_bits(a["kv_cache"][a["block_table"][0][0], 0])
    np.testing.assert_array_equal(o[0, 1], np.broadcast_to(k[:512], (2, 512)))
    assert np.all(o[1] == 0) and np.all(l[1] == -np.inf)


def test_head_permutation_equivariance():
    c = _case(batch=2, s_q=1, h_q=6, seqlens=(90, 33))
    a = W.oracle_arrays(c)
    o, l = _run(a)
    perm = np.array([3, 0, 5, 1, 4, 2])
    o2, l2 = _run(a, q_bits=a["q_bits"][:, :, perm].copy())
    np.testing.assert_array_equal(o2, o[:, :, perm])
    np.testing.assert_array_equal(l2, l[:, :, perm])


# ---------------------------------------------------------------------------
# planted mistakes: each mutant must fail at least one pin
# ---------------------------------------------------------------------------

def _mutant(kind):
    def gather(kv_cache, fmt, row, L):
        K = om.gather_keys(kv_cache, fmt, row, L)
        if kind == "drop_rope":
            K = K.copy()
            K[:, 512:] = 0
        return K

    def decode(q_bits, kv_cache, fmt, block_table, cache_seqlens, softmax_scale, causal):
        B, s_q, h_q, _ = q_bits.shape
        out = np.zeros((B, s_q, h_q, 512))
        lse = np.full((B, s_q, h_q), -np.inf)
        for b in range(B):
            L = int(cache_seqlens[b])
            q = om.decode_bf16_bits(q_bits[b])
            K = gather(kv_cache, fmt, block_table[b], L)
            for i in range(s_q):
                n = om.visible_keys(L, s_q, i, causal)
                if kind == "causal_off_by_one" and causal:
                    n = max(0, min(L, L - s_q + i))
                if n == 0:
                    continue
                x = softmax_scale * (q[i] @ K[:n].T)
                if kind == "log2_lse":
                    m = x.max(1)
                    l_ = m + np.log2(np.exp(x - m[:, None]).sum(1))
                    w = np.exp(x - (m + np.log(np.exp(x - m[:, None]).sum(1)))[:, None])
                else:
                    m = x.max(1)
                    l_ = m + np.log(np.exp(x - m[:, None]).sum(1))
                    w = np.exp(x - l_[:, None])
                V = K[:n, 64:576] if kind == "value_tail" else K[:n, :512]
                out[b, i] = w @ V
                lse[b, i] = l_
        return out, lse
    return decode


@pytest.mark.parametrize("kind", ["drop_rope", "causal_off_by_one", "log2_lse", "value_tail"])
def test_planted_mistakes_are_caught(kind):
    bad = _mutant(kind)
    caught = []
    # pin 1: single token -> exact value, lse = scale q.k
    c = _case(batch=1, s_q=1, h_q=2, seqlens=(1,))
    a = W.oracle_arrays(c)
    o, l = bad(**{k: a[k] for k in ("q_bits", "kv_cache", "fmt", "block_table", "cache_seqlens", "softmax_scale", "causal")})
    k = om.decode_bf16_bits(a["kv_cache"][a["block_table"][0][0], 0])
    q = om.decode_bf16_bits(a["q_bits"][0, 0])
    caught.append(not (np.array_equal(o[0, 0], np.broadcast_to(k[:512], (2, 512)))
                       and np.allclose(l[0, 0], a["softmax_scale"] * (q @ k), atol=1e-12)))
    # pin 2: brute force with the causal two-query case
    c = _case(batch=1, s_q=2, h_q=2, seqlens=(20,), causal=True)
    a = W.oracle_arrays(c)
    o, l = bad(**{k: a[k] for k in ("q_bits", "kv_cache", "fmt", "block_table", "cache_seqlens", "softmax_scale", "causal")})
    bo, bl = _brute(a)
    caught.append(not (np.allclose(o, bo, atol=1e-12) and np.allclose(l, bl, atol=1e-12)))
    # pin 3: equal logits -> lse = ln L
    c = _case(batch=1, s_q=1, h_q=1, seqlens=(50,))
    a = W.oracle_arrays(c)
    a["q_bits"] = np.zeros_like(a["q_bits"])
    o, l = bad(**{k: a[k] for k in ("q_bits", "kv_cache", "fmt", "block_table", "cache_seqlens", "softmax_scale", "causal")})
    caught.append(not np.allclose(l, math.log(50), atol=1e-12))
    assert any(caught), f"mutant {kind} passed every pin"
