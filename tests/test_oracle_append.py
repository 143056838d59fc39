"""Pins for the oracle's cache-append side (CPU only): the E4M3 encoder, the
656-byte quantiser and the placement of new tokens through the page table.

Each test checks the oracle against something other than itself: the E4M3
decoder (itself pinned against torch's float8_e4m3fn), torch's own
round-to-nearest-even float8 conversion, the torch-based packer of the input
generator, the error bound of a 3-bit mantissa, and the page-table rule read
back through the oracle's own gather.  The mutation tests at the end plant
plausible mistakes in copies of these functions and check that a pin catches
each of them.
"""

import numpy as np
import pytest
import torch

import oracle
from oracle import mla as om
import workloads as W


def _rand_bf16_bits(shape, seed, scale=1.0):
    g = torch.Generator().manual_seed(seed)
    x = (torch.randn(shape, generator=g, dtype=torch.float32) * scale).to(torch.bfloat16)
    return x.view(torch.int16).numpy().view(np.uint16)


def _torch_e4m3_codes(y):
    t = torch.from_numpy(np.asarray(y, dtype=np.float32))
    return t.to(torch.float8_e4m3fn).view(torch.uint8).numpy()


# ---------------------------------------------------------------------------
# E4M3 encoder
# ---------------------------------------------------------------------------

def test_encoder_round_trips_every_finite_code():
    codes = np.array([c for c in range(256) if (c & 0x7F) != 0x7F], dtype=np.uint8)
    vals = om.decode_e4m3(codes).astype(np.float32)
    back = oracle.encode_e4m3_rne(vals)
    # +0 and -0 keep their sign bit; every other code maps to itself
    np.testing.assert_array_equal(back, codes)


def test_encoder_midpoints_go_to_the_even_code():
    mags = om.decode_e4m3(np.arange(0x7F, dtype=np.uint8))
    for k in range(0x7E):
        mid = np.float32((mags[k] + mags[k + 1]) / 2)
        assert float(mid) == (mags[k] + mags[k + 1]) / 2  # exact in binary32
        even = k if k % 2 == 0 else k + 1
        assert oracle.encode_e4m3_rne([mid])[0] == even, k
        assert oracle.encode_e4m3_rne([-mid])[0] == even | 0x80, k
        # just off the midpoint the nearer neighbour wins
        lo = np.nextafter(mid, np.float32(-np.inf), dtype=np.float32)
        hi = np.nextafter(mid, np.float32(np.inf), dtype=np.float32)
        assert oracle.encode_e4m3_rne([lo])[0] == k
        assert oracle.encode_e4m3_rne([hi])[0] == k + 1


def test_encoder_saturates_at_448():
    y = np.array([448.0, 449.0, 464.0, 465.0, 1e30, -500.0, -1e30], dtype=np.float32)
    np.testing.assert_array_equal(oracle.encode_e4m3_rne(y), [0x7E, 0x7E, 0x7E, 0x7E, 0x7E, 0xFE, 0xFE])


def test_encoder_matches_torch_float8_conversion():
    g = torch.Generator().manual_seed(5)
    y = torch.cat([torch.randn(20000, generator=g) * 100,
                   torch.randn(20000, generator=g) * 1e-2,   # subnormal range and below
                   torch.rand(20000, generator=g) * 896 - 448]).clamp(-448, 448).numpy()
    np.testing.assert_array_equal(oracle.encode_e4m3_rne(y), _torch_e4m3_codes(y))


# ---------------------------------------------------------------------------
# quantiser
# ---------------------------------------------------------------------------

def _tokens(n, seed):
    lat = _rand_bf16_bits((n, 512), seed)
    rope = _rand_bf16_bits((n, 64), seed + 1)
    lat[0, 128:256] = 0          # an all-zero group: scale 0, codes 0
    lat[1, 0:128] = 0x8000       # -0.0 everywhere: amax 0 as well
    lat[2, 256:384] = _rand_bf16_bits((128,), seed + 2, scale=1e-6)  # tiny group
    lat[3, 384] = np.float32(300.0).view(np.uint32) >> 16             # one outlier
    return lat, rope


def test_quantizer_matches_the_torch_packer():
    lat, rope = _tokens(64, 11)
    ref = W.quantize_fp8_656(torch.from_numpy(lat.view(np.int16)).view(torch.bfloat16),
                             torch.from_numpy(rope.view(np.int16)).view(torch.bfloat16)).numpy()
    np.testing.assert_array_equal(oracle.quantize_fp8_656(lat, rope), ref)


def test_quantizer_layout_and_zero_groups():
    lat, rope = _tokens(4, 3)
    q = oracle.quantize_fp8_656(lat, rope)
    assert q.shape == (4, 656) and q.dtype == np.uint8
    scales = np.ascontiguousarray(q[:, 512:528]).view("<f4")
    assert scales[0, 1] == 0 and not q[0, 128:256].any()
    assert scales[1, 0] == 0 and not q[1, 0:128].any()
    np.testing.assert_array_equal(np.ascontiguousarray(q[:, 528:]).view("<u2"), rope)
    # the scale is amax / 448 in binary32
    x = om.decode_bf16_bits(lat).astype(np.float32).reshape(4, 4, 128)
    np.testing.assert_array_equal(scales, (np.abs(x).max(-1) / np.float32(448)).astype(np.float32))


def test_dequantized_token_is_within_half_an_e4m3_step():
    lat, rope = _tokens(32, 7)
    q = oracle.quantize_fp8_656(lat, rope)
    deq = oracle.unpack_fp8_656(q)
    x = om.decode_bf16_bits(lat)
    scales = np.ascontiguousarray(q[:, 512:528]).view("<f4").astype(np.float64)
    s = np.repeat(scales, 128, axis=1)
    # 3 mantissa bits: half a step is 2^-4 of the magnitude for normals and
    # 2^-10 * scale in the subnormal range; the binary32 division adds ~2^-24
    bound = np.maximum(np.abs(x) * 2.0 ** -4, s * 2.0 ** -10) * (1 + 2.0 ** -20)
    assert np.all(np.abs(deq[:, :512] - x) <= bound)
    np.testing.assert_array_equal(deq[:, 512:], om.decode_bf16_bits(rope))
    # each group's largest magnitude lands on code +-448
    codes = q[:, :512].reshape(32, 4, 128)
    xm = np.abs(x).reshape(32, 4, 128)
    for i in range(32):
        for gidx in range(4):
            if xm[i, gidx].max() > 0:
                assert (codes[i, gidx, xm[i, gidx].argmax()] & 0x7F) == 0x7E


# ---------------------------------------------------------------------------
# placement through the page table
# ---------------------------------------------------------------------------

def _append_case(fmt, seqlens=(70, 3, 128), s_new=3, seed=2):
    w = W.Workload("t", len(seqlens), 1, 1, (1, 1), fmt=fmt, seed=seed)
    c = W.make_case(w, seqlens=list(seqlens), poison=True)
    a = W.oracle_arrays(c)
    new = _rand_bf16_bits((len(seqlens), s_new, 576), seed + 100)
    return a, new


@pytest.mark.parametrize("fmt", ["bf16", "fp8_656"])
def test_appended_tokens_read_back_at_the_last_positions(fmt):
    a, new = _append_case(fmt)
    kv1 = oracle.append_tokens(a["kv_cache"], fmt, new, a["block_table"], a["cache_seqlens"])
    s_new = new.shape[1]
    written = set()
    for b, L in enumerate(a["cache_seqlens"]):
        L = int(L)
        K0 = oracle.gather_keys(a["kv_cache"], fmt, a["block_table"][b], L)
        K1 = oracle.gather_keys(kv1, fmt, a["block_table"][b], L)
        np.testing.assert_array_equal(K1[:L - s_new], K0[:L - s_new])  # earlier tokens untouched
        if fmt == "bf16":
            expect = om.decode_bf16_bits(new[b])
        else:
            expect = oracle.unpack_fp8_656(oracle.quantize_fp8_656(new[b, :, :512], new[b, :, 512:]))
        np.testing.assert_array_equal(K1[L - s_new:], expect)
        for p in range(L - s_new, L):
            written.add((int(a["block_table"][b][p // 64]), p % 64))
    # nothing else in the cache changed (poisoned slots and spare blocks included)
    mask = np.ones(kv1.shape[:2], dtype=bool)
    for blk, slot in written:
        mask[blk, slot] = False
    np.testing.assert_array_equal(kv1[mask], a["kv_cache"][mask])


def test_invalid_rows_are_skipped():
    a, new = _append_case("bf16", seqlens=(2, 70), s_new=3)
    bt = a["block_table"].copy()
    bt[1, 1] = -5  # token 67..69 of request 1 live on page 1
    kv1 = oracle.append_tokens(a["kv_cache"], "bf16", new, bt, a["cache_seqlens"])
    # request 0 has L = 2 < s_new: its first new token has position -1
    K = oracle.gather_keys(kv1, "bf16", bt[0], 2)
    np.testing.assert_array_equal(K, om.decode_bf16_bits(new[0, 1:]))
    np.testing.assert_array_equal(kv1[bt[1, 0]], a["kv_cache"][bt[1, 0]])  # page 0 of request 1 untouched
    changed = np.any(kv1 != a["kv_cache"], axis=-1)
    assert changed.sum() == 2  # only request 0's two valid rows


# ---------------------------------------------------------------------------
# planted mistakes
# ---------------------------------------------------------------------------

def _mutant_encoder(kind):
    def enc(y):
        v = np.asarray(y, dtype=np.float32).astype(np.float64)
        mags = om.decode_e4m3(np.arange(0x7F, dtype=np.uint8))
        a = np.minimum(np.abs(v), mags[-1])
        hi = np.clip(np.searchsorted(mags, a, side="left"), 0, 126)
        lo = np.clip(hi - 1, 0, 126)
        if kind == "ties_away":
            pick = (mags[hi] - a) <= (a - mags[lo])
        elif kind == "truncate":
            pick = mags[hi] == a
        else:
            pick = ((mags[hi] - a) < (a - mags[lo])) | (((mags[hi] - a) == (a - mags[lo])) & (hi % 2 == 0))
        code = np.where(pick, hi, lo).astype(np.uint8)
        if kind == "no_sign":
            return code
        return np.where(np.signbit(v), code | 0x80, code).astype(np.uint8)
    return enc


def _mutant_quantizer(kind):
    def quant(lat, rope):
        n = lat.shape[0]
        x = om.decode_bf16_bits(lat).astype(np.float32).reshape(n, 4, 128)
        amax = np.abs(x).max(-1)
        scale = (amax / np.float32(240.0 if kind == "max240" else 448.0)).astype(np.float32)
        codes = np.zeros((n, 4, 128), dtype=np.uint8)
        for i in range(n):
            for g in range(4):
                if scale[i, g] > 0:
                    yy = (x[i, g] * scale[i, g]) if kind == "multiply" else (x[i, g] / scale[i, g])
                    codes[i, g] = oracle.encode_e4m3_rne(yy.astype(np.float32))
        out = np.empty((n, 656), dtype=np.uint8)
        out[:, :512] = codes.reshape(n, 512)
        out[:, 512:528] = np.ascontiguousarray(scale.astype("<f4")).view(np.uint8).reshape(n, 16)
        out[:, 528:] = np.ascontiguousarray(rope.astype("<u2")).view(np.uint8).reshape(n, 128)
        return out
    return quant


def _mutant_append(kind):
    def app(kv, fmt, new, bt, seqlens):
        out = np.array(kv, copy=True)
        B, s_new, _ = new.shape
        for b in range(B):
            L = int(seqlens[b])
            for t in range(s_new):
                p = L + t if kind == "after_length" else L - s_new + t
                if p < 0 or p // 64 >= bt.shape[1]:
                    continue
                blk = int(bt[b, t // 64]) if kind == "page_of_t" else int(bt[b, p // 64])
                if 0 <= blk < out.shape[0]:
                    out[blk, p % 64] = new[b, t]
        return out
    return app


@pytest.mark.parametrize("kind", ["ties_away", "truncate", "no_sign"])
def test_planted_encoder_mistakes_are_caught(kind):
    enc = _mutant_encoder(kind)
    codes = np.array([c for c in range(256) if (c & 0x7F) != 0x7F], dtype=np.uint8)
    rt = np.array_equal(enc(om.decode_e4m3(codes).astype(np.float32)), codes)
    g = torch.Generator().manual_seed(9)
    y = (torch.randn(5000, generator=g) * 50).clamp(-448, 448).numpy()
    lib = np.array_equal(enc(y), _torch_e4m3_codes(y))
    mags = om.decode_e4m3(np.arange(0x7F, dtype=np.uint8))
    mids = np.float32((mags[:-1] + mags[1:]) / 2)
    even = np.array([k if k % 2 == 0 else k + 1 for k in range(126)])
    mid = np.array_equal(enc(mids), even)
    assert not (rt and lib and mid), f"mutant {kind} passed every pin"


@pytest.mark.parametrize("kind", ["max240", "multiply"])
def test_planted_quantizer_mistakes_are_caught(kind):
    lat, rope = _tokens(16, 4)
    ref = W.quantize_fp8_656(torch.from_numpy(lat.view(np.int16)).view(torch.bfloat16),
                             torch.from_numpy(rope.view(np.int16)).view(torch.bfloat16)).numpy()
    assert not np.array_equal(_mutant_quantizer(kind)(lat, rope), ref)


@pytest.mark.parametrize("kind", ["after_length", "page_of_t"])
def test_planted_append_mistakes_are_caught(kind):
    a, new = _append_case("bf16")
    kv1 = _mutant_append(kind)(a["kv_cache"], "bf16", new, a["block_table"], a["cache_seqlens"])
    ok = True
    for b, L in enumerate(a["cache_seqlens"]):
        L = int(L)
        if L < new.shape[1]:
            continue
        K1 = oracle.gather_keys(kv1, "bf16", a["block_table"][b], L)
        ok &= np.array_equal(K1[L - new.shape[1]:], om.decode_bf16_bits(new[b]))
    assert not ok, f"mutant {kind} passed the read-back pin"
