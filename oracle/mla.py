"""Plain float64 restatement of MLA decoding over a paged KV cache.

TEST INFRASTRUCTURE ONLY (see the package docstring): the product path never
imports this module, and this module imports nothing from the product.

What is computed (MLA decode, FlashMLA pages):
  * Many query heads attend to ONE shared latent KV head (MQA-like sharing with
    a compressed latent, Novita AI page, "Was ist MLA?" and the MHA/MQA/GQA/MLA
    table).  Each cached token is a 576-wide key: a 512-d latent followed by a
    64-d decoupled-RoPE slice.  The value of a token is the first 512 dims of
    its key (the latent).
  * The cache is paged with 64 tokens per block and requests have variable
    lengths (DeepSeek launch tweet, 8bitnewsroom page).
  * Two cache formats: BF16 (576 x 2 = 1152 bytes per token) and FP8 at 656
    bytes per token with the RoPE slice kept in BF16 (menfem.com DeepSeek
    page, "Key Contributions").

Readings taken where the pages are silent (each is a plain reading):
  R1 lse is the natural-log log-sum-exp of the scaled logits, one per
     (request, query token, head).
  R2 Causal alignment for s_q > 1 is bottom-right: query token i of a request
     with L cached tokens sees keys j <= L - s_q + i (the s_q query tokens are
     the last s_q positions of the sequence, as in speculative decoding).
  R3 A query row with no visible key returns out = 0 and lse = -inf (the
     log of an empty sum).
  R4 656-byte token layout: bytes [0,512) are 512 E4M3 latent codes, bytes
     [512,528) are four little-endian fp32 scales, one per 128-wide latent
     group, bytes [528,656) are the 64 RoPE values as little-endian bf16.
     512 + 4*4 + 64*2 = 656, the page's per-token figure.
  R5 E4M3 is the OCP FP8 E4M3 ("FN") encoding: 1 sign, 4 exponent bits with
     bias 7, 3 mantissa bits, subnormals at exponent 0, no infinities, NaN only
     for S.1111.111; the CUTLASS discussion page names "E4M3" as the format.
  R6 The page-table maps logical page p of request b to physical block
     block_table[b, p]; token j lives in slot j mod 64 of page j // 64.
     Slots at or beyond L, blocks not referenced, and block_table entries at
     or beyond ceil(L/64) are never read and may hold any bits.
  R7 softmax_scale multiplies the fp64 logits q . k; it is not folded into q.
"""

from __future__ import annotations

import math

import numpy as np

D_LATENT = 512
D_ROPE = 64
D_QK = D_LATENT + D_ROPE  # 576
D_V = D_LATENT  # 512: the value is the latent part of the key
PAGE_SIZE = 64
BF16_TOKEN_BYTES = 2 * D_QK  # 1152
FP8_GROUP = 128
FP8_NUM_SCALES = D_LATENT // FP8_GROUP  # 4
FP8_TOKEN_BYTES = D_LATENT + 4 * FP8_NUM_SCALES + 2 * D_ROPE  # 656


# ---------------------------------------------------------------------------
# Number formats
# ---------------------------------------------------------------------------

def decode_bf16_bits(bits: np.ndarray) -> np.ndarray:
    """bf16 bit patterns (uint16) -> exact float64 values.

    A bf16 number is the upper half of an IEEE binary32, so the value is the
    binary32 whose top 16 bits are `bits` and whose low 16 bits are zero.
    Every bf16 value (NaN and Inf included) is exact in float64.
    """
    b = np.asarray(bits).astype(np.uint16)
    with np.errstate(invalid="ignore"):
        return (b.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)


def decode_e4m3(codes: np.ndarray) -> np.ndarray:
    """E4M3 codes (uint8) -> exact float64 values, reading R5.

    sign s = bit 7, exponent e = bits 6..3, mantissa m = bits 2..0:
      e == 0            -> (-1)^s * (m / 8) * 2^-6          (zero / subnormal)
      e == 15 and m == 7 -> NaN
      otherwise         -> (-1)^s * (1 + m / 8) * 2^(e - 7)
    """
    c = np.asarray(codes).astype(np.int64)
    s = (c >> 7) & 1
    e = (c >> 3) & 0xF
    m = c & 0x7
    mag = np.where(
        e == 0,
        (m / 8.0) * 2.0 ** -6,
        (1.0 + m / 8.0) * np.power(2.0, (e - 7).astype(np.float64)),
    )
    val = np.where(s == 1, -mag, mag)
    return np.where((e == 15) & (m == 7), np.nan, val).astype(np.float64)


def unpack_fp8_656(tokens: np.ndarray) -> np.ndarray:
    """656-byte FP8 tokens (uint8[..., 656]) -> float64 keys [..., 576].

    key[d] = e4m3(byte d) * scale[d // 128]    for d < 512   (R4, R5)
    key[d] = bf16 RoPE value d - 512           for d >= 512
    The product is formed exactly in float64; how a kernel rounds it is that
    kernel's business (the FP8 parity tests additionally feed the oracle the
    keys rounded the way the kernel rounds them, as a BF16 cache).
    """
    t = np.ascontiguousarray(np.asarray(tokens, dtype=np.uint8))
    assert t.shape[-1] == FP8_TOKEN_BYTES
    lead = t.shape[:-1]
    flat = t.reshape(-1, FP8_TOKEN_BYTES)
    codes = flat[:, :D_LATENT]
    scales = np.ascontiguousarray(flat[:, D_LATENT:D_LATENT + 16]).view("<f4").astype(np.float64)
    rope_bits = np.ascontiguousarray(flat[:, D_LATENT + 16:]).view("<u2")
    out = np.empty((flat.shape[0], D_QK), dtype=np.float64)
    # decode_e4m3 evaluated once per code value and looked up: the same values
    # as calling it on every byte, without redoing the arithmetic per byte
    lat = decode_e4m3(np.arange(256, dtype=np.uint8))[codes]
    group = np.arange(D_LATENT) // FP8_GROUP
    out[:, :D_LATENT] = lat * scales[:, group]
    out[:, D_LATENT:] = decode_bf16_bits(rope_bits)
    return out.reshape(*lead, D_QK)


# ---------------------------------------------------------------------------
# Paging
# ---------------------------------------------------------------------------

def gather_keys(kv_cache: np.ndarray, fmt: str, block_table_row: np.ndarray, L: int) -> np.ndarray:
    """Dense float64 keys [L, 576] of one request, read through its page table.

    fmt "bf16":    kv_cache is uint16 bit patterns [num_blocks, 64, 576].
    fmt "fp8_656": kv_cache is uint8 [num_blocks, 64, 656].
    Token j is slot j % 64 of physical block block_table_row[j // 64] (R6).
    Only the ceil(L/64) referenced pages and the first L tokens are touched.
    """
    n_pages = (L + PAGE_SIZE - 1) // PAGE_SIZE
    if L == 0:
        return np.zeros((0, D_QK), dtype=np.float64)
    phys = np.asarray(block_table_row[:n_pages], dtype=np.int64)
    num_blocks = kv_cache.shape[0]
    if np.any(phys < 0) or np.any(phys >= num_blocks):
        raise ValueError("block_table references a block outside the cache")
    pages = kv_cache[phys]  # [n_pages, 64, width]
    rows = pages.reshape(n_pages * PAGE_SIZE, pages.shape[-1])[:L]
    if fmt == "bf16":
        return decode_bf16_bits(rows)
    if fmt == "fp8_656":
        return unpack_fp8_656(rows)
    raise ValueError(f"unknown cache format {fmt!r}")


def visible_keys(L: int, s_q: int, i: int, causal: bool) -> int:
    """Number of keys visible to query token i: they are always keys [0, n).

    Without the causal mask a query sees all L keys; with it, reading R2,
    query i sees keys j <= L - s_q + i, i.e. n = clamp(L - s_q + i + 1, 0, L).
    """
    if not causal:
        return L
    return max(0, min(L, L - s_q + i + 1))


# ---------------------------------------------------------------------------
# Attention
# ---------------------------------------------------------------------------

def _softmax_rows(x: np.ndarray):
    """Row-wise (lse, weights) of logits x [R, n] by the explicit definition.

    lse = m + ln sum_j exp(x_j - m) with m = max_j x_j;  w_j = exp(x_j - lse).
    An empty row (n == 0) has lse = -inf and no weights (R3).
    """
    R, n = x.shape
    if n == 0:
        return np.full(R, -np.inf), np.zeros((R, 0))
    m = x.max(axis=1)
    lse = m + np.log(np.exp(x - m[:, None]).sum(axis=1))
    return lse, np.exp(x - lse[:, None])


def mla_decode_partial(q: np.ndarray, keys: np.ndarray, L: int, softmax_scale: float,
                       causal: bool, j0: int, j1: int):
    """Attention of one request restricted to the key range [j0, j1).

    q: float64 [s_q, h_q, 576]; keys: float64 [>= j1, 576].
    Returns (o [s_q, h_q, 512], lse [s_q, h_q]) where o is normalised within
    the range and lse is the log-sum-exp over the visible keys of the range
    (-inf and o = 0 when the range holds none).  These are the per-split
    partial results that the split-KV combine merges.
    """
    s_q, h_q, _ = q.shape
    o = np.zeros((s_q, h_q, D_V))
    lse = np.full((s_q, h_q), -np.inf)
    for i in range(s_q):
        hi = min(j1, visible_keys(L, s_q, i, causal))
        if hi <= j0:
            continue
        k = keys[j0:hi]
        x = softmax_scale * (q[i] @ k.T)  # [h_q, n]
        lse_i, w = _softmax_rows(x)
        lse[i] = lse_i
        o[i] = w @ k[:, :D_V]
    return o, lse


def combine_splits(lse_parts: np.ndarray, o_parts: np.ndarray):
    """Merge per-split partials: lse = ln sum_s e^{lse_s}, out = sum_s e^{lse_s - lse} o_s.

    lse_parts [S, ...], o_parts [S, ..., 512].  Splits with lse_s = -inf carry
    no weight; if every split is empty the result is out = 0, lse = -inf.
    """
    lse_parts = np.asarray(lse_parts, dtype=np.float64)
    o_parts = np.asarray(o_parts, dtype=np.float64)
    m = lse_parts.max(axis=0)
    finite = np.isfinite(m)
    m_safe = np.where(finite, m, 0.0)
    ssum = np.exp(lse_parts - m_safe[None]).sum(axis=0)
    lse = np.where(finite, m_safe + np.log(np.where(finite, ssum, 1.0)), -np.inf)
    w = np.where(finite[None], np.exp(lse_parts - np.where(finite, lse, 0.0)[None]), 0.0)
    out = (w[..., None] * o_parts).sum(axis=0)
    return out, lse


def mla_decode_rows(q_bits: np.ndarray, kv_cache: np.ndarray, fmt: str, block_table: np.ndarray,
                    cache_seqlens: np.ndarray, softmax_scale: float, causal: bool, requests):
    """Oracle output for a subset of requests (used for sampled full-size checks).

    Returns dict b -> (out [s_q, h_q, 512], lse [s_q, h_q]) in float64.
    """
    res = {}
    for b in requests:
        L = int(cache_seqlens[b])
        q = decode_bf16_bits(q_bits[b])  # [s_q, h_q, 576]
        keys = gather_keys(kv_cache, fmt, block_table[b], L)
        res[b] = mla_decode_partial(q, keys, L, softmax_scale, causal, 0, L)
    return res


def mla_decode(q_bits: np.ndarray, kv_cache: np.ndarray, fmt: str, block_table: np.ndarray,
               cache_seqlens: np.ndarray, softmax_scale: float, causal: bool):
    """MLA decode of a whole batch, by the definition.

    q_bits        uint16 bf16 patterns [b, s_q, h_q, 576]
    kv_cache      uint16 [num_blocks, 64, 576] (fmt "bf16") or uint8
                  [num_blocks, 64, 656] (fmt "fp8_656")
    block_table   int32 [b, max_pages]
    cache_seqlens int32 [b]
    Returns out float64 [b, s_q, h_q, 512] and lse float64 [b, s_q, h_q]:
      x_j   = softmax_scale * sum_{d<576} q[d] * K_j[d]   over visible keys j
      lse   = ln sum_j e^{x_j}                             (R1, R3)
      out   = sum_j e^{x_j - lse} * K_j[:512]              (value = latent)
    """
    B, s_q, h_q, d = q_bits.shape
    assert d == D_QK
    out = np.zeros((B, s_q, h_q, D_V))
    lse = np.full((B, s_q, h_q), -np.inf)
    rows = mla_decode_rows(q_bits, kv_cache, fmt, block_table, cache_seqlens,
                           softmax_scale, causal, range(B))
    for b, (o, l) in rows.items():
        out[b] = o
        lse[b] = l
    return out, lse


def mla_sparse_decode(q_bits: np.ndarray, kv_cache: np.ndarray, fmt: str, block_table: np.ndarray,
                      cache_seqlens: np.ndarray, indices: np.ndarray, softmax_scale: float):
    """Sparse MLA decode: every query token attends only to its listed tokens.

    The menfem.com DeepSeek page ("Key Contributions") names a sparse decode
    kernel over the same 656-byte FP8 cache without defining it.  Reading R11:
      indices int32 [b, s_q, topk] holds, for query token i of request b, the
      positions j (0 <= j < L_b, the same positions the dense decode reads
      through block_table) of the keys it attends to.  Entries outside
      [0, L_b) are padding and are not keys.  Every valid entry is one term of
      the softmax, so a position listed twice counts twice.  No causal mask:
      the list alone decides what is visible.  A row with no valid entry gets
      out = 0 and lse = -inf (R3).
    For each head h:  x_k = softmax_scale * q[b,i,h] . K_{idx_k};
      lse = ln sum_k e^{x_k};  out = sum_k e^{x_k - lse} K_{idx_k}[:512].
    Returns out float64 [b, s_q, h_q, 512] and lse float64 [b, s_q, h_q].
    """
    B, s_q, h_q, d = q_bits.shape
    assert d == D_QK
    idx = np.asarray(indices, dtype=np.int64)
    assert idx.shape[:2] == (B, s_q)
    out = np.zeros((B, s_q, h_q, D_V))
    lse = np.full((B, s_q, h_q), -np.inf)
    for b in range(B):
        L = int(cache_seqlens[b])
        keys = gather_keys(kv_cache, fmt, block_table[b], L)  # [L, 576]
        q = decode_bf16_bits(q_bits[b])  # [s_q, h_q, 576]
        for i in range(s_q):
            sel = idx[b, i]
            sel = sel[(sel >= 0) & (sel < L)]
            if sel.size == 0:
                continue
            k = keys[sel]  # [n, 576], duplicates kept
            x = softmax_scale * (q[i] @ k.T)  # [h_q, n]
            lse_i, w = _softmax_rows(x)
            lse[b, i] = lse_i
            out[b, i] = w @ k[:, :D_V]
    return out, lse


def default_softmax_scale() -> float:
    """576^-0.5, the scale every configured workload uses."""
    return 1.0 / math.sqrt(D_QK)


# ---------------------------------------------------------------------------
# Cache append: writing new tokens into the paged cache
# ---------------------------------------------------------------------------
#
# The pages fix the FP8 token at 656 bytes with the RoPE slice kept in BF16
# (menfem.com DeepSeek page, "Key Contributions") and name E4M3 (CUTLASS
# discussion page); how a token is quantised into it is not printed.  Reading
# R9 (the plainest one the layout R4 supports): per 128-wide latent group g,
#   scale_g = fp32(amax_g / 448)                (448 = largest finite E4M3)
#   code_d  = E4M3 round-to-nearest-even of fp32(x_d / scale_g), saturated
#             to +-448
# with both divisions IEEE binary32 (correctly rounded); a group with
# amax_g == 0 gets scale 0 and all codes 0.  The new token's values are finite.

def _e4m3_finite_magnitudes() -> np.ndarray:
    """Values of the non-negative finite E4M3 codes 0x00..0x7E, ascending."""
    return decode_e4m3(np.arange(0x7F, dtype=np.uint8))


def encode_e4m3_rne(y: np.ndarray) -> np.ndarray:
    """float32 values -> E4M3 codes (uint8), round to nearest, ties to even.

    Written from the format definition (R5): the result is the finite E4M3
    value nearest to y; at an exact midpoint between two neighbours the one
    with an even code (mantissa LSB 0) wins.  Magnitudes beyond 448 saturate
    to 448.  The sign bit is y's sign bit, so -0.0 and negative values that
    round to zero give 0x80.  NaN is outside the supported inputs.
    """
    v = np.asarray(y, dtype=np.float32).astype(np.float64)
    mags = _e4m3_finite_magnitudes()  # 127 values, strictly increasing
    a = np.minimum(np.abs(v), mags[-1])
    hi = np.clip(np.searchsorted(mags, a, side="left"), 0, mags.size - 1)
    lo = np.clip(hi - 1, 0, mags.size - 1)
    d_lo = a - mags[lo]
    d_hi = mags[hi] - a
    pick_hi = (d_hi < d_lo) | ((d_hi == d_lo) & (hi % 2 == 0))
    code = np.where(pick_hi, hi, lo).astype(np.uint8)
    return np.where(np.signbit(v), code | np.uint8(0x80), code).astype(np.uint8)


def quantize_fp8_656(latent_bits: np.ndarray, rope_bits: np.ndarray) -> np.ndarray:
    """New tokens -> 656-byte FP8 rows (reading R9 above, layout R4).

    latent_bits uint16 [n, 512] and rope_bits uint16 [n, 64] are bf16 bit
    patterns; the result is uint8 [n, 656]: 512 codes, four little-endian fp32
    scales, the 64 RoPE bf16 values unchanged.
    """
    lat = np.asarray(latent_bits, dtype=np.uint16)
    n = lat.shape[0]
    x = decode_bf16_bits(lat).astype(np.float32).reshape(n, FP8_NUM_SCALES, FP8_GROUP)
    amax = np.abs(x).max(axis=-1)  # exact
    scale = (amax / np.float32(448.0)).astype(np.float32)  # one IEEE binary32 division
    codes = np.zeros((n, FP8_NUM_SCALES, FP8_GROUP), dtype=np.uint8)
    for i in range(n):
        for g in range(FP8_NUM_SCALES):
            if scale[i, g] > 0:
                y = (x[i, g] / scale[i, g]).astype(np.float32)  # IEEE binary32 divisions
                codes[i, g] = encode_e4m3_rne(y)
    out = np.empty((n, FP8_TOKEN_BYTES), dtype=np.uint8)
    out[:, :D_LATENT] = codes.reshape(n, D_LATENT)
    out[:, D_LATENT:D_LATENT + 16] = np.ascontiguousarray(scale.astype("<f4")).view(np.uint8).reshape(n, 16)
    out[:, D_LATENT + 16:] = np.ascontiguousarray(np.asarray(rope_bits, dtype="<u2")).view(np.uint8).reshape(n, 128)
    return out


def append_tokens(kv_cache: np.ndarray, fmt: str, new_bits: np.ndarray, block_table: np.ndarray,
                  cache_seqlens: np.ndarray) -> np.ndarray:
    """The cache after appending new tokens (returns a modified copy).

    new_bits uint16 [batch, s_new, 576]: bf16 bit patterns of the new keys.
    cache_seqlens [batch] are the lengths after the append (the ones the next
    decode call takes), so new token t of request b is token
    p = L_b - s_new + t of the request and lands in slot p % 64 of physical
    block block_table[b, p // 64] (R6).  "bf16" stores the bit patterns,
    "fp8_656" the quantised row (R9).  Rows with p < 0, a page at or beyond
    the block-table row, or a block index outside the cache are skipped.
    """
    out = np.array(kv_cache, copy=True)
    new = np.asarray(new_bits, dtype=np.uint16)
    B, s_new, _ = new.shape
    bt = np.asarray(block_table)
    num_blocks = out.shape[0]
    for b in range(B):
        L = int(cache_seqlens[b])
        rows = new[b]
        if fmt == "fp8_656":
            rows = quantize_fp8_656(rows[:, :D_LATENT], rows[:, D_LATENT:])
        for t in range(s_new):
            p = L - s_new + t
            if p < 0 or p // PAGE_SIZE >= bt.shape[1]:
                continue
            blk = int(bt[b, p // PAGE_SIZE])
            if blk < 0 or blk >= num_blocks:
                continue
            out[blk, p % PAGE_SIZE] = rows[t]
    return out
