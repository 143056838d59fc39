"""Float64 CPU oracle for MLA decoding over a paged KV cache.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path may import, call or
execute this package: only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` use it.  It shares
no code with the CUDA path (no kernels, headers, helpers or constant tables);
the only thing both sides see is the seeded input generator in ``workloads``,
which holds none of the method's arithmetic.

Every function is a plain restatement of what the method computes, written
from the descriptions of FlashMLA (an MLA decoding kernel for Hopper GPUs
over a BF16 cache paged in 64-token blocks, DeepSeek launch tweet on the
8bitnewsroom page; MLA's shared latent KV with decoupled RoPE, Novita AI
page, section "Was ist MLA?" and its MHA/MQA/GQA/MLA table; the 656-byte FP8
cache format, menfem.com DeepSeek page, "Key Contributions").  Where those
pages are silent the reading taken is stated in the docstring.

Parity status per function (what pins it, see tests/test_oracle.py):
  decode_bf16_bits / decode_e4m3      closed forms + library cross-check
  unpack_fp8_656                      byte-layout arithmetic + round trip
  gather_keys                         block-permutation invariance, poison
  mla_decode                          brute force, SDPA (library), closed forms
  mla_decode_partial + combine_splits split == unsplit, closed forms
  mla_sparse_decode                   the full index list equals the dense
                                      decode; permutation and padding
                                      invariance; duplicate and single-key
                                      closed forms; brute force
  encode_e4m3_rne                     every code round-trips, midpoints go to the
                                      even code, saturation; library cross-check
  quantize_fp8_656 / append_tokens    library cross-check of the codes, error
                                      bound of the dequantised token, placement
                                      through the page table
"""

from .mla import (  # noqa: F401
    D_QK,
    D_V,
    D_ROPE,
    PAGE_SIZE,
    FP8_TOKEN_BYTES,
    BF16_TOKEN_BYTES,
    decode_bf16_bits,
    decode_e4m3,
    unpack_fp8_656,
    gather_keys,
    visible_keys,
    mla_decode,
    mla_decode_partial,
    combine_splits,
    mla_decode_rows,
    mla_sparse_decode,
    encode_e4m3_rne,
    quantize_fp8_656,
    append_tokens,
)
