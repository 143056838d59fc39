"""Seeded synthetic inputs for MLA paged-KV decoding.

This module is shared by the oracle-side tests and the CUDA-side tests and
bench.  It holds none of the method's arithmetic: it only draws random
numbers, lays them out in the cache formats and builds page tables.

The five workloads follow the configured benchmark set (tiny; uniform BF16;
variable-length speculative BF16; FP8 656-byte cache; long context).  The
pages describe no dataset, only batches of variable-length sequences over a
cache paged in 64-token blocks (DeepSeek launch tweet, 8bitnewsroom page) and a Novita
AI sweep over batch size, sequence length and head count whose charts did not
survive; these generators stand in for all of them.

Recipe (all draws from one torch.Generator seeded with `seed`, default 0):
  1. cache_seqlens: fixed, or integers uniform on [lo, hi] inclusive.
  2. Pages: request b owns ceil(L_b / 64) pages.  The pool holds exactly the
     sum of those plus ceil(5%) spare blocks; torch.randperm of the pool gives
     the physical block of every (request, page) in row-major order, the
     rest are spares.  block_table entries past a request's last page are -1.
  3. q and the BF16 cache: N(0, 1) drawn in fp32 and rounded to bf16 (RNE).
  4. FP8 656-byte cache: latents drawn as for BF16, then per 128-wide group
     scale = fp32(amax / 448) and code = e4m3_rne(clamp(x / scale, +-448));
     a group with amax 0 gets scale 0 and codes 0.  RoPE slice N(0,1) bf16.
  5. Poison (default on): tail slots of each request's last page and all
     spare blocks are filled with NaN/Inf patterns; they must never be read.
  6. Sparse workloads (topk > 0): for every (request b, query token i) an
     index list of topk positions: a uniformly random set of topk distinct
     positions of [0, L_b) in increasing order (the form a top-k selector
     returns), or, when L_b < topk, every position followed by -1 padding.
     The selector itself is not modelled (it needs trained weights).
"""

from __future__ import annotations

import dataclasses
import math

import numpy as np
import torch

PAGE = 64
D_QK = 576
D_LAT = 512
FP8_BYTES = 656


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    batch: int
    s_q: int
    h_q: int
    seqlen: tuple  # (lo, hi) inclusive; lo == hi for a fixed length
    fmt: str = "bf16"  # "bf16" | "fp8_656"
    causal: bool = False
    seed: int = 0
    spare_frac: float = 0.05
    topk: int = 0  # > 0: a sparse decode with index lists of topk entries

    @property
    def softmax_scale(self) -> float:
        return 1.0 / math.sqrt(D_QK)

    def describe(self) -> str:
        lo, hi = self.seqlen
        L = f"{lo}" if lo == hi else f"U[{lo},{hi}]"
        return (f"{self.name}: b={self.batch} s_q={self.s_q} h_q={self.h_q} L={L} "
                f"{self.fmt}{' causal' if self.causal else ''}{f' topk={self.topk}' if self.topk else ''}")


WORKLOADS = {
    "tiny": Workload("tiny", 1, 1, 16, (256, 256)),
    "uniform_bf16": Workload("uniform_bf16", 64, 1, 128, (4096, 4096)),
    "varlen_spec_bf16": Workload("varlen_spec_bf16", 128, 2, 64, (1, 8192), causal=True),
    "fp8_656": Workload("fp8_656", 128, 1, 128, (16384, 32768), fmt="fp8_656"),
    "long_ctx_bf16": Workload("long_ctx_bf16", 8, 1, 128, (131072, 131072)),
    # the sparse decode over the FP8 workload's cache: 2048 listed tokens per query
    "sparse_fp8": Workload("sparse_fp8", 128, 1, 128, (16384, 32768), fmt="fp8_656", topk=2048),
}
ORDER = ["tiny", "uniform_bf16", "varlen_spec_bf16", "fp8_656", "long_ctx_bf16"]
SPARSE_ORDER = ["sparse_fp8"]


def make_sparse_indices(cache_seqlens, s_q: int, topk: int, seed: int = 0, device="cpu", pad: int = 0,
                        dup: int = 0, oob: int = 0):
    """Index lists int32 [batch, s_q, topk] (recipe step 6).

    Optional edge cases for tests, per list: `dup` entries overwritten with a
    repeat of another entry, `pad` with -1, `oob` with positions >= L_b.
    """
    gen = torch.Generator()
    gen.manual_seed(seed + 12345)
    L = [int(x) for x in torch.as_tensor(cache_seqlens).cpu().tolist()]
    B = len(L)
    idx = torch.full((B, s_q, topk), -1, dtype=torch.int32)
    for b in range(B):
        for i in range(s_q):
            n = min(topk, L[b])
            if n > 0:
                sel = torch.randperm(L[b], generator=gen)[:n] if L[b] > topk else torch.arange(L[b])
                idx[b, i, :n] = torch.sort(sel.to(torch.int32)).values
            row = idx[b, i]
            slots = torch.randperm(topk, generator=gen)
            k = 0
            for _ in range(min(dup, n)):
                src = int(torch.randint(0, n, (1,), generator=gen))
                row[int(slots[k])] = row[src] if int(row[src]) >= 0 else 0
                k += 1
            for _ in range(pad):
                if k < topk:
                    row[int(slots[k])] = -1
                    k += 1
            for _ in range(oob):
                if k < topk:
                    row[int(slots[k])] = L[b] + int(torch.randint(0, 1000, (1,), generator=gen))
                    k += 1
    return idx.to(device)

# NaN / Inf bit patterns used as poison.
_BF16_POISON = (0x7FC0, 0xFF80, 0xFFFF, 0x7F80)


def _randn_bf16(shape, gen, device, chunk_rows=1 << 16):
    """N(0,1) drawn in fp32, rounded to bf16; generated in row chunks."""
    out = torch.empty(shape, dtype=torch.bfloat16, device=device)
    flat = out.view(-1, shape[-1])
    for r0 in range(0, flat.shape[0], chunk_rows):
        r1 = min(flat.shape[0], r0 + chunk_rows)
        flat[r0:r1] = torch.randn((r1 - r0, shape[-1]), generator=gen, device=device,
                                  dtype=torch.float32).to(torch.bfloat16)
    return out


def quantize_fp8_656(latent_bf16: torch.Tensor, rope_bf16: torch.Tensor) -> torch.Tensor:
    """Pack tokens into the 656-byte layout (input preparation, recipe step 4).

    latent_bf16 [n, 512], rope_bf16 [n, 64] -> uint8 [n, 656]:
    bytes [0,512) e4m3 codes, [512,528) four fp32 scales, [528,656) bf16 RoPE.
    """
    n = latent_bf16.shape[0]
    x = latent_bf16.float().view(n, 4, 128)
    amax = x.abs().amax(dim=-1)  # [n, 4]
    scale = (amax / 448.0).to(torch.float32)
    safe = torch.where(scale > 0, scale, torch.ones_like(scale))
    y = torch.where(scale[..., None] > 0, x / safe[..., None], torch.zeros_like(x))
    codes = y.clamp(-448.0, 448.0).to(torch.float8_e4m3fn).view(torch.uint8).view(n, 512)
    out = torch.empty((n, FP8_BYTES), dtype=torch.uint8, device=latent_bf16.device)
    out[:, :512] = codes
    out[:, 512:528] = scale.contiguous().view(torch.uint8).view(n, 16)
    out[:, 528:] = rope_bf16.contiguous().view(torch.uint8).view(n, 128)
    return out


def make_case(w: Workload, seed: int | None = None, device="cpu", poison: bool = True,
              seqlens=None):
    """Build one seeded case of workload `w` on `device`.

    `seqlens` (optional list of ints) overrides the drawn lengths, for edge
    cases.  Returns a dict of torch tensors plus the scalar arguments.
    """
    seed = w.seed if seed is None else seed
    device = torch.device(device)
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    lo, hi = w.seqlen
    if seqlens is not None:
        L = torch.tensor(list(seqlens), dtype=torch.int32)
    elif lo == hi:
        L = torch.full((w.batch,), lo, dtype=torch.int32)
    else:
        L = torch.randint(lo, hi + 1, (w.batch,), generator=gen, device=device).to(torch.int32).cpu()
    B = int(L.numel())
    n_pages = [(int(x) + PAGE - 1) // PAGE for x in L.tolist()]
    total = sum(n_pages)
    spare = int(math.ceil(w.spare_frac * total)) if total > 0 else 1
    num_blocks = max(1, total + spare)
    perm = torch.randperm(num_blocks, generator=gen, device=device).cpu().to(torch.int32)
    max_pages = max(1, max(n_pages) if n_pages else 1)
    bt = torch.full((B, max_pages), -1, dtype=torch.int32)
    k = 0
    for b in range(B):
        if n_pages[b]:
            bt[b, :n_pages[b]] = perm[k:k + n_pages[b]]
            k += n_pages[b]
    spare_blocks = perm[total:]

    q = _randn_bf16((B, w.s_q, w.h_q, D_QK), gen, device)
    if w.fmt == "bf16":
        kv = _randn_bf16((num_blocks, PAGE, D_QK), gen, device)
    elif w.fmt == "fp8_656":
        kv = torch.empty((num_blocks, PAGE, FP8_BYTES), dtype=torch.uint8, device=device)
        flat = kv.view(num_blocks * PAGE, FP8_BYTES)
        rows = 1 << 18
        for r0 in range(0, flat.shape[0], rows):
            r1 = min(flat.shape[0], r0 + rows)
            lat = _randn_bf16((r1 - r0, D_LAT), gen, device)
            rope = _randn_bf16((r1 - r0, D_QK - D_LAT), gen, device)
            flat[r0:r1] = quantize_fp8_656(lat, rope)
    else:
        raise ValueError(w.fmt)

    if poison:
        _poison(kv, w.fmt, bt, L, spare_blocks)

    case = dict(
        workload=w, q=q, kv_cache=kv, block_table=bt.to(device), cache_seqlens=L.to(device),
        softmax_scale=w.softmax_scale, causal=w.causal, fmt=w.fmt, num_blocks=num_blocks,
        s_q=w.s_q, h_q=w.h_q, batch=B,
    )
    if w.topk:
        case["indices"] = make_sparse_indices(L, w.s_q, w.topk, seed=seed, device=device)
    return case


def _poison(kv, fmt, bt, L, spare_blocks):
    """Fill never-read slots with NaN/Inf patterns (recipe step 5)."""
    dev = kv.device
    if fmt == "bf16":
        pat = torch.tensor(_BF16_POISON, dtype=torch.int32).to(torch.int16)
        page = pat.repeat(PAGE * D_QK // len(_BF16_POISON)).view(PAGE, D_QK).to(dev)
        target = kv.view(torch.int16)
    else:
        page = torch.full((PAGE, FP8_BYTES), 0xFF, dtype=torch.uint8, device=dev)
        target = kv
    for b in range(bt.shape[0]):
        Lb = int(L[b])
        if Lb % PAGE:
            target[int(bt[b, (Lb - 1) // PAGE]), Lb % PAGE:] = page[Lb % PAGE:]
    if spare_blocks.numel():
        target[spare_blocks.to(device=dev, dtype=torch.long)] = page


def oracle_arrays(case):
    """Numpy views of a case's inputs for the oracle (bit patterns, no arithmetic)."""
    q = case["q"].detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)
    kv = case["kv_cache"].detach().cpu().contiguous()
    if case["fmt"] == "bf16":
        kv = kv.view(torch.int16).numpy().view(np.uint16)
    else:
        kv = kv.numpy()
    return dict(q_bits=q, kv_cache=kv, fmt=case["fmt"],
                block_table=case["block_table"].cpu().numpy(),
                cache_seqlens=case["cache_seqlens"].cpu().numpy(),
                softmax_scale=case["softmax_scale"], causal=case["causal"])


def oracle_arrays_for(case, requests):
    """Like oracle_arrays but only copies the pages the given requests use.

    Returns (arrays, remap) where block_table rows of the listed requests are
    rewritten to index a compact cache holding just their pages.
    """
    bt = case["block_table"].cpu()
    L = case["cache_seqlens"].cpu()
    blocks = []
    for b in requests:
        n = (int(L[b]) + PAGE - 1) // PAGE
        blocks.extend(bt[b, :n].tolist())
    uniq = sorted(set(blocks)) or [0]
    index = {blk: i for i, blk in enumerate(uniq)}
    sub = case["kv_cache"][torch.tensor(uniq, dtype=torch.long, device=case["kv_cache"].device)].cpu().contiguous()
    new_bt = bt.clone()
    for b in requests:
        n = (int(L[b]) + PAGE - 1) // PAGE
        for p in range(n):
            new_bt[b, p] = index[int(bt[b, p])]
    q = case["q"].detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)
    kv = sub.view(torch.int16).numpy().view(np.uint16) if case["fmt"] == "bf16" else sub.numpy()
    return dict(q_bits=q, kv_cache=kv, fmt=case["fmt"], block_table=new_bt.numpy(),
                cache_seqlens=L.numpy(), softmax_scale=case["softmax_scale"],
                causal=case["causal"])
