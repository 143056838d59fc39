"""Python binding of the B200 MLA paged-KV decoding library (libmla_b200.so).

Argument marshalling only: every step of the computation runs in the CUDA
kernels behind the C ABI declared in include/mla.h.  PyTorch supplies device
memory and streams.  There is no fallback: if the shared library is missing
or the device is not an sm_100 part, calls raise.

Names follow the C ABI:
  mla_default_num_sm_parts, mla_metadata_size, mla_get_metadata,
  mla_workspace_size, mla_decode_fwd, mla_decode_fwd_noalloc, mla_kv_append, mla_last_device_status,
  mla_clear_device_status, mla_status_string
plus `decode(...)`, a convenience wrapper that allocates the outputs, the
schedule and the workspace.
"""

from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmla_b200.so")

MLA_KV_BF16 = 0
MLA_KV_FP8_656 = 1
FORMATS = {"bf16": MLA_KV_BF16, "fp8_656": MLA_KV_FP8_656}
STATUS = {0: "MLA_OK", 1: "MLA_ERR_INVALID_ARG", 2: "MLA_ERR_UNSUPPORTED", 3: "MLA_ERR_WORKSPACE",
          4: "MLA_ERR_CUDA", 5: "MLA_ERR_TIMEOUT", 6: "MLA_ERR_BAD_BLOCK_INDEX"}

_lib = None


class MLAError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {STATUS.get(status, status)}")


def load_library():
    """Load libmla_b200.so (built in-tree by `build.build()`); raise if absent."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"{LIB_PATH} is missing: build it with mla_paged_kv_04_b200.build.build()")
    lib = ctypes.CDLL(LIB_PATH)
    c_int, c_size, vp, c_float, c_i64 = ctypes.c_int, ctypes.c_size_t, ctypes.c_void_p, ctypes.c_float, ctypes.c_int64
    lib.mla_status_string.restype = ctypes.c_char_p
    lib.mla_status_string.argtypes = [c_int]
    lib.mla_default_num_sm_parts.restype = c_int
    lib.mla_default_num_sm_parts.argtypes = [c_int]
    lib.mla_metadata_size.restype = c_size
    lib.mla_metadata_size.argtypes = [c_int, c_int]
    lib.mla_get_metadata.restype = c_int
    lib.mla_get_metadata.argtypes = [vp, c_int, c_int, c_int, c_int, vp, vp, vp]
    lib.mla_workspace_size.restype = c_size
    lib.mla_workspace_size.argtypes = [c_int, c_int, c_int, c_int]
    lib.mla_decode_fwd.restype = c_int
    lib.mla_decode_fwd.argtypes = [vp, vp, c_int, c_i64, vp, c_int, vp, c_int, c_int, c_int, c_float, c_int,
                                   vp, vp, c_int, vp, vp, vp, c_size, vp]
    lib.mla_decode_fwd_noalloc.restype = c_int
    lib.mla_decode_fwd_noalloc.argtypes = [vp, vp, c_int, c_i64, vp, c_int, vp, c_int, c_int, c_int, c_float, c_int,
                                           vp, vp, c_int, vp, vp, vp]
    lib.mla_kv_append.restype = c_int
    lib.mla_kv_append.argtypes = [vp, c_int, c_int, vp, vp, c_int, vp, c_int, c_i64, vp, c_size, vp]
    lib.mla_last_device_status.restype = c_int
    lib.mla_last_device_status.argtypes = [vp, vp]
    lib.mla_clear_device_status.restype = c_int
    lib.mla_clear_device_status.argtypes = [vp, vp]
    _lib = lib
    return lib


def _stream(stream=None) -> int:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream


def _check(status: int, where: str):
    if status != 0:
        raise MLAError(status, where)


def _check_cache(kv_cache: torch.Tensor, fmt: str):
    """The cache tensor must be what `fmt` says, since the kernels address it
    as [num_blocks, 64, token bytes] from its first dimension alone."""
    if fmt not in FORMATS:
        raise ValueError(f"unknown cache format {fmt!r}")
    want = (torch.bfloat16, 576) if fmt == "bf16" else (torch.uint8, 656)
    if kv_cache.dtype != want[0] or kv_cache.dim() != 3 or tuple(kv_cache.shape[1:]) != (64, want[1]):
        raise ValueError(f"{fmt} cache must be {want[0]} [num_blocks, 64, {want[1]}], "
                         f"got {kv_cache.dtype} {tuple(kv_cache.shape)}")
    if not kv_cache.is_contiguous():
        raise ValueError("the cache must be contiguous")


def mla_status_string(status: int) -> str:
    return load_library().mla_status_string(status).decode()


def mla_default_num_sm_parts(device=None) -> int:
    dev = torch.cuda.current_device() if device is None else torch.device(device).index or 0
    n = load_library().mla_default_num_sm_parts(dev)
    if n <= 0:
        raise MLAError(4, "mla_default_num_sm_parts")
    return n


def mla_metadata_size(batch: int, num_sm_parts: int) -> int:
    return load_library().mla_metadata_size(batch, num_sm_parts)


def mla_workspace_size(batch: int, s_q: int, h_q: int, num_sm_parts: int) -> int:
    return load_library().mla_workspace_size(batch, s_q, h_q, num_sm_parts)


def mla_get_metadata(cache_seqlens: torch.Tensor, s_q: int, h_q: int, num_sm_parts: int | None = None,
                     sched: torch.Tensor | None = None, num_splits: torch.Tensor | None = None, stream=None):
    """Split-KV schedule for `cache_seqlens` (device int32 [batch]) -> (sched, num_splits)."""
    lib = load_library()
    assert cache_seqlens.is_cuda and cache_seqlens.dtype == torch.int32 and cache_seqlens.is_contiguous()
    batch = cache_seqlens.numel()
    parts = mla_default_num_sm_parts(cache_seqlens.device) if num_sm_parts is None else int(num_sm_parts)
    nbytes = lib.mla_metadata_size(batch, parts)
    if sched is None:
        sched = torch.empty(max(nbytes // 4, 1), dtype=torch.int32, device=cache_seqlens.device)
    if num_splits is None:
        num_splits = torch.empty(batch + 1, dtype=torch.int32, device=cache_seqlens.device)
    if sched.numel() * 4 < nbytes:
        raise MLAError(3, "mla_get_metadata")
    _check(lib.mla_get_metadata(cache_seqlens.data_ptr(), batch, s_q, h_q, parts, sched.data_ptr(),
                                num_splits.data_ptr(), _stream(stream)), "mla_get_metadata")
    return sched, num_splits


def alloc_workspace(batch: int, s_q: int, h_q: int, num_sm_parts: int, device) -> torch.Tensor:
    """Zero-filled workspace (the zero fill clears the device status word)."""
    n = mla_workspace_size(batch, s_q, h_q, num_sm_parts)
    if n == 0:
        raise MLAError(2, "mla_workspace_size")
    return torch.zeros(n, dtype=torch.uint8, device=device)


def mla_decode_fwd(q: torch.Tensor, kv_cache: torch.Tensor, fmt: str, block_table: torch.Tensor,
                   cache_seqlens: torch.Tensor, softmax_scale: float, causal: bool, sched: torch.Tensor,
                   num_splits: torch.Tensor, num_sm_parts: int, out: torch.Tensor, lse: torch.Tensor,
                   workspace: torch.Tensor, stream=None):
    """Enqueue the decode (and, where needed, the split-KV combine) on `stream`."""
    lib = load_library()
    B, s_q, h_q, d = q.shape
    assert d == 576 and q.dtype == torch.bfloat16 and q.is_contiguous()
    _check_cache(kv_cache, fmt)
    assert block_table.is_contiguous() and block_table.dtype == torch.int32 and block_table.shape[0] == B
    assert out.shape == (B, s_q, h_q, 512) and out.dtype == torch.bfloat16 and out.is_contiguous()
    assert lse.shape == (B, s_q, h_q) and lse.dtype == torch.float32 and lse.is_contiguous()
    assert cache_seqlens.dtype == torch.int32 and cache_seqlens.is_contiguous() and cache_seqlens.numel() == B
    num_blocks = kv_cache.shape[0]
    _check(lib.mla_decode_fwd(q.data_ptr(), kv_cache.data_ptr(), FORMATS[fmt], num_blocks, block_table.data_ptr(),
                              block_table.shape[1], cache_seqlens.data_ptr(), B, s_q, h_q, float(softmax_scale),
                              1 if causal else 0, sched.data_ptr(), num_splits.data_ptr(), int(num_sm_parts),
                              out.data_ptr(), lse.data_ptr(), workspace.data_ptr(),
                              workspace.numel() * workspace.element_size(), _stream(stream)), "mla_decode_fwd")
    return out, lse


def mla_decode_fwd_noalloc(q: torch.Tensor, kv_cache: torch.Tensor, fmt: str, block_table: torch.Tensor,
                           cache_seqlens: torch.Tensor, softmax_scale: float, causal: bool, sched: torch.Tensor,
                           num_splits: torch.Tensor, num_sm_parts: int, out: torch.Tensor, lse: torch.Tensor,
                           stream=None):
    """mla_decode_fwd without a workspace: the split-KV scratch is the library's
    static per-device array (see include/mla.h for its size limit and sharing)."""
    lib = load_library()
    B, s_q, h_q, d = q.shape
    assert d == 576 and q.dtype == torch.bfloat16 and q.is_contiguous()
    _check_cache(kv_cache, fmt)
    assert block_table.is_contiguous() and block_table.dtype == torch.int32 and block_table.shape[0] == B
    assert out.shape == (B, s_q, h_q, 512) and out.dtype == torch.bfloat16 and out.is_contiguous()
    assert lse.shape == (B, s_q, h_q) and lse.dtype == torch.float32 and lse.is_contiguous()
    assert cache_seqlens.dtype == torch.int32 and cache_seqlens.is_contiguous() and cache_seqlens.numel() == B
    _check(lib.mla_decode_fwd_noalloc(q.data_ptr(), kv_cache.data_ptr(), FORMATS[fmt], kv_cache.shape[0],
                                      block_table.data_ptr(), block_table.shape[1], cache_seqlens.data_ptr(), B, s_q,
                                      h_q, float(softmax_scale), 1 if causal else 0, sched.data_ptr(),
                                      num_splits.data_ptr(), int(num_sm_parts), out.data_ptr(), lse.data_ptr(),
                                      _stream(stream)), "mla_decode_fwd_noalloc")
    return out, lse


def mla_kv_append(kv_new: torch.Tensor, kv_cache: torch.Tensor, fmt: str, block_table: torch.Tensor,
                  cache_seqlens: torch.Tensor, workspace: torch.Tensor, stream=None):
    """Enqueue the append of kv_new (bf16 [batch, s_new, 576]) into the paged cache on `stream`.

    cache_seqlens are the lengths after the append; new token t of request b
    lands at position cache_seqlens[b] - s_new + t (see include/mla.h).
    """
    lib = load_library()
    B, s_new, d = kv_new.shape
    assert d == 576 and kv_new.dtype == torch.bfloat16 and kv_new.is_contiguous()
    _check_cache(kv_cache, fmt)
    assert block_table.is_contiguous() and block_table.dtype == torch.int32 and block_table.shape[0] == B
    assert cache_seqlens.dtype == torch.int32 and cache_seqlens.is_contiguous() and cache_seqlens.numel() == B
    _check(lib.mla_kv_append(kv_new.data_ptr(), B, s_new, cache_seqlens.data_ptr(), block_table.data_ptr(),
                             block_table.shape[1], kv_cache.data_ptr(), FORMATS[fmt], kv_cache.shape[0],
                             workspace.data_ptr(), workspace.numel() * workspace.element_size(), _stream(stream)),
           "mla_kv_append")
    return kv_cache


def mla_last_device_status(workspace: torch.Tensor, stream=None) -> int:
    """Synchronise the stream and return the device status code (0 = MLA_OK)."""
    return load_library().mla_last_device_status(workspace.data_ptr(), _stream(stream))


def mla_clear_device_status(workspace: torch.Tensor, stream=None):
    _check(load_library().mla_clear_device_status(workspace.data_ptr(), _stream(stream)), "mla_clear_device_status")


def decode(q, kv_cache, block_table, cache_seqlens, softmax_scale, causal=False, fmt="bf16", num_sm_parts=None,
           stream=None):
    """One-shot decode: schedule + workspace + outputs allocated here -> (out, lse)."""
    B, s_q, h_q, _ = q.shape
    parts = mla_default_num_sm_parts(q.device) if num_sm_parts is None else int(num_sm_parts)
    sched, num_splits = mla_get_metadata(cache_seqlens, s_q, h_q, parts, stream=stream)
    ws = alloc_workspace(B, s_q, h_q, parts, q.device)
    out = torch.empty((B, s_q, h_q, 512), dtype=torch.bfloat16, device=q.device)
    lse = torch.empty((B, s_q, h_q), dtype=torch.float32, device=q.device)
    mla_decode_fwd(q, kv_cache, fmt, block_table, cache_seqlens, softmax_scale, causal, sched, num_splits, parts,
                   out, lse, ws, stream=stream)
    return out, lse
