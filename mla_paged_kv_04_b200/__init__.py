"""Python binding of the B200 MLA paged-KV decoding library (libmla_b200.so).

Argument marshalling only: every step of the computation runs in the CUDA
kernels behind the C ABI declared in include/mla.h.  PyTorch supplies device
memory and streams.  There is no fallback: if the shared library is missing
or the device is not an sm_100 part, calls raise.

Names follow the C ABI:
  mla_default_num_sm_parts, mla_metadata_size, mla_get_metadata,
  mla_workspace_size, mla_decode_fwd, mla_decode_fwd_noalloc,
  mla_noalloc_last_device_status, mla_kv_append, mla_last_device_status,
  mla_clear_device_status, mla_status_string, mla_set_wait_timeout_ns,
  mla_debug_trace_bytes, mla_debug_set_trace_buffer, mla_debug_hold_at_tile,
  mla_get_sparse_metadata, mla_sparse_workspace_size, mla_sparse_decode_fwd
plus `decode(...)` and `sparse_decode(...)`, convenience wrappers that
allocate the outputs, the schedule and the workspace.  Every tensor argument is checked (device, dtype,
shape, size) before its pointer reaches the C ABI.
"""

from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmla_b200.so")
TRACE_LIB_PATH = os.path.join(_HERE, "libmla_b200_trace.so")

MLA_KV_BF16 = 0
MLA_KV_FP8_656 = 1
FORMATS = {"bf16": MLA_KV_BF16, "fp8_656": MLA_KV_FP8_656}
STATUS = {0: "MLA_OK", 1: "MLA_ERR_INVALID_ARG", 2: "MLA_ERR_UNSUPPORTED", 3: "MLA_ERR_WORKSPACE",
          4: "MLA_ERR_CUDA", 5: "MLA_ERR_TIMEOUT", 6: "MLA_ERR_BAD_BLOCK_INDEX"}

_lib = None
_trace_lib = None


class MLAError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {STATUS.get(status, status)}")


def load_library(trace: bool = False):
    """Load libmla_b200.so (built in-tree by `build.build()`); raise if absent.

    trace=True loads the timestamp-recording build (libmla_b200_trace.so,
    `build.build(trace=True)`) instead; see trace.py.
    """
    global _lib, _trace_lib
    if (_trace_lib if trace else _lib) is not None:
        return _trace_lib if trace else _lib
    path = TRACE_LIB_PATH if trace else LIB_PATH
    if not os.path.exists(path):
        raise RuntimeError(f"{path} is missing: build it with mla_paged_kv_04_b200.build.build(trace={trace})")
    lib = ctypes.CDLL(path)
    c_int, c_size, vp, c_float, c_i64 = ctypes.c_int, ctypes.c_size_t, ctypes.c_void_p, ctypes.c_float, ctypes.c_int64
    lib.mla_status_string.restype = ctypes.c_char_p
    lib.mla_status_string.argtypes = [c_int]
    lib.mla_default_num_sm_parts.restype = c_int
    lib.mla_default_num_sm_parts.argtypes = [c_int]
    lib.mla_metadata_size.restype = c_size
    lib.mla_metadata_size.argtypes = [c_int, c_int, c_int, c_int]
    lib.mla_num_splits_len.restype = c_int
    lib.mla_num_splits_len.argtypes = [c_int, c_int, c_int]
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
    lib.mla_sparse_num_splits_len.restype = c_int
    lib.mla_sparse_num_splits_len.argtypes = [c_int, c_int, c_int]
    lib.mla_sparse_metadata_size.restype = c_size
    lib.mla_sparse_metadata_size.argtypes = [c_int, c_int, c_int, c_int]
    lib.mla_sparse_workspace_size.restype = c_size
    lib.mla_sparse_workspace_size.argtypes = [c_int, c_int, c_int, c_int]
    lib.mla_get_sparse_metadata.restype = c_int
    lib.mla_get_sparse_metadata.argtypes = [c_int, c_int, c_int, c_int, c_int, vp, vp, vp]
    lib.mla_sparse_decode_fwd.restype = c_int
    lib.mla_sparse_decode_fwd.argtypes = [vp, vp, c_i64, vp, c_int, vp, vp, c_int, c_int, c_int, c_int, c_float,
                                          vp, vp, c_int, vp, vp, vp, c_size, vp]
    lib.mla_kv_append.restype = c_int
    lib.mla_kv_append.argtypes = [vp, c_int, c_int, vp, vp, c_int, vp, c_int, c_i64, vp, c_size, vp]
    lib.mla_last_device_status.restype = c_int
    lib.mla_last_device_status.argtypes = [vp, vp]
    lib.mla_clear_device_status.restype = c_int
    lib.mla_clear_device_status.argtypes = [vp, vp]
    lib.mla_noalloc_last_device_status.restype = c_int
    lib.mla_noalloc_last_device_status.argtypes = [vp]
    lib.mla_set_wait_timeout_ns.restype = ctypes.c_uint64
    lib.mla_set_wait_timeout_ns.argtypes = [ctypes.c_uint64]
    lib.mla_debug_trace_bytes.restype = c_size
    lib.mla_debug_trace_bytes.argtypes = []
    lib.mla_debug_set_trace_buffer.restype = c_int
    lib.mla_debug_set_trace_buffer.argtypes = [vp, c_size]
    lib.mla_debug_hold_at_tile.restype = c_int
    lib.mla_debug_hold_at_tile.argtypes = [vp, c_int]
    if trace:
        _trace_lib = lib
    else:
        _lib = lib
    return lib


def _active_lib():
    """The library the calls go through: the product one, unless only the
    trace build has been loaded (trace.py does that)."""
    if _lib is None and _trace_lib is not None:
        return _trace_lib
    return load_library()


def _stream(stream=None) -> int:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream


def _check(status: int, where: str):
    if status != 0:
        raise MLAError(status, where)


def _on_device(device: torch.device, **tensors):
    """Every tensor must live on `device` (a CUDA device) and be contiguous:
    the C ABI receives bare pointers and cannot tell."""
    if device.type != "cuda":
        raise ValueError(f"tensors must be CUDA tensors, got {device}")
    if device.index is None:
        device = torch.device("cuda", torch.cuda.current_device())
    for name, t in tensors.items():
        if not isinstance(t, torch.Tensor):
            raise TypeError(f"{name} must be a torch.Tensor")
        if t.device != device:
            raise ValueError(f"{name} is on {t.device}, expected {device}")
        if not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous")


def _nbytes(t: torch.Tensor) -> int:
    return t.numel() * t.element_size()


def _check_decode_tensors(q, kv_cache, fmt, block_table, cache_seqlens, sched, num_splits, num_sm_parts, out,
                          lse, workspace=None):
    """Shapes, dtypes, devices and sizes of a decode call's tensors."""
    if q.dim() != 4 or q.shape[3] != 576 or q.dtype != torch.bfloat16:
        raise ValueError(f"q must be bf16 [batch, s_q, h_q, 576], got {q.dtype} {tuple(q.shape)}")
    B, s_q, h_q, _ = q.shape
    tensors = dict(q=q, kv_cache=kv_cache, block_table=block_table, cache_seqlens=cache_seqlens, sched=sched,
                   num_splits=num_splits, out=out, lse=lse)
    if workspace is not None:
        tensors["workspace"] = workspace
    _on_device(q.device, **tensors)
    _check_cache(kv_cache, fmt)
    if block_table.dtype != torch.int32 or block_table.dim() != 2 or block_table.shape[0] != B:
        raise ValueError(f"block_table must be int32 [batch={B}, max_pages], got {block_table.dtype} "
                         f"{tuple(block_table.shape)}")
    if cache_seqlens.dtype != torch.int32 or cache_seqlens.numel() != B:
        raise ValueError(f"cache_seqlens must be int32 [{B}]")
    if out.shape != (B, s_q, h_q, 512) or out.dtype != torch.bfloat16:
        raise ValueError(f"out must be bf16 {(B, s_q, h_q, 512)}, got {out.dtype} {tuple(out.shape)}")
    if lse.shape != (B, s_q, h_q) or lse.dtype != torch.float32:
        raise ValueError(f"lse must be fp32 {(B, s_q, h_q)}, got {lse.dtype} {tuple(lse.shape)}")
    if sched.dtype != torch.int32 or _nbytes(sched) < mla_metadata_size(B, s_q, h_q, int(num_sm_parts)):
        raise ValueError(f"sched must be int32 of >= mla_metadata_size({B}, {s_q}, {h_q}, {num_sm_parts}) bytes")
    n_len = mla_num_splits_len(B, s_q, h_q)
    if num_splits.dtype != torch.int32 or num_splits.numel() < n_len:
        raise ValueError(f"num_splits must be int32 [>= {n_len}]")


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
    return _active_lib().mla_status_string(status).decode()


def mla_default_num_sm_parts(device=None) -> int:
    dev = torch.cuda.current_device() if device is None else torch.device(device).index or 0
    n = _active_lib().mla_default_num_sm_parts(dev)
    if n <= 0:
        raise MLAError(4, "mla_default_num_sm_parts")
    return n


def mla_metadata_size(batch: int, s_q: int, h_q: int, num_sm_parts: int) -> int:
    return _active_lib().mla_metadata_size(batch, s_q, h_q, num_sm_parts)


def mla_num_splits_len(batch: int, s_q: int, h_q: int) -> int:
    return _active_lib().mla_num_splits_len(batch, s_q, h_q)


def mla_workspace_size(batch: int, s_q: int, h_q: int, num_sm_parts: int) -> int:
    return _active_lib().mla_workspace_size(batch, s_q, h_q, num_sm_parts)


def mla_get_metadata(cache_seqlens: torch.Tensor, s_q: int, h_q: int, num_sm_parts: int | None = None,
                     sched: torch.Tensor | None = None, num_splits: torch.Tensor | None = None, stream=None):
    """Split-KV schedule for `cache_seqlens` (device int32 [batch]) -> (sched, num_splits)."""
    lib = _active_lib()
    if not cache_seqlens.is_cuda or cache_seqlens.dtype != torch.int32:
        raise ValueError("cache_seqlens must be a CUDA int32 tensor")
    batch = cache_seqlens.numel()
    parts = mla_default_num_sm_parts(cache_seqlens.device) if num_sm_parts is None else int(num_sm_parts)
    nbytes = lib.mla_metadata_size(batch, s_q, h_q, parts)
    n_len = lib.mla_num_splits_len(batch, s_q, h_q)
    if nbytes == 0 or n_len == 0:
        raise MLAError(2, "mla_get_metadata")
    if sched is None:
        sched = torch.empty(max(nbytes // 4, 1), dtype=torch.int32, device=cache_seqlens.device)
    if num_splits is None:
        num_splits = torch.empty(n_len, dtype=torch.int32, device=cache_seqlens.device)
    _on_device(cache_seqlens.device, cache_seqlens=cache_seqlens, sched=sched, num_splits=num_splits)
    if sched.dtype != torch.int32 or num_splits.dtype != torch.int32 or num_splits.numel() < n_len:
        raise ValueError(f"sched and num_splits must be int32, num_splits of >= {n_len} entries")
    if _nbytes(sched) < nbytes:
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
    lib = _active_lib()
    _check_decode_tensors(q, kv_cache, fmt, block_table, cache_seqlens, sched, num_splits, num_sm_parts, out, lse,
                          workspace)
    B, s_q, h_q, _ = q.shape
    num_blocks = kv_cache.shape[0]
    _check(lib.mla_decode_fwd(q.data_ptr(), kv_cache.data_ptr(), FORMATS[fmt], num_blocks, block_table.data_ptr(),
                              block_table.shape[1], cache_seqlens.data_ptr(), B, s_q, h_q, float(softmax_scale),
                              1 if causal else 0, sched.data_ptr(), num_splits.data_ptr(), int(num_sm_parts),
                              out.data_ptr(), lse.data_ptr(), workspace.data_ptr(),
                              _nbytes(workspace), _stream(stream)), "mla_decode_fwd")
    return out, lse


def mla_decode_fwd_noalloc(q: torch.Tensor, kv_cache: torch.Tensor, fmt: str, block_table: torch.Tensor,
                           cache_seqlens: torch.Tensor, softmax_scale: float, causal: bool, sched: torch.Tensor,
                           num_splits: torch.Tensor, num_sm_parts: int, out: torch.Tensor, lse: torch.Tensor,
                           stream=None):
    """mla_decode_fwd without a workspace: the split-KV scratch is the library's
    static per-device array (see include/mla.h for its size limit and sharing)."""
    lib = _active_lib()
    _check_decode_tensors(q, kv_cache, fmt, block_table, cache_seqlens, sched, num_splits, num_sm_parts, out, lse)
    B, s_q, h_q, _ = q.shape
    _check(lib.mla_decode_fwd_noalloc(q.data_ptr(), kv_cache.data_ptr(), FORMATS[fmt], kv_cache.shape[0],
                                      block_table.data_ptr(), block_table.shape[1], cache_seqlens.data_ptr(), B, s_q,
                                      h_q, float(softmax_scale), 1 if causal else 0, sched.data_ptr(),
                                      num_splits.data_ptr(), int(num_sm_parts), out.data_ptr(), lse.data_ptr(),
                                      _stream(stream)), "mla_decode_fwd_noalloc")
    return out, lse


def mla_get_sparse_metadata(batch: int, s_q: int, h_q: int, topk: int, num_sm_parts: int | None = None,
                            device=None, sched: torch.Tensor | None = None, num_splits: torch.Tensor | None = None,
                            stream=None):
    """Split-KV schedule of a sparse decode: batch * s_q units of h_q rows,
    each attending to topk list entries -> (sched, num_splits)."""
    lib = _active_lib()
    device = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    parts = mla_default_num_sm_parts(device) if num_sm_parts is None else int(num_sm_parts)
    nbytes = lib.mla_sparse_metadata_size(batch, s_q, h_q, parts)
    n_len = lib.mla_sparse_num_splits_len(batch, s_q, h_q)
    if nbytes == 0 or n_len == 0:
        raise MLAError(2, "mla_get_sparse_metadata")
    if sched is None:
        sched = torch.empty(max(nbytes // 4, 1), dtype=torch.int32, device=device)
    if num_splits is None:
        num_splits = torch.empty(n_len, dtype=torch.int32, device=device)
    _on_device(device, sched=sched, num_splits=num_splits)
    if sched.dtype != torch.int32 or num_splits.dtype != torch.int32 or num_splits.numel() < n_len or \
            _nbytes(sched) < nbytes:
        raise ValueError(f"sched (int32, >= {nbytes} bytes) and num_splits (int32, >= {n_len}) too small")
    _check(lib.mla_get_sparse_metadata(batch, s_q, h_q, int(topk), parts, sched.data_ptr(), num_splits.data_ptr(),
                                       _stream(stream)), "mla_get_sparse_metadata")
    return sched, num_splits


def mla_sparse_workspace_size(batch: int, s_q: int, h_q: int, num_sm_parts: int) -> int:
    return _active_lib().mla_sparse_workspace_size(batch, s_q, h_q, num_sm_parts)


def mla_sparse_metadata_size_bytes(batch: int, s_q: int, h_q: int, num_sm_parts: int) -> int:
    return _active_lib().mla_sparse_metadata_size(batch, s_q, h_q, num_sm_parts)


def mla_sparse_num_splits_len(batch: int, s_q: int, h_q: int) -> int:
    return _active_lib().mla_sparse_num_splits_len(batch, s_q, h_q)


def mla_sparse_decode_fwd(q: torch.Tensor, kv_cache: torch.Tensor, block_table: torch.Tensor,
                          cache_seqlens: torch.Tensor, indices: torch.Tensor, softmax_scale: float,
                          sched: torch.Tensor, num_splits: torch.Tensor, num_sm_parts: int, out: torch.Tensor,
                          lse: torch.Tensor, workspace: torch.Tensor, stream=None):
    """Enqueue the sparse decode (FP8 656-byte cache): query token i of request
    b attends to the positions indices[b, i, :] (entries outside [0, L) are
    padding); see include/mla.h."""
    lib = _active_lib()
    if q.dim() != 4 or q.shape[3] != 576 or q.dtype != torch.bfloat16:
        raise ValueError(f"q must be bf16 [batch, s_q, h_q, 576], got {q.dtype} {tuple(q.shape)}")
    B, s_q, h_q, _ = q.shape
    _on_device(q.device, q=q, kv_cache=kv_cache, block_table=block_table, cache_seqlens=cache_seqlens,
               indices=indices, sched=sched, num_splits=num_splits, out=out, lse=lse, workspace=workspace)
    _check_cache(kv_cache, "fp8_656")
    if indices.dtype != torch.int32 or indices.dim() != 3 or tuple(indices.shape[:2]) != (B, s_q):
        raise ValueError(f"indices must be int32 [{B}, {s_q}, topk], got {indices.dtype} {tuple(indices.shape)}")
    topk = indices.shape[2]
    if block_table.dtype != torch.int32 or block_table.dim() != 2 or block_table.shape[0] != B:
        raise ValueError(f"block_table must be int32 [batch={B}, max_pages]")
    if cache_seqlens.dtype != torch.int32 or cache_seqlens.numel() != B:
        raise ValueError(f"cache_seqlens must be int32 [{B}]")
    if out.shape != (B, s_q, h_q, 512) or out.dtype != torch.bfloat16:
        raise ValueError(f"out must be bf16 {(B, s_q, h_q, 512)}")
    if lse.shape != (B, s_q, h_q) or lse.dtype != torch.float32:
        raise ValueError(f"lse must be fp32 {(B, s_q, h_q)}")
    nbytes = lib.mla_sparse_metadata_size(B, s_q, h_q, int(num_sm_parts))
    if sched.dtype != torch.int32 or _nbytes(sched) < nbytes or num_splits.dtype != torch.int32 or \
            num_splits.numel() < lib.mla_sparse_num_splits_len(B, s_q, h_q):
        raise ValueError("sched / num_splits do not fit this shape (use mla_get_sparse_metadata)")
    _check(lib.mla_sparse_decode_fwd(q.data_ptr(), kv_cache.data_ptr(), kv_cache.shape[0], block_table.data_ptr(),
                                     block_table.shape[1], cache_seqlens.data_ptr(), indices.data_ptr(), topk, B,
                                     s_q, h_q, float(softmax_scale), sched.data_ptr(), num_splits.data_ptr(),
                                     int(num_sm_parts), out.data_ptr(), lse.data_ptr(), workspace.data_ptr(),
                                     _nbytes(workspace), _stream(stream)), "mla_sparse_decode_fwd")
    return out, lse


def sparse_decode(q, kv_cache, block_table, cache_seqlens, indices, softmax_scale, num_sm_parts=None, stream=None):
    """One-shot sparse decode: schedule + workspace + outputs allocated here -> (out, lse)."""
    B, s_q, h_q, _ = q.shape
    parts = mla_default_num_sm_parts(q.device) if num_sm_parts is None else int(num_sm_parts)
    sched, num_splits = mla_get_sparse_metadata(B, s_q, h_q, indices.shape[2], parts, device=q.device,
                                                stream=stream)
    n = mla_sparse_workspace_size(B, s_q, h_q, parts)
    if n == 0:
        raise MLAError(2, "mla_sparse_workspace_size")
    ws = torch.zeros(n, dtype=torch.uint8, device=q.device)
    out = torch.empty((B, s_q, h_q, 512), dtype=torch.bfloat16, device=q.device)
    lse = torch.empty((B, s_q, h_q), dtype=torch.float32, device=q.device)
    mla_sparse_decode_fwd(q, kv_cache, block_table, cache_seqlens, indices, softmax_scale, sched, num_splits, parts,
                          out, lse, ws, stream=stream)
    return out, lse


def mla_noalloc_last_device_status(stream=None) -> int:
    """Synchronise the stream and return the device status of the last
    mla_decode_fwd_noalloc call on the current device (0 = MLA_OK)."""
    return _active_lib().mla_noalloc_last_device_status(_stream(stream))


def mla_set_wait_timeout_ns(ns: int) -> int:
    """Limit of every wait inside later decode kernels (0 = the 2 s default);
    returns the previous limit."""
    return int(_active_lib().mla_set_wait_timeout_ns(int(ns)))


def mla_debug_trace_bytes() -> int:
    return int(_active_lib().mla_debug_trace_bytes())


def mla_debug_set_trace_buffer(buffer: torch.Tensor | None) -> int:
    """Point the trace build's timestamp recording at `buffer` (None stops it).
    Returns the status (MLA_ERR_UNSUPPORTED from the product library)."""
    lib = _active_lib()
    if buffer is None:
        return lib.mla_debug_set_trace_buffer(None, 0)
    _on_device(buffer.device, buffer=buffer)
    return lib.mla_debug_set_trace_buffer(buffer.data_ptr(), _nbytes(buffer))


def mla_debug_hold_at_tile(flag: torch.Tensor | None, tile: int = -1):
    """Make later decode calls wait at tile `tile` until the device int32
    `flag` is non-zero (bounded by the wait timeout); None turns it off."""
    lib = _active_lib()
    if flag is None:
        _check(lib.mla_debug_hold_at_tile(None, -1), "mla_debug_hold_at_tile")
        return
    _on_device(flag.device, flag=flag)
    if flag.dtype != torch.int32 or flag.numel() < 1:
        raise ValueError("flag must be a device int32 tensor")
    _check(lib.mla_debug_hold_at_tile(flag.data_ptr(), int(tile)), "mla_debug_hold_at_tile")


def mla_kv_append(kv_new: torch.Tensor, kv_cache: torch.Tensor, fmt: str, block_table: torch.Tensor,
                  cache_seqlens: torch.Tensor, workspace: torch.Tensor, stream=None):
    """Enqueue the append of kv_new (bf16 [batch, s_new, 576]) into the paged cache on `stream`.

    cache_seqlens are the lengths after the append; new token t of request b
    lands at position cache_seqlens[b] - s_new + t (see include/mla.h).
    """
    lib = _active_lib()
    if kv_new.dim() != 3 or kv_new.shape[2] != 576 or kv_new.dtype != torch.bfloat16:
        raise ValueError(f"kv_new must be bf16 [batch, s_new, 576], got {kv_new.dtype} {tuple(kv_new.shape)}")
    B, s_new, _ = kv_new.shape
    _on_device(kv_new.device, kv_new=kv_new, kv_cache=kv_cache, block_table=block_table,
               cache_seqlens=cache_seqlens, workspace=workspace)
    _check_cache(kv_cache, fmt)
    if block_table.dtype != torch.int32 or block_table.dim() != 2 or block_table.shape[0] != B:
        raise ValueError(f"block_table must be int32 [batch={B}, max_pages]")
    if cache_seqlens.dtype != torch.int32 or cache_seqlens.numel() != B:
        raise ValueError(f"cache_seqlens must be int32 [{B}]")
    _check(lib.mla_kv_append(kv_new.data_ptr(), B, s_new, cache_seqlens.data_ptr(), block_table.data_ptr(),
                             block_table.shape[1], kv_cache.data_ptr(), FORMATS[fmt], kv_cache.shape[0],
                             workspace.data_ptr(), _nbytes(workspace), _stream(stream)),
           "mla_kv_append")
    return kv_cache


def mla_last_device_status(workspace: torch.Tensor, stream=None) -> int:
    """Synchronise the stream and return the device status code (0 = MLA_OK)."""
    _on_device(workspace.device, workspace=workspace)
    return _active_lib().mla_last_device_status(workspace.data_ptr(), _stream(stream))


def mla_clear_device_status(workspace: torch.Tensor, stream=None):
    _on_device(workspace.device, workspace=workspace)
    _check(_active_lib().mla_clear_device_status(workspace.data_ptr(), _stream(stream)), "mla_clear_device_status")


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
