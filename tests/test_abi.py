"""The C-ABI shared library, without a GPU: it builds, loads, exports every
entry point that include/mla.h declares, and rejects bad arguments with the
documented status before touching the device."""

import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "mla.h")


@pytest.fixture(scope="module")
def lib():
    from mla_paged_kv_04_b200 import build
    build.build()
    import mla_paged_kv_04_b200 as mla
    return mla.load_library()


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(mla_[a-z0-9_]+)\s*\(", src)))


def test_header_declares_the_hot_path_calls():
    names = declared_functions()
    for required in ("mla_get_metadata", "mla_decode_fwd", "mla_workspace_size", "mla_metadata_size"):
        assert required in names


def test_every_declared_symbol_is_exported(lib):
    for name in declared_functions():
        assert hasattr(lib, name), f"{name} not exported"


def test_status_strings(lib):
    import mla_paged_kv_04_b200 as mla
    for code, name in mla.STATUS.items():
        assert mla.mla_status_string(code) == name


def test_sizes(lib):
    import mla_paged_kv_04_b200 as mla
    from mla_paged_kv_04_b200 import schedule
    assert mla.mla_metadata_size(64, 1, 128, 74) == 4 * schedule.sched_ints(64, 74)
    assert mla.mla_metadata_size(64, 2, 128, 74) == 4 * schedule.sched_ints(128, 74)   # two row tiles
    assert mla.mla_metadata_size(0, 1, 128, 74) == 0
    assert mla.mla_num_splits_len(64, 1, 128) == 65
    assert mla.mla_num_splits_len(64, 3, 128) == 64 * 3 + 1
    assert mla.mla_num_splits_len(64, 9, 128) == 0                                     # M = 1152 > 1024
    w1 = mla.mla_workspace_size(64, 1, 128, 74)
    w2 = mla.mla_workspace_size(64, 1, 128, 148)
    assert w1 >= 256 + (64 + 74) * 128 * 513 * 4 and w2 > w1
    w3 = mla.mla_workspace_size(1, 2, 128, 74)      # M = 256: two row tiles of 128 rows
    assert w3 >= 256 + (2 + 74) * 128 * 513 * 4
    assert mla.mla_workspace_size(1, 8, 128, 74) > 0
    assert mla.mla_workspace_size(1, 9, 128, 74) == 0  # M = 1152 > 1024 unsupported
    assert mla.mla_workspace_size(4096, 8, 128, 74) == 0  # 32768 row tiles > 16384


def _call_decode(lib, **over):
    args = dict(q=16, kv=16, fmt=0, num_blocks=10, bt=16, max_pages=4, seqlens=16, batch=2, s_q=1, h_q=16,
                scale=0.0417, causal=0, sched=16, ns=16, parts=74, out=16, lse=16, ws=256, ws_bytes=1 << 30,
                stream=None)
    args.update(over)
    return lib.mla_decode_fwd(args["q"], args["kv"], args["fmt"], args["num_blocks"], args["bt"],
                              args["max_pages"], args["seqlens"], args["batch"], args["s_q"], args["h_q"],
                              args["scale"], args["causal"], args["sched"], args["ns"], args["parts"],
                              args["out"], args["lse"], args["ws"], args["ws_bytes"], args["stream"])


def test_decode_argument_validation(lib):
    INVALID, UNSUPPORTED, WORKSPACE = 1, 2, 3
    assert _call_decode(lib, q=None) == INVALID
    assert _call_decode(lib, kv=None) == INVALID
    assert _call_decode(lib, q=8) == INVALID            # misaligned
    assert _call_decode(lib, ws=128) == INVALID         # workspace not 256-aligned
    assert _call_decode(lib, fmt=7) == INVALID
    assert _call_decode(lib, num_blocks=0) == INVALID
    assert _call_decode(lib, max_pages=0) == INVALID
    assert _call_decode(lib, scale=float("nan")) == INVALID
    assert _call_decode(lib, scale=float("inf")) == INVALID
    assert _call_decode(lib, batch=0) == INVALID
    assert _call_decode(lib, s_q=9, h_q=128) == UNSUPPORTED   # M = 1152 > 1024
    assert _call_decode(lib, s_q=2, h_q=128, ws_bytes=1024) == WORKSPACE   # M = 256 is supported
    assert _call_decode(lib, batch=20000) == UNSUPPORTED
    assert _call_decode(lib, ws_bytes=1024) == WORKSPACE


def _call_append(lib, **over):
    args = dict(new=16, batch=2, s_new=1, seqlens=16, bt=16, max_pages=4, kv=16, fmt=1, num_blocks=10, ws=16,
                ws_bytes=256, stream=None)
    args.update(over)
    return lib.mla_kv_append(args["new"], args["batch"], args["s_new"], args["seqlens"], args["bt"],
                             args["max_pages"], args["kv"], args["fmt"], args["num_blocks"], args["ws"],
                             args["ws_bytes"], args["stream"])


def test_append_argument_validation(lib):
    INVALID, UNSUPPORTED, WORKSPACE = 1, 2, 3
    assert _call_append(lib, new=None) == INVALID
    assert _call_append(lib, kv=None) == INVALID
    assert _call_append(lib, ws=None) == INVALID
    assert _call_append(lib, new=8) == INVALID           # misaligned rows
    assert _call_append(lib, kv=4) == INVALID
    assert _call_append(lib, seqlens=2) == INVALID
    assert _call_append(lib, fmt=3) == INVALID
    assert _call_append(lib, batch=0) == INVALID
    assert _call_append(lib, s_new=0) == INVALID
    assert _call_append(lib, max_pages=0) == INVALID
    assert _call_append(lib, num_blocks=0) == INVALID
    assert _call_append(lib, num_blocks=1 << 30) == INVALID
    assert _call_append(lib, batch=1 << 30, s_new=1 << 10) == UNSUPPORTED
    assert _call_append(lib, ws_bytes=2) == WORKSPACE


def test_metadata_argument_validation(lib):
    INVALID, UNSUPPORTED = 1, 2
    f = lib.mla_get_metadata
    assert f(None, 4, 1, 128, 74, 16, 16, None) == INVALID
    assert f(16, 4, 1, 128, 0, 16, 16, None) == INVALID
    assert f(16, 4, 1, 128, 74, 8, 16, None) == INVALID   # sched must be 16-byte aligned
    assert f(16, 0, 1, 128, 74, 16, 16, None) == INVALID
    assert f(16, 4, 17, 64, 74, 16, 16, None) == UNSUPPORTED   # M = 1088 > 1024


def test_product_has_no_oracle_dependency():
    pkg = os.path.join(ROOT, "mla_paged_kv_04_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                src = open(os.path.join(dirpath, f)).read()
                assert "import oracle" not in src and "from oracle" not in src, f


def test_binding_rejects_a_cache_that_does_not_match_its_format():
    import torch
    import mla_paged_kv_04_b200 as mla
    mla._check_cache(torch.zeros((2, 64, 576), dtype=torch.bfloat16), "bf16")
    mla._check_cache(torch.zeros((2, 64, 656), dtype=torch.uint8), "fp8_656")
    for bad, fmt in [(torch.zeros((2, 64, 576), dtype=torch.uint8), "bf16"),
                     (torch.zeros((2, 64, 656), dtype=torch.uint8), "bf16"),
                     (torch.zeros((2, 64, 576), dtype=torch.bfloat16), "fp8_656"),
                     (torch.zeros((2, 32, 656), dtype=torch.uint8), "fp8_656"),
                     (torch.zeros((2, 576, 64), dtype=torch.bfloat16).transpose(1, 2), "bf16"),
                     (torch.zeros((2, 64, 576), dtype=torch.bfloat16), "fp16")]:
        with pytest.raises(ValueError):
            mla._check_cache(bad, fmt)


def test_noalloc_argument_validation(lib):
    # Every host-side check returns before anything is enqueued; on this
    # GPU-less host the fake pointers are never dereferenced.
    INVALID, UNSUPPORTED, WORKSPACE = 1, 2, 3
    f = lib.mla_decode_fwd_noalloc

    def call(**over):
        a = dict(q=16, kv=16, fmt=0, nb=10, bt=16, mp=4, L=16, batch=2, s_q=1, h_q=16, scale=0.0417, causal=0,
                 sched=16, ns=16, parts=74, out=16, lse=16)
        a.update(over)
        return f(a["q"], a["kv"], a["fmt"], a["nb"], a["bt"], a["mp"], a["L"], a["batch"], a["s_q"], a["h_q"],
                 a["scale"], a["causal"], a["sched"], a["ns"], a["parts"], a["out"], a["lse"], None)

    assert call(q=None) == INVALID
    assert call(parts=0) == INVALID           # same code as mla_decode_fwd
    assert call(q=8) == INVALID
    assert call(scale=float("nan")) == INVALID
    assert call(s_q=9, h_q=128) == UNSUPPORTED
    assert call(batch=16384, h_q=128) == WORKSPACE   # beyond the static scratch


def test_wait_timeout_knob(lib):
    import mla_paged_kv_04_b200 as mla
    default = 2_000_000_000
    first = mla.mla_set_wait_timeout_ns(5)
    assert first == default
    assert mla.mla_set_wait_timeout_ns(0) == 5        # 0 restores the default
    assert mla.mla_set_wait_timeout_ns(0) == default


def test_diagnostic_hooks_on_the_product_library(lib):
    import mla_paged_kv_04_b200 as mla
    UNSUPPORTED, INVALID = 2, 1
    assert lib.mla_debug_trace_bytes() == 4 * 7 * 128 * 16 * 8
    assert lib.mla_debug_set_trace_buffer(16, 1 << 20) == UNSUPPORTED   # records only in the trace build
    assert lib.mla_debug_hold_at_tile(2, 3) == INVALID                 # misaligned flag
    assert lib.mla_debug_hold_at_tile(None, -1) == 0
    assert mla.mla_debug_trace_bytes() == 4 * 7 * 128 * 16 * 8


def test_binding_rejects_host_tensors_before_the_c_abi():
    import torch
    import mla_paged_kv_04_b200 as mla
    B = 2
    q = torch.zeros((B, 1, 16, 576), dtype=torch.bfloat16)
    kv = torch.zeros((3, 64, 576), dtype=torch.bfloat16)
    bt = torch.zeros((B, 1), dtype=torch.int32)
    L = torch.ones(B, dtype=torch.int32)
    sched = torch.zeros(mla.mla_metadata_size(B, 1, 16, 74) // 4, dtype=torch.int32)
    ns = torch.zeros(B + 1, dtype=torch.int32)
    out = torch.zeros((B, 1, 16, 512), dtype=torch.bfloat16)
    lse = torch.zeros((B, 1, 16), dtype=torch.float32)
    ws = torch.zeros(mla.mla_workspace_size(B, 1, 16, 74), dtype=torch.uint8)
    with pytest.raises(ValueError):
        mla.mla_decode_fwd(q, kv, "bf16", bt, L, 0.04, False, sched, ns, 74, out, lse, ws)
    with pytest.raises(ValueError):
        mla.mla_decode_fwd_noalloc(q, kv, "bf16", bt, L, 0.04, False, sched, ns, 74, out, lse)
    with pytest.raises(ValueError):
        mla.mla_kv_append(torch.zeros((B, 1, 576), dtype=torch.bfloat16), kv, "bf16", bt, L, ws)
    with pytest.raises(ValueError):
        mla.mla_get_metadata(L, 1, 16, 74)


def test_binding_device_check_resolves_an_unindexed_cuda_device(monkeypatch):
    # torch.device("cuda") names the current device, while tensors report
    # cuda:<index>; the check compares against the resolved index (and still
    # rejects a host tensor, naming that device).
    import torch
    import mla_paged_kv_04_b200 as mla
    monkeypatch.setattr(torch.cuda, "current_device", lambda: 0)
    with pytest.raises(ValueError, match="cuda:0"):
        mla._on_device(torch.device("cuda"), t=torch.zeros(4))
