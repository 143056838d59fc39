"""Helpers shared by the GPU parity tests: run the CUDA path, run the oracle,
and compare with the tolerances of the method's accuracy contract:
  out: max |err| <= 2e-2 and mean |err| <= 2e-3  (bf16 output vs float64)
  lse: max |err| <= 1e-3
"""

import numpy as np
import torch

import oracle
import workloads as W

OUT_MAX_TOL = 2e-2
OUT_MEAN_TOL = 2e-3
LSE_TOL = 1e-3


def run_gpu(case, num_sm_parts=None, workspace=None):
    import mla_paged_kv_04_b200 as mla
    dev = torch.device("cuda")
    q = case["q"].to(dev)
    kv = case["kv_cache"].to(dev)
    bt = case["block_table"].to(dev)
    L = case["cache_seqlens"].to(dev)
    B, s_q, h_q, _ = q.shape
    parts = mla.mla_default_num_sm_parts() if num_sm_parts is None else num_sm_parts
    sched, ns = mla.mla_get_metadata(L, s_q, h_q, parts)
    ws = mla.alloc_workspace(B, s_q, h_q, parts, dev) if workspace is None else workspace
    out = torch.empty((B, s_q, h_q, 512), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((B, s_q, h_q), dtype=torch.float32, device=dev)
    mla.mla_decode_fwd(q, kv, case["fmt"], bt, L, case["softmax_scale"], case["causal"], sched, ns, parts,
                       out, lse, ws)
    status = mla.mla_last_device_status(ws)
    return out.float().cpu().double().numpy(), lse.cpu().double().numpy(), status


def fp8_cache_as_bf16(kv_u8: torch.Tensor) -> torch.Tensor:
    """The dequantised cache the kernel computes on: bf16(fp32(e4m3) * fp32(scale)).

    Test-side input preparation (torch on CPU) so that the FP8 parity check can
    feed the oracle "the same dequantised cache" as the GPU path.
    """
    kv = kv_u8.cpu()
    nb = kv.shape[0]
    flat = kv.reshape(-1, 656)
    codes = flat[:, :512].contiguous().view(torch.float8_e4m3fn).float()
    scales = flat[:, 512:528].contiguous().view(torch.float32)
    lat = (codes.view(-1, 4, 128) * scales[:, :, None]).view(-1, 512).to(torch.bfloat16)
    rope = flat[:, 528:].contiguous().view(torch.bfloat16)
    return torch.cat([lat, rope], dim=1).view(nb, 64, 576)


def oracle_for(case, requests=None, dequant_bf16=False):
    """Oracle (float64) outputs for all or some requests of a case."""
    if dequant_bf16 and case["fmt"] == "fp8_656":
        case = dict(case)
        case["kv_cache"] = fp8_cache_as_bf16(case["kv_cache"])
        case["fmt"] = "bf16"
    if requests is None:
        a = W.oracle_arrays(case)
        return oracle.mla_decode(a["q_bits"], a["kv_cache"], a["fmt"], a["block_table"], a["cache_seqlens"],
                                 a["softmax_scale"], a["causal"])
    a = W.oracle_arrays_for(case, requests)
    res = oracle.mla_decode_rows(a["q_bits"], a["kv_cache"], a["fmt"], a["block_table"], a["cache_seqlens"],
                                 a["softmax_scale"], a["causal"], requests)
    return res


def oracle_chunked(case, dequant_bf16=False, chunk=16):
    """Oracle outputs of every request of a (possibly full-size) case, computed
    a few requests at a time on compact copies of their pages, so that host
    memory stays bounded.  Returns out [B, s_q, h_q, 512], lse [B, s_q, h_q]."""
    B = case["batch"]
    out = np.zeros((B, case["s_q"], case["h_q"], 512))
    lse = np.full((B, case["s_q"], case["h_q"]), -np.inf)
    for b0 in range(0, B, chunk):
        reqs = list(range(b0, min(B, b0 + chunk)))
        a = W.oracle_arrays_for(case, reqs)
        if dequant_bf16 and a["fmt"] == "fp8_656":
            kv = fp8_cache_as_bf16(torch.from_numpy(a["kv_cache"]))
            a["kv_cache"] = kv.view(torch.int16).numpy().view(np.uint16)
            a["fmt"] = "bf16"
        res = oracle.mla_decode_rows(a["q_bits"], a["kv_cache"], a["fmt"], a["block_table"], a["cache_seqlens"],
                                     a["softmax_scale"], a["causal"], reqs)
        for b in reqs:
            out[b], lse[b] = res[b]
    return out, lse


def run_gpu_sparse(case, indices, num_sm_parts=None, workspace=None):
    """The sparse decode through the C ABI -> (out, lse, status) as float64 numpy."""
    import mla_paged_kv_04_b200 as mla
    dev = torch.device("cuda")
    q = case["q"].to(dev)
    kv = case["kv_cache"].to(dev)
    bt = case["block_table"].to(dev)
    L = case["cache_seqlens"].to(dev)
    idx = indices.to(dev)
    B, s_q, h_q, _ = q.shape
    parts = mla.mla_default_num_sm_parts() if num_sm_parts is None else num_sm_parts
    sched, ns = mla.mla_get_sparse_metadata(B, s_q, h_q, idx.shape[2], parts, device=dev)
    if workspace is None:
        workspace = torch.zeros(mla.mla_sparse_workspace_size(B, s_q, h_q, parts), dtype=torch.uint8, device=dev)
    out = torch.empty((B, s_q, h_q, 512), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((B, s_q, h_q), dtype=torch.float32, device=dev)
    mla.mla_sparse_decode_fwd(q, kv, bt, L, idx, case["softmax_scale"], sched, ns, parts, out, lse, workspace)
    status = mla.mla_last_device_status(workspace)
    return out.float().cpu().double().numpy(), lse.cpu().double().numpy(), status


def oracle_sparse(case, indices, dequant_bf16=False, chunk=16):
    """Sparse-decode oracle outputs for every request, a few requests at a time
    on compact copies of their pages."""
    B = case["batch"]
    idx = indices.cpu().numpy()
    out = np.zeros((B, case["s_q"], case["h_q"], 512))
    lse = np.full((B, case["s_q"], case["h_q"]), -np.inf)
    for b0 in range(0, B, chunk):
        reqs = list(range(b0, min(B, b0 + chunk)))
        a = W.oracle_arrays_for(case, reqs)
        if dequant_bf16 and a["fmt"] == "fp8_656":
            kv = fp8_cache_as_bf16(torch.from_numpy(a["kv_cache"]))
            a["kv_cache"] = kv.view(torch.int16).numpy().view(np.uint16)
            a["fmt"] = "bf16"
        o, l = oracle.mla_sparse_decode(a["q_bits"][reqs], a["kv_cache"], a["fmt"], a["block_table"][reqs],
                                        a["cache_seqlens"][reqs], idx[reqs], a["softmax_scale"])
        out[b0:b0 + len(reqs)] = o
        lse[b0:b0 + len(reqs)] = l
    return out, lse


def check(out, lse, ref_out, ref_lse, what=""):
    """Element-wise comparison; -inf lse must match exactly (empty rows)."""
    err = np.abs(out - ref_out)
    assert np.all(np.isfinite(out)), f"{what}: non-finite output"
    assert err.max() <= OUT_MAX_TOL, f"{what}: out max err {err.max():.3g}"
    assert err.mean() <= OUT_MEAN_TOL, f"{what}: out mean err {err.mean():.3g}"
    inf_ref = np.isneginf(ref_lse)
    assert np.array_equal(np.isneginf(lse), inf_ref), f"{what}: -inf lse pattern differs"
    if (~inf_ref).any():
        lerr = np.abs(lse[~inf_ref] - ref_lse[~inf_ref])
        assert lerr.max() <= LSE_TOL, f"{what}: lse max err {lerr.max():.3g}"
    return float(err.max()), float(err.mean())
