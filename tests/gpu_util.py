"""Shared helpers of the GPU parity tests: upload seeded host inputs, call the library through
its C ABI, and compare with the CPU oracle at the stated tolerance.

Tolerance (the attention outputs are O(1e-3) at million-token lengths, so an elementwise
relative bound is ill-posed near zero): for every (sequence, query head) row,
max_d |out - ref| <= 2e-3 * max_d |ref|, and |lse - ref_lse| <= 1e-4 absolute; an empty
row must give exactly 0 and -inf.
"""
from __future__ import annotations

import concurrent.futures as cf
import os

import numpy as np

OUT_RTOL = 2e-3
LSE_ATOL = 1e-4


def device_tensor(arr: np.ndarray, dtype: str):
    import torch

    if dtype == "bf16":
        return torch.from_numpy(np.ascontiguousarray(arr).view(np.int16)).view(torch.bfloat16).cuda()
    return torch.from_numpy(np.ascontiguousarray(arr, dtype=np.float32)).cuda()


def empty_outputs(B: int, Hq: int, D: int):
    import torch

    out = torch.full((B, Hq, D), float("nan"), dtype=torch.float32, device="cuda")
    lse = torch.full((B, Hq), float("nan"), dtype=torch.float32, device="cuda")
    return out, lse


def new_workspace(nbytes: int):
    import torch

    import exact_long_context_split_b200 as ta

    ws = torch.empty(max(nbytes, 256), dtype=torch.uint8, device="cuda")
    ta.tree_attn_workspace_init(ws)
    return ws


def decode_gpu(inp, spec, opts=None, entry: str = "ex", ws=None):
    """Run one decode through the C ABI; returns (out, lse) as numpy float32 arrays."""
    import torch

    import exact_long_context_split_b200 as ta

    B, Hq, Hkv, D = spec.batch, spec.n_q_heads, spec.n_kv_heads, spec.head_dim
    q = device_tensor(inp["q"], spec.dtype)
    k = device_tensor(inp["k"], spec.dtype)
    v = device_tensor(inp["v"], spec.dtype)
    out, lse = empty_outputs(B, Hq, D)
    seqlens = [int(s) for s in spec.seqlens]
    if entry == "ex":
        if ws is None:
            ws = new_workspace(ta.tree_attn_workspace_size(seqlens, Hq, Hkv, D, spec.dtype, opts))
        ta.tree_attn_decode_ex(spec.dtype, q, k, v, seqlens, Hq, Hkv, D, spec.scale, out, lse, opts, ws)
        status = ta.tree_attn_check(ws)
        assert status == ta.TA_OK, ta.tree_attn_status_string(status)
    elif spec.dtype == "bf16":
        ta.tree_attn_decode(q, k, v, seqlens, Hq, Hkv, D, spec.scale, out, lse)
    else:
        ta.tree_attn_decode_f32(q, k, v, seqlens, Hq, Hkv, D, spec.scale, out, lse)
    torch.cuda.synchronize()
    return out.cpu().numpy(), lse.cpu().numpy()


def compare(out, lse, ref_out, ref_lse, pairs=None):
    """Assert the tolerance on the given (b, h) rows (all rows if None); return the worst errors."""
    if pairs is None:
        pairs = [(b, h) for b in range(ref_out.shape[0]) for h in range(ref_out.shape[1])]
    worst_rel, worst_lse = 0.0, 0.0
    for b, h in pairs:
        r, g = ref_out[b, h], out[b, h].astype(np.float64)
        if ref_lse[b, h] == -np.inf:
            assert np.all(g == 0.0) and lse[b, h] == -np.inf, f"empty row {(b, h)}: {g[:4]}, {lse[b, h]}"
            continue
        assert np.all(np.isfinite(g)), f"non-finite output at {(b, h)}"
        rel = float(np.max(np.abs(g - r)) / np.max(np.abs(r)))
        le = abs(float(lse[b, h]) - float(ref_lse[b, h]))
        worst_rel, worst_lse = max(worst_rel, rel), max(worst_lse, le)
        assert rel <= OUT_RTOL, f"out row {(b, h)}: inf-norm relative error {rel:.3g} > {OUT_RTOL}"
        assert le <= LSE_ATOL, f"lse {(b, h)}: |{lse[b, h]} - {ref_lse[b, h]}| = {le:.3g} > {LSE_ATOL}"
    return worst_rel, worst_lse


def oracle_parallel(fn, tasks, workers: int = 0):
    """Run fn(task) -> (out, lse) over disjoint row subsets in a thread pool and combine them.

    Each call computes only its rows and leaves NaN elsewhere; the combined arrays take every
    non-NaN entry.  numpy releases the GIL in the oracle's array operations (the widening of
    the cache, the products, exp), so the row groups run side by side on the host cores; BLAS
    is held to one thread per call meanwhile.  The oracle itself is unchanged.
    """
    import threadpoolctl

    workers = workers or max(1, min(8, len(tasks), os.cpu_count() or 1))
    with threadpoolctl.threadpool_limits(1), cf.ThreadPoolExecutor(workers) as ex:
        results = list(ex.map(fn, tasks))
    out, lse = (np.array(x, copy=True) for x in results[0])
    for o, l in results[1:]:
        mo, ml = ~np.isnan(o), ~np.isnan(l)
        out[mo] = o[mo]
        lse[ml] = l[ml]
    return out, lse
