"""The no-allocation entry point, through the C ABI, against the allocating one.

tree_attn_decode_noalloc serves callers that may not allocate device memory while they
run (runtimes that own all of HBM through their own pools, latency-critical paths): it
uses a fixed scratch array inside the library instead of a per-call workspace.  Its
results must match tree_attn_decode_ex within the parity tolerance, on consecutive calls
that reuse the same array.  This file is collected last so that a failure here does not
hide the other GPU tests.
"""
import ctypes

import numpy as np
import pytest

import synth
from gpu_util import compare, device_tensor, empty_outputs, new_workspace

pytestmark = pytest.mark.gpu


def _inputs():
    sp = synth.DecodeSpec("noalloc", [5000, 77, 0, 2100, 40000], 32, 8, 128, seed=31, spike_frac=0.001)
    inp = synth.make_decode_inputs(sp)
    return sp, {n: device_tensor(inp[n], "bf16") for n in ("q", "k", "v")}


def test_noalloc_matches_workspace_entry_point_on_two_calls():
    import torch

    import exact_long_context_split_b200 as ta

    sp, d = _inputs()
    seqlens = [int(s) for s in sp.seqlens]
    B, Hq, Hkv, D = sp.batch, sp.n_q_heads, sp.n_kv_heads, sp.head_dim
    ref_out, ref_lse = empty_outputs(B, Hq, D)
    ws = new_workspace(ta.tree_attn_workspace_size(seqlens, Hq, Hkv, D))
    ta.tree_attn_decode_ex("bf16", d["q"], d["k"], d["v"], seqlens, Hq, Hkv, D, sp.scale, ref_out, ref_lse, None, ws)
    assert ta.tree_attn_check(ws) == ta.TA_OK
    ro = ref_out.cpu().numpy().astype(np.float64)
    rl = ref_lse.cpu().numpy().astype(np.float64)
    for _ in range(2):
        out, lse = empty_outputs(B, Hq, D)
        ta.tree_attn_decode_noalloc(d["q"], d["k"], d["v"], seqlens, Hq, Hkv, D, sp.scale, out, lse)
        torch.cuda.synchronize()
        compare(out.cpu().numpy(), lse.cpu().numpy(), ro, rl)


def test_noalloc_rejects_problems_beyond_its_scratch():
    """128 sequences x 64 KV heads need more than the fixed 4 MiB: rejected before any launch."""
    import torch

    import exact_long_context_split_b200 as ta

    dummy = torch.zeros(64, dtype=torch.float32, device="cuda")
    lens = (ctypes.c_int64 * 128)(*([1] * 128))
    p = dummy.data_ptr()
    status = ta.lib().tree_attn_decode_noalloc(p, p, p, lens, 128, 64, 64, 128, 0.1, p, p, None)
    assert status == ta.TA_ERR_SCRATCH_LIMIT
    assert "4 MiB" in ta.tree_attn_status_string(status)
