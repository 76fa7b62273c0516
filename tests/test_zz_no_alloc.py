"""The no-allocation entry point, through the C ABI, against the CPU oracle.

tree_attn_decode_noalloc serves callers that may not allocate device memory while they
run (runtimes that own all of HBM through their own pools, latency-critical paths where an
allocation call can block): it uses a fixed scratch array inside the library instead of a
per-call workspace.  Its results must match the oracle within the parity tolerance, on
consecutive calls that reuse the same array, and agree bit for bit with tree_attn_decode_ex
(the same kernel and plan); a problem whose workspace is just under the array's 4 MiB must
work too.  tree_attn_noalloc_check reads the array's error word.  This file is collected
last so that a failure here does not hide the other GPU tests.
"""
import ctypes

import numpy as np
import pytest

import oracle
import synth
from gpu_util import compare, device_tensor, empty_outputs, new_workspace

pytestmark = pytest.mark.gpu

LIMIT = 4 << 20


def _run_noalloc(ta, d, sp):
    import torch

    seqlens = [int(s) for s in sp.seqlens]
    out, lse = empty_outputs(sp.batch, sp.n_q_heads, sp.head_dim)
    ta.tree_attn_decode_noalloc(d["q"], d["k"], d["v"], seqlens, sp.n_q_heads, sp.n_kv_heads, sp.head_dim, sp.scale,
                                out, lse)
    assert ta.tree_attn_noalloc_check() == ta.TA_OK
    torch.cuda.synchronize()
    return out.cpu().numpy(), lse.cpu().numpy()


def test_noalloc_matches_oracle_on_two_calls():
    import exact_long_context_split_b200 as ta

    sp = synth.DecodeSpec("noalloc", [5000, 77, 0, 2100, 40000], 32, 8, 128, seed=31, spike_frac=0.001)
    inp = synth.make_decode_inputs(sp)
    d = {n: device_tensor(inp[n], "bf16") for n in ("q", "k", "v")}
    ro, rl = oracle.decode_attention(inp["q"], inp["k"], inp["v"], sp.seqlens, 32, 8, 128, sp.scale)
    first = _run_noalloc(ta, d, sp)
    compare(*first, ro, rl)
    second = _run_noalloc(ta, d, sp)
    compare(*second, ro, rl)
    # the same kernel and plan as the workspace entry point: identical bits
    seqlens = [int(s) for s in sp.seqlens]
    out, lse = empty_outputs(sp.batch, 32, 128)
    ws = new_workspace(ta.tree_attn_workspace_size(seqlens, 32, 8, 128))
    ta.tree_attn_decode_ex("bf16", d["q"], d["k"], d["v"], seqlens, 32, 8, 128, sp.scale, out, lse, None, ws)
    assert ta.tree_attn_check(ws) == ta.TA_OK
    assert np.array_equal(out.cpu().numpy().view(np.uint32), second[0].view(np.uint32))
    assert np.array_equal(lse.cpu().numpy().view(np.uint32), second[1].view(np.uint32))


def test_noalloc_just_under_its_limit():
    """The largest batch of short sequences whose workspace still fits the 4 MiB array: its
    partial slots reach the end of the array."""
    import exact_long_context_split_b200 as ta

    Hq, Hkv, D = 8, 8, 128

    def lens(B):
        return [1 + (37 * b) % 300 for b in range(B)]

    B = 1
    while ta.tree_attn_workspace_size(lens(B + 1), Hq, Hkv, D) <= LIMIT:
        B += 1
    need = ta.tree_attn_workspace_size(lens(B), Hq, Hkv, D)
    assert LIMIT - 64 * 1024 < need <= LIMIT, need
    # inputs for B + 1 sequences; the first B are a prefix of every packed tensor
    big = synth.DecodeSpec("noalloc_limit", lens(B + 1), Hq, Hkv, D, seed=32)
    inp = synth.make_decode_inputs(big)
    d = {n: device_tensor(inp[n], "bf16") for n in ("q", "k", "v")}
    sp = synth.DecodeSpec("noalloc_limit", lens(B), Hq, Hkv, D, seed=32)
    ro, rl = oracle.decode_attention(inp["q"][:B], inp["k"], inp["v"], sp.seqlens, Hq, Hkv, D, sp.scale)
    for _ in range(2):
        compare(*_run_noalloc(ta, d, sp), ro, rl)
    # one more sequence no longer fits: rejected before anything is launched
    out, lse = empty_outputs(B + 1, Hq, D)
    with pytest.raises(ta.TreeAttnError) as e:
        ta.tree_attn_decode_noalloc(d["q"], d["k"], d["v"], lens(B + 1), Hq, Hkv, D, big.scale, out, lse)
    assert e.value.status == ta.TA_ERR_SCRATCH_LIMIT


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
