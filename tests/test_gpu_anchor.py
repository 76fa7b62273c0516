"""GPU parity of context encoding with anchor blocks (Star Attention article, "Two-phase
inference under Star Attention", "Phase 1: context encoding") against the CPU oracle, through
the C ABI; and the tensor-core kernel's bounded waits running out on purpose (a K tile that is
never loaded), in this form and in the several-query-tokens form."""
import numpy as np
import pytest

import oracle
import synth
from gpu_util import compare, device_tensor, new_workspace

pytestmark = pytest.mark.gpu


def anchor_gpu(inp, sp, opts=None, ws=None):
    import torch

    import exact_long_context_split_b200 as ta

    S, Hq, Hkv, D = sp.seq_len, sp.n_q_heads, sp.n_kv_heads, sp.head_dim
    q = device_tensor(inp["q"], "bf16")
    k = device_tensor(inp["k"], "bf16")
    v = device_tensor(inp["v"], "bf16")
    out = torch.full((S, Hq, D), float("nan"), device="cuda")
    lse = torch.full((S, Hq), float("nan"), device="cuda")
    ws = new_workspace(256) if ws is None else ws
    ta.tree_attn_anchor_prefill(q, k, v, S, sp.block_size, Hq, Hkv, D, sp.scale, out, lse, opts, ws)
    status = ta.tree_attn_check(ws)
    torch.cuda.synchronize()
    return out.cpu().numpy(), lse.cpu().numpy(), status


def oracle_anchor(inp, sp, rows=None):
    return oracle.anchor_block_attention(inp["q"], inp["k"], inp["v"], sp.seq_len, sp.block_size, sp.n_q_heads,
                                         sp.n_kv_heads, sp.head_dim, sp.scale, rows=rows)


# (seq_len, block_size, Hq, Hkv): every G (16 to 128 positions per query tile), a partial last
# query tile and block, an anchor of one key tile, a block longer than the context (plain causal
# attention), many short blocks, a single token.
CASES = [
    (1000, 256, 8, 2),
    (777, 128, 32, 8),
    (600, 384, 8, 8),
    (300, 1024, 16, 2),
    (2050, 128, 4, 2),
    (1, 128, 8, 2),
    (4096, 1024, 32, 8),
]


@pytest.mark.parametrize("S,B,Hq,Hkv", CASES)
def test_anchor_prefill_against_oracle(S, B, Hq, Hkv):
    import exact_long_context_split_b200 as ta

    sp = synth.AnchorSpec("case", S, B, Hq, Hkv, 128, seed=41)
    inp = synth.make_anchor_inputs(sp)
    out, lse, status = anchor_gpu(inp, sp)
    assert status == ta.TA_OK
    ref_out, ref_lse = oracle_anchor(inp, sp)
    compare(out, lse, ref_out, ref_lse)


def test_anchor_prefill_bit_identical_across_runs():
    sp = synth.AnchorSpec("case", 3000, 512, 32, 8, 128, seed=42)
    inp = synth.make_anchor_inputs(sp)
    a = anchor_gpu(inp, sp)
    b = anchor_gpu(inp, sp)
    assert np.array_equal(a[0].view(np.uint32), b[0].view(np.uint32))
    assert np.array_equal(a[1].view(np.uint32), b[1].view(np.uint32))


def test_anchor_prefill_workload_sampled():
    """The 32K-token workload (8K blocks, 32/8 heads): every query head of positions at block
    and query-tile edges and spread inside each block."""
    from gpu_util import oracle_parallel

    sp = synth.anchor_configs()["star_prefill_32k"]
    inp = synth.make_anchor_inputs(sp)
    out, lse, status = anchor_gpu(inp, sp)
    assert status == 0
    assert np.all(np.isfinite(out)) and np.all(np.isfinite(lse))
    B, S = sp.block_size, sp.seq_len
    positions = sorted({p for i0 in range(0, S, B) for p in (i0, i0 + 1, i0 + 31, i0 + 32, i0 + B // 2 + 7,
                                                              i0 + B - 33, i0 + B - 1) if p < S})
    tasks = [[(p, h) for h in range(sp.n_q_heads)] for p in positions]
    ref_out, ref_lse = oracle_parallel(lambda rows: oracle_anchor(inp, sp, rows=rows), tasks)
    pairs = [r for t in tasks for r in t]
    compare(out, lse, ref_out, ref_lse, pairs=pairs)


def test_anchor_prefill_arguments():
    import torch

    import exact_long_context_split_b200 as ta

    z = torch.zeros(1 << 16, dtype=torch.bfloat16, device="cuda")
    o = torch.zeros(1 << 16, dtype=torch.float32, device="cuda")
    ws = new_workspace(256)
    for (S, B, Hq, Hkv, D), status in [((100, 100, 8, 2, 128), ta.TA_ERR_UNSUPPORTED),  # block not a tile multiple
                                       ((100, 128, 8, 2, 64), ta.TA_ERR_UNSUPPORTED),
                                       ((100, 128, 32, 2, 128), ta.TA_ERR_UNSUPPORTED),  # G = 16
                                       ((100, 128, 6, 4, 128), ta.TA_ERR_INVALID_ARG),
                                       ((-1, 128, 8, 2, 128), ta.TA_ERR_INVALID_ARG),
                                       ((100, 0, 8, 2, 128), ta.TA_ERR_INVALID_ARG)]:
        with pytest.raises(ta.TreeAttnError) as e:
            ta.tree_attn_anchor_prefill(z, z, z, S, B, Hq, Hkv, D, 0.1, o, o, None, ws)
        assert e.value.status == status, (S, B, Hq, Hkv, D)
    with pytest.raises(ta.TreeAttnError) as e:
        ta.tree_attn_anchor_prefill(z, z, z, 100, 128, 8, 2, 128, 0.1, o, o, None, ws, 128)
    assert e.value.status == ta.TA_ERR_WORKSPACE
    ta.tree_attn_anchor_prefill(z, z, z, 0, 128, 8, 2, 128, 0.1, o, o, None, ws)  # nothing to do


def test_tensor_core_bounded_wait_runs_out_and_context_survives():
    """A K tile that CTA (0, 0, 0) never loads (test hook): the MMA thread's wait runs out after
    20 ms, the CTA aborts, drains its copies and products and frees its tensor memory; the call
    reports TA_ERR_TIMEOUT with that CTA's rows NaN and the others exact, and the next call works."""
    import exact_long_context_split_b200 as ta

    sp = synth.AnchorSpec("case", 1000, 256, 8, 2, 128, seed=43)
    inp = synth.make_anchor_inputs(sp)
    G, n_pos = 4, 32
    ws = new_workspace(256)
    opts = ta.make_options(wait_limit_us=20000, debug_skip_tile=1)
    out, lse, status = anchor_gpu(inp, sp, opts, ws)
    assert status == ta.TA_ERR_TIMEOUT
    # CTA (0, 0, 0) holds the last query tile (launched first) of KV head 0
    last0 = (sp.seq_len - 1) // n_pos * n_pos
    assert np.isnan(out[last0:, :G]).all() and np.isnan(lse[last0:, :G]).all()
    ref_out, ref_lse = oracle_anchor(inp, sp)
    pairs = [(p, h) for p in range(last0) for h in range(sp.n_q_heads)] + \
            [(p, h) for p in range(last0, sp.seq_len) for h in range(G, sp.n_q_heads)]
    compare(out, lse, ref_out, ref_lse, pairs=pairs)
    ta.tree_attn_workspace_init(ws)
    out, lse, status = anchor_gpu(inp, sp, None, ws)
    assert status == ta.TA_OK
    compare(out, lse, ref_out, ref_lse)


def test_tensor_core_multi_query_bounded_wait_runs_out():
    """The same hook in the several-query-tokens form: TA_ERR_TIMEOUT, NaN outputs, then a
    correct call on the re-initialised workspace."""
    import torch

    import exact_long_context_split_b200 as ta

    sp = synth.DecodeSpec("multi", [3000, 700], 32, 8, 128, seed=44, n_queries=4)
    inp = synth.make_decode_inputs(sp)
    q, k, v = (device_tensor(inp[n], "bf16") for n in ("q", "k", "v"))
    out = torch.empty(2, 4, 32, 128, device="cuda")
    lse = torch.empty(2, 4, 32, device="cuda")
    lens = [3000, 700]
    for opts, expect in ((ta.make_options(wait_limit_us=20000, debug_skip_tile=1, prefix_path=1), ta.TA_ERR_TIMEOUT),
                         (ta.make_options(prefix_path=1), ta.TA_OK)):
        ws = new_workspace(ta.tree_attn_multi_workspace_size(lens, 4, 32, 8, 128, "bf16", opts))
        ta.tree_attn_decode_multi_ex("bf16", q, k, v, lens, 4, 32, 8, 128, sp.scale, out, lse, opts, ws)
        assert ta.tree_attn_check(ws) == expect
        if expect == ta.TA_ERR_TIMEOUT:
            assert torch.isnan(out).all()
    ref_out, ref_lse = oracle.multi_query_attention(inp["q"], inp["k"], inp["v"], lens, 4, 32, 8, 128, sp.scale)
    compare(out.cpu().numpy().reshape(8, 32, 128), lse.cpu().numpy().reshape(8, 32),
            ref_out.reshape(8, 32, 128), ref_lse.reshape(8, 32))


def test_shared_prefix_bounded_wait_runs_out():
    """The hook in the shared-prefix tensor-core pass (two M tiles per CTA): CTA (0, 0, 0) never
    loads K tile 0, its waits run out, the suffix pass sees the error word and writes NaN for
    every row; after re-initialising the workspace the same call is exact."""
    import torch

    import exact_long_context_split_b200 as ta

    sp = synth.BifurcatedSpec("case", 3000, [5, 0, 300, 40], 32, 8, 128, seed=45)
    inp = synth.make_bifurcated_inputs(sp)
    q, kp, vp, ks, vs = (device_tensor(inp[n], "bf16") for n in ("q", "k_prefix", "v_prefix", "k_suffix", "v_suffix"))
    lens = [int(s) for s in sp.suffix_lens]
    out = torch.empty(4, 32, 128, device="cuda")
    lse = torch.empty(4, 32, device="cuda")
    for opts, expect in ((ta.make_options(wait_limit_us=20000, debug_skip_tile=0, prefix_path=1, split_tiles=3),
                          ta.TA_ERR_TIMEOUT),
                         (ta.make_options(prefix_path=1, split_tiles=3), ta.TA_OK)):
        ws = new_workspace(ta.tree_attn_bifurcated_workspace_size(3000, lens, 32, 8, 128, opts))
        ta.tree_attn_decode_bifurcated_ex(q, kp, vp, 3000, ks, vs, lens, 32, 8, 128, sp.scale, out, lse, opts, ws)
        assert ta.tree_attn_check(ws) == expect
        if expect == ta.TA_ERR_TIMEOUT:
            assert torch.isnan(out).all() and torch.isnan(lse).all()
    ref = oracle.bifurcated_attention(inp["q"], inp["k_prefix"], inp["v_prefix"], 3000, inp["k_suffix"],
                                      inp["v_suffix"], lens, 32, 8, 128, sp.scale)
    compare(out.cpu().numpy(), lse.cpu().numpy(), *ref)


@pytest.mark.parametrize("call", ["decode", "g8_decode", "bifurcated", "anchor"])
def test_profile_events_bracket_the_main_kernel(call):
    """tree_attn_profile_events: the library records the events on the call's stream around its
    main kernel; the span lies inside the whole call's span, and turning the hook off stops the
    recording."""
    import torch

    import exact_long_context_split_b200 as ta

    outer = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
    inner = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
    for e in inner:
        e.record()  # torch creates the CUDA event on its first record
    torch.cuda.synchronize()
    if call in ("decode", "g8_decode"):
        Hq = 32 if call == "decode" else 64
        sp = synth.DecodeSpec("p", [20000, 3000], Hq, 8, 128, seed=46)
        inp = synth.make_decode_inputs(sp)
        q, k, v = (device_tensor(inp[n], "bf16") for n in ("q", "k", "v"))
        out, lse = torch.empty(2, Hq, 128, device="cuda"), torch.empty(2, Hq, device="cuda")
        ws = new_workspace(ta.tree_attn_workspace_size([20000, 3000], Hq, 8, 128))
        run = lambda: ta.tree_attn_decode_ex("bf16", q, k, v, [20000, 3000], Hq, 8, 128, sp.scale, out, lse,  # noqa: E731
                                             None, ws)
    elif call == "bifurcated":
        sp = synth.BifurcatedSpec("p", 5000, [100] * 40, 32, 8, 128, seed=47)
        inp = synth.make_bifurcated_inputs(sp)
        d = {n: device_tensor(inp[n], "bf16") for n in ("q", "k_prefix", "v_prefix", "k_suffix", "v_suffix")}
        out, lse = torch.empty(40, 32, 128, device="cuda"), torch.empty(40, 32, device="cuda")
        ws = new_workspace(ta.tree_attn_bifurcated_workspace_size(5000, [100] * 40, 32, 8, 128))
        run = lambda: ta.tree_attn_decode_bifurcated_ex(d["q"], d["k_prefix"], d["v_prefix"], 5000,  # noqa: E731
                                                        d["k_suffix"], d["v_suffix"], [100] * 40, 32, 8, 128,
                                                        sp.scale, out, lse, None, ws)
    else:
        sp = synth.AnchorSpec("p", 4096, 1024, 32, 8, 128, seed=48)
        inp = synth.make_anchor_inputs(sp)
        q, k, v = (device_tensor(inp[n], "bf16") for n in ("q", "k", "v"))
        out, lse = torch.empty(4096, 32, 128, device="cuda"), torch.empty(4096, 32, device="cuda")
        ws = new_workspace(256)
        run = lambda: ta.tree_attn_anchor_prefill(q, k, v, 4096, 1024, 32, 8, 128, sp.scale, out, lse,  # noqa: E731
                                                  None, ws)
    run()  # warm (first-call set-up outside the spans)
    ta.tree_attn_profile_events(inner[0], inner[1])
    outer[0].record()
    run()
    outer[1].record()
    ta.tree_attn_profile_events()
    torch.cuda.synchronize()
    assert ta.tree_attn_check(ws) == ta.TA_OK
    whole = outer[0].elapsed_time(outer[1])
    kernel = inner[0].elapsed_time(inner[1])
    assert 0.0 < kernel <= whole
    assert outer[0].elapsed_time(inner[0]) >= 0.0 and inner[1].elapsed_time(outer[1]) >= 0.0
    # hook off: the next call leaves the events where they were
    stamp = inner[1].elapsed_time(outer[1])
    run()
    torch.cuda.synchronize()
    assert inner[1].elapsed_time(outer[1]) == stamp
