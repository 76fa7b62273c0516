"""GPU parity of split decode attention against the CPU oracle, through the C ABI.

Every case, the full-size workloads included, is compared on every output row.
"""
import numpy as np
import pytest

import oracle
import synth
from gpu_util import compare, decode_gpu, empty_outputs, new_workspace

pytestmark = pytest.mark.gpu


def spec(seqlens, Hq, Hkv, D, dtype="bf16", seed=11, spike_frac=0.0):
    return synth.DecodeSpec("case", list(seqlens), Hq, Hkv, D, dtype=dtype, seed=seed, spike_frac=spike_frac)


def oracle_of(inp, sp, pairs=None):
    return oracle.decode_attention(inp["q"], inp["k"], inp["v"], sp.seqlens, sp.n_q_heads, sp.n_kv_heads,
                                   sp.head_dim, sp.scale, dtype=sp.dtype, pairs=pairs)


# Every kernel instance (dtype x D x G) on a ragged batch with lengths around the tile sizes
# (bf16 D=128: 64 tokens, bf16 D=64: 128, f32 D=64: 64, f32 D=128: 32), an empty sequence,
# a one-token sequence and a multi-tile one.
RAGGED = [1, 0, 31, 33, 64, 65, 127, 129, 1000, 3001]


@pytest.mark.parametrize("tiles", [1, 2])  # long and short tile configurations
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("G", [1, 2, 4, 8])
def test_every_instance_ragged(dtype, D, G, tiles):
    import exact_long_context_split_b200 as ta

    Hkv = 2
    sp = spec(RAGGED, G * Hkv, Hkv, D, dtype=dtype, seed=100 + G + D)
    inp = synth.make_decode_inputs(sp)
    out, lse = decode_gpu(inp, sp, ta.make_options(split_tiles=tiles, prefix_path=ta.PREFIX_SPLIT_KV))
    ref_out, ref_lse = oracle_of(inp, sp)
    compare(out, lse, ref_out, ref_lse)


@pytest.mark.parametrize("Hq,Hkv", [(16, 2), (64, 8), (8, 1)])
def test_g8_decode_on_tensor_cores(Hq, Hkv):
    """G = 8 bf16 decode (head_dim 128) runs on the tensor cores by default: ragged lengths with
    an empty and a one-token sequence against the oracle, bit-identical across runs, and within
    the tolerance of the split kernel (prefix_path 2)."""
    import exact_long_context_split_b200 as ta

    sp = spec([1, 0, 129, 1000, 20000], Hq, Hkv, 128, seed=14, spike_frac=0.001)
    inp = synth.make_decode_inputs(sp)
    out, lse = decode_gpu(inp, sp)
    ref_out, ref_lse = oracle_of(inp, sp)
    compare(out, lse, ref_out, ref_lse)
    out2, lse2 = decode_gpu(inp, sp)
    assert np.array_equal(out.view(np.uint32), out2.view(np.uint32))
    assert np.array_equal(lse.view(np.uint32), lse2.view(np.uint32))
    s_out, s_lse = decode_gpu(inp, sp, ta.make_options(prefix_path=ta.PREFIX_SPLIT_KV))
    compare(s_out, s_lse, ref_out, ref_lse)
    a_out, a_lse = decode_gpu(inp, sp, entry="alloc")
    assert np.array_equal(out.view(np.uint32), a_out.view(np.uint32))


def test_tensor_core_decode_forced_for_g4():
    """prefix_path 1 sends G = 4 bf16 decode to the tensor cores as well."""
    import exact_long_context_split_b200 as ta

    sp = spec([3000, 5, 0], 32, 8, 128, seed=15)
    inp = synth.make_decode_inputs(sp)
    out, lse = decode_gpu(inp, sp, ta.make_options(prefix_path=ta.PREFIX_TENSOR_CORE))
    compare(out, lse, *oracle_of(inp, sp))


@pytest.mark.parametrize("tiles", [1, 2])
@pytest.mark.parametrize("num_ctas", [1, 2, 7, 37, 148, 1000, 100000])
def test_grid_sizes_and_merge_trees(num_ctas, tiles):
    """From one CTA doing every tile (no merge) to one tile per CTA (deep merge trees)."""
    sp = spec([5000, 77, 0, 2100], 16, 4, 128, seed=5)
    inp = synth.make_decode_inputs(sp)
    import exact_long_context_split_b200 as ta

    opts = ta.make_options(num_ctas=num_ctas, split_tiles=tiles)
    out, lse = decode_gpu(inp, sp, opts)
    ref_out, ref_lse = oracle_of(inp, sp)
    compare(out, lse, ref_out, ref_lse)
    out2, lse2 = decode_gpu(inp, sp, opts)
    assert np.array_equal(out.view(np.uint32), out2.view(np.uint32)), "not bit-identical across runs"
    assert np.array_equal(lse.view(np.uint32), lse2.view(np.uint32))


def test_bit_identical_across_runs_and_entry_points():
    sp = spec([40000, 12345], 32, 8, 128, seed=6)
    inp = synth.make_decode_inputs(sp)
    a = decode_gpu(inp, sp)
    b = decode_gpu(inp, sp)
    c = decode_gpu(inp, sp, entry="alloc")
    for x, y in [(a, b), (a, c)]:
        assert np.array_equal(x[0].view(np.uint32), y[0].view(np.uint32))
        assert np.array_equal(x[1].view(np.uint32), y[1].view(np.uint32))
    compare(a[0], a[1], *oracle_of(inp, sp))


def test_f32_alloc_entry_point():
    sp = spec([4096, 100], 4, 4, 64, dtype="f32", seed=7)
    inp = synth.make_decode_inputs(sp)
    out, lse = decode_gpu(inp, sp, entry="alloc")
    compare(out, lse, *oracle_of(inp, sp))


@pytest.mark.parametrize("seqlens", [[0], [1], [0, 0, 0], [0, 5, 0], [64], [65], [1, 1, 1, 1]])
def test_edge_lengths(seqlens):
    sp = spec(seqlens, 8, 2, 128, seed=8)
    inp = synth.make_decode_inputs(sp)
    out, lse = decode_gpu(inp, sp)
    compare(out, lse, *oracle_of(inp, sp))


def test_many_sequences_span_several_launches():
    """More than 128 sequences: the batch is planned as several launches."""
    rng = np.random.default_rng(3)
    seqlens = [int(x) for x in rng.integers(0, 700, size=300)]
    sp = spec(seqlens, 8, 8, 64, seed=9)
    inp = synth.make_decode_inputs(sp)
    out, lse = decode_gpu(inp, sp)
    compare(out, lse, *oracle_of(inp, sp))


@pytest.mark.parametrize("scale", [0.0, -0.3, 2.0])
def test_scales(scale):
    import dataclasses

    sp = dataclasses.replace(spec([3000, 10], 8, 2, 128, seed=10), scale_value=scale)
    inp = synth.make_decode_inputs(sp)
    out, lse = decode_gpu(inp, sp)
    compare(out, lse, *oracle_of(inp, sp))


def test_spiky_keys():
    """Keys scaled by 4 on 1% of rows: large score gaps exercise the rescaling path."""
    sp = spec([20000, 3000], 32, 8, 128, seed=12, spike_frac=0.01)
    inp = synth.make_decode_inputs(sp)
    out, lse = decode_gpu(inp, sp)
    compare(out, lse, *oracle_of(inp, sp))


def test_bounded_wait_reports_timeout_and_context_survives():
    """A tile that is never loaded (test hook) makes CTA 0's consumers' wait run out: the call
    records TA_ERR_TIMEOUT, the affected rows are NaN, and the next call works."""
    import torch

    import exact_long_context_split_b200 as ta

    sp = spec([20000], 8, 2, 128, seed=13)
    inp = synth.make_decode_inputs(sp)
    seqlens = list(sp.seqlens)
    opts = ta.make_options(wait_limit_us=20000, debug_skip_tile=0)
    ws = new_workspace(ta.tree_attn_workspace_size(seqlens, 8, 2, 128, "bf16", opts))
    from gpu_util import device_tensor

    q, k, v = (device_tensor(inp[n], "bf16") for n in ("q", "k", "v"))
    out, lse = empty_outputs(1, 8, 128)
    ta.tree_attn_decode_ex("bf16", q, k, v, seqlens, 8, 2, 128, sp.scale, out, lse, opts, ws)
    assert ta.tree_attn_check(ws) == ta.TA_ERR_TIMEOUT
    assert torch.isnan(out[0, 0]).all()
    ta.tree_attn_workspace_init(ws)
    ta.tree_attn_decode_ex("bf16", q, k, v, seqlens, 8, 2, 128, sp.scale, out, lse, None, ws)
    assert ta.tree_attn_check(ws) == ta.TA_OK
    compare(out.cpu().numpy(), lse.cpu().numpy(), *oracle_of(inp, sp))


# ----------------------------------------------------------------------------------------------
# The workloads at full size
# ----------------------------------------------------------------------------------------------


def test_config_tiny_full():
    sp = synth.decode_configs()["tiny"]
    inp = synth.make_decode_inputs(sp)
    out, lse = decode_gpu(inp, sp)
    compare(out, lse, *oracle_of(inp, sp))


def test_config_llama3_8b_gqa_full():
    sp = synth.decode_configs()["llama3_8b_gqa"]
    inp = synth.make_decode_inputs(sp)
    out, lse = decode_gpu(inp, sp)
    compare(out, lse, *oracle_of(inp, sp))


def _full_size(name, workers=0):
    """A full-size workload: every (sequence, query head) row against the oracle, the row groups
    of one (sequence, KV head) computed side by side on the host cores."""
    from gpu_util import oracle_parallel

    sp = {**synth.decode_configs(), **synth.gqa8_configs()}[name]
    inp = synth.make_decode_inputs(sp)
    out, lse = decode_gpu(inp, sp)
    assert np.all(np.isfinite(out)) and np.all(np.isfinite(lse))
    G = sp.n_q_heads // sp.n_kv_heads
    tasks = [[(b, g * G + i) for i in range(G)] for b in range(sp.batch) for g in range(sp.n_kv_heads)]
    ref_out, ref_lse = oracle_parallel(lambda pairs: oracle_of(inp, sp, pairs=pairs), tasks, workers)
    return compare(out, lse, ref_out, ref_lse)


def test_config_long_1m_all_rows():
    _full_size("long_1m")


def test_config_extreme_5m_all_rows():
    _full_size("extreme_5m", workers=4)


def test_config_extreme_ragged_all_rows():
    _full_size("extreme_ragged", workers=4)


def test_config_long_1m_g8_all_rows():
    """64 query heads over 8 KV heads at 1M tokens: the tensor-core decode path."""
    _full_size("long_1m_g8")
