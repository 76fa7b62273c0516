"""GPU parity of multi-query decode (several query tokens per sequence, causal among
themselves) against the CPU oracle, through the C ABI."""
import numpy as np
import pytest

import oracle
import synth
from gpu_util import LSE_ATOL, OUT_RTOL, device_tensor, new_workspace

pytestmark = pytest.mark.gpu


def spec(seqlens, n, Hq, Hkv, D, dtype="bf16", seed=31):
    return synth.DecodeSpec("multi", list(seqlens), Hq, Hkv, D, dtype=dtype, seed=seed, n_queries=n)


def multi_gpu(inp, sp, opts=None, entry="ex"):
    import torch

    import exact_long_context_split_b200 as ta

    B, n, Hq, Hkv, D = sp.batch, sp.n_queries, sp.n_q_heads, sp.n_kv_heads, sp.head_dim
    q = device_tensor(inp["q"], sp.dtype)
    k = device_tensor(inp["k"], sp.dtype)
    v = device_tensor(inp["v"], sp.dtype)
    out = torch.full((B, n, Hq, D), float("nan"), device="cuda")
    lse = torch.full((B, n, Hq), float("nan"), device="cuda")
    lens = [int(s) for s in sp.seqlens]
    if entry == "ex":
        ws = new_workspace(ta.tree_attn_multi_workspace_size(lens, n, Hq, Hkv, D, sp.dtype, opts))
        ta.tree_attn_decode_multi_ex(sp.dtype, q, k, v, lens, n, Hq, Hkv, D, sp.scale, out, lse, opts, ws)
        assert ta.tree_attn_check(ws) == ta.TA_OK
    else:
        ta.tree_attn_decode_multi(q, k, v, lens, n, Hq, Hkv, D, sp.scale, out, lse)
    torch.cuda.synchronize()
    return out.cpu().numpy(), lse.cpu().numpy()


def check(out, lse, inp, sp, rows=None):
    ref_out, ref_lse = oracle.multi_query_attention(inp["q"], inp["k"], inp["v"], sp.seqlens, sp.n_queries,
                                                    sp.n_q_heads, sp.n_kv_heads, sp.head_dim, sp.scale,
                                                    dtype=sp.dtype, rows=rows)
    todo = rows if rows is not None else [(b, j, h) for b in range(sp.batch) for j in range(sp.n_queries)
                                          for h in range(sp.n_q_heads)]
    for (b, j, h) in todo:
        g, r = out[b, j, h].astype(np.float64), ref_out[b, j, h]
        rel = float(np.max(np.abs(g - r)) / np.max(np.abs(r)))
        assert rel <= OUT_RTOL, f"row {(b, j, h)}: inf-norm relative error {rel:.3g}"
        assert abs(float(lse[b, j, h]) - ref_lse[b, j, h]) <= LSE_ATOL, f"lse {(b, j, h)}"


# (seqlens, n, Hq, Hkv, D, dtype): single passes (G n <= 8), several passes (G n > 8, and n not a
# power of two), sequences exactly n long (query 0 sees one key) and tails shorter than n.
CASES = [
    ([37, 300, 1000], 2, 8, 2, 128, "bf16"),
    ([5, 129, 2049], 3, 4, 2, 64, "bf16"),
    ([4, 4, 70, 513], 4, 8, 2, 128, "bf16"),
    ([8, 100, 3000], 8, 2, 2, 64, "f32"),
    ([6, 1500], 5, 16, 2, 128, "bf16"),
    ([2, 65, 66, 67, 4099], 2, 32, 8, 128, "bf16"),
]


def tc_eligible(n, Hq, Hkv, D, dtype):
    return dtype == "bf16" and D == 128 and (Hq // Hkv) * n <= 128


# path: 0 automatic (tensor cores when bf16, D = 128 and 8 <= G n <= 128), 1 tensor-core form,
# 2 split-KV passes (with long or short tiles).
@pytest.mark.parametrize("path,tiles", [(0, 0), (1, 0), (2, 1), (2, 2)])
@pytest.mark.parametrize("case", CASES, ids=[f"n{c[1]}_G{c[2] // c[3]}_D{c[4]}_{c[5]}" for c in CASES])
def test_multi_query_against_oracle(case, path, tiles):
    import exact_long_context_split_b200 as ta

    seqlens, n, Hq, Hkv, D, dtype = case
    sp = spec(seqlens, n, Hq, Hkv, D, dtype=dtype, seed=40 + n + D)
    inp = synth.make_decode_inputs(sp)
    opts = ta.make_options(split_tiles=tiles, prefix_path=path)
    if path == 1 and not tc_eligible(n, Hq, Hkv, D, dtype):
        with pytest.raises(ta.TreeAttnError) as e:
            multi_gpu(inp, sp, opts)
        assert e.value.status == ta.TA_ERR_UNSUPPORTED
        return
    out, lse = multi_gpu(inp, sp, opts)
    check(out, lse, inp, sp)


# Tensor-core form: shorter than one 128-key tile, on and next to tile boundaries, G n = 128
# rows, and more than 128 sequences (two launch groups with their own chunk counts).
TC_CASES = [
    ([5, 128, 129, 256, 257], 4, 16, 4, 1),
    ([3000, 16], 16, 64, 8, 3),
    ([70] * 130 + [5000], 2, 8, 2, 5),
    ([1000, 40000], 3, 32, 8, 7),
]


@pytest.mark.parametrize("case", TC_CASES, ids=["tile_edges", "rows128", "two_groups", "long"])
def test_tensor_core_multi_query(case):
    import exact_long_context_split_b200 as ta

    seqlens, n, Hq, Hkv, seed = case
    sp = spec(seqlens, n, Hq, Hkv, 128, seed=seed)
    inp = synth.make_decode_inputs(sp)
    opts = ta.make_options(prefix_path=1)
    out, lse = multi_gpu(inp, sp, opts)
    r = np.random.default_rng(seed)
    rows = None
    if sp.batch * n * Hq > 400:
        rows = sorted({(int(r.integers(sp.batch)), int(r.integers(n)), int(r.integers(Hq))) for _ in range(150)} |
                      {(sp.batch - 1, j, h) for j in range(n) for h in (0, Hq - 1)})
    check(out, lse, inp, sp, rows=rows)
    out2, lse2 = multi_gpu(inp, sp, opts)
    assert np.array_equal(out.view(np.uint32), out2.view(np.uint32)), "not bit-identical across runs"
    assert np.array_equal(lse.view(np.uint32), lse2.view(np.uint32))


@pytest.mark.parametrize("num_ctas", [1, 3, 148, 100000])
def test_masked_tail_alone_in_a_cta(num_ctas):
    """Split-KV passes with one tile per CTA: the CTA holding a sequence's last tile (2 tokens)
    sees no key for the query tokens that precede them, and sends an empty partial."""
    import exact_long_context_split_b200 as ta

    sp = spec([130, 66], 4, 8, 2, 128, seed=77)
    inp = synth.make_decode_inputs(sp)
    opts = ta.make_options(num_ctas=num_ctas, split_tiles=2, prefix_path=2)
    out, lse = multi_gpu(inp, sp, opts)
    check(out, lse, inp, sp)
    out2, lse2 = multi_gpu(inp, sp, opts)
    assert np.array_equal(out.view(np.uint32), out2.view(np.uint32)), "not bit-identical across runs"


def test_one_query_equals_decode():
    """n = 1 runs the decode kernels with the same plan: bit-identical to tree_attn_decode_ex."""
    from gpu_util import decode_gpu

    import exact_long_context_split_b200 as ta

    sp1 = spec([17, 2000, 40000], 1, 32, 8, 128, seed=5)
    inp = synth.make_decode_inputs(sp1)
    out, lse = multi_gpu(inp, sp1, ta.make_options(prefix_path=2))
    sp = synth.DecodeSpec("plain", [17, 2000, 40000], 32, 8, 128, seed=5)
    ref_out, ref_lse = decode_gpu(synth.make_decode_inputs(sp), sp)
    assert np.array_equal(out[:, 0].view(np.uint32), ref_out.view(np.uint32))
    assert np.array_equal(lse[:, 0].view(np.uint32), ref_lse.view(np.uint32))


def test_allocating_entry_point():
    sp = spec([300, 5], 3, 8, 2, 128, seed=9)
    inp = synth.make_decode_inputs(sp)
    out, lse = multi_gpu(inp, sp, entry="alloc")
    check(out, lse, inp, sp)


@pytest.mark.parametrize("name", ["spec_decode_2", "spec_decode_4"])
def test_spec_decode_workload_sampled(name):
    """The bench workloads (8 x 32K tokens, 32/8 heads): every row of every query token."""
    sp = synth.multi_query_configs()[name]
    inp = synth.make_decode_inputs(sp)
    out, lse = multi_gpu(inp, sp)
    assert np.all(np.isfinite(out)) and np.all(np.isfinite(lse))
    check(out, lse, inp, sp)


def test_invalid_arguments():
    import torch

    import exact_long_context_split_b200 as ta

    q = torch.zeros(2 * 3 * 8 * 128, dtype=torch.bfloat16, device="cuda")
    kv = torch.zeros(8 * 2 * 128 * 10, dtype=torch.bfloat16, device="cuda")
    out = torch.empty(2 * 3 * 8 * 128, device="cuda")
    lse = torch.empty(2 * 3 * 8, device="cuda")
    for lens, n in (([2, 5], 3), ([5, 5], 0)):
        with pytest.raises(ta.TreeAttnError) as e:
            ta.tree_attn_decode_multi(q, kv, kv, lens, n, 8, 2, 128, 0.1, out, lse)
        assert e.value.status == ta.TA_ERR_INVALID_ARG
