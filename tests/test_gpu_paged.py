"""GPU parity of decode over a paged KV cache (block table) against the CPU oracle, through
the C ABI.  Unused page rows hold NaN, so any read through a wrong entry shows up."""
import numpy as np
import pytest

import oracle
import synth
from gpu_util import compare, decode_gpu, device_tensor, new_workspace

pytestmark = pytest.mark.gpu

NAN = {"bf16": np.uint16(0x7FC0), "f32": np.float32("nan")}


def paged_case(seqlens, Hq, Hkv, D, dtype, ps, seed, spare=3):
    sp = synth.DecodeSpec("paged", list(seqlens), Hq, Hkv, D, dtype=dtype, seed=seed)
    inp = synth.make_decode_inputs(sp)
    table, n_pages = synth.page_table(seed, seqlens, ps, spare=spare)
    kp = synth.scatter_pages(inp["k"], seqlens, Hkv, D, ps, table, n_pages, NAN[dtype])
    vp = synth.scatter_pages(inp["v"], seqlens, Hkv, D, ps, table, n_pages, NAN[dtype])
    return sp, inp, table, n_pages, kp, vp


def paged_gpu(sp, inp, table, n_pages, kp, vp, ps, opts=None, entry="ex", expect=None):
    import torch

    import exact_long_context_split_b200 as ta

    B, Hq, Hkv, D = sp.batch, sp.n_q_heads, sp.n_kv_heads, sp.head_dim
    q = device_tensor(inp["q"], sp.dtype)
    k = device_tensor(kp.reshape(-1), sp.dtype)
    v = device_tensor(vp.reshape(-1), sp.dtype)
    bt = torch.from_numpy(np.ascontiguousarray(table)).cuda()
    out = torch.full((B, Hq, D), float("nan"), device="cuda")
    lse = torch.full((B, Hq), float("nan"), device="cuda")
    lens = [int(s) for s in sp.seqlens]
    if entry == "ex":
        ws = new_workspace(ta.tree_attn_workspace_size(lens, Hq, Hkv, D, sp.dtype, opts))
        ta.tree_attn_decode_paged_ex(sp.dtype, q, k, v, n_pages, ps, bt, table.shape[1], lens, Hq, Hkv, D, sp.scale,
                                     out, lse, opts, ws)
        status = ta.tree_attn_check(ws)
        assert status == (ta.TA_OK if expect is None else expect), ta.tree_attn_status_string(status)
    else:
        ta.tree_attn_decode_paged(q, k, v, n_pages, ps, bt, table.shape[1], lens, Hq, Hkv, D, sp.scale, out, lse)
    torch.cuda.synchronize()
    return out.cpu().numpy(), lse.cpu().numpy()


def oracle_paged(sp, inp, table, kp, vp, ps, pairs=None):
    return oracle.paged_decode_attention(inp["q"], kp.reshape(-1), vp.reshape(-1), table, sp.seqlens, ps,
                                         sp.n_q_heads, sp.n_kv_heads, sp.head_dim, sp.scale, dtype=sp.dtype,
                                         pairs=pairs)


CASES = [
    ([1, 0, 17, 33, 64, 200, 1000, 3001], 8, 2, 128, "bf16", 16),
    ([5, 129, 2049], 4, 4, 64, "bf16", 32),
    ([300, 20000], 32, 4, 128, "bf16", 256),
    ([100, 4097], 8, 2, 64, "f32", 64),
    ([1024, 5, 1500], 16, 4, 128, "bf16", 1024),
]


@pytest.mark.parametrize("tiles", [1, 2])
@pytest.mark.parametrize("case", CASES, ids=[f"ps{c[5]}_G{c[1] // c[2]}_D{c[3]}_{c[4]}" for c in CASES])
def test_paged_against_oracle(case, tiles):
    import exact_long_context_split_b200 as ta

    seqlens, Hq, Hkv, D, dtype, ps = case
    sp, inp, table, n_pages, kp, vp = paged_case(seqlens, Hq, Hkv, D, dtype, ps, seed=50 + ps + D)
    out, lse = paged_gpu(sp, inp, table, n_pages, kp, vp, ps, ta.make_options(split_tiles=tiles))
    ref_out, ref_lse = oracle_paged(sp, inp, table, kp, vp, ps)
    compare(out, lse, ref_out, ref_lse)


@pytest.mark.parametrize("num_ctas", [1, 7, 148, 100000])
def test_paged_bit_identical_to_contiguous(num_ctas):
    """The paged layout changes where tiles come from, not what is computed."""
    import exact_long_context_split_b200 as ta

    seqlens = [5000, 77, 0, 2100]
    sp, inp, table, n_pages, kp, vp = paged_case(seqlens, 16, 4, 128, "bf16", 16, seed=5)
    opts = ta.make_options(num_ctas=num_ctas)
    out, lse = paged_gpu(sp, inp, table, n_pages, kp, vp, 16, opts)
    ref_out, ref_lse = decode_gpu(inp, sp, opts)
    assert np.array_equal(out.view(np.uint32), ref_out.view(np.uint32))
    assert np.array_equal(lse.view(np.uint32), ref_lse.view(np.uint32))


def test_shared_prefix_blocks():
    """Two sequences whose tables share their first blocks (a common prompt prefix)."""
    seqlens = [160, 100]
    sp, inp, table, n_pages, kp, vp = paged_case(seqlens, 8, 2, 128, "bf16", 32, seed=8)
    table = table.copy()
    table[1, :3] = table[0, :3]  # sequence 1 reads sequence 0's first 96 tokens
    out, lse = paged_gpu(sp, inp, table, n_pages, kp, vp, 32)
    ref_out, ref_lse = oracle_paged(sp, inp, table, kp, vp, 32)
    compare(out, lse, ref_out, ref_lse)


def test_allocating_entry_point():
    sp, inp, table, n_pages, kp, vp = paged_case([300, 5, 1000], 8, 2, 128, "bf16", 16, seed=9)
    out, lse = paged_gpu(sp, inp, table, n_pages, kp, vp, 16, entry="alloc")
    ref_out, ref_lse = oracle_paged(sp, inp, table, kp, vp, 16)
    compare(out, lse, ref_out, ref_lse)


def test_bad_block_table_entry_is_reported():
    """An entry outside [0, num_pages) is caught on the device before any read through it: the
    call reports TA_ERR_BAD_PAGE, the poisoned rows are NaN, and the next call succeeds."""
    import exact_long_context_split_b200 as ta

    seqlens = [300, 70]
    sp, inp, table, n_pages, kp, vp = paged_case(seqlens, 8, 2, 128, "bf16", 16, seed=10, spare=0)
    bad = table.copy()
    bad[0, 5] = n_pages  # one past the last physical block
    out, lse = paged_gpu(sp, inp, bad, n_pages, kp, vp, 16, expect=ta.TA_ERR_BAD_PAGE)
    assert np.isnan(out[0]).all() and np.isnan(lse[0]).all()
    bad[0, 5] = -1
    paged_gpu(sp, inp, bad, n_pages, kp, vp, 16, expect=ta.TA_ERR_BAD_PAGE)
    out, lse = paged_gpu(sp, inp, table, n_pages, kp, vp, 16)
    ref_out, ref_lse = oracle_paged(sp, inp, table, kp, vp, 16)
    compare(out, lse, ref_out, ref_lse)


def test_invalid_page_size():
    import torch

    import exact_long_context_split_b200 as ta

    z = torch.zeros(4096, dtype=torch.bfloat16, device="cuda")
    bt = torch.zeros(8, dtype=torch.int32, device="cuda")
    o = torch.empty(8 * 128, device="cuda")
    for ps in (8, 24, 0):
        with pytest.raises(ta.TreeAttnError) as e:
            ta.tree_attn_decode_paged(z, z, z, 1, ps, bt, 8, [5], 8, 2, 128, 0.1, o, o)
        assert e.value.status == ta.TA_ERR_INVALID_ARG


def test_long_1m_paged_all_rows():
    """The bench workload: 1M tokens in 16-token blocks at random places, every row."""
    import torch

    import exact_long_context_split_b200 as ta

    sp = synth.paged_configs()["long_1m_paged"]
    inp = synth.make_decode_inputs(sp)
    S, Hkv, D, ps = sp.seqlens[0], sp.n_kv_heads, sp.head_dim, sp.page_size
    table, n_pages = synth.page_table(sp.seed, sp.seqlens, ps)
    bt = torch.from_numpy(table).cuda()
    idx = bt[0].long()
    pages = {}
    for name in ("k", "v"):
        c = device_tensor(inp[name], "bf16").view(Hkv, S // ps, ps, D).permute(1, 0, 2, 3)
        pg = torch.empty(n_pages, Hkv, ps, D, dtype=torch.bfloat16, device="cuda")
        pg[idx] = c
        pages[name] = pg
    q = device_tensor(inp["q"], "bf16")
    out = torch.empty(1, 32, D, device="cuda")
    lse = torch.empty(1, 32, device="cuda")
    ws = new_workspace(ta.tree_attn_workspace_size([S], 32, Hkv, D))
    ta.tree_attn_decode_paged_ex("bf16", q, pages["k"], pages["v"], n_pages, ps, bt, table.shape[1], [S], 32, Hkv, D,
                                 sp.scale, out, lse, None, ws)
    assert ta.tree_attn_check(ws) == ta.TA_OK
    out, lse = out.cpu().numpy(), lse.cpu().numpy()
    # the paged cache holds the contiguous cache's rows (pinned on the CPU), so the oracle reads
    # the contiguous one: every row, a KV head's query heads per task
    from gpu_util import oracle_parallel

    G = 32 // Hkv
    tasks = [[(0, g * G + i) for i in range(G)] for g in range(Hkv)]
    ref_out, ref_lse = oracle_parallel(
        lambda pairs: oracle.decode_attention(inp["q"], inp["k"], inp["v"], sp.seqlens, 32, Hkv, D, sp.scale,
                                              pairs=pairs), tasks)
    compare(out, lse, ref_out, ref_lse)


# Several query tokens per sequence over a paged cache: the tensor-core form (one TMA box per
# page segment of a 128-key tile) and the split-KV passes (paged instances).
MULTI_CASES = [
    ([5, 129, 2049], 4, 16, 4, 16),      # 16 rows, 16-token pages (8 boxes per key tile)
    ([300, 40, 1000], 2, 32, 8, 64),     # 8 rows, 64-token pages
    ([700, 4], 4, 8, 2, 256),            # pages larger than a key tile
    ([3000, 16], 16, 64, 8, 32),         # 128 rows
]


@pytest.mark.parametrize("path", [1, 2])
@pytest.mark.parametrize("case", MULTI_CASES, ids=["ps16", "ps64", "ps256", "rows128"])
def test_multi_query_paged_against_oracle(case, path):
    import torch

    import exact_long_context_split_b200 as ta

    seqlens, n, Hq, Hkv, ps = case
    sp = synth.DecodeSpec("mpaged", list(seqlens), Hq, Hkv, 128, seed=60 + ps, n_queries=n)
    inp = synth.make_decode_inputs(sp)
    table, n_pages = synth.page_table(sp.seed, seqlens, ps, spare=2)
    kp = synth.scatter_pages(inp["k"], seqlens, Hkv, 128, ps, table, n_pages, NAN["bf16"])
    vp = synth.scatter_pages(inp["v"], seqlens, Hkv, 128, ps, table, n_pages, NAN["bf16"])
    B = sp.batch
    out = torch.full((B, n, Hq, 128), float("nan"), device="cuda")
    lse = torch.full((B, n, Hq), float("nan"), device="cuda")
    opts = ta.make_options(prefix_path=path)
    ws = new_workspace(ta.tree_attn_multi_workspace_size(list(seqlens), n, Hq, Hkv, 128, "bf16", opts))
    ta.tree_attn_decode_multi_paged_ex("bf16", device_tensor(inp["q"], "bf16"), device_tensor(kp.reshape(-1), "bf16"),
                                       device_tensor(vp.reshape(-1), "bf16"), n_pages, ps,
                                       torch.from_numpy(table).cuda(), table.shape[1], list(seqlens), n, Hq, Hkv,
                                       128, sp.scale, out, lse, opts, ws)
    assert ta.tree_attn_check(ws) == ta.TA_OK
    o, l = out.cpu().numpy(), lse.cpu().numpy()
    ref_out, ref_lse = oracle.paged_multi_query_attention(inp["q"], kp.reshape(-1), vp.reshape(-1), table, seqlens,
                                                          ps, n, Hq, Hkv, 128, sp.scale)
    compare(o.reshape(B * n, Hq, 128), l.reshape(B * n, Hq), ref_out.reshape(B * n, Hq, 128),
            ref_lse.reshape(B * n, Hq))


def test_multi_query_paged_bad_entry():
    """A bad block-table entry in the tensor-core form: TA_ERR_BAD_PAGE, NaN rows, no read."""
    import torch

    import exact_long_context_split_b200 as ta

    seqlens, n, Hq, Hkv, ps = [300, 70], 2, 8, 2, 16
    sp = synth.DecodeSpec("mpaged_bad", seqlens, Hq, Hkv, 128, seed=61, n_queries=n)
    inp = synth.make_decode_inputs(sp)
    table, n_pages = synth.page_table(sp.seed, seqlens, ps)
    kp = synth.scatter_pages(inp["k"], seqlens, Hkv, 128, ps, table, n_pages, NAN["bf16"])
    bad = table.copy()
    bad[0, 3] = n_pages
    out = torch.empty(2, n, Hq, 128, device="cuda")
    lse = torch.empty(2, n, Hq, device="cuda")
    opts = ta.make_options(prefix_path=1)
    ws = new_workspace(ta.tree_attn_multi_workspace_size(seqlens, n, Hq, Hkv, 128, "bf16", opts))
    k = device_tensor(kp.reshape(-1), "bf16")
    ta.tree_attn_decode_multi_paged_ex("bf16", device_tensor(inp["q"], "bf16"), k, k, n_pages, ps,
                                       torch.from_numpy(bad).cuda(), bad.shape[1], seqlens, n, Hq, Hkv, 128, sp.scale,
                                       out, lse, opts, ws)
    assert ta.tree_attn_check(ws) == ta.TA_ERR_BAD_PAGE
    assert np.isnan(out[0].cpu().numpy()).all()


@pytest.mark.parametrize("path", [0, 2])
@pytest.mark.parametrize("ps", [16, 64, 256])
def test_paged_g8_decode(ps, path):
    """G = 8 bf16 decode over pages runs on the paged tensor-core form by default (one query token)
    and on the split kernel with prefix_path 2; both against the oracle, unused page rows NaN."""
    import exact_long_context_split_b200 as ta

    sp, inp, table, n_pages, kp, vp = paged_case([1, 0, 300, 5000, 129], 16, 2, 128, "bf16", ps, seed=11)
    opts = ta.make_options(prefix_path=path) if path else None
    out, lse = paged_gpu(sp, inp, table, n_pages, kp, vp, ps, opts)
    compare(out, lse, *oracle_paged(sp, inp, table, kp, vp, ps))


def test_paged_g8_bad_entry_and_allocating_entry():
    """On the tensor-core route a bad block-table entry is reported (TA_ERR_BAD_PAGE, NaN outputs)
    and the allocating entry point sizes its workspace for that route."""
    import exact_long_context_split_b200 as ta

    sp, inp, table, n_pages, kp, vp = paged_case([700, 33], 64, 8, 128, "bf16", 16, seed=12, spare=0)
    bad = table.copy()
    bad[0, 7] = n_pages
    out, lse = paged_gpu(sp, inp, bad, n_pages, kp, vp, 16, expect=ta.TA_ERR_BAD_PAGE)
    assert np.isnan(out).all() and np.isnan(lse).all()
    out, lse = paged_gpu(sp, inp, table, n_pages, kp, vp, 16, entry="alloc")
    compare(out, lse, *oracle_paged(sp, inp, table, kp, vp, 16))
