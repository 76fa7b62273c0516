"""GPU parity of sequence-sharded decode on one GPU: the cache is cut into W contiguous shards
per sequence, each shard decoded by the library, and the W results merged by
tree_attn_merge_shards; compared with the CPU oracle over the whole cache."""
import numpy as np
import pytest

import oracle
import synth
from gpu_util import compare, device_tensor, new_workspace

pytestmark = pytest.mark.gpu


def shard_inputs(inp, sp, W, r):
    from exact_long_context_split_b200.sharded import shard_bounds

    Hkv, D = sp.n_kv_heads, sp.head_dim
    lens, ks, vs, off = [], [], [], 0
    for S in sp.seqlens:
        t0, t1 = shard_bounds(S, W, r)
        lens.append(t1 - t0)
        ks.append(inp["k"][off:off + Hkv * S * D].reshape(Hkv, S, D)[:, t0:t1].reshape(-1))
        vs.append(inp["v"][off:off + Hkv * S * D].reshape(Hkv, S, D)[:, t0:t1].reshape(-1))
        off += Hkv * S * D
    return lens, np.concatenate(ks), np.concatenate(vs)


@pytest.mark.parametrize("W", [1, 2, 3, 5, 8])
def test_sharded_merge_against_oracle(W):
    import torch

    import exact_long_context_split_b200 as ta

    sp = synth.DecodeSpec("sharded", [3, 100, 5000, 0, 70000], 32, 8, 128, seed=21)
    inp = synth.make_decode_inputs(sp)
    B, Hq, Hkv, D = sp.batch, 32, 8, 128
    rows = B * Hq
    outs = torch.empty(W, rows, D, device="cuda")
    lses = torch.empty(W, rows, device="cuda")
    q = device_tensor(inp["q"], "bf16")
    for r in range(W):
        lens, k, v = shard_inputs(inp, sp, W, r)
        ws = new_workspace(ta.tree_attn_workspace_size(lens, Hq, Hkv, D))
        ta.tree_attn_decode_ex("bf16", q, device_tensor(k, "bf16") if k.size else None,
                               device_tensor(v, "bf16") if v.size else None, lens, Hq, Hkv, D, sp.scale, outs[r],
                               lses[r], None, ws)
        assert ta.tree_attn_check(ws) == ta.TA_OK
    out = torch.empty(B, Hq, D, device="cuda")
    lse = torch.empty(B, Hq, device="cuda")
    ta.tree_attn_merge_shards(outs, lses, W, rows, D, out, lse)
    out2 = torch.empty_like(out)
    lse2 = torch.empty_like(lse)
    ta.tree_attn_merge_shards(outs, lses, W, rows, D, out2, lse2)
    torch.cuda.synchronize()
    o, l = out.cpu().numpy(), lse.cpu().numpy()
    assert np.array_equal(o.view(np.uint32), out2.cpu().numpy().view(np.uint32)), "merge not bit-identical"
    if W == 1:
        assert np.array_equal(o.reshape(-1).view(np.uint32), outs.cpu().numpy().reshape(-1).view(np.uint32))
    ref_out, ref_lse = oracle.decode_attention(inp["q"], inp["k"], inp["v"], sp.seqlens, Hq, Hkv, D, sp.scale)
    compare(o, l, ref_out, ref_lse)


def test_merge_shards_invalid_arguments():
    import torch

    import exact_long_context_split_b200 as ta

    x = torch.zeros(16, device="cuda")
    for n in (0, 65537):
        with pytest.raises(ta.TreeAttnError) as e:
            ta.tree_attn_merge_shards(x, x, n, 1, 8, x, x)
        assert e.value.status == ta.TA_ERR_INVALID_ARG
