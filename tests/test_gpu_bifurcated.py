"""GPU parity of bifurcated (shared-prefix) decode against the CPU oracle, through the C ABI."""
import numpy as np
import pytest

import oracle
import synth
from gpu_util import compare, device_tensor, empty_outputs, new_workspace

pytestmark = pytest.mark.gpu


def bif_gpu(inp, sp, entry="ex", prefix_path=0, split_tiles=0, num_ctas=0):
    import torch

    import exact_long_context_split_b200 as ta

    N, Hq, Hkv, D, P = sp.n_samples, sp.n_q_heads, sp.n_kv_heads, sp.head_dim, sp.prefix_len
    q = device_tensor(inp["q"], "bf16")
    kp, vp = device_tensor(inp["k_prefix"], "bf16"), device_tensor(inp["v_prefix"], "bf16")
    ks, vs = device_tensor(inp["k_suffix"], "bf16"), device_tensor(inp["v_suffix"], "bf16")
    out, lse = empty_outputs(N, Hq, D)
    lens = [int(s) for s in sp.suffix_lens]
    if entry == "ex":
        opts = ta.make_options(num_ctas=num_ctas, prefix_path=prefix_path, split_tiles=split_tiles)
        ws = new_workspace(ta.tree_attn_bifurcated_workspace_size(P, lens, Hq, Hkv, D, opts))
        ta.tree_attn_decode_bifurcated_ex(q, kp, vp, P, ks, vs, lens, Hq, Hkv, D, sp.scale, out, lse, opts, ws)
        assert ta.tree_attn_check(ws) == ta.TA_OK
    else:
        ta.tree_attn_decode_bifurcated(q, kp, vp, P, ks, vs, lens, Hq, Hkv, D, sp.scale, out, lse)
    torch.cuda.synchronize()
    return out.cpu().numpy(), lse.cpu().numpy()


def oracle_bif(inp, sp, pairs=None):
    return oracle.bifurcated_attention(inp["q"], inp["k_prefix"], inp["v_prefix"], sp.prefix_len, inp["k_suffix"],
                                       inp["v_suffix"], sp.suffix_lens, sp.n_q_heads, sp.n_kv_heads, sp.head_dim,
                                       sp.scale, dtype="bf16", pairs=pairs)


@pytest.mark.parametrize(
    "prefix_len,suffix_lens,Hq,Hkv,D",
    [
        (1000, [5, 0, 64, 130], 32, 8, 128),
        (0, [100, 3], 8, 2, 128),
        (4097, [0, 0], 8, 8, 64),
        (256, [1] * 20, 16, 2, 128),
    ],
)
@pytest.mark.parametrize("entry", ["ex", "alloc"])
def test_bifurcated_small(prefix_len, suffix_lens, Hq, Hkv, D, entry):
    sp = synth.BifurcatedSpec("case", prefix_len, suffix_lens, Hq, Hkv, D, seed=21)
    inp = synth.make_bifurcated_inputs(sp)
    out, lse = bif_gpu(inp, sp, entry)
    compare(out, lse, *oracle_bif(inp, sp))


# Tensor-core prefix pass (prefix_path 1) and the split-KV pass per sample (2) on shapes with
# several 128-row tiles (N * G > 128), a partial last row tile, partial 64-key tiles, one tile,
# and more chunks than tiles.
TC_CASES = [
    (65, [3, 70], 8, 2, 128),          # 8 rows, 2 key tiles (one partial)
    (1000, [5, 0, 64, 130], 32, 8, 128),
    (4097, [1] * 40, 16, 4, 128),      # 160 rows: two row tiles, the second partial
    (300, [9] * 64, 16, 2, 128),       # 512 rows: four row tiles
    (64, [0, 2], 8, 8, 128),           # G = 1, exactly one key tile
    (12345, [100] * 20, 32, 8, 128),
]


@pytest.mark.parametrize("prefix_path", [1, 2])
@pytest.mark.parametrize("prefix_len,suffix_lens,Hq,Hkv,D", TC_CASES)
def test_bifurcated_prefix_paths(prefix_len, suffix_lens, Hq, Hkv, D, prefix_path):
    sp = synth.BifurcatedSpec("case", prefix_len, suffix_lens, Hq, Hkv, D, seed=23)
    inp = synth.make_bifurcated_inputs(sp)
    out, lse = bif_gpu(inp, sp, "ex", prefix_path)
    compare(out, lse, *oracle_bif(inp, sp))


# The suffix pass on the short-unit kernel (one CTA per sample and KV head, the prefix chunks'
# statistics folded into each row): ragged suffixes with empty and one-token ones, every G, more
# than 128 samples (two launches).
SHORT_CASES = [
    (1000, [0, 1, 31, 32, 33, 300, 2047, 5], 32, 8, 128),
    (65, [3, 70], 8, 2, 128),
    (300, [9] * 64, 16, 2, 128),
    (64, [0, 2, 128], 8, 8, 128),
    (4097, [100] * 140, 16, 8, 128),
]


@pytest.mark.parametrize("prefix_len,suffix_lens,Hq,Hkv,D", SHORT_CASES)
def test_short_unit_suffix_pass(prefix_len, suffix_lens, Hq, Hkv, D):
    sp = synth.BifurcatedSpec("case", prefix_len, suffix_lens, Hq, Hkv, D, seed=25)
    inp = synth.make_bifurcated_inputs(sp)
    out, lse = bif_gpu(inp, sp, "ex", prefix_path=1, split_tiles=3)
    compare(out, lse, *oracle_bif(inp, sp))
    again = bif_gpu(inp, sp, "ex", prefix_path=1, split_tiles=3)
    assert np.array_equal(out.view(np.uint32), again[0].view(np.uint32))


@pytest.mark.parametrize("num_ctas", [1, 3, 7, 40])
def test_short_unit_suffix_grid_sizes(num_ctas):
    """Fewer persistent CTAs than units: each CTA streams several ragged units through its stage
    ring (wrapping it many times, units with 0, 1 and partial stages), against the oracle."""
    sp = synth.BifurcatedSpec("case", 700, [0, 1, 31, 32, 33, 255, 256, 257, 600, 5] * 3, 32, 8, 128, seed=26)
    inp = synth.make_bifurcated_inputs(sp)
    out, lse = bif_gpu(inp, sp, "ex", prefix_path=1, split_tiles=3, num_ctas=num_ctas)
    compare(out, lse, *oracle_bif(inp, sp))


def test_short_unit_suffix_stage_never_loaded():
    """The suffix kernel's bounded waits: with a stage of CTA 0 never loaded, the call reports
    TA_ERR_TIMEOUT, CTA 0's first unit (sample 0, KV head 0) comes out NaN, and the next call on
    the same stream is correct."""
    import torch

    import exact_long_context_split_b200 as ta

    sp = synth.BifurcatedSpec("case", 1000, [300, 40, 7, 128], 32, 8, 128, seed=27)
    inp = synth.make_bifurcated_inputs(sp)
    q = device_tensor(inp["q"], "bf16")
    kp, vp = device_tensor(inp["k_prefix"], "bf16"), device_tensor(inp["v_prefix"], "bf16")
    ks, vs = device_tensor(inp["k_suffix"], "bf16"), device_tensor(inp["v_suffix"], "bf16")
    lens = [int(s) for s in sp.suffix_lens]
    for skip in (1, 3, 9):
        out, lse = torch.zeros(4, 32, 128, device="cuda"), torch.zeros(4, 32, device="cuda")
        opts = ta.make_options(wait_limit_us=20000, prefix_path=1, split_tiles=3, debug_skip_stage=skip)
        ws = new_workspace(ta.tree_attn_bifurcated_workspace_size(1000, lens, 32, 8, 128, opts))
        ta.tree_attn_decode_bifurcated_ex(q, kp, vp, 1000, ks, vs, lens, 32, 8, 128, sp.scale, out, lse, opts, ws)
        assert ta.tree_attn_check(ws) == ta.TA_ERR_TIMEOUT
        assert torch.isnan(out[0, :4]).all() and torch.isnan(lse[0, :4]).all()
    out, lse = bif_gpu(inp, sp, "ex", prefix_path=1, split_tiles=3)
    compare(out, lse, *oracle_bif(inp, sp))


def test_tensor_core_prefix_is_deterministic():
    sp = synth.BifurcatedSpec("case", 20000, [50] * 32, 32, 8, 128, seed=24)
    inp = synth.make_bifurcated_inputs(sp)
    a = bif_gpu(inp, sp, "ex", 1)
    b = bif_gpu(inp, sp, "ex", 1)
    assert np.array_equal(a[0].view(np.uint32), b[0].view(np.uint32))
    assert np.array_equal(a[1].view(np.uint32), b[1].view(np.uint32))


def test_tensor_core_prefix_unsupported_shape():
    import exact_long_context_split_b200 as ta

    with pytest.raises(ta.TreeAttnError):
        ta.tree_attn_bifurcated_workspace_size(100, [1, 2], 8, 2, 64, ta.make_options(prefix_path=1))


def test_bifurcated_equals_plain_decode_of_concatenation():
    """Exactness of the split: the GPU bifurcated result (prefix and suffix parts merged) matches
    the GPU plain decode of each sample's concatenated cache [prefix ; suffix_n] within the
    tolerance, and both match the oracle."""
    sp = synth.BifurcatedSpec("case", 3000, [7, 300], 8, 2, 128, seed=22)
    inp = synth.make_bifurcated_inputs(sp)
    out, lse = bif_gpu(inp, sp)
    ref = oracle_bif(inp, sp)
    compare(out, lse, *ref)
    # the same samples as plain decode: sequence n's cache is [prefix ; suffix_n] per KV head
    P, Hkv, D, lens = sp.prefix_len, sp.n_kv_heads, sp.head_dim, list(sp.suffix_lens)
    kp = inp["k_prefix"].reshape(Hkv, P, D)
    vp = inp["v_prefix"].reshape(Hkv, P, D)
    ks, vs, off = [], [], 0
    for S in lens:
        ks.append(np.concatenate([kp, inp["k_suffix"][off:off + Hkv * S * D].reshape(Hkv, S, D)], axis=1))
        vs.append(np.concatenate([vp, inp["v_suffix"][off:off + Hkv * S * D].reshape(Hkv, S, D)], axis=1))
        off += Hkv * S * D
    dec = synth.DecodeSpec("concat", [P + S for S in lens], sp.n_q_heads, Hkv, D, seed=22)
    dinp = {"q": inp["q"], "k": np.concatenate([x.reshape(-1) for x in ks]),
            "v": np.concatenate([x.reshape(-1) for x in vs])}
    from gpu_util import decode_gpu

    plain_out, plain_lse = decode_gpu(dinp, dec)
    compare(plain_out, plain_lse, *ref)
    compare(out, lse, plain_out.astype(np.float64), plain_lse.astype(np.float64))


@pytest.mark.parametrize("prefix_path,split_tiles", [(1, 0), (1, 1), (2, 0)])
def test_bifurcated_config_sampled(prefix_path, split_tiles):
    """The shared-prefix workload (64 samples, 65,536 + 256 tokens): every query head of 17
    samples spread over the batch; the suffix pass on the short-unit kernel (automatic), on the
    split kernel (split_tiles 1), and the all-split path (prefix_path 2)."""
    from gpu_util import oracle_parallel

    sp = synth.bifurcated_configs()["shared_prefix"]
    inp = synth.make_bifurcated_inputs(sp)
    out, lse = bif_gpu(inp, sp, "ex", prefix_path, split_tiles)
    assert np.all(np.isfinite(out)) and np.all(np.isfinite(lse))
    samples = list(range(0, sp.n_samples, 4)) + [sp.n_samples - 1]
    tasks = [[(n, h) for h in range(sp.n_q_heads)] for n in samples]
    ref_out, ref_lse = oracle_parallel(lambda pairs: oracle_bif(inp, sp, pairs=pairs), tasks, workers=4)
    pairs = [p for t in tasks for p in t]
    compare(out, lse, ref_out, ref_lse, pairs=pairs)
