"""Sequence-sharded decode over the ranks of a torch.distributed process group.

Tree Attention article (m.srwj168.com.cn, "The energy view of attention"): max and
logsumexp are associative, so the attention each device computes over its slice of the
cache combines exactly with the others'; across devices the combination is a tree
all-reduce.  Star Attention phase 2 (tiaojiaomugou.com): each host attends over its local
cache and the query host combines the softmax statistics.

Here rank r holds the contiguous token range shard_bounds(S_b, W, r) of every sequence b,
runs ordinary decode over it (the library's split-KV kernels) to get (out_r, lse_r), the
ranks all-gather those B * Hq * (D + 1) floats in one collective, and every rank merges them
with tree_attn_merge_shards (a fixed pairwise tree over the ranks).  The only data-path
collective is that all-gather; the decode and the merge run in the library's kernels.
"""
from __future__ import annotations

from typing import Callable, Optional, Sequence, Tuple

from . import tree_attn_decode, tree_attn_decode_f32, tree_attn_merge_shards


def shard_bounds(seqlen: int, n_shards: int, shard: int) -> Tuple[int, int]:
    """Token range [t0, t1) that rank `shard` of `n_shards` holds of a sequence of seqlen tokens:
    t0 = floor(shard * S / n), t1 = floor((shard + 1) * S / n) (contiguous, covering [0, S))."""
    S = int(seqlen)
    return shard * S // n_shards, (shard + 1) * S // n_shards


def _decode(dtype, q, k, v, lens, Hq, Hkv, D, scale, out, lse):
    fn = tree_attn_decode if dtype == "bf16" else tree_attn_decode_f32
    fn(q, k, v, lens, Hq, Hkv, D, scale, out, lse)


def decode_sharded(q, k_shard, v_shard, shard_lens: Sequence[int], n_q_heads: int, n_kv_heads: int, head_dim: int,
                   scale: float, out, lse, group=None, dtype: str = "bf16", decode: Optional[Callable] = None,
                   merge: Optional[Callable] = None) -> None:
    """Decode over a cache sharded by token range across the group's ranks.

    Every rank passes the same q ([B][Hq][D]) and its own shard of every sequence's cache
    (packed like tree_attn_decode's k/v, sequence b holding shard_lens[b] tokens); on return
    out ([B][Hq][D] f32) and lse ([B][Hq] f32) hold the result over the whole cache on every
    rank.  `decode` / `merge` replace the library calls (same arguments as _decode and
    tree_attn_merge_shards); the host-side tests use that to run the exchange on CPU ranks.
    """
    import torch
    import torch.distributed as dist

    world = dist.get_world_size(group)
    rows = len(shard_lens) * n_q_heads
    n_out = rows * head_dim
    local = torch.empty(n_out + rows, dtype=torch.float32, device=out.device)  # out then lse: one collective
    (decode or _decode)(dtype, q, k_shard, v_shard, list(shard_lens), n_q_heads, n_kv_heads, head_dim, scale,
                        local[:n_out], local[n_out:])
    gathered = torch.empty(world, n_out + rows, dtype=torch.float32, device=out.device)
    if dist.get_backend(group) == "nccl":
        dist.all_gather_into_tensor(gathered, local, group=group)
    else:
        dist.all_gather(list(gathered.unbind(0)), local, group=group)
    outs = gathered[:, :n_out].contiguous()
    lses = gathered[:, n_out:].contiguous()
    (merge or tree_attn_merge_shards)(outs, lses, world, rows, head_dim, out, lse)
