"""CPU oracle for exact split decode attention.

TEST INFRASTRUCTURE.  This module is the correctness reference for the CUDA
library.  Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg
of ``bench.py`` may import or call it; the library never does, and it shares no
code with the library (it reads the same host input bytes, nothing else).

Everything is computed in float64 on the exact input values (bf16 and float32
inputs widen to float64 without rounding).

Sources (the web pages this method is taken from):

* [AttnAccel] "Attention acceleration" (compassingai.com, concept page
  attention-acceleration), section "Technical principles": part 1 "Self-attention
  recap" gives S = Q K^T / sqrt(d_k), P = softmax(S), O = P V; part 2.1
  "Tiling and online softmax" gives m(x) = max_j x_j, l(x) = sum_j exp(x_j - m(x))
  and the block update of m, l and O.
* [TreeAttn] Tree Attention article (m.srwj168.com.cn, keji312/12691), section
  "The energy view of attention": attention is the gradient, at zeta = 0, of a
  scalar energy F(K, Q, V, zeta); logsumexp and max are associative, so the
  per-device pieces can be combined in any order (tree all-reduce).
* [Bifurcated] Bifurcated attention summary (briefgpt.xyz, 2403.08845), TL;DR:
  decode attention over a shared prefilled context plus per-sample decoded
  tokens is split into two GEMMs and stays exact.
* [StarAttn] Star Attention article (tiaojiaomugou.com, 242533), "Phase 2: query
  encoding and token generation": each host attends over its local cache and the
  query host combines the softmax statistics into global attention; "Phase 1: context
  encoding": the context is cut into blocks, each prefixed with the anchor block.

Readings taken where the pages are silent or garbled (each also listed in the
design notes):

1. The decode energy formula did not survive extraction.  It is read as
   F(zeta) = log sum_t exp(s * q.k_t + zeta.v_t); then dF/dzeta at 0 = output.
2. lse is the natural logarithm of sum_t exp(s * q.k_t) (scaled scores).
3. The online-softmax output update of [AttnAccel] 2.1 is printed in the
   normalised form with an undefined "block_result"; it is read as
   sum_{j in block} exp(x_j - m_new) v_j.  The split path keeps O unnormalised
   (the partial (m, l, o)), which is algebraically the same.
4. An empty sequence gives out = 0 and lse = -inf.
5. GQA: query head h reads KV head h // (Hq / Hkv) (consecutive groups).
6. The bifurcated result for sample n is plain attention over the concatenation
   [prefix ; suffix_n]; no mask (the query is the last position).
7. Several query tokens per sequence ([StarAttn], "How Star Attention cuts the cost of
   inference" and phase 2): a short query of n tokens follows the cached context, and its
   tokens' keys and values are written to the cache at its end before attention.  Query
   token j (0-based) sits at position S - n + j and attends to every key at or before it,
   i.e. to the first S - n + j + 1 keys (all preceding context, causal among the n new
   tokens).  n = 1 is ordinary decode.
8. Paged cache ([AttnAccel] part 3, "PagedAttention (vLLM)"): the cache is cut into blocks of
   a fixed number of tokens and a table maps each sequence's logical blocks to physical ones
   (which sequences may share).  Layout read here: physical block p holds, for each KV head
   h, page_size consecutive token rows [p][h][0..page_size)[D]; logical block i of sequence b
   (its tokens i * page_size ...) is physical block table[b][i].
9. Sequence-sharded decode ([TreeAttn], tree all-reduce across devices; [StarAttn] phase 2,
   the query host combining the hosts' softmax statistics): device r holds the contiguous
   token range shard_bounds(S, W, r) of every sequence and computes ordinary decode attention
   over it, i.e. (out_r, lse_r); the results combine exactly as partials (m = lse_r, l = 1,
   o = out_r) merged in a fixed pairwise tree over r.  A shard with no token gives (0, -inf).
10. Context encoding with anchor blocks ([StarAttn], "Two-phase inference under Star Attention",
   "Phase 1: context encoding"): the context of S tokens is cut into blocks of block_size
   tokens (the last one may be shorter); every block except the first is prefixed with the
   first block (the anchor block) and each host attends over its [anchor ; own block]
   sequence.  Read here, as the page does not spell it out: attention inside that augmented
   sequence is the usual causal rule, so the token at position p of block i (i = p //
   block_size) attends to keys [0, p] when i = 0 and to keys [0, block_size) and
   [i * block_size, p] when i > 0; the anchor block is the first block, of block_size tokens.
   Only the non-anchor rows of each host are kept, so every position has exactly one output.
"""
from __future__ import annotations

import math
from typing import Iterable, List, Optional, Sequence, Tuple

import numpy as np

Partial = Tuple[float, float, np.ndarray]  # (m, l, o): running max, sum of exponentials, unnormalised output

# Rows of K and V widened to float64 at a time when a cache is decoded in pieces
# (memory only: every score and every sum term is the same as with one piece).
ROWS_PER_PIECE = 1 << 20


# ------------------------------------------------------------------------------------------
# Input decoding
# ------------------------------------------------------------------------------------------


def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    """bf16 bit patterns (uint16) to float64: the bf16 value is the float32 whose
    upper 16 bits are the pattern and whose lower 16 bits are zero (exact)."""
    b = np.asarray(bits, dtype=np.uint16)
    return (b.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)


def to_f64(a: np.ndarray, dtype: str) -> np.ndarray:
    if dtype == "bf16":
        return bf16_to_f64(a)
    if dtype == "f32":
        return np.asarray(a, dtype=np.float32).astype(np.float64)
    if dtype == "f64":
        return np.asarray(a, dtype=np.float64)
    raise ValueError(dtype)


def sequence_block(flat: np.ndarray, seqlens: Sequence[int], b: int, n_kv_heads: int, head_dim: int) -> np.ndarray:
    """View of sequence b's [Hkv][S_b][D] block in a cache packed sequence after sequence."""
    start = int(sum(int(s) for s in seqlens[:b])) * n_kv_heads * head_dim
    S = int(seqlens[b])
    return flat[start : start + n_kv_heads * S * head_dim].reshape(n_kv_heads, S, head_dim)


# ------------------------------------------------------------------------------------------
# The definition ([AttnAccel] part 1, one decode query)
# ------------------------------------------------------------------------------------------


def attention_one(q: np.ndarray, K: np.ndarray, V: np.ndarray, scale: float) -> Tuple[np.ndarray, float]:
    """softmax(scale * K q) V and its log-sum-exp, two passes, float64.

    q: [D]; K, V: [S][D] float64.  Pass 1 forms every score x_t = scale * q.k_t
    and their maximum m; pass 2 forms l = sum_t exp(x_t - m) and
    sum_t exp(x_t - m) v_t.  Returns (out = that sum / l, lse = m + ln l).
    """
    S, D = K.shape
    if S == 0:
        return np.zeros(D), -math.inf
    x = scale * (K @ q)
    m = float(np.max(x))
    e = np.exp(x - m)
    l = float(np.sum(e))
    out = (e @ V) / l
    return out, m + math.log(l)


def attention_heads_cache(Q: np.ndarray, Kbits: np.ndarray, Vbits: np.ndarray, scale: float,
                          dtype: str = "bf16") -> Tuple[np.ndarray, np.ndarray]:
    """attention_one for several query rows over one long cache kept in its storage format.

    Q: [H][D] float64 (the query heads that read this cache); Kbits, Vbits: [S][D] bf16 bits
    or float32.  The cache is widened to float64 ROWS_PER_PIECE rows at a time.  For every
    row h the arithmetic is the definition's: pass 1 forms every score x_t = scale * q_h.k_t
    (one product K Q^T serves all rows) and their maximum m_h before pass 2 forms
    l_h = sum_t exp(x_t - m_h) and sum_t exp(x_t - m_h) v_t.  Returns (out [H][D], lse [H]).
    """
    Q = np.atleast_2d(np.asarray(Q, dtype=np.float64))
    S = Kbits.shape[0]
    H, D = Q.shape
    if S == 0:
        return np.zeros((H, D)), np.full(H, -math.inf)
    x = np.empty((S, H))
    for r0 in range(0, S, ROWS_PER_PIECE):
        r1 = min(S, r0 + ROWS_PER_PIECE)
        x[r0:r1] = scale * (to_f64(Kbits[r0:r1], dtype) @ Q.T)
    m = np.max(x, axis=0)
    e = np.exp(x - m)
    l = np.sum(e, axis=0)
    acc = np.zeros((H, D))
    for r0 in range(0, S, ROWS_PER_PIECE):
        r1 = min(S, r0 + ROWS_PER_PIECE)
        acc += e[r0:r1].T @ to_f64(Vbits[r0:r1], dtype)
    return acc / l[:, None], m + np.log(l)


def attention_one_bf16_cache(q: np.ndarray, Kbits: np.ndarray, Vbits: np.ndarray, scale: float,
                             dtype: str = "bf16") -> Tuple[np.ndarray, float]:
    """attention_one for one query row over a cache kept in its storage format ([S][D] bf16
    bits or float32): attention_heads_cache with a single row."""
    out, lse = attention_heads_cache(np.asarray(q, dtype=np.float64)[None, :], Kbits, Vbits, scale, dtype)
    return out[0], float(lse[0])


def decode_attention(q, k_cache, v_cache, seqlens: Sequence[int], n_q_heads: int, n_kv_heads: int,
                     head_dim: int, scale: float, dtype: str = "bf16",
                     pairs: Optional[Iterable[Tuple[int, int]]] = None):
    """Decode attention for a batch with a packed, ragged KV cache.

    q: [B][Hq][D] (storage format); k_cache, v_cache: flat arrays, sequence b's
    block is [Hkv][S_b][D], blocks back to back.  Query head h of sequence b
    attends over KV head h // (Hq / Hkv) of sequence b (reading 5).

    Returns (out [B][Hq][D] float64, lse [B][Hq] float64).  With `pairs`, only
    those (b, h) entries are computed; the rest are NaN.
    """
    B = len(seqlens)
    Hq, Hkv, D = n_q_heads, n_kv_heads, head_dim
    if Hq % Hkv != 0:
        raise ValueError("n_q_heads must be a multiple of n_kv_heads")
    G = Hq // Hkv
    qf = to_f64(np.asarray(q).reshape(B, Hq, D), dtype)
    out = np.full((B, Hq, D), np.nan)
    lse = np.full((B, Hq), np.nan)
    todo = sorted(set(pairs)) if pairs is not None else [(b, h) for b in range(B) for h in range(Hq)]
    for b in sorted({p[0] for p in todo}):
        Kb = sequence_block(k_cache, seqlens, b, Hkv, D)
        Vb = sequence_block(v_cache, seqlens, b, Hkv, D)
        for g in sorted({h // G for (bb, h) in todo if bb == b}):
            heads = [h for (bb, h) in todo if bb == b and h // G == g]
            out[b, heads], lse[b, heads] = attention_heads_cache(qf[b, heads], Kb[g], Vb[g], scale, dtype)
    return out, lse


# ------------------------------------------------------------------------------------------
# The method's steps: chunk partials and their merge
# ------------------------------------------------------------------------------------------


def chunk_partial(q: np.ndarray, K: np.ndarray, V: np.ndarray, scale: float) -> Partial:
    """Softmax statistics of one chunk of the cache ([StarAttn] phase 2; [AttnAccel] 2.1).

    m = max_t x_t, l = sum_t exp(x_t - m), o = sum_t exp(x_t - m) v_t (o is not
    divided by l).  An empty chunk gives (-inf, 0, 0).
    """
    D = q.shape[0]
    if K.shape[0] == 0:
        return -math.inf, 0.0, np.zeros(D)
    x = scale * (K @ q)
    m = float(np.max(x))
    e = np.exp(x - m)
    return m, float(np.sum(e)), e @ V


def merge(a: Partial, b: Partial) -> Partial:
    """Combine the statistics of two disjoint chunks ([TreeAttn]: max and logsumexp are associative).

    m = max(m_a, m_b); each side is rescaled by exp(m_side - m) before l and o
    are added, as in the l_new update of [AttnAccel] 2.1.
    """
    ma, la, oa = a
    mb, lb, ob = b
    if ma == -math.inf and mb == -math.inf:
        return -math.inf, 0.0, np.zeros_like(oa)
    m = max(ma, mb)
    ca = math.exp(ma - m) if ma != -math.inf else 0.0
    cb = math.exp(mb - m) if mb != -math.inf else 0.0
    return m, la * ca + lb * cb, oa * ca + ob * cb


def finalize(p: Partial) -> Tuple[np.ndarray, float]:
    """out = o / l and lse = m + ln l; (-inf, 0, 0) gives (0, -inf) (reading 4)."""
    m, l, o = p
    if l == 0.0:
        return np.zeros_like(o), -math.inf
    return o / l, m + math.log(l)


def merge_tree(parts: List[Partial]) -> Partial:
    """Merge partials pairwise, level by level: depth ceil(log2 n) ([TreeAttn] tree all-reduce)."""
    if not parts:
        raise ValueError("no partials")
    level = list(parts)
    while len(level) > 1:
        nxt = [merge(level[i], level[i + 1]) for i in range(0, len(level) - 1, 2)]
        if len(level) % 2:
            nxt.append(level[-1])
        level = nxt
    return level[0]


def split_attention(q: np.ndarray, K: np.ndarray, V: np.ndarray, scale: float,
                    bounds: Sequence[int]) -> Tuple[np.ndarray, float]:
    """Attention computed chunk by chunk: chunk c covers rows [bounds[c], bounds[c+1])."""
    parts = [chunk_partial(q, K[t0:t1], V[t0:t1], scale) for t0, t1 in zip(bounds[:-1], bounds[1:])]
    return finalize(merge_tree(parts))


def online_softmax(q: np.ndarray, K: np.ndarray, V: np.ndarray, scale: float, block: int) -> Tuple[np.ndarray, float]:
    """[AttnAccel] 2.1 as printed: blocks of `block` keys, normalised running output.

    m_new = max(m_old, m_block); l_new = l_old exp(m_old - m_new) + sum_block exp(x - m_new);
    O_new = (O_old l_old exp(m_old - m_new) + sum_block exp(x - m_new) v) / l_new.
    """
    S, D = K.shape
    m, l, O = -math.inf, 0.0, np.zeros(D)
    for t0 in range(0, S, block):
        x = scale * (K[t0 : t0 + block] @ q)
        m_new = max(m, float(np.max(x)))
        carry = math.exp(m - m_new) if m != -math.inf else 0.0
        e = np.exp(x - m_new)
        l_new = l * carry + float(np.sum(e))
        O = (O * l * carry + e @ V[t0 : t0 + block]) / l_new
        m, l = m_new, l_new
    if l == 0.0:
        return np.zeros(D), -math.inf
    return O, m + math.log(l)


def energy(q: np.ndarray, K: np.ndarray, V: np.ndarray, scale: float, zeta: np.ndarray) -> float:
    """F(zeta) = log sum_t exp(scale * q.k_t + zeta.v_t)  ([TreeAttn], reading 1)."""
    z = scale * (K @ q) + V @ zeta
    zm = float(np.max(z))
    return zm + math.log(float(np.sum(np.exp(z - zm))))


# ------------------------------------------------------------------------------------------
# Bifurcated (shared-prefix) decode
# ------------------------------------------------------------------------------------------


def bifurcated_attention(q, k_prefix, v_prefix, prefix_len: int, k_suffix, v_suffix,
                         suffix_lens: Sequence[int], n_q_heads: int, n_kv_heads: int, head_dim: int,
                         scale: float, dtype: str = "bf16",
                         pairs: Optional[Iterable[Tuple[int, int]]] = None):
    """Sample n, query head h attends over [prefix ; suffix_n] of KV head h // G (reading 6).

    q: [N][Hq][D]; k_prefix, v_prefix: [Hkv][P][D]; k_suffix, v_suffix: packed
    per sample ([Hkv][S_n][D] blocks back to back).  Returns (out, lse) as
    decode_attention does.
    """
    N = len(suffix_lens)
    Hq, Hkv, D, P = n_q_heads, n_kv_heads, head_dim, prefix_len
    G = Hq // Hkv
    qf = to_f64(np.asarray(q).reshape(N, Hq, D), dtype)
    Kp = to_f64(np.asarray(k_prefix).reshape(Hkv, P, D), dtype)
    Vp = to_f64(np.asarray(v_prefix).reshape(Hkv, P, D), dtype)
    out = np.full((N, Hq, D), np.nan)
    lse = np.full((N, Hq), np.nan)
    todo = sorted(set(pairs)) if pairs is not None else [(n, h) for n in range(N) for h in range(Hq)]
    for n in sorted({p[0] for p in todo}):
        Ks = to_f64(sequence_block(k_suffix, suffix_lens, n, Hkv, D), dtype)
        Vs = to_f64(sequence_block(v_suffix, suffix_lens, n, Hkv, D), dtype)
        for g in sorted({h // G for (nn, h) in todo if nn == n}):
            heads = [h for (nn, h) in todo if nn == n and h // G == g]
            K = np.concatenate([Kp[g], Ks[g]], axis=0)
            V = np.concatenate([Vp[g], Vs[g]], axis=0)
            out[n, heads], lse[n, heads] = attention_heads_cache(qf[n, heads], K, V, scale, "f64")
    return out, lse


def multi_query_attention(q, k_cache, v_cache, seqlens: Sequence[int], n_queries: int, n_q_heads: int,
                          n_kv_heads: int, head_dim: int, scale: float, dtype: str = "bf16",
                          rows: Optional[Iterable[Tuple[int, int, int]]] = None):
    """n query tokens per sequence, causal among themselves (reading 7).

    q: [B][n][Hq][D] (storage format); k_cache, v_cache packed as for decode_attention, each
    sequence's block already holding the n query tokens' keys and values as its last n rows.
    Row (b, j, h) is attention over the first S_b - n + j + 1 keys of KV head h // G.

    Returns (out [B][n][Hq][D], lse [B][n][Hq]) in float64.  With `rows`, only those
    (b, j, h) entries are computed; the rest are NaN.
    """
    B, n = len(seqlens), n_queries
    Hq, Hkv, D = n_q_heads, n_kv_heads, head_dim
    if Hq % Hkv != 0:
        raise ValueError("n_q_heads must be a multiple of n_kv_heads")
    if n < 1 or any(int(S) < n for S in seqlens):
        raise ValueError("every sequence must hold its n query tokens")
    G = Hq // Hkv
    qf = to_f64(np.asarray(q).reshape(B, n, Hq, D), dtype)
    out = np.full((B, n, Hq, D), np.nan)
    lse = np.full((B, n, Hq), np.nan)
    todo = sorted(set(rows)) if rows is not None else [(b, j, h) for b in range(B) for j in range(n)
                                                         for h in range(Hq)]
    for b in sorted({r[0] for r in todo}):
        Kb = sequence_block(k_cache, seqlens, b, Hkv, D)
        Vb = sequence_block(v_cache, seqlens, b, Hkv, D)
        S = int(seqlens[b])
        for (j, g) in sorted({(r[1], r[2] // G) for r in todo if r[0] == b}):
            heads = [h for (bb, jj, h) in todo if bb == b and jj == j and h // G == g]
            visible = S - n + j + 1
            out[b, j, heads], lse[b, j, heads] = attention_heads_cache(qf[b, j, heads], Kb[g][:visible],
                                                                       Vb[g][:visible], scale, dtype)
    return out, lse


def gather_paged_sequence(pages, block_row, seqlen: int, n_kv_heads: int, page_size: int, head_dim: int):
    """Sequence b's [Hkv][S][D] block read through its row of the block table (reading 8):
    token t of KV head h is row t % page_size of head h in physical block block_row[t // page_size]."""
    S, Hkv, ps, D = int(seqlen), n_kv_heads, page_size, head_dim
    pages = np.asarray(pages).reshape(-1, Hkv, ps, D)
    out = np.empty((Hkv, S, D), dtype=pages.dtype)
    for t in range(S):
        out[:, t, :] = pages[int(block_row[t // ps]), :, t % ps, :]
    return out


def paged_decode_attention(q, k_pages, v_pages, block_table, seqlens: Sequence[int], page_size: int,
                           n_q_heads: int, n_kv_heads: int, head_dim: int, scale: float, dtype: str = "bf16",
                           pairs: Optional[Iterable[Tuple[int, int]]] = None):
    """Decode attention over a paged cache (reading 8): each sequence's cache is gathered through
    its block-table row, then attended exactly as decode_attention does.  block_table: [B][*]."""
    B = len(seqlens)
    Hkv, D = n_kv_heads, head_dim
    blocks = [gather_paged_sequence(k_pages, block_table[b], seqlens[b], Hkv, page_size, D) for b in range(B)]
    kc = np.concatenate([x.reshape(-1) for x in blocks]) if B else np.zeros(0, dtype=np.asarray(k_pages).dtype)
    blocks = [gather_paged_sequence(v_pages, block_table[b], seqlens[b], Hkv, page_size, D) for b in range(B)]
    vc = np.concatenate([x.reshape(-1) for x in blocks]) if B else np.zeros(0, dtype=np.asarray(v_pages).dtype)
    return decode_attention(q, kc, vc, seqlens, n_q_heads, n_kv_heads, head_dim, scale, dtype=dtype, pairs=pairs)


def shard_bounds(seqlen: int, n_shards: int, shard: int) -> Tuple[int, int]:
    """Token range [t0, t1) of shard `shard` of n_shards contiguous shards of a sequence
    (reading 9): t0 = floor(shard * S / n), t1 = floor((shard + 1) * S / n)."""
    S = int(seqlen)
    return shard * S // n_shards, (shard + 1) * S // n_shards


def merge_shard_results(outs, lses):
    """Combine the (out, lse) of every shard of one row (reading 9): each is the partial
    (lse, 1, out) in natural-log units; a fixed pairwise tree over the shards, then finalize."""
    parts = [(float(l), 1.0 if l != -math.inf else 0.0, np.asarray(o, dtype=np.float64) if l != -math.inf
              else np.zeros_like(np.asarray(o, dtype=np.float64))) for o, l in zip(outs, lses)]
    return finalize(merge_tree(parts))


def paged_multi_query_attention(q, k_pages, v_pages, block_table, seqlens: Sequence[int], page_size: int,
                                n_queries: int, n_q_heads: int, n_kv_heads: int, head_dim: int, scale: float,
                                dtype: str = "bf16", rows: Optional[Iterable[Tuple[int, int, int]]] = None):
    """Several query tokens per sequence (reading 7) over a paged cache (reading 8): each
    sequence's cache gathered through its block-table row, then multi_query_attention."""
    B, Hkv, D = len(seqlens), n_kv_heads, head_dim
    kc = np.concatenate([gather_paged_sequence(k_pages, block_table[b], seqlens[b], Hkv, page_size, D).reshape(-1)
                         for b in range(B)])
    vc = np.concatenate([gather_paged_sequence(v_pages, block_table[b], seqlens[b], Hkv, page_size, D).reshape(-1)
                         for b in range(B)])
    return multi_query_attention(q, kc, vc, seqlens, n_queries, n_q_heads, n_kv_heads, head_dim, scale, dtype=dtype,
                                 rows=rows)


def anchor_visible_keys(position: int, block_size: int) -> np.ndarray:
    """Key indices the token at `position` attends to in context encoding (reading 10): the
    anchor block's keys [0, block_size) (for blocks after the first) and its own block's keys up
    to and including itself."""
    i = position // block_size
    own = np.arange(i * block_size, position + 1)
    if i == 0:
        return own
    return np.concatenate([np.arange(block_size), own])


def anchor_block_attention(q, k, v, seq_len: int, block_size: int, n_q_heads: int, n_kv_heads: int,
                           head_dim: int, scale: float, dtype: str = "bf16",
                           rows: Optional[Iterable[Tuple[int, int]]] = None):
    """Star Attention phase 1 (context encoding with anchor blocks, reading 10) for one context.

    q: [S][Hq][D] (the S context tokens' queries, storage format); k, v: [Hkv][S][D].  Query
    head h of position p attends over KV head h // G at the keys anchor_visible_keys(p, B).
    Returns (out [S][Hq][D], lse [S][Hq]) in float64.  With `rows`, only those (p, h) entries
    are computed; the rest are NaN.
    """
    S, Hq, Hkv, D, B = int(seq_len), n_q_heads, n_kv_heads, head_dim, int(block_size)
    if Hq % Hkv != 0:
        raise ValueError("n_q_heads must be a multiple of n_kv_heads")
    if B < 1:
        raise ValueError("block_size must be positive")
    G = Hq // Hkv
    qf = to_f64(np.asarray(q).reshape(S, Hq, D), dtype)
    K = np.asarray(k).reshape(Hkv, S, D)
    V = np.asarray(v).reshape(Hkv, S, D)
    out = np.full((S, Hq, D), np.nan)
    lse = np.full((S, Hq), np.nan)
    todo = sorted(set(rows)) if rows is not None else [(p, h) for p in range(S) for h in range(Hq)]
    for p in sorted({r[0] for r in todo}):
        keys = anchor_visible_keys(p, B)
        for g in sorted({h // G for (pp, h) in todo if pp == p}):
            heads = [h for (pp, h) in todo if pp == p and h // G == g]
            out[p, heads], lse[p, heads] = attention_heads_cache(qf[p, heads], K[g][keys], V[g][keys], scale, dtype)
    return out, lse
