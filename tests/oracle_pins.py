"""Pins for the CPU oracle: facts fixed by the pages and by the mathematics.

Each ``pin_*`` takes an oracle module (the real one, or a copy with a planted
mistake) and raises AssertionError when the module disagrees with a fact that
does not come from the oracle itself: a closed form, an invariance, a library
routine (torch / scipy), brute force over every chunking and merge tree, a
finite-difference gradient, or the bit layout of bf16.

Sources: [AttnAccel] "Attention acceleration" concept page, Technical principles
part 1 (S = QK^T/sqrt(d_k), P = softmax(S), O = PV) and part 2.1 (online
softmax m, l and O updates); [TreeAttn] Tree Attention article, "The energy view
of attention" (attention = dF/dzeta at zeta = 0; logsumexp and max are
associative); [Bifurcated] Bifurcated attention TL;DR (two GEMMs, exact);
[StarAttn] Star Attention article, phase 2 (global attention from combined
softmax statistics).
"""
from __future__ import annotations

import itertools
import math

import numpy as np

RTOL = 1e-12


def _rng(seed):
    return np.random.default_rng(seed)


def _close(a, b, rtol=RTOL, atol=0.0, what=""):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    assert a.shape == b.shape, f"{what}: shape {a.shape} vs {b.shape}"
    if not np.allclose(a, b, rtol=rtol, atol=atol, equal_nan=False):
        err = np.max(np.abs(a - b))
        raise AssertionError(f"{what}: max abs diff {err:g} (rtol {rtol}, atol {atol})")


# --------------------------------------------------------------------------------------------
# Storage format
# --------------------------------------------------------------------------------------------


def pin_bf16_decoding(O):
    """bf16 = sign, 8-bit exponent (bias 127), 7-bit fraction: the top half of a float32."""
    bits = np.array([0x3F80, 0xC000, 0x3E80, 0x4049, 0x0001, 0x7F80, 0x8000, 0x3F81], dtype=np.uint16)
    want = [1.0, -2.0, 0.25, 3.140625, 2.0 ** -133, math.inf, -0.0, 1.0 + 2.0 ** -7]
    got = O.bf16_to_f64(bits)
    for g, w in zip(got, want):
        assert g == w, f"bf16 decode {g} != {w}"


# --------------------------------------------------------------------------------------------
# Closed forms of the definition ([AttnAccel] part 1)
# --------------------------------------------------------------------------------------------


def pin_identical_keys(O):
    """All keys equal k: softmax is uniform, out = mean_t v_t, lse = s q.k + ln S."""
    r = _rng(1)
    for S, D in [(1, 4), (7, 8), (64, 16), (300, 8)]:
        q, k = r.standard_normal(D), r.standard_normal(D)
        K = np.tile(k, (S, 1))
        V = r.standard_normal((S, D))
        s = 0.37
        out, lse = O.attention_one(q, K, V, s)
        _close(out, V.mean(axis=0), rtol=1e-12, atol=1e-14, what="identical keys out")
        _close(lse, s * float(q @ k) + math.log(S), what="identical keys lse")


def pin_dominant_key(O):
    """One score exceeds all others by >= 60: out = that row of V to e^-60, lse = its score."""
    r = _rng(2)
    S, D = 50, 8
    q = r.standard_normal(D)
    q /= np.linalg.norm(q)
    K = 0.1 * r.standard_normal((S, D))
    j = 17
    K[j] = 200.0 * q
    V = r.standard_normal((S, D))
    s = 0.5
    out, lse = O.attention_one(q, K, V, s)
    x = s * (K @ q)
    assert x[j] - np.max(np.delete(x, j)) >= 60
    _close(out, V[j], rtol=1e-20, atol=1e-20 + 60 * math.exp(-60), what="dominant key out")
    _close(lse, x[j], rtol=1e-14, what="dominant key lse")


def pin_single_key(O):
    """S = 1: out = v_0 and lse = x_0 exactly."""
    r = _rng(3)
    q, K, V = r.standard_normal(5), r.standard_normal((1, 5)), r.standard_normal((1, 5))
    out, lse = O.attention_one(q, K, V, 0.8)
    _close(out, V[0], rtol=1e-15, what="S=1 out")
    _close(lse, 0.8 * float(K[0] @ q), rtol=1e-15, what="S=1 lse")


def pin_zero_scale(O):
    """scale = 0: uniform weights, out = mean v, lse = ln S."""
    r = _rng(4)
    S, D = 33, 6
    q, K, V = r.standard_normal(D), r.standard_normal((S, D)), r.standard_normal((S, D))
    out, lse = O.attention_one(q, K, V, 0.0)
    _close(out, V.mean(axis=0), rtol=1e-12, atol=1e-15, what="scale 0 out")
    _close(lse, math.log(S), what="scale 0 lse")


def pin_constant_values(O):
    """Every v_t = c: the weights sum to one, so out = c whatever the scores."""
    r = _rng(5)
    S, D = 40, 7
    q, K = r.standard_normal(D), 3.0 * r.standard_normal((S, D))
    c = r.standard_normal(D)
    out, _ = O.attention_one(q, K, np.tile(c, (S, 1)), 0.6)
    _close(out, c, rtol=1e-13, atol=1e-15, what="constant V")


def pin_two_keys(O):
    """S = 2: out = sigmoid(x1 - x2) v1 + sigmoid(x2 - x1) v2, lse = logaddexp(x1, x2)."""
    r = _rng(6)
    D = 4
    q, K, V = r.standard_normal(D), r.standard_normal((2, D)), r.standard_normal((2, D))
    s = 1.3
    x1, x2 = s * float(K[0] @ q), s * float(K[1] @ q)
    sig = lambda z: 1.0 / (1.0 + math.exp(-z))  # noqa: E731
    out, lse = O.attention_one(q, K, V, s)
    _close(out, sig(x1 - x2) * V[0] + sig(x2 - x1) * V[1], rtol=1e-13, atol=1e-15, what="two keys out")
    _close(lse, max(x1, x2) + math.log1p(math.exp(-abs(x1 - x2))), rtol=1e-14, what="two keys lse")


def pin_library_routines(O):
    """General inputs against torch's scaled_dot_product_attention and scipy's logsumexp (float64)."""
    import scipy.special
    import torch

    r = _rng(7)
    for S, D, s in [(5, 4, 0.5), (129, 16, 0.25), (1000, 64, 0.125)]:
        q, K, V = r.standard_normal(D), r.standard_normal((S, D)), r.standard_normal((S, D))
        out, lse = O.attention_one(q, K, V, s)
        tq = torch.from_numpy(q).view(1, 1, 1, D)
        tk = torch.from_numpy(K).view(1, 1, S, D)
        tv = torch.from_numpy(V).view(1, 1, S, D)
        ref = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, scale=s).view(D).numpy()
        _close(out, ref, rtol=1e-11, atol=1e-13, what="torch sdpa")
        _close(lse, scipy.special.logsumexp(s * np.einsum("td,d->t", K, q)), rtol=1e-13, what="scipy lse")


# --------------------------------------------------------------------------------------------
# Invariances
# --------------------------------------------------------------------------------------------


def pin_permutation(O):
    """Attention is a sum over keys: permuting (k_t, v_t) pairs jointly changes nothing."""
    r = _rng(8)
    S, D = 31, 8
    q, K, V = r.standard_normal(D), r.standard_normal((S, D)), r.standard_normal((S, D))
    p = r.permutation(S)
    o1, l1 = O.attention_one(q, K, V, 0.3)
    o2, l2 = O.attention_one(q, K[p], V[p], 0.3)
    _close(o1, o2, rtol=1e-12, what="permutation out")
    _close(l1, l2, rtol=1e-13, what="permutation lse")


def pin_score_shift(O):
    """Appending component b to every key and a to q shifts every score by c = s a b:
    lse moves by exactly c, out does not move."""
    r = _rng(9)
    S, D = 20, 6
    q, K, V = r.standard_normal(D), r.standard_normal((S, D)), r.standard_normal((S, D))
    s, a, b = 0.4, 2.5, 1.5
    o1, l1 = O.attention_one(q, K, V, s)
    o2, l2 = O.attention_one(np.append(q, a), np.hstack([K, np.full((S, 1), b)]), V, s)
    _close(o1, o2, rtol=1e-12, what="shift out")
    _close(l2 - l1, s * a * b, rtol=1e-12, what="shift lse")


# --------------------------------------------------------------------------------------------
# The energy view ([TreeAttn])
# --------------------------------------------------------------------------------------------


def pin_energy_gradient(O):
    """Central differences of F(zeta) = log sum exp(s q.k_t + zeta.v_t) at zeta = 0 equal out."""
    r = _rng(10)
    for S, D in [(3, 2), (16, 4), (64, 8)]:
        q, K, V = r.standard_normal(D), r.standard_normal((S, D)), r.standard_normal((S, D))
        s = 0.7
        out, lse = O.attention_one(q, K, V, s)
        h = 1e-5
        grad = np.empty(D)
        for d in range(D):
            e = np.zeros(D)
            e[d] = h
            grad[d] = (O.energy(q, K, V, s, e) - O.energy(q, K, V, s, -e)) / (2 * h)
        _close(grad, out, rtol=0.0, atol=1e-7, what="dF/dzeta")
        _close(O.energy(q, K, V, s, np.zeros(D)), lse, rtol=1e-14, what="F(0) = lse")


# --------------------------------------------------------------------------------------------
# Chunk partials and their merge ([TreeAttn] associativity, [StarAttn] phase 2)
# --------------------------------------------------------------------------------------------


def _compositions(n, kmax):
    """Every way to cut range(n) into 1..kmax contiguous non-empty chunks, as boundary lists."""
    for k in range(1, kmax + 1):
        for cuts in itertools.combinations(range(1, n), k - 1):
            yield [0, *cuts, n]


def _all_trees(items):
    """Every binary merge tree over an ordered list of partials (Catalan many)."""
    if len(items) == 1:
        yield items[0]
        return
    for i in range(1, len(items)):
        for left in _all_trees(items[:i]):
            for right in _all_trees(items[i:]):
                yield ("node", left, right)


def _eval_tree(O, t):
    if isinstance(t, tuple) and len(t) == 3 and t[0] == "node":
        return O.merge(_eval_tree(O, t[1]), _eval_tree(O, t[2]))
    return t


def pin_merge_brute_force(O):
    """Every chunking of S <= 12 keys into <= 4 chunks, every chunk order and every merge tree
    gives the unchunked result (max and logsumexp are associative and commutative)."""
    r = _rng(11)
    for S in [1, 2, 5, 9, 12]:
        D = 3
        q, K, V = r.standard_normal(D), 2.0 * r.standard_normal((S, D)), r.standard_normal((S, D))
        s = 0.9
        ref_out, ref_lse = O.attention_one(q, K, V, s)
        for bounds in _compositions(S, 4):
            parts = [O.chunk_partial(q, K[a:b], V[a:b], s) for a, b in zip(bounds[:-1], bounds[1:])]
            for order in itertools.permutations(range(len(parts))):
                for tree in _all_trees([parts[i] for i in order]):
                    out, lse = O.finalize(_eval_tree(O, tree))
                    _close(out, ref_out, rtol=1e-13, atol=1e-15, what=f"merge S={S} {bounds}")
                    _close(lse, ref_lse, rtol=1e-13, atol=1e-15, what=f"merge lse S={S} {bounds}")
            out, lse = O.finalize(O.merge_tree(parts))
            _close(out, ref_out, rtol=1e-13, atol=1e-15, what="merge_tree")
            _close(lse, ref_lse, rtol=1e-13, atol=1e-15, what="merge_tree lse")
            out, lse = O.split_attention(q, K, V, s, bounds)
            _close(out, ref_out, rtol=1e-13, atol=1e-15, what="split_attention")


def pin_empty_chunks(O):
    """An empty chunk has (m, l, o) = (-inf, 0, 0) and is the identity of the merge;
    an empty sequence gives out = 0 and lse = -inf."""
    r = _rng(12)
    D = 4
    q, K, V = r.standard_normal(D), r.standard_normal((6, D)), r.standard_normal((6, D))
    e = O.chunk_partial(q, K[:0], V[:0], 0.5)
    assert e[0] == -math.inf and e[1] == 0.0 and np.all(e[2] == 0.0)
    p = O.chunk_partial(q, K, V, 0.5)
    for m in (O.merge(e, p), O.merge(p, e)):
        assert m[0] == p[0] and m[1] == p[1] and np.array_equal(m[2], p[2])
    out, lse = O.finalize(O.merge(e, e))
    assert lse == -math.inf and np.all(out == 0.0)
    out, lse = O.attention_one(q, K[:0], V[:0], 0.5)
    assert lse == -math.inf and np.all(out == 0.0)


def pin_online_softmax(O):
    """The block recurrence printed in [AttnAccel] 2.1 gives the two-pass result for any block size."""
    r = _rng(13)
    S, D = 97, 8
    q, K, V = r.standard_normal(D), 2.0 * r.standard_normal((S, D)), r.standard_normal((S, D))
    ref_out, ref_lse = O.attention_one(q, K, V, 0.45)
    for block in [1, 2, 7, 32, 97, 200]:
        out, lse = O.online_softmax(q, K, V, 0.45, block)
        _close(out, ref_out, rtol=1e-12, atol=1e-14, what=f"online block {block}")
        _close(lse, ref_lse, rtol=1e-13, what=f"online lse block {block}")


# --------------------------------------------------------------------------------------------
# Batch layout, GQA and the bifurcated form
# --------------------------------------------------------------------------------------------


def pin_gqa_mapping(O):
    """Hq = 4, Hkv = 2: query heads 0, 1 read KV head 0 (identical keys, so out = mean V_0) and
    heads 2, 3 read KV head 1 (constant rows c, so out = c)."""
    r = _rng(14)
    S, D = 10, 4
    k = r.standard_normal(D)
    K0, V0 = np.tile(k, (S, 1)), r.standard_normal((S, D))
    c = r.standard_normal(D)
    K1, V1 = r.standard_normal((S, D)), np.tile(c, (S, 1))
    kc = np.stack([K0, K1]).reshape(-1)
    vc = np.stack([V0, V1]).reshape(-1)
    q = r.standard_normal((1, 4, D))
    out, lse = O.decode_attention(q, kc, vc, [S], 4, 2, D, 0.5, dtype="f64")
    for h in (0, 1):
        _close(out[0, h], V0.mean(axis=0), rtol=1e-12, atol=1e-14, what=f"gqa head {h}")
        _close(lse[0, h], 0.5 * float(q[0, h] @ k) + math.log(S), what=f"gqa lse {h}")
    for h in (2, 3):
        _close(out[0, h], c, rtol=1e-12, atol=1e-14, what=f"gqa head {h}")


def pin_packed_layout(O):
    """Ragged batch [3, 0, 5, 1] packed sequence after sequence, 2 KV heads each: every
    (sequence, head) block is found where the layout puts it (closed forms per block)."""
    r = _rng(15)
    D, Hkv, Hq = 4, 2, 2
    seqlens = [3, 0, 5, 1]
    blocks_k, blocks_v, want = [], [], {}
    q = r.standard_normal((4, Hq, D))
    for b, S in enumerate(seqlens):
        for h in range(Hkv):
            c = r.standard_normal(D) + 10 * b + h
            k = r.standard_normal(D)
            blocks_k.append(np.tile(k, (S, 1)))
            blocks_v.append(np.tile(c, (S, 1)))
            want[(b, h)] = (c, 0.25 * float(q[b, h] @ k) + (math.log(S) if S else -math.inf))
    kc = np.concatenate([x.reshape(-1) for x in blocks_k])
    vc = np.concatenate([x.reshape(-1) for x in blocks_v])
    out, lse = O.decode_attention(q, kc, vc, seqlens, Hq, Hkv, D, 0.25, dtype="f64")
    for (b, h), (c, l) in want.items():
        if seqlens[b] == 0:
            assert np.all(out[b, h] == 0.0) and lse[b, h] == -math.inf, "empty sequence"
        else:
            _close(out[b, h], c, rtol=1e-13, what=f"layout out {b},{h}")
            _close(lse[b, h], l, rtol=1e-13, what=f"layout lse {b},{h}")


def pin_bifurcated(O):
    """[Bifurcated]: sample n attends over [prefix ; suffix_n].  (i) With every key identical, out
    is the mean of the P + S_n value rows of that sample; (ii) the result equals the merge of a
    prefix partial and a suffix partial formed by two separate products (the page's two GEMMs)."""
    r = _rng(16)
    D, Hkv, Hq, P = 4, 2, 4, 6
    suffix_lens = [2, 5, 1]
    N = len(suffix_lens)
    k = r.standard_normal(D)
    kp = np.tile(k, (Hkv, P, 1))
    vp = r.standard_normal((Hkv, P, D))
    ks = np.concatenate([np.tile(k, (Hkv, S, 1)).reshape(-1) for S in suffix_lens])
    vs_blocks = [r.standard_normal((Hkv, S, D)) for S in suffix_lens]
    vs = np.concatenate([x.reshape(-1) for x in vs_blocks])
    q = r.standard_normal((N, Hq, D))
    out, lse = O.bifurcated_attention(q, kp.reshape(-1), vp.reshape(-1), P, ks, vs, suffix_lens, Hq, Hkv, D,
                                      0.5, dtype="f64")
    G = Hq // Hkv
    for n in range(N):
        for h in range(Hq):
            g = h // G
            rows = np.concatenate([vp[g], vs_blocks[n][g]])
            _close(out[n, h], rows.mean(axis=0), rtol=1e-12, atol=1e-14, what=f"bifurcated mean {n},{h}")
            _close(lse[n, h], 0.5 * float(q[n, h] @ k) + math.log(P + suffix_lens[n]), what="bifurcated lse")
    # (ii) general values, two products merged
    kp = r.standard_normal((Hkv, P, D))
    ks_blocks = [r.standard_normal((Hkv, S, D)) for S in suffix_lens]
    ks = np.concatenate([x.reshape(-1) for x in ks_blocks])
    out, lse = O.bifurcated_attention(q, kp.reshape(-1), vp.reshape(-1), P, ks, vs, suffix_lens, Hq, Hkv, D,
                                      0.5, dtype="f64")
    for n in range(N):
        for h in range(Hq):
            g = h // G
            xp = 0.5 * (kp[g] @ q[n, h])
            xs = 0.5 * (ks_blocks[n][g] @ q[n, h])
            m = max(xp.max(), xs.max())
            ep, es = np.exp(xp - m), np.exp(xs - m)
            l = ep.sum() + es.sum()
            want = (ep @ vp[g] + es @ vs_blocks[n][g]) / l
            _close(out[n, h], want, rtol=1e-12, atol=1e-14, what=f"bifurcated split {n},{h}")
            _close(lse[n, h], m + math.log(l), rtol=1e-13, what="bifurcated split lse")


def pin_long_cache_pieces(O):
    """The storage-format path (cache widened in pieces) equals the definition on the whole cache,
    for bf16 and float32 storage, with a piece boundary inside the cache."""
    r = _rng(17)
    S, D = 2500, 8
    mod = getattr(O, "attention", O)  # the package keeps the setting in its submodule
    saved = mod.ROWS_PER_PIECE
    try:
        mod.ROWS_PER_PIECE = 1000
        Kf = r.standard_normal((S, D)).astype(np.float32)
        Vf = r.standard_normal((S, D)).astype(np.float32)
        q = r.standard_normal(D)
        o1, l1 = O.attention_one_bf16_cache(q, Kf, Vf, 0.3, dtype="f32")
        o2, l2 = O.attention_one(q, Kf.astype(np.float64), Vf.astype(np.float64), 0.3)
        _close(o1, o2, rtol=1e-12, atol=1e-15, what="pieces f32")
        _close(l1, l2, rtol=1e-14, what="pieces f32 lse")
        Kb = (Kf.view(np.uint32) >> 16).astype(np.uint16)
        Vb = (Vf.view(np.uint32) >> 16).astype(np.uint16)
        o1, l1 = O.attention_one_bf16_cache(q, Kb, Vb, 0.3, dtype="bf16")
        o2, l2 = O.attention_one(q, O.bf16_to_f64(Kb), O.bf16_to_f64(Vb), 0.3)
        _close(o1, o2, rtol=1e-12, atol=1e-15, what="pieces bf16")
        # several query rows in one pass: each row is the definition applied to that row alone
        Q = r.standard_normal((3, D))
        Q[2] = -2.0 * Q[0]
        oh, lh = O.attention_heads_cache(Q, Kb, Vb, 0.3, dtype="bf16")
        for h in range(3):
            o2, l2 = O.attention_one(Q[h], O.bf16_to_f64(Kb), O.bf16_to_f64(Vb), 0.3)
            _close(oh[h], o2, rtol=1e-12, atol=1e-15, what=f"pieces bf16 row {h}")
            _close(lh[h], l2, rtol=1e-14, what=f"pieces bf16 lse row {h}")
    finally:
        mod.ROWS_PER_PIECE = saved


def pin_multi_query(O):
    """[StarAttn] query tokens attend to all preceding context (reading 7).  (i) A masked score
    matrix built independently (the n x S scores of all query tokens with -inf above the
    staircase from np.triu, row softmax by exp / sum) gives every row; (ii) with identical keys
    query j's out is the mean of its S - n + j + 1 visible value rows and lse = s q.k + ln of
    that count; (iii) one query per sequence is plain decode of the whole cache."""
    r = _rng(21)
    D, Hkv, Hq, n = 4, 2, 4, 3
    seqlens = [3, 7, 5]
    G = Hq // Hkv
    B = len(seqlens)
    kb = [r.standard_normal((Hkv, S, D)) for S in seqlens]
    vb = [r.standard_normal((Hkv, S, D)) for S in seqlens]
    k = np.concatenate([x.reshape(-1) for x in kb])
    v = np.concatenate([x.reshape(-1) for x in vb])
    q = r.standard_normal((B, n, Hq, D))
    out, lse = O.multi_query_attention(q, k, v, seqlens, n, Hq, Hkv, D, 0.7, dtype="f64")
    for b, S in enumerate(seqlens):
        # query token j is cache position S - n + j; key t is hidden from it when t > S - n + j
        hidden = np.triu(np.ones((n, S), dtype=bool), k=S - n + 1)
        for h in range(Hq):
            g = h // G
            X = 0.7 * (q[b, :, h, :] @ kb[b][g].T)
            X[hidden] = -np.inf
            mx = X.max(axis=1, keepdims=True)
            E = np.exp(X - mx)
            L = E.sum(axis=1)
            want = (E @ vb[b][g]) / L[:, None]
            _close(out[b, :, h], want, rtol=1e-12, atol=1e-14, what=f"multi-query rows {b},{h}")
            _close(lse[b, :, h], mx[:, 0] + np.log(L), rtol=1e-13, what=f"multi-query lse {b},{h}")
    # (ii) identical keys: the visible count decides both outputs
    kc = r.standard_normal(D)
    k_same = np.concatenate([np.tile(kc, (Hkv, S, 1)).reshape(-1) for S in seqlens])
    out, lse = O.multi_query_attention(q, k_same, v, seqlens, n, Hq, Hkv, D, 0.7, dtype="f64")
    for b, S in enumerate(seqlens):
        for j in range(n):
            cnt = S - n + j + 1
            for h in range(Hq):
                g = h // G
                _close(out[b, j, h], vb[b][g][:cnt].mean(axis=0), rtol=1e-12, atol=1e-14,
                       what=f"multi-query mean {b},{j},{h}")
                _close(lse[b, j, h], 0.7 * float(q[b, j, h] @ kc) + math.log(cnt), rtol=1e-13,
                       what="multi-query lse count")
    # (iii) n = 1 over the whole cache, against the textbook formula
    out1, lse1 = O.multi_query_attention(q[:, :1], k, v, seqlens, 1, Hq, Hkv, D, 0.7, dtype="f64")
    for b, S in enumerate(seqlens):
        for h in range(Hq):
            x = 0.7 * (kb[b][h // G] @ q[b, 0, h])
            e = np.exp(x - x.max())
            _close(out1[b, 0, h], (e @ vb[b][h // G]) / e.sum(), rtol=1e-12, atol=1e-14, what="n = 1")
            _close(lse1[b, 0, h], x.max() + math.log(e.sum()), rtol=1e-13, what="n = 1 lse")


def pin_paged_cache(O):
    """[AttnAccel] part 3 (reading 8): a contiguous cache scattered into pages through a random
    block table (numpy fancy indexing, page by page, independent of the oracle's token loop)
    gives back every sequence's cache, and paged decode then equals decode of the contiguous
    cache; two sequences whose tables share their first blocks see the same prefix rows."""
    r = _rng(23)
    D, Hkv, Hq, ps = 4, 2, 4, 4
    seqlens = [9, 4, 13, 1]
    blocks_per = [-(-S // ps) for S in seqlens]
    n_pages = sum(blocks_per) + 3
    perm = r.permutation(n_pages)
    table = np.full((len(seqlens), max(blocks_per)), -1, dtype=np.int64)
    pages_k = r.standard_normal((n_pages, Hkv, ps, D))
    pages_v = r.standard_normal((n_pages, Hkv, ps, D))
    caches_k, caches_v = [], []
    used = 0
    for b, S in enumerate(seqlens):
        kb = r.standard_normal((Hkv, S, D))
        vb = r.standard_normal((Hkv, S, D))
        caches_k.append(kb)
        caches_v.append(vb)
        for i in range(blocks_per[b]):
            p = int(perm[used])
            used += 1
            table[b, i] = p
            n = min(ps, S - i * ps)
            pages_k[p, :, :n, :] = kb[:, i * ps:i * ps + n, :]
            pages_v[p, :, :n, :] = vb[:, i * ps:i * ps + n, :]
    for b, S in enumerate(seqlens):
        got = O.gather_paged_sequence(pages_k.reshape(-1), table[b], S, Hkv, ps, D)
        _close(got, caches_k[b], rtol=0.0, what=f"gathered cache {b}")
    q = r.standard_normal((len(seqlens), Hq, D))
    out, lse = O.paged_decode_attention(q, pages_k.reshape(-1), pages_v.reshape(-1), table, seqlens, ps, Hq, Hkv, D,
                                        0.6, dtype="f64")
    G = Hq // Hkv
    for b, S in enumerate(seqlens):
        for h in range(Hq):
            x = 0.6 * (caches_k[b][h // G] @ q[b, h])
            e = np.exp(x - x.max())
            _close(out[b, h], (e @ caches_v[b][h // G]) / e.sum(), rtol=1e-12, atol=1e-14, what=f"paged {b},{h}")
            _close(lse[b, h], x.max() + math.log(e.sum()), rtol=1e-13, what=f"paged lse {b},{h}")
    # shared prefix blocks: sequence 1 reuses sequence 0's first block
    shared = table.copy()
    shared[1, 0] = table[0, 0]
    g0 = O.gather_paged_sequence(pages_v.reshape(-1), shared[0], seqlens[0], Hkv, ps, D)
    g1 = O.gather_paged_sequence(pages_v.reshape(-1), shared[1], seqlens[1], Hkv, ps, D)
    _close(g1[:, :ps], g0[:, :ps], rtol=0.0, what="shared block")


def pin_sharded_decode(O):
    """[TreeAttn] across devices (reading 9): a cache cut into W contiguous shards (some empty),
    each shard's own attention (out, lse) merged by merge_shard_results equals the textbook
    attention over the whole cache; the shard bounds tile [0, S) exactly."""
    r = _rng(27)
    D = 5
    for S, W in ((11, 3), (3, 4), (16, 8), (1, 2)):
        bounds = [O.shard_bounds(S, W, i) for i in range(W)]
        assert bounds[0][0] == 0 and bounds[-1][1] == S
        assert all(bounds[i][1] == bounds[i + 1][0] for i in range(W - 1))
        K = r.standard_normal((S, D))
        V = r.standard_normal((S, D))
        q = r.standard_normal(D)
        outs, lses = [], []
        for t0, t1 in bounds:
            x = 0.9 * (K[t0:t1] @ q)
            if t1 == t0:
                outs.append(np.zeros(D))
                lses.append(-math.inf)
                continue
            e = np.exp(x - x.max())
            outs.append((e @ V[t0:t1]) / e.sum())
            lses.append(x.max() + math.log(e.sum()))
        out, lse = O.merge_shard_results(outs, lses)
        x = 0.9 * (K @ q)
        e = np.exp(x - x.max())
        _close(out, (e @ V) / e.sum(), rtol=1e-12, atol=1e-14, what=f"sharded out S={S} W={W}")
        _close(lse, x.max() + math.log(e.sum()), rtol=1e-13, what=f"sharded lse S={S} W={W}")


def pin_paged_multi_query(O):
    """[AttnAccel] part 3 with reading 7: several query tokens over a paged cache.  Contiguous
    caches are scattered into pages through a random block table with plain numpy fancy
    indexing (whole pages at once); every row must equal a staircase-masked softmax written
    here from the contiguous cache (scores of all n query tokens, -inf above the staircase,
    row softmax).  Two sequences whose tables share their first block read the same rows."""
    r = _rng(31)
    D, Hkv, Hq, ps, n = 4, 2, 4, 4, 3
    seqlens = [9, 3, 14, 5]
    G, B = Hq // Hkv, len(seqlens)
    nblk = [-(-S // ps) for S in seqlens]
    n_pages = sum(nblk) + 2
    perm = r.permutation(n_pages)
    table = np.zeros((B, max(nblk)), dtype=np.int64)
    pk = np.full((n_pages, Hkv, ps, D), np.nan)
    pv = np.full((n_pages, Hkv, ps, D), np.nan)
    kb, vb = [], []
    used = 0
    for b, S in enumerate(seqlens):
        kk = r.standard_normal((Hkv, nblk[b] * ps, D))
        vv = r.standard_normal((Hkv, nblk[b] * ps, D))
        kk[:, S:] = np.nan  # rows past the sequence never enter the result
        vv[:, S:] = np.nan
        kb.append(kk[:, :S])
        vb.append(vv[:, :S])
        table[b, :nblk[b]] = perm[used:used + nblk[b]]
        used += nblk[b]
        pk[table[b, :nblk[b]]] = kk.reshape(Hkv, nblk[b], ps, D).transpose(1, 0, 2, 3)
        pv[table[b, :nblk[b]]] = vv.reshape(Hkv, nblk[b], ps, D).transpose(1, 0, 2, 3)
    q = r.standard_normal((B, n, Hq, D))
    out, lse = O.paged_multi_query_attention(q, pk.reshape(-1), pv.reshape(-1), table, seqlens, ps, n, Hq, Hkv, D,
                                             0.8, dtype="f64")
    for b, S in enumerate(seqlens):
        hidden = np.triu(np.ones((n, S), dtype=bool), k=S - n + 1)
        for h in range(Hq):
            X = 0.8 * (q[b, :, h, :] @ kb[b][h // G].T)
            X[hidden] = -np.inf
            mx = X.max(axis=1, keepdims=True)
            E = np.exp(X - mx)
            L = E.sum(axis=1)
            _close(out[b, :, h], (E @ vb[b][h // G]) / L[:, None], rtol=1e-12, atol=1e-14,
                   what=f"paged multi-query {b},{h}")
            _close(lse[b, :, h], mx[:, 0] + np.log(L), rtol=1e-13, what=f"paged multi-query lse {b},{h}")
    # sequence 1 shares sequence 0's first block: its rows are sequence 0's first rows
    shared = table.copy()
    shared[1, 0] = table[0, 0]
    lens = [ps, ps]
    q2 = np.repeat(q[:1, :1], 2, axis=0)
    o2, l2 = O.paged_multi_query_attention(q2, pk.reshape(-1), pv.reshape(-1), shared[:2], lens, ps, 1, Hq, Hkv, D,
                                           0.8, dtype="f64")
    _close(o2[1], o2[0], rtol=0.0, what="shared first block")
    _close(l2[1], l2[0], rtol=0.0, what="shared first block lse")


def pin_anchor_blocks(O):
    """[StarAttn] phase 1 (reading 10) as the page describes it: each block after the first is
    prefixed with the anchor block and the host runs ordinary causal attention over that
    augmented sequence, keeping the rows of its own block.  Computed here with torch's
    scaled_dot_product_attention (is_causal) per augmented block; the first block is causal
    attention over itself.  Also: a block at least as long as the context is plain causal
    attention, and with identical keys every row is the mean of its visible value rows."""
    import torch

    r = _rng(33)
    D, Hkv, Hq = 8, 2, 4
    G = Hq // Hkv
    for S, Bsz in ((23, 6), (16, 4), (9, 9), (7, 20)):
        q = r.standard_normal((S, Hq, D))
        k = r.standard_normal((Hkv, S, D))
        v = r.standard_normal((Hkv, S, D))
        out, lse = O.anchor_block_attention(q, k.reshape(-1), v.reshape(-1), S, Bsz, Hq, Hkv, D, 0.45, dtype="f64")
        for i0 in range(0, S, Bsz):
            i1 = min(S, i0 + Bsz)
            idx = np.arange(i0, i1) if i0 == 0 else np.concatenate([np.arange(min(Bsz, S)), np.arange(i0, i1)])
            keep = slice(len(idx) - (i1 - i0), len(idx))
            for h in range(Hq):
                g = h // G
                tq = torch.from_numpy(q[idx, h, :]).view(1, 1, len(idx), D)
                tk = torch.from_numpy(k[g][idx]).view(1, 1, len(idx), D)
                tv = torch.from_numpy(v[g][idx]).view(1, 1, len(idx), D)
                ref = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, is_causal=True, scale=0.45)
                _close(out[i0:i1, h], ref.view(len(idx), D).numpy()[keep], rtol=1e-11, atol=1e-13,
                       what=f"anchor S={S} B={Bsz} block {i0} head {h}")
                X = 0.45 * (q[idx, h, :] @ k[g][idx].T)
                X[np.triu(np.ones((len(idx), len(idx)), dtype=bool), k=1)] = -np.inf
                import scipy.special
                _close(lse[i0:i1, h], scipy.special.logsumexp(X, axis=1)[keep], rtol=1e-13,
                       what=f"anchor lse S={S} B={Bsz} block {i0} head {h}")
        if Bsz >= S:  # one block: plain causal attention
            for h in range(Hq):
                X = 0.45 * (q[:, h, :] @ k[h // G].T)
                X[np.triu(np.ones((S, S), dtype=bool), k=1)] = -np.inf
                E = np.exp(X - X.max(axis=1, keepdims=True))
                _close(out[:, h], (E @ v[h // G]) / E.sum(axis=1, keepdims=True), rtol=1e-12, atol=1e-14,
                       what="one block is causal attention")
    # identical keys: out = mean of the visible value rows, lse = s q.k + ln(count)
    S, Bsz = 13, 4
    kc = r.standard_normal(D)
    k = np.tile(kc, (Hkv, S, 1))
    v = r.standard_normal((Hkv, S, D))
    q = r.standard_normal((S, Hq, D))
    out, lse = O.anchor_block_attention(q, k.reshape(-1), v.reshape(-1), S, Bsz, Hq, Hkv, D, 0.3, dtype="f64")
    for p in range(S):
        i = p // Bsz
        vis = list(range(i * Bsz, p + 1)) if i == 0 else list(range(Bsz)) + list(range(i * Bsz, p + 1))
        for h in range(Hq):
            _close(out[p, h], v[h // G][vis].mean(axis=0), rtol=1e-12, atol=1e-14, what=f"anchor mean {p},{h}")
            _close(lse[p, h], 0.3 * float(q[p, h] @ kc) + math.log(len(vis)), rtol=1e-13, what=f"anchor count {p}")


ALL_PINS = [
    pin_bf16_decoding,
    pin_identical_keys,
    pin_dominant_key,
    pin_single_key,
    pin_zero_scale,
    pin_constant_values,
    pin_two_keys,
    pin_library_routines,
    pin_permutation,
    pin_score_shift,
    pin_energy_gradient,
    pin_merge_brute_force,
    pin_empty_chunks,
    pin_online_softmax,
    pin_gqa_mapping,
    pin_packed_layout,
    pin_bifurcated,
    pin_long_cache_pieces,
    pin_multi_query,
    pin_paged_cache,
    pin_sharded_decode,
    pin_paged_multi_query,
    pin_anchor_blocks,
]
