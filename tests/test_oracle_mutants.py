"""Planted mistakes in a copy of the oracle must each fail at least one pin (CPU only).

Each mutant is the oracle's source with one plausible slip: a dropped term, a wrong
index, a transposed operand, a wrong sign.  The mistake is planted in a private copy
of the oracle module on the CPU; the real oracle is not touched.
"""
import os
import types

import pytest

import oracle_pins

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "oracle", "attention.py")

MUTANTS = {
    "scale dropped": ("    x = scale * (K @ q)\n    m = float(np.max(x))\n    e = np.exp(x - m)\n    l = float(np.sum(e))\n    out = (e @ V) / l",
                      "    x = (K @ q)\n    m = float(np.max(x))\n    e = np.exp(x - m)\n    l = float(np.sum(e))\n    out = (e @ V) / l"),
    "K rows misaligned with V": ("    x = scale * (K @ q)\n    m = float(np.max(x))\n    e = np.exp(x - m)\n    l = float(np.sum(e))\n    out = (e @ V) / l",
                                 "    x = scale * (K[::-1] @ q)\n    m = float(np.max(x))\n    e = np.exp(x - m)\n    l = float(np.sum(e))\n    out = (e @ V) / l"),
    "normalisation dropped": ("    out = (e @ V) / l\n", "    out = (e @ V)\n"),
    "max dropped from lse": ("    return out, m + math.log(l)\n", "    return out, math.log(l)\n"),
    "log2 instead of ln": ("    return out, m + math.log(l)\n", "    return out, m + math.log2(l)\n"),
    "gqa modulo mapping": ("if bb == b and h // G == g]", "if bb == b and h % Hkv == g]"),
    "layout offset missing heads": ("* n_kv_heads * head_dim\n    S = int(seqlens[b])", "* head_dim\n    S = int(seqlens[b])"),
    "merge forgets rescale of l": ("return m, la * ca + lb * cb, oa * ca + ob * cb", "return m, la + lb, oa * ca + ob * cb"),
    "merge swaps o factors": ("return m, la * ca + lb * cb, oa * ca + ob * cb", "return m, la * ca + lb * cb, oa * cb + ob * ca"),
    "finalize skips division": ("    return o / l, m + math.log(l)", "    return o, m + math.log(l)"),
    "online drops l_old": ("        O = (O * l * carry + e @ V[t0 : t0 + block]) / l_new",
                           "        O = (O * carry + e @ V[t0 : t0 + block]) / l_new"),
    "energy sign": ("    z = scale * (K @ q) + V @ zeta", "    z = scale * (K @ q) - V @ zeta"),
    "bf16 shift": ("<< np.uint32(16)", "<< np.uint32(15)"),
    "bifurcated ignores suffix": ("            K = np.concatenate([Kp[g], Ks[g]], axis=0)\n            V = np.concatenate([Vp[g], Vs[g]], axis=0)",
                                  "            K = Kp[g]\n            V = Vp[g]"),
    "bifurcated wrong sample suffix": ("Ks = to_f64(sequence_block(k_suffix, suffix_lens, n, Hkv, D), dtype)\n        Vs = to_f64(sequence_block(v_suffix, suffix_lens, n, Hkv, D), dtype)",
                                       "Ks = to_f64(sequence_block(k_suffix, suffix_lens, 0, Hkv, D), dtype)\n        Vs = to_f64(sequence_block(v_suffix, suffix_lens, 0, Hkv, D), dtype)"),
    "multi-query mask one short": ("            visible = S - n + j + 1\n", "            visible = S - n + j\n"),
    "multi-query mask reversed": ("            visible = S - n + j + 1\n", "            visible = S - j\n"),
    "paged block index off by one": ("pages[int(block_row[t // ps]), :, t % ps, :]", "pages[int(block_row[t // ps + (t >= ps)]), :, t % ps, :]"),
    "paged rows ignore the head": ("pages[int(block_row[t // ps]), :, t % ps, :]", "pages[int(block_row[t // ps]), :1, t % ps, :]"),
    "shard bounds overlap": ("    return shard * S // n_shards, (shard + 1) * S // n_shards", "    return shard * S // n_shards, min(S, (shard + 1) * S // n_shards + 1)"),
    "shard merge ignores lse": ("    parts = [(float(l), 1.0 if l != -math.inf", "    parts = [(0.0 if l != -math.inf else l, 1.0 if l != -math.inf"),
    "pieces skip last rows": ("        acc += e[r0:r1].T @ to_f64(Vbits[r0:r1], dtype)", "        acc += e[r0:r1 - (r1 == S)].T @ to_f64(Vbits[r0:r1 - (r1 == S)], dtype)"),
    "heads' lse takes the first row's max": ("    return acc / l[:, None], m + np.log(l)", "    return acc / l[:, None], m[0] + np.log(l)"),
    "heads read each other's scores": ("    x = np.empty((S, H))\n", "    x = np.empty((S, H))\n    Q = Q[::-1]\n"),
    "paged multi-query reads table row 0": ("kc = np.concatenate([gather_paged_sequence(k_pages, block_table[b],",
                                            "kc = np.concatenate([gather_paged_sequence(k_pages, block_table[0],"),
    "paged multi-query V from K pages": ("vc = np.concatenate([gather_paged_sequence(v_pages,", "vc = np.concatenate([gather_paged_sequence(k_pages,"),
    "paged multi-query cache one row short": ("    return multi_query_attention(q, kc, vc, seqlens, n_queries,",
                                              "    return multi_query_attention(q, kc, vc, [int(s) - 1 for s in seqlens], n_queries,"),
    "anchor dropped": ("    if i == 0:\n        return own\n", "    if True:\n        return own\n"),
    "anchor is the previous block": ("np.concatenate([np.arange(block_size), own])",
                                     "np.concatenate([np.arange(max(0, i - 1) * block_size, i * block_size), own])"),
    "own block excludes itself": ("    own = np.arange(i * block_size, position + 1)", "    own = np.arange(i * block_size, position)"),
    "block index off by one": ("    i = position // block_size\n", "    i = (position + 1) // block_size\n"),
    "anchor sees the whole own block": ("    own = np.arange(i * block_size, position + 1)",
                                        "    own = np.arange(i * block_size, (i + 1) * block_size)"),
}


def _mutant(name):
    before, after = MUTANTS[name]
    src = open(SRC).read()
    assert src.count(before) == 1, f"mutation site for '{name}' not found exactly once"
    mod = types.ModuleType("oracle_mutant")
    mod.__file__ = SRC
    exec(compile(src.replace(before, after), SRC + f" [{name}]", "exec"), mod.__dict__)
    return mod


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name):
    mod = _mutant(name)
    failed = []
    for pin in oracle_pins.ALL_PINS:
        try:
            pin(mod)
        except (AssertionError, ValueError, IndexError, TypeError):
            failed.append(pin.__name__)
    assert failed, f"no pin catches the planted mistake '{name}'"


def test_unmutated_copy_passes():
    src = open(SRC).read()
    mod = types.ModuleType("oracle_copy")
    exec(compile(src, SRC, "exec"), mod.__dict__)
    for pin in oracle_pins.ALL_PINS:
        pin(mod)
