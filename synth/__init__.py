"""Seeded synthetic inputs for split decode attention.

A module of its own: it serves the tests, the benchmark and the CPU oracle's
callers alike and holds none of the attention arithmetic.  Every tensor is a
pure function of (seed, tensor id, element index) computed by ``gen.c``
(SplitMix64 words, Box-Muller normals, round-to-nearest-even to float32 and
then to bf16), so a slice can be rebuilt on its own.

Layouts (shared with the C ABI of the library under test):

* ``q``       ``[B][Hq][D]``
* ``k``, ``v`` packed per sequence: sequence ``b`` is a ``[Hkv][S_b][D]`` block,
  blocks stored back to back in batch order (one flat array).
* bf16 tensors are carried on the host as ``numpy.uint16`` bit patterns.
"""
from __future__ import annotations

import ctypes
import dataclasses
import math
import os
import subprocess
from typing import Dict, List, Optional, Sequence

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "gen.c")
_LIB = os.path.join(_HERE, "libsynth.so")

# Tensor ids of the counter-based streams.
TID_Q, TID_K, TID_V, TID_SPIKE, TID_K_SUFFIX, TID_V_SUFFIX, TID_PAGES = 0, 1, 2, 3, 4, 5, 6


def build(force: bool = False) -> str:
    """Compile gen.c into libsynth.so next to it (plain C, OpenMP)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        subprocess.check_call(
            ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-ffp-contract=off", "-o", _LIB, _SRC, "-lm"]
        )
    return _LIB


_lib = None


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB)
        u64, u32, i64, i32 = ctypes.c_uint64, ctypes.c_uint32, ctypes.c_int64, ctypes.c_int32
        vp = ctypes.c_void_p
        lib.synth_word.argtypes = [u64, u32, u64]
        lib.synth_word.restype = u64
        lib.synth_normal_bf16.argtypes = [u64, u32, u64, u64, vp]
        lib.synth_normal_bf16.restype = None
        lib.synth_normal_f32.argtypes = [u64, u32, u64, u64, vp]
        lib.synth_normal_f32.restype = None
        lib.synth_spike_rows_bf16.argtypes = [u64, u32, u64, vp, i64, i32, i64, ctypes.c_float, vp]
        lib.synth_spike_rows_bf16.restype = ctypes.c_int
        _lib = lib
    return _lib


def word(seed: int, tid: int, index: int) -> int:
    return int(_load().synth_word(seed, tid, index))


def normal_bf16(seed: int, tid: int, n: int, start: int = 0, out: Optional[np.ndarray] = None) -> np.ndarray:
    """n ~N(0,1) values of stream (seed, tid) from element `start`, as bf16 bit patterns."""
    if out is None:
        out = np.empty(n, dtype=np.uint16)
    assert out.dtype == np.uint16 and out.flags.c_contiguous and out.size == n
    if n:
        _load().synth_normal_bf16(seed, tid, start, n, out.ctypes.data)
    return out


def normal_f32(seed: int, tid: int, n: int, start: int = 0, out: Optional[np.ndarray] = None) -> np.ndarray:
    if out is None:
        out = np.empty(n, dtype=np.float32)
    assert out.dtype == np.float32 and out.flags.c_contiguous and out.size == n
    if n:
        _load().synth_normal_f32(seed, tid, start, n, out.ctypes.data)
    return out


def spike_rows_bf16(mat: np.ndarray, seed: int, stream: int, n_spikes: int, factor: float = 4.0) -> np.ndarray:
    """Scale exactly `n_spikes` seeded distinct rows of a C-contiguous [rows][dim] bf16 matrix in place."""
    assert mat.dtype == np.uint16 and mat.ndim == 2 and mat.flags.c_contiguous
    chosen = np.empty(max(n_spikes, 1), dtype=np.int64)
    rc = _load().synth_spike_rows_bf16(
        seed, TID_SPIKE, stream, mat.ctypes.data, mat.shape[0], mat.shape[1], n_spikes, factor, chosen.ctypes.data
    )
    if rc != 0:
        raise ValueError("spike_rows_bf16: bad arguments")
    return chosen[:n_spikes]


def bf16_bits_from_f32(a: np.ndarray) -> np.ndarray:
    """Round float32 values to bf16 (nearest even) and return the bit patterns."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return u.astype(np.uint16)


# --------------------------------------------------------------------------------------------
# Workload recipes
# --------------------------------------------------------------------------------------------


@dataclasses.dataclass(frozen=True)
class DecodeSpec:
    """One decode step: B sequences, n_queries query tokens per (sequence, query head) (the
    last n_queries cache rows are those tokens' keys and values)."""

    name: str
    seqlens: Sequence[int]
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    dtype: str = "bf16"  # "bf16" or "f32" for q, K and V
    seed: int = 0
    spike_frac: float = 0.0  # fraction of keys per KV head scaled by spike_factor
    spike_factor: float = 4.0
    scale_value: Optional[float] = None  # softmax scale; default 1/sqrt(head_dim) rounded to float32
    n_queries: int = 1
    page_size: int = 0  # > 0: the cache is paged (blocks of page_size tokens, seeded placement)

    @property
    def batch(self) -> int:
        return len(self.seqlens)

    @property
    def scale(self) -> float:
        if self.scale_value is not None:
            return float(np.float32(self.scale_value))
        return float(np.float32(1.0 / math.sqrt(self.head_dim)))

    @property
    def elem_bytes(self) -> int:
        return 2 if self.dtype == "bf16" else 4

    def n_spikes(self, seqlen: int) -> int:
        return int(round(self.spike_frac * seqlen))

    @property
    def kv_elems(self) -> int:
        return sum(self.seqlens) * self.n_kv_heads * self.head_dim

    @property
    def kv_bytes(self) -> int:
        """Algorithmic bytes of one step: every K and V element read once."""
        return 2 * self.kv_elems * self.elem_bytes

    @property
    def tokens(self) -> int:
        return int(sum(self.seqlens))


@dataclasses.dataclass(frozen=True)
class BifurcatedSpec:
    """Shared-prefix sampling: N samples share one prefix cache and own a private suffix each."""

    name: str
    prefix_len: int
    suffix_lens: Sequence[int]
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    seed: int = 0

    @property
    def n_samples(self) -> int:
        return len(self.suffix_lens)

    @property
    def scale(self) -> float:
        return float(np.float32(1.0 / math.sqrt(self.head_dim)))

    @property
    def kv_bytes(self) -> int:
        return 2 * 2 * self.n_kv_heads * self.head_dim * (self.prefix_len + sum(self.suffix_lens))


def decode_configs() -> Dict[str, DecodeSpec]:
    """The decode workloads at full size."""
    M = 1_048_576
    return {
        "tiny": DecodeSpec("tiny", [4096], 1, 1, 64, dtype="f32", seed=1),
        "llama3_8b_gqa": DecodeSpec("llama3_8b_gqa", [32768] * 8, 32, 8, 128, seed=2),
        "long_1m": DecodeSpec("long_1m", [M], 32, 8, 128, seed=3, spike_frac=0.001),
        "extreme_5m": DecodeSpec("extreme_5m", [5_120_000], 32, 8, 128, seed=4),
        "extreme_ragged": DecodeSpec("extreme_ragged", [5_120_000, M, 262_144, 4096], 32, 8, 128, seed=4),
    }


def gqa8_configs() -> Dict[str, DecodeSpec]:
    """Decode with 8 query heads per KV head (Llama-3-70B-shaped: 64 query heads, 8 KV heads,
    head_dim 128) over long_1m's recipe: 1,048,576 tokens, bf16, 0.1% of keys scaled x4."""
    return {"long_1m_g8": DecodeSpec("long_1m_g8", [1_048_576], 64, 8, 128, seed=12, spike_frac=0.001)}


def multi_query_configs() -> Dict[str, DecodeSpec]:
    """Several query tokens per sequence (speculative decode verifying draft tokens): the
    32K x 8 batch of llama3_8b_gqa with 2 and with 4 query tokens per sequence."""
    return {
        "spec_decode_2": DecodeSpec("spec_decode_2", [32768] * 8, 32, 8, 128, seed=7, n_queries=2),
        "spec_decode_4": DecodeSpec("spec_decode_4", [32768] * 8, 32, 8, 128, seed=8, n_queries=4),
    }


def capture_configs():
    """Smaller versions of workloads for profiler captures: the long-context decode at 1/4 of the
    length (same recipe, 1.07 GB of K/V, still far larger than the 126 MB L2), and context
    encoding over 8K tokens in 2K blocks."""
    return {"long_256k": DecodeSpec("long_256k", [262_144], 32, 8, 128, seed=3, spike_frac=0.001),
            "star_prefill_8k": AnchorSpec("star_prefill_8k", 8_192, 2_048, 32, 8, 128, seed=11)}


def bifurcated_configs() -> Dict[str, BifurcatedSpec]:
    return {"shared_prefix": BifurcatedSpec("shared_prefix", 65_536, [256] * 64, 32, 8, 128, seed=5)}


def make_decode_inputs(spec: DecodeSpec) -> Dict[str, np.ndarray]:
    """Host buffers for one decode step (bf16 as uint16 bits, f32 as float32)."""
    B, Hq, Hkv, D = spec.batch, spec.n_q_heads, spec.n_kv_heads, spec.head_dim
    n = spec.n_queries
    nq = B * n * Hq * D
    if spec.dtype == "bf16":
        q = normal_bf16(spec.seed, TID_Q, nq)
        k = normal_bf16(spec.seed, TID_K, spec.kv_elems)
        v = normal_bf16(spec.seed, TID_V, spec.kv_elems)
    elif spec.dtype == "f32":
        q = normal_f32(spec.seed, TID_Q, nq)
        k = normal_f32(spec.seed, TID_K, spec.kv_elems)
        v = normal_f32(spec.seed, TID_V, spec.kv_elems)
    else:
        raise ValueError(spec.dtype)
    spikes: List[np.ndarray] = []
    if spec.spike_frac > 0:
        if spec.dtype != "bf16":
            raise ValueError("spikes are defined for bf16 caches")
        off = 0
        for b, S in enumerate(spec.seqlens):
            for h in range(Hkv):
                rows = k[off : off + S * D].reshape(S, D)
                spikes.append(spike_rows_bf16(rows, spec.seed, b * Hkv + h, spec.n_spikes(S), spec.spike_factor))
                off += S * D
    return {
        "q": q.reshape(B, Hq, D) if n == 1 else q.reshape(B, n, Hq, D),
        "k": k,
        "v": v,
        "seqlens": np.asarray(spec.seqlens, dtype=np.int64),
        "spikes": spikes,
    }


def page_table(seed: int, seqlens: Sequence[int], page_size: int, spare: int = 0):
    """Block table placing each logical block of each sequence in a distinct physical block, in a
    seeded random order, with `spare` physical blocks left unused.  Returns (table [B][max
    blocks] int32, number of physical blocks)."""
    blocks = [-(-int(S) // page_size) for S in seqlens]
    n = sum(blocks) + spare
    perm = np.random.default_rng([seed, TID_PAGES]).permutation(n).astype(np.int32)
    table = np.zeros((len(seqlens), max([1] + blocks)), dtype=np.int32)
    used = 0
    for b, nb in enumerate(blocks):
        table[b, :nb] = perm[used:used + nb]
        used += nb
    return table, n


def scatter_pages(cache, seqlens: Sequence[int], n_kv_heads: int, head_dim: int, page_size: int, table,
                  num_pages: int, fill):
    """Lay a packed cache ([Hkv][S_b][D] blocks back to back) out as physical blocks
    [num_pages][Hkv][page_size][D] through `table`; rows no token maps to hold `fill`."""
    Hkv, D, ps = n_kv_heads, head_dim, page_size
    pages = np.full((num_pages, Hkv, ps, D), fill, dtype=cache.dtype)
    off = 0
    for b, S in enumerate(seqlens):
        S = int(S)
        blk = cache[off:off + Hkv * S * D].reshape(Hkv, S, D)
        off += Hkv * S * D
        for i in range(-(-S // ps)):
            n = min(ps, S - i * ps)
            pages[table[b, i], :, :n, :] = blk[:, i * ps:i * ps + n, :]
    return pages


def paged_configs() -> Dict[str, DecodeSpec]:
    """long_1m's cache, and spec_decode_4's, in 16-token blocks placed at random (the common
    serving block size)."""
    return {"long_1m_paged": DecodeSpec("long_1m_paged", [1_048_576], 32, 8, 128, seed=3, spike_frac=0.001,
                                        page_size=16),
            "spec_decode_4_paged": DecodeSpec("spec_decode_4_paged", [32768] * 8, 32, 8, 128, seed=8, n_queries=4,
                                              page_size=16)}


def make_bifurcated_inputs(spec: BifurcatedSpec) -> Dict[str, np.ndarray]:
    N, Hq, Hkv, D, P = spec.n_samples, spec.n_q_heads, spec.n_kv_heads, spec.head_dim, spec.prefix_len
    n_suffix = sum(spec.suffix_lens) * Hkv * D
    return {
        "q": normal_bf16(spec.seed, TID_Q, N * Hq * D).reshape(N, Hq, D),
        "k_prefix": normal_bf16(spec.seed, TID_K, Hkv * P * D),
        "v_prefix": normal_bf16(spec.seed, TID_V, Hkv * P * D),
        "k_suffix": normal_bf16(spec.seed, TID_K_SUFFIX, n_suffix),
        "v_suffix": normal_bf16(spec.seed, TID_V_SUFFIX, n_suffix),
        "suffix_lens": np.asarray(spec.suffix_lens, dtype=np.int64),
    }


@dataclasses.dataclass(frozen=True)
class AnchorSpec:
    """Context encoding with anchor blocks: one context of seq_len tokens in blocks of
    block_size, every block after the first prefixed with the first (anchor) block."""

    name: str
    seq_len: int
    block_size: int
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    seed: int = 0

    @property
    def scale(self) -> float:
        return float(np.float32(1.0 / math.sqrt(self.head_dim)))

    @property
    def visible_keys(self) -> int:
        """Sum over positions of the keys each one attends to (anchor block plus its own block up
        to itself; the first block has no anchor)."""
        S, B = self.seq_len, self.block_size
        total = 0
        for i0 in range(0, S, B):
            L = min(B, S - i0)
            total += L * (B if i0 > 0 else 0) + L * (L + 1) // 2
        return total

    @property
    def flops(self) -> int:
        """Algorithmic FLOPs: for every (position, query head) and visible key, a D-long dot
        product for the score and a D-long multiply-add for the output (2 D each)."""
        return 4 * self.head_dim * self.n_q_heads * self.visible_keys

    @property
    def kv_bytes(self) -> int:
        return 2 * 2 * self.n_kv_heads * self.seq_len * self.head_dim


def anchor_configs() -> Dict[str, AnchorSpec]:
    """Llama-3-8B-shaped context encoding (32/8 heads, head_dim 128) with the block a quarter of
    the context: 32K tokens in 8K blocks, and 128K tokens in 32K blocks."""
    return {
        "star_prefill_32k": AnchorSpec("star_prefill_32k", 32_768, 8_192, 32, 8, 128, seed=9),
        "star_prefill_128k": AnchorSpec("star_prefill_128k", 131_072, 32_768, 32, 8, 128, seed=10),
    }


def make_anchor_inputs(spec: AnchorSpec) -> Dict[str, np.ndarray]:
    """q [S][Hq][D], k and v [Hkv][S][D], bf16 bits, ~N(0,1)."""
    S, Hq, Hkv, D = spec.seq_len, spec.n_q_heads, spec.n_kv_heads, spec.head_dim
    return {
        "q": normal_bf16(spec.seed, TID_Q, S * Hq * D).reshape(S, Hq, D),
        "k": normal_bf16(spec.seed, TID_K, Hkv * S * D),
        "v": normal_bf16(spec.seed, TID_V, Hkv * S * D),
    }
