"""Exact split decode attention on B200 — Python binding of the C ABI in include/tree_attn.h.

Argument marshalling only: every step of the computation runs in the CUDA
kernels of ``libtree_attn.so``.  Functions take torch tensors (device memory)
or raw integer device pointers, keep the C names, and raise ``TreeAttnError``
on any status other than ``TA_OK``.  There is no CPU fallback: if the library
is missing, loading fails loudly.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence

from . import _build
from ._build import LIB, build  # noqa: F401

TA_OK, TA_ERR_INVALID_ARG, TA_ERR_UNSUPPORTED, TA_ERR_WORKSPACE, TA_ERR_CUDA, TA_ERR_TIMEOUT = range(6)
TA_ERR_SCRATCH_LIMIT = 6
TA_ERR_BAD_PAGE = 7
TA_BF16, TA_F32 = 0, 1
_DTYPES = {"bf16": TA_BF16, "f32": TA_F32}

EXPORTED = [
    "tree_attn_build_id",
    "tree_attn_profile_events",
    "tree_attn_status_string",
    "tree_attn_last_cuda_error",
    "tree_attn_workspace_size",
    "tree_attn_workspace_init",
    "tree_attn_decode",
    "tree_attn_decode_f32",
    "tree_attn_decode_ex",
    "tree_attn_decode_bifurcated",
    "tree_attn_bifurcated_workspace_size",
    "tree_attn_decode_bifurcated_ex",
    "tree_attn_check",
    "tree_attn_decode_noalloc",
    "tree_attn_noalloc_check",
    "tree_attn_multi_workspace_size",
    "tree_attn_decode_multi_ex",
    "tree_attn_decode_multi",
    "tree_attn_decode_paged_ex",
    "tree_attn_decode_paged",
    "tree_attn_merge_shards",
    "tree_attn_decode_multi_paged_ex",
    "tree_attn_anchor_prefill",
]


class TreeAttnError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        msg = f"{where}: {tree_attn_status_string(status)} (status {status})"
        if status == TA_ERR_CUDA:
            msg += f", cudaError {lib().tree_attn_last_cuda_error()}"
        super().__init__(msg)


class ta_options(ctypes.Structure):
    _fields_ = [
        ("num_ctas", ctypes.c_int32),
        ("wait_limit_us", ctypes.c_int32),
        ("debug_skip_tile", ctypes.c_int32),
        ("prefix_path", ctypes.c_int32),
        ("split_tiles", ctypes.c_int32),
        ("debug_skip_stage", ctypes.c_int32),
        ("reserved", ctypes.c_int32 * 2),
    ]


PREFIX_AUTO, PREFIX_TENSOR_CORE, PREFIX_SPLIT_KV = 0, 1, 2


TILES_AUTO, TILES_LONG, TILES_SHORT = 0, 1, 2


def make_options(num_ctas: int = 0, wait_limit_us: int = 0, debug_skip_tile: int = -1,
                 prefix_path: int = PREFIX_AUTO, split_tiles: int = TILES_AUTO,
                 debug_skip_stage: int = 0) -> ta_options:
    return ta_options(num_ctas, wait_limit_us, debug_skip_tile, prefix_path, split_tiles, debug_skip_stage,
                      (ctypes.c_int32 * 2)())


_lib = None


def lib() -> ctypes.CDLL:
    """The loaded library.  Raises if it is missing, or if it was not built from the sources in
    the tree (its build id, a hash of every source and header, differs from theirs)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB):
            raise ImportError(f"{LIB} is missing: build it with exact_long_context_split_b200.build()")
        L = ctypes.CDLL(LIB)
        L.tree_attn_build_id.argtypes = []
        L.tree_attn_build_id.restype = ctypes.c_char_p
        built, current = L.tree_attn_build_id().decode(), _build.source_hash()
        if built != current:
            raise ImportError(f"{LIB} was built from other sources (build id {built}, sources {current}): "
                              "rebuild it with exact_long_context_split_b200.build()")
        vp, i32, i64, f32, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_float, ctypes.c_size_t
        pi64 = ctypes.POINTER(ctypes.c_int64)
        popt = ctypes.POINTER(ta_options)
        psz = ctypes.POINTER(ctypes.c_size_t)
        sigs = {
            "tree_attn_status_string": ([ctypes.c_int], ctypes.c_char_p),
            "tree_attn_last_cuda_error": ([], i32),
            "tree_attn_profile_events": ([vp, vp], None),
            "tree_attn_workspace_size": ([pi64, i32, i32, i32, i32, ctypes.c_int, popt, psz], ctypes.c_int),
            "tree_attn_workspace_init": ([vp, sz, vp], ctypes.c_int),
            "tree_attn_decode": ([vp, vp, vp, pi64, i32, i32, i32, i32, f32, vp, vp, vp], ctypes.c_int),
            "tree_attn_decode_f32": ([vp, vp, vp, pi64, i32, i32, i32, i32, f32, vp, vp, vp], ctypes.c_int),
            "tree_attn_decode_ex": (
                [ctypes.c_int, vp, vp, vp, pi64, i32, i32, i32, i32, f32, vp, vp, popt, vp, sz, vp],
                ctypes.c_int,
            ),
            "tree_attn_decode_bifurcated": (
                [vp, vp, vp, i64, vp, vp, pi64, i32, i32, i32, i32, f32, vp, vp, vp],
                ctypes.c_int,
            ),
            "tree_attn_bifurcated_workspace_size": ([i64, pi64, i32, i32, i32, i32, popt, psz], ctypes.c_int),
            "tree_attn_decode_bifurcated_ex": (
                [vp, vp, vp, i64, vp, vp, pi64, i32, i32, i32, i32, f32, vp, vp, popt, vp, sz, vp],
                ctypes.c_int,
            ),
            "tree_attn_check": ([vp, vp], ctypes.c_int),
            "tree_attn_decode_noalloc": ([vp, vp, vp, pi64, i32, i32, i32, i32, f32, vp, vp, vp], ctypes.c_int),
            "tree_attn_noalloc_check": ([vp], ctypes.c_int),
            "tree_attn_multi_workspace_size": ([pi64, i32, i32, i32, i32, i32, ctypes.c_int, popt, psz], ctypes.c_int),
            "tree_attn_decode_multi_ex": (
                [ctypes.c_int, vp, vp, vp, pi64, i32, i32, i32, i32, i32, f32, vp, vp, popt, vp, sz, vp],
                ctypes.c_int,
            ),
            "tree_attn_decode_multi": ([vp, vp, vp, pi64, i32, i32, i32, i32, i32, f32, vp, vp, vp], ctypes.c_int),
            "tree_attn_decode_paged_ex": (
                [ctypes.c_int, vp, vp, vp, i64, i32, vp, i64, pi64, i32, i32, i32, i32, f32, vp, vp, popt, vp, sz, vp],
                ctypes.c_int,
            ),
            "tree_attn_merge_shards": ([vp, vp, i32, i64, i32, vp, vp, vp], ctypes.c_int),
            "tree_attn_decode_multi_paged_ex": (
                [ctypes.c_int, vp, vp, vp, i64, i32, vp, i64, pi64, i32, i32, i32, i32, i32, f32, vp, vp, popt, vp, sz,
                 vp],
                ctypes.c_int,
            ),
            "tree_attn_anchor_prefill": (
                [vp, vp, vp, i64, i64, i32, i32, i32, f32, vp, vp, popt, vp, sz, vp], ctypes.c_int),
            "tree_attn_decode_paged": (
                [vp, vp, vp, i64, i32, vp, i64, pi64, i32, i32, i32, i32, f32, vp, vp, vp], ctypes.c_int),
        }
        for name, (args, res) in sigs.items():
            fn = getattr(L, name)
            fn.argtypes = args
            fn.restype = res
        _lib = L
    return _lib


# ----------------------------------------------------------------------------------------------
# Marshalling helpers
# ----------------------------------------------------------------------------------------------


def _ptr(x) -> Optional[int]:
    if x is None:
        return None
    if isinstance(x, int):
        return x
    return x.data_ptr()


def _lens(seqlens: Sequence[int]):
    n = len(seqlens)
    arr = (ctypes.c_int64 * max(n, 1))(*[int(s) for s in seqlens])
    return arr, n


def _stream(stream, *tensors) -> Optional[int]:
    if stream is not None:
        return stream if isinstance(stream, int) else stream.cuda_stream
    for t in tensors:
        if t is not None and not isinstance(t, int) and getattr(t, "is_cuda", False):
            import torch

            return torch.cuda.current_stream(t.device).cuda_stream
    return None


def _opts(opts: Optional[ta_options]):
    return ctypes.byref(opts) if opts is not None else None


def _check(status: int, where: str) -> None:
    if status != TA_OK:
        raise TreeAttnError(status, where)


# ----------------------------------------------------------------------------------------------
# The C ABI, one Python function per entry point
# ----------------------------------------------------------------------------------------------


def tree_attn_build_id() -> str:
    """Hash of the sources and headers the loaded library was built from."""
    return lib().tree_attn_build_id().decode()


def tree_attn_profile_events(start=None, stop=None) -> None:
    """Record these CUDA events (torch.cuda.Event, recorded once so that they exist, or raw
    cudaEvent_t handles) around the main kernel of every following call on this thread; no
    arguments turns it off."""
    def handle(e):
        if e is None:
            return None
        return e if isinstance(e, int) else e.cuda_event
    lib().tree_attn_profile_events(handle(start), handle(stop))


def tree_attn_status_string(status: int) -> str:
    return lib().tree_attn_status_string(status).decode()


def tree_attn_workspace_size(seqlens, n_q_heads, n_kv_heads, head_dim, dtype="bf16", opts=None) -> int:
    arr, n = _lens(seqlens)
    out = ctypes.c_size_t(0)
    _check(lib().tree_attn_workspace_size(arr, n, n_q_heads, n_kv_heads, head_dim, _DTYPES[dtype], _opts(opts),
                                          ctypes.byref(out)), "tree_attn_workspace_size")
    return out.value


def tree_attn_workspace_init(workspace, nbytes: Optional[int] = None, stream=None) -> None:
    if nbytes is None:
        nbytes = workspace.numel() * workspace.element_size()
    _check(lib().tree_attn_workspace_init(_ptr(workspace), nbytes, _stream(stream, workspace)),
           "tree_attn_workspace_init")


def tree_attn_decode(q, k_cache, v_cache, seqlens, n_q_heads, n_kv_heads, head_dim, scale, out, lse,
                     stream=None) -> None:
    arr, n = _lens(seqlens)
    _check(lib().tree_attn_decode(_ptr(q), _ptr(k_cache), _ptr(v_cache), arr, n, n_q_heads, n_kv_heads, head_dim,
                                  scale, _ptr(out), _ptr(lse), _stream(stream, q, out)), "tree_attn_decode")


def tree_attn_decode_f32(q, k_cache, v_cache, seqlens, n_q_heads, n_kv_heads, head_dim, scale, out, lse,
                         stream=None) -> None:
    arr, n = _lens(seqlens)
    _check(lib().tree_attn_decode_f32(_ptr(q), _ptr(k_cache), _ptr(v_cache), arr, n, n_q_heads, n_kv_heads,
                                      head_dim, scale, _ptr(out), _ptr(lse), _stream(stream, q, out)),
           "tree_attn_decode_f32")


def tree_attn_decode_ex(dtype, q, k_cache, v_cache, seqlens, n_q_heads, n_kv_heads, head_dim, scale, out, lse,
                        opts, workspace, workspace_bytes: Optional[int] = None, stream=None) -> None:
    arr, n = _lens(seqlens)
    if workspace_bytes is None:
        workspace_bytes = workspace.numel() * workspace.element_size()
    _check(lib().tree_attn_decode_ex(_DTYPES[dtype], _ptr(q), _ptr(k_cache), _ptr(v_cache), arr, n, n_q_heads,
                                     n_kv_heads, head_dim, scale, _ptr(out), _ptr(lse), _opts(opts), _ptr(workspace),
                                     workspace_bytes, _stream(stream, q, out)), "tree_attn_decode_ex")


def tree_attn_decode_bifurcated(q, k_prefix, v_prefix, prefix_len, k_suffix, v_suffix, suffix_lens, n_q_heads,
                                n_kv_heads, head_dim, scale, out, lse, stream=None) -> None:
    arr, n = _lens(suffix_lens)
    _check(lib().tree_attn_decode_bifurcated(_ptr(q), _ptr(k_prefix), _ptr(v_prefix), prefix_len, _ptr(k_suffix),
                                             _ptr(v_suffix), arr, n, n_q_heads, n_kv_heads, head_dim, scale,
                                             _ptr(out), _ptr(lse), _stream(stream, q, out)),
           "tree_attn_decode_bifurcated")


def tree_attn_bifurcated_workspace_size(prefix_len, suffix_lens, n_q_heads, n_kv_heads, head_dim, opts=None) -> int:
    arr, n = _lens(suffix_lens)
    out = ctypes.c_size_t(0)
    _check(lib().tree_attn_bifurcated_workspace_size(prefix_len, arr, n, n_q_heads, n_kv_heads, head_dim,
                                                     _opts(opts), ctypes.byref(out)),
           "tree_attn_bifurcated_workspace_size")
    return out.value


def tree_attn_decode_bifurcated_ex(q, k_prefix, v_prefix, prefix_len, k_suffix, v_suffix, suffix_lens, n_q_heads,
                                   n_kv_heads, head_dim, scale, out, lse, opts, workspace,
                                   workspace_bytes: Optional[int] = None, stream=None) -> None:
    arr, n = _lens(suffix_lens)
    if workspace_bytes is None:
        workspace_bytes = workspace.numel() * workspace.element_size()
    _check(lib().tree_attn_decode_bifurcated_ex(_ptr(q), _ptr(k_prefix), _ptr(v_prefix), prefix_len, _ptr(k_suffix),
                                                _ptr(v_suffix), arr, n, n_q_heads, n_kv_heads, head_dim, scale,
                                                _ptr(out), _ptr(lse), _opts(opts), _ptr(workspace), workspace_bytes,
                                                _stream(stream, q, out)), "tree_attn_decode_bifurcated_ex")


def tree_attn_check(workspace, stream=None) -> int:
    """Synchronise the stream and return the workspace's status (TA_OK or TA_ERR_TIMEOUT); does not raise."""
    return lib().tree_attn_check(_ptr(workspace), _stream(stream, workspace))


def tree_attn_decode_noalloc(q, k_cache, v_cache, seqlens, n_q_heads, n_kv_heads, head_dim, scale, out, lse,
                             stream=None) -> None:
    """tree_attn_decode without any device allocation: the library's fixed 4 MiB scratch array
    serves as workspace (for callers that may not allocate while they run).  Calls that overlap
    on the GPU share that array and must be serialised by the caller."""
    arr, n = _lens(seqlens)
    _check(lib().tree_attn_decode_noalloc(_ptr(q), _ptr(k_cache), _ptr(v_cache), arr, n, n_q_heads, n_kv_heads,
                                          head_dim, scale, _ptr(out), _ptr(lse), _stream(stream, q, out)),
           "tree_attn_decode_noalloc")


def tree_attn_noalloc_check(stream=None) -> int:
    """Synchronise the stream and return the no-allocation scratch array's status (TA_OK or
    TA_ERR_TIMEOUT); does not raise."""
    return lib().tree_attn_noalloc_check(_stream(stream))


def tree_attn_multi_workspace_size(seqlens, n_queries, n_q_heads, n_kv_heads, head_dim, dtype="bf16",
                                   opts=None) -> int:
    arr, n = _lens(seqlens)
    out = ctypes.c_size_t(0)
    _check(lib().tree_attn_multi_workspace_size(arr, n, n_queries, n_q_heads, n_kv_heads, head_dim, _DTYPES[dtype],
                                                _opts(opts), ctypes.byref(out)), "tree_attn_multi_workspace_size")
    return out.value


def tree_attn_decode_multi_ex(dtype, q, k_cache, v_cache, seqlens, n_queries, n_q_heads, n_kv_heads, head_dim,
                              scale, out, lse, opts, workspace, workspace_bytes: Optional[int] = None,
                              stream=None) -> None:
    """n query tokens per sequence, causal among themselves: q, out [B][n][Hq][D], lse [B][n][Hq]."""
    arr, n = _lens(seqlens)
    if workspace_bytes is None:
        workspace_bytes = workspace.numel() * workspace.element_size()
    _check(lib().tree_attn_decode_multi_ex(_DTYPES[dtype], _ptr(q), _ptr(k_cache), _ptr(v_cache), arr, n, n_queries,
                                           n_q_heads, n_kv_heads, head_dim, scale, _ptr(out), _ptr(lse), _opts(opts),
                                           _ptr(workspace), workspace_bytes, _stream(stream, q, out)),
           "tree_attn_decode_multi_ex")


def tree_attn_decode_multi(q, k_cache, v_cache, seqlens, n_queries, n_q_heads, n_kv_heads, head_dim, scale, out,
                           lse, stream=None) -> None:
    arr, n = _lens(seqlens)
    _check(lib().tree_attn_decode_multi(_ptr(q), _ptr(k_cache), _ptr(v_cache), arr, n, n_queries, n_q_heads,
                                        n_kv_heads, head_dim, scale, _ptr(out), _ptr(lse), _stream(stream, q, out)),
           "tree_attn_decode_multi")


def tree_attn_decode_paged_ex(dtype, q, k_pages, v_pages, num_pages, page_size, block_table, block_table_stride,
                              seqlens, n_q_heads, n_kv_heads, head_dim, scale, out, lse, opts, workspace,
                              workspace_bytes: Optional[int] = None, stream=None) -> None:
    """Decode over a paged cache: pages [num_pages][Hkv][page_size][D], a device int32 block table."""
    arr, n = _lens(seqlens)
    if workspace_bytes is None:
        workspace_bytes = workspace.numel() * workspace.element_size()
    _check(lib().tree_attn_decode_paged_ex(_DTYPES[dtype], _ptr(q), _ptr(k_pages), _ptr(v_pages), num_pages,
                                           page_size, _ptr(block_table), block_table_stride, arr, n, n_q_heads,
                                           n_kv_heads, head_dim, scale, _ptr(out), _ptr(lse), _opts(opts),
                                           _ptr(workspace), workspace_bytes, _stream(stream, q, out)),
           "tree_attn_decode_paged_ex")


def tree_attn_decode_paged(q, k_pages, v_pages, num_pages, page_size, block_table, block_table_stride, seqlens,
                           n_q_heads, n_kv_heads, head_dim, scale, out, lse, stream=None) -> None:
    arr, n = _lens(seqlens)
    _check(lib().tree_attn_decode_paged(_ptr(q), _ptr(k_pages), _ptr(v_pages), num_pages, page_size,
                                        _ptr(block_table), block_table_stride, arr, n, n_q_heads, n_kv_heads,
                                        head_dim, scale, _ptr(out), _ptr(lse), _stream(stream, q, out)),
           "tree_attn_decode_paged")


def tree_attn_merge_shards(outs, lses, n_shards, rows, head_dim, out, lse, stream=None) -> None:
    """Merge (out, lse) computed over n_shards slices of every sequence: outs [n_shards][rows][D]."""
    _check(lib().tree_attn_merge_shards(_ptr(outs), _ptr(lses), n_shards, rows, head_dim, _ptr(out), _ptr(lse),
                                        _stream(stream, outs, out)), "tree_attn_merge_shards")


def tree_attn_decode_multi_paged_ex(dtype, q, k_pages, v_pages, num_pages, page_size, block_table,
                                    block_table_stride, seqlens, n_queries, n_q_heads, n_kv_heads, head_dim, scale,
                                    out, lse, opts, workspace, workspace_bytes: Optional[int] = None,
                                    stream=None) -> None:
    """Several query tokens per sequence over a paged cache: q, out [B][n][Hq][D]."""
    arr, n = _lens(seqlens)
    if workspace_bytes is None:
        workspace_bytes = workspace.numel() * workspace.element_size()
    _check(lib().tree_attn_decode_multi_paged_ex(_DTYPES[dtype], _ptr(q), _ptr(k_pages), _ptr(v_pages), num_pages,
                                                 page_size, _ptr(block_table), block_table_stride, arr, n, n_queries,
                                                 n_q_heads, n_kv_heads, head_dim, scale, _ptr(out), _ptr(lse),
                                                 _opts(opts), _ptr(workspace), workspace_bytes,
                                                 _stream(stream, q, out)), "tree_attn_decode_multi_paged_ex")


def tree_attn_anchor_prefill(q, k, v, seq_len, block_size, n_q_heads, n_kv_heads, head_dim, scale, out, lse,
                             opts, workspace, workspace_bytes: Optional[int] = None, stream=None) -> None:
    """Context encoding with anchor blocks: q, out [S][Hq][D], k, v [Hkv][S][D], lse [S][Hq]."""
    if workspace_bytes is None:
        workspace_bytes = workspace.numel() * workspace.element_size()
    _check(lib().tree_attn_anchor_prefill(_ptr(q), _ptr(k), _ptr(v), seq_len, block_size, n_q_heads, n_kv_heads,
                                          head_dim, scale, _ptr(out), _ptr(lse), _opts(opts), _ptr(workspace),
                                          workspace_bytes, _stream(stream, q, out)), "tree_attn_anchor_prefill")
