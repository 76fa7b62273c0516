"""The C ABI without a GPU: the library loads, exports every declared entry point, and
rejects bad arguments with the documented status before any CUDA call (CPU only)."""
import ctypes
import math
import os
import re

import pytest

import exact_long_context_split_b200 as ta

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "tree_attn.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?\w+\**\s+\**(tree_attn_\w+)\s*\(", text, flags=re.M)))


def test_library_exports_every_declared_symbol():
    ta.build()
    L = ta.lib()
    names = declared_functions()
    assert len(names) >= 11, names
    for n in names:
        assert hasattr(L, n), f"{n} is declared in tree_attn.h but not exported"
    assert sorted(ta.EXPORTED) == names


def test_status_strings():
    for s in range(6):
        assert ta.tree_attn_status_string(s)
    assert ta.tree_attn_status_string(99) == "unknown status"


A = 0x10000  # a 256-byte aligned stand-in address; never dereferenced on these paths


def call_ex(seqlens=(8,), Hq=4, Hkv=2, D=128, scale=0.1, q=A, k=A, v=A, out=A, lse=A, opts=None, dtype="bf16",
            ws=A, ws_bytes=1 << 30):
    arr = (ctypes.c_int64 * max(1, len(seqlens)))(*seqlens)
    return ta.lib().tree_attn_decode_ex(ta._DTYPES[dtype], q, k, v, arr, len(seqlens), Hq, Hkv, D, scale, out, lse,
                                        ctypes.byref(opts) if opts else None, ws, ws_bytes, None)


@pytest.mark.parametrize(
    "kwargs,status",
    [
        (dict(Hq=6, Hkv=4), ta.TA_ERR_INVALID_ARG),  # Hq % Hkv != 0
        (dict(Hq=0), ta.TA_ERR_INVALID_ARG),
        (dict(Hkv=0), ta.TA_ERR_INVALID_ARG),
        (dict(D=96), ta.TA_ERR_UNSUPPORTED),
        (dict(D=256), ta.TA_ERR_UNSUPPORTED),
        (dict(Hq=12, Hkv=4), ta.TA_ERR_UNSUPPORTED),  # G = 3
        (dict(Hq=32, Hkv=2), ta.TA_ERR_UNSUPPORTED),  # G = 16
        (dict(seqlens=(5, -1)), ta.TA_ERR_INVALID_ARG),
        (dict(scale=math.inf), ta.TA_ERR_INVALID_ARG),
        (dict(scale=math.nan), ta.TA_ERR_INVALID_ARG),
        (dict(q=0), ta.TA_ERR_INVALID_ARG),
        (dict(k=0), ta.TA_ERR_INVALID_ARG),
        (dict(out=0), ta.TA_ERR_INVALID_ARG),
        (dict(lse=0), ta.TA_ERR_INVALID_ARG),
        (dict(q=A + 8), ta.TA_ERR_INVALID_ARG),  # 16-byte alignment of q/K/V
        (dict(v=A + 2), ta.TA_ERR_INVALID_ARG),
        (dict(out=A + 2), ta.TA_ERR_INVALID_ARG),
        (dict(ws=0), ta.TA_ERR_WORKSPACE),
        (dict(ws=A + 16), ta.TA_ERR_WORKSPACE),  # 256-byte alignment
        (dict(opts=ta.make_options(num_ctas=-1)), ta.TA_ERR_INVALID_ARG),
        (dict(opts=ta.make_options(debug_skip_tile=-2)), ta.TA_ERR_INVALID_ARG),
    ],
)
def test_decode_ex_rejects(kwargs, status):
    assert call_ex(**kwargs) == status


def test_reserved_options_must_be_zero():
    o = ta.make_options()
    o.reserved[1] = 1
    assert call_ex(opts=o) == ta.TA_ERR_INVALID_ARG
    assert call_ex(opts=ta.make_options(debug_skip_stage=-1)) == ta.TA_ERR_INVALID_ARG


def test_bad_dtype_rejected():
    arr = (ctypes.c_int64 * 1)(8)
    assert ta.lib().tree_attn_decode_ex(7, A, A, A, arr, 1, 4, 2, 128, 0.1, A, A, None, A, 1 << 20, None) == \
        ta.TA_ERR_INVALID_ARG


def test_empty_batch_is_a_no_op():
    assert call_ex(seqlens=()) == ta.TA_OK


def test_allocating_entry_points_validate_first():
    arr = (ctypes.c_int64 * 1)(8)
    L = ta.lib()
    assert L.tree_attn_decode(A, A, A, arr, 1, 6, 4, 128, 0.1, A, A, None) == ta.TA_ERR_INVALID_ARG
    assert L.tree_attn_decode_f32(A, A, A, arr, 1, 4, 4, 80, 0.1, A, A, None) == ta.TA_ERR_UNSUPPORTED
    assert L.tree_attn_decode(A, A, A, None, 1, 4, 4, 128, 0.1, A, A, None) == ta.TA_ERR_INVALID_ARG


def test_bifurcated_validation():
    L = ta.lib()
    arr = (ctypes.c_int64 * 2)(4, 5)
    bad = (ctypes.c_int64 * 2)(4, -5)
    args = lambda lens, P=16, Hq=8, Hkv=2, D=128, ks=A: (A, A, A, P, ks, A, lens, 2, Hq, Hkv, D, 0.1, A, A)  # noqa
    assert L.tree_attn_decode_bifurcated(*args(bad), None) == ta.TA_ERR_INVALID_ARG
    assert L.tree_attn_decode_bifurcated(*args(arr, P=-1), None) == ta.TA_ERR_INVALID_ARG
    assert L.tree_attn_decode_bifurcated(*args(arr, D=32), None) == ta.TA_ERR_UNSUPPORTED
    assert L.tree_attn_decode_bifurcated(*args(arr, ks=A + 4), None) == ta.TA_ERR_INVALID_ARG
    assert L.tree_attn_decode_bifurcated_ex(*args(arr, Hq=8, Hkv=3), None, A, 1 << 20, None) == ta.TA_ERR_INVALID_ARG
    assert L.tree_attn_decode_bifurcated_ex(*args(arr), None, 0, 1 << 20, None) == ta.TA_ERR_WORKSPACE


def test_workspace_entry_points_validate():
    L = ta.lib()
    assert L.tree_attn_workspace_init(None, 1024, None) == ta.TA_ERR_WORKSPACE
    assert L.tree_attn_workspace_init(A + 8, 1024, None) == ta.TA_ERR_WORKSPACE
    assert L.tree_attn_check(None, None) == ta.TA_ERR_WORKSPACE
    arr = (ctypes.c_int64 * 1)(8)
    sz = ctypes.c_size_t(0)
    assert L.tree_attn_workspace_size(arr, 1, 6, 4, 128, 0, None, ctypes.byref(sz)) == ta.TA_ERR_INVALID_ARG
    assert L.tree_attn_workspace_size(arr, 1, 4, 4, 128, 0, None, None) == ta.TA_ERR_INVALID_ARG


def test_build_id_does_not_depend_on_where_the_tree_sits(tmp_path):
    """The library carries a hash of its sources; a copy of the tree at another absolute path
    (as on a GPU machine) must hash the same, or the loaded library would be refused there."""
    import shutil
    import subprocess
    import sys

    shutil.copytree(os.path.join(ROOT, "exact_long_context_split_b200"), tmp_path / "exact_long_context_split_b200",
                    ignore=shutil.ignore_patterns("_build", "*.so", "*.hash", "__pycache__"))
    shutil.copytree(os.path.join(ROOT, "include"), tmp_path / "include")
    code = "import sys; sys.path.insert(0, sys.argv[1]); from exact_long_context_split_b200 import _build; " \
           "print(_build.source_hash())"
    there = subprocess.run([sys.executable, "-c", code, str(tmp_path)], capture_output=True, text=True, check=True)
    from exact_long_context_split_b200 import _build

    assert there.stdout.strip() == _build.source_hash() == ta.tree_attn_build_id()
