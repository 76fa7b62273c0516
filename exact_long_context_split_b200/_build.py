"""Builds the CUDA library in-tree: csrc/*.cu -> _build/*.o -> libtree_attn.so (sm_100a).

Each translation unit compiles to its own object (in parallel, and only when it or a header
it includes changed); the objects link into one shared library.
"""
from __future__ import annotations

import concurrent.futures as cf
import glob
import os
import re
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
LIB = os.path.join(HERE, "libtree_attn.so")
OBJ_DIR = os.path.join(HERE, "_build")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")

CFLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC",
    "--expt-relaxed-constexpr",
    "-I", os.path.join(ROOT, "include"),
]
# Kept for callers that compile the sources in one command.
FLAGS = CFLAGS + ["-shared"]

_INCLUDE = re.compile(r'^\s*#\s*include\s+"([^"]+)"', re.M)


def sources(src_dir: str = os.path.join(HERE, "csrc")):
    return sorted(glob.glob(os.path.join(src_dir, "*.cu")))


def _deps(path: str, seen=None) -> set:
    """The file and every quoted include it reaches (relative to the including file)."""
    seen = set() if seen is None else seen
    path = os.path.normpath(path)
    if path in seen or not os.path.exists(path):
        return seen
    seen.add(path)
    with open(path) as fh:
        for inc in _INCLUDE.findall(fh.read()):
            _deps(os.path.join(os.path.dirname(path), inc), seen)
    return seen


def _obj(src: str, obj_dir: str) -> str:
    return os.path.join(obj_dir, os.path.splitext(os.path.basename(src))[0] + ".o")


def _stale(target: str, deps) -> bool:
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    return any(os.path.getmtime(d) > t for d in deps)


def stale() -> bool:
    srcs = sources()
    return any(_stale(_obj(s, OBJ_DIR), _deps(s)) for s in srcs) or _stale(LIB, [_obj(s, OBJ_DIR) for s in srcs])


def compile_objects(srcs, obj_dir: str, force: bool = False, verbose_ptxas: bool = False, extra=()) -> list:
    os.makedirs(obj_dir, exist_ok=True)
    todo = [s for s in srcs if force or _stale(_obj(s, obj_dir), _deps(s))]

    def one(src):
        cmd = [NVCC, *CFLAGS, *extra, *(["-Xptxas", "-v"] if verbose_ptxas else []), "-c", "-o", _obj(src, obj_dir),
               src]
        subprocess.check_call(cmd)

    if todo:
        with cf.ThreadPoolExecutor(max(1, min(len(todo), os.cpu_count() or 1))) as ex:
            list(ex.map(one, todo))
    return [_obj(s, obj_dir) for s in srcs]


def link(objs, out: str) -> str:
    subprocess.check_call([NVCC, "-gencode", "arch=compute_100a,code=sm_100a", "-shared", "-Xcompiler", "-fPIC",
                           "-o", out, *objs])
    return out


def build(force: bool = False, verbose_ptxas: bool = False) -> str:
    if force or stale():
        objs = compile_objects(sources(), OBJ_DIR, force=force, verbose_ptxas=verbose_ptxas)
        link(objs, LIB)
    return LIB


if __name__ == "__main__":
    import sys

    print(build(force="-f" in sys.argv or "-v" in sys.argv, verbose_ptxas="-v" in sys.argv))
