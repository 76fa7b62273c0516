"""Builds the CUDA library in-tree: csrc/*.cu -> _build/*.o -> libtree_attn.so (sm_100a).

Each translation unit compiles to its own object (in parallel); an object is rebuilt when the
content hash of its source, the headers it includes and the compiler flags differs from the
hash recorded beside it.  The library carries the hash of every source and header it was built
from (``tree_attn_build_id()``, compiled from a generated one-line unit), so a loaded binary can
be checked against the sources in the tree.
"""
from __future__ import annotations

import concurrent.futures as cf
import glob
import hashlib
import os
import re
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
LIB = os.path.join(HERE, "libtree_attn.so")
OBJ_DIR = os.path.join(HERE, "_build")
SRC_DIR = os.path.join(HERE, "csrc")
INC_DIR = os.path.join(ROOT, "include")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")

CFLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC",
    "--expt-relaxed-constexpr",
    "-I", INC_DIR,
]
# Kept for callers that compile the sources in one command.
FLAGS = CFLAGS + ["-shared"]

_INCLUDE = re.compile(r'^\s*#\s*include\s+"([^"]+)"', re.M)


def sources(src_dir: str = SRC_DIR):
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


def _hash_files(paths, extra=()) -> str:
    """Hash of the files (by path relative to the repository root) and of the flags, with the
    include directory written relative too: the same tree gives the same hash wherever it sits."""
    h = hashlib.sha256()
    for f in sorted(paths, key=lambda f: os.path.relpath(f, ROOT)):
        h.update(os.path.relpath(f, ROOT).encode())
        with open(f, "rb") as fh:
            h.update(fh.read())
    for x in extra:
        h.update((os.path.relpath(x, ROOT) if os.path.isabs(x) else x).encode())
    return h.hexdigest()[:32]


def source_hash() -> str:
    """Hash of every library source and public header, and the compiler flags."""
    files = [f for f in glob.glob(os.path.join(SRC_DIR, "*")) if f.endswith((".cu", ".cuh", ".h"))]
    files += glob.glob(os.path.join(INC_DIR, "*.h"))
    return _hash_files(files, CFLAGS)


def _obj(src: str, obj_dir: str) -> str:
    return os.path.join(obj_dir, os.path.splitext(os.path.basename(src))[0] + ".o")


def _obj_hash(src: str, extra=()) -> str:
    return _hash_files(_deps(src), [*CFLAGS, *extra])


def _stale_obj(src: str, obj_dir: str, extra=()) -> bool:
    o = _obj(src, obj_dir)
    try:
        with open(o + ".hash") as fh:
            return fh.read().strip() != _obj_hash(src, extra) or not os.path.exists(o)
    except OSError:
        return True


def built_hash() -> str:
    """The source hash recorded when libtree_attn.so was last linked ('' if none)."""
    try:
        with open(LIB + ".hash") as fh:
            return fh.read().strip()
    except OSError:
        return ""


def stale() -> bool:
    return not os.path.exists(LIB) or built_hash() != source_hash()


def compile_objects(srcs, obj_dir: str, force: bool = False, verbose_ptxas: bool = False, extra=()) -> list:
    os.makedirs(obj_dir, exist_ok=True)
    todo = [s for s in srcs if force or _stale_obj(s, obj_dir, extra)]

    def one(src):
        o = _obj(src, obj_dir)
        digest = _obj_hash(src, extra)  # taken before compiling: an edit made meanwhile stays stale
        cmd = [NVCC, *CFLAGS, *extra, *(["-Xptxas", "-v"] if verbose_ptxas else []), "-c", "-o", o, src]
        subprocess.check_call(cmd)
        with open(o + ".hash", "w") as fh:
            fh.write(digest)

    if todo:
        with cf.ThreadPoolExecutor(max(1, min(len(todo), os.cpu_count() or 1))) as ex:
            list(ex.map(one, todo))
    return [_obj(s, obj_dir) for s in srcs]


def _build_id_object(obj_dir: str, digest: str) -> str:
    """A one-function unit returning the source hash the library is linked from."""
    src = os.path.join(obj_dir, "build_id.cu")
    with open(src, "w") as fh:
        fh.write('extern "C" const char* tree_attn_build_id(void) { return "%s"; }\n' % digest)
    obj = os.path.join(obj_dir, "build_id.o")
    subprocess.check_call([NVCC, *CFLAGS, "-c", "-o", obj, src])
    return obj


def link(objs, out: str) -> str:
    subprocess.check_call([NVCC, "-gencode", "arch=compute_100a,code=sm_100a", "-shared", "-Xcompiler", "-fPIC",
                           "-o", out, *objs])
    return out


def build(force: bool = False, verbose_ptxas: bool = False) -> str:
    if force or stale():
        digest = source_hash()
        objs = compile_objects(sources(), OBJ_DIR, force=force, verbose_ptxas=verbose_ptxas)
        link(objs + [_build_id_object(OBJ_DIR, digest)], LIB)
        with open(LIB + ".hash", "w") as fh:
            fh.write(digest)
    return LIB


if __name__ == "__main__":
    import sys

    print(build(force="-f" in sys.argv or "-v" in sys.argv, verbose_ptxas="-v" in sys.argv))
