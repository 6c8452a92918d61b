"""Build libtaylor_attn.so in-tree with nvcc for sm_100a.

    python -m recurrent_states_b200.build [--force]

Compiles every ``csrc/*.cu`` for ``sm_100a`` only (``-gencode
arch=compute_100a,code=sm_100a``) into ``_build/`` (one object per source,
in parallel), links them with the CUDA runtime statically and writes
``recurrent_states_b200/libtaylor_attn.so``.  An object is rebuilt when its
source, a header or this script is newer than it."""
from __future__ import annotations

import glob
import os
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libtaylor_attn.so")
OBJ_DIR = os.path.join(HERE, "_build")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = [
    *ARCH,
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC,-fvisibility=hidden",
    "--expt-relaxed-constexpr", "--extended-lambda",
    "-I", os.path.join(ROOT, "include"),
]


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _headers():
    return sorted(glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.h"))) + [
        os.path.join(ROOT, "include", "taylor_attn.h"), os.path.abspath(__file__)]


def _obj(src: str) -> str:
    return os.path.join(OBJ_DIR, os.path.splitext(os.path.basename(src))[0] + ".o")


def _deps(src: str, headers) -> list:
    """The files an object depends on: the dependency list nvcc wrote when it
    last compiled the source (-MD), else every header of the library."""
    dep = _obj(src)[:-2] + ".d"
    if os.path.exists(dep):
        with open(dep) as f:
            text = f.read().replace("\\\n", " ")
        files = []
        for t in text.split(":", 1)[-1].split():
            # nvcc writes paths as it was given them: relative ones are taken
            # against the package and the repository roots
            for c in ([t] if os.path.isabs(t) else [os.path.join(HERE, t), os.path.join(ROOT, t), t]):
                if os.path.exists(c):
                    files.append(c)
                    break
        if files:
            return [src, *files, os.path.abspath(__file__)]
    return [src, *headers]


def _stale(target: str, deps) -> bool:
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    return any(os.path.getmtime(p) > t for p in deps)


def up_to_date() -> bool:
    return not _stale(LIB, sources() + _headers())


def build(force: bool = False, verbose: bool = False, extra=()) -> str:
    if not force and up_to_date():
        return LIB
    os.makedirs(OBJ_DIR, exist_ok=True)
    headers = _headers()
    todo = [s for s in sources() if force or extra or _stale(_obj(s), _deps(s, headers))]

    def compile_one(src):
        dep = _obj(src)[:-2] + ".d"
        cmd = [NVCC, *FLAGS, *extra, "-MD", "-MF", dep, "-c", "-o", _obj(src), src]
        if verbose:
            print(" ".join(cmd), flush=True)
        return subprocess.run(cmd, capture_output=True, text=True)

    with ThreadPoolExecutor(max_workers=max(1, min(len(todo), os.cpu_count() or 1))) as pool:
        results = list(pool.map(compile_one, todo))
    for src, r in zip(todo, results):
        if r.stdout or r.stderr:
            sys.stderr.write(r.stdout + r.stderr)
        if r.returncode != 0:
            raise subprocess.CalledProcessError(r.returncode, f"nvcc {os.path.basename(src)}")
    # objects of sources that no longer exist are not linked
    objs = [_obj(s) for s in sources()]
    tmp = LIB + ".tmp"
    cmd = [NVCC, *ARCH, "-shared", "-cudart", "static", "-o", tmp, *objs]
    if verbose:
        print(" ".join(cmd), flush=True)
    subprocess.run(cmd, check=True)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose=True,
                extra=["-Xptxas", "-v"] if "--ptxas-v" in sys.argv else []))
