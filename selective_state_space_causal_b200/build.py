"""Build the CUDA library (sm_100a) in-tree: libssm_causal.so next to this file.

Run ``python selective_state_space_causal_b200/build.py`` (by path: importing
the package needs the built library) or call ``build_library()``. nvcc
cross-compiles for sm_100a without a GPU. Each ``csrc/*.cu`` compiles to its
own object under ``_build/`` (in parallel; a file is recompiled when it or a
file it includes is newer than its object), and the objects are linked into the shared
library.
"""

from __future__ import annotations

import glob
import re
import os
import shutil
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(ROOT, "include")
OBJDIR = os.path.join(ROOT, "_build")
LIBRARY = os.path.join(HERE, "libssm_causal.so")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-lineinfo", "-std=c++17", "--expt-relaxed-constexpr", "-Xcompiler", "-fPIC"]


def nvcc_path() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def sources() -> list[str]:
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _headers() -> list[str]:
    return glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.h")) + \
        glob.glob(os.path.join(INCLUDE, "*.h"))


def _inputs() -> list[str]:
    return sources() + _headers()


def _mtime(path: str) -> float:
    return os.path.getmtime(path) if os.path.exists(path) else -1.0


def up_to_date() -> bool:
    if not os.path.exists(LIBRARY):
        return False
    t = os.path.getmtime(LIBRARY)
    return all(os.path.getmtime(f) <= t for f in _inputs())


def _deps(path: str, seen: set | None = None) -> set:
    """The file and every file it reaches through quoted #include lines."""
    seen = set() if seen is None else seen
    path = os.path.normpath(path)
    if path in seen or not os.path.exists(path):
        return seen
    seen.add(path)
    for line in open(path, encoding="utf-8", errors="replace"):
        m = re.match(r'\s*#\s*include\s+"([^"]+)"', line)
        if m:
            _deps(os.path.join(os.path.dirname(path), m.group(1)), seen)
    return seen


def _object(src: str) -> str:
    return os.path.join(OBJDIR, os.path.basename(src)[:-3] + ".o")


def build_library(force: bool = False, verbose: bool = False, extra: list[str] | None = None) -> str:
    if not force and up_to_date():
        return LIBRARY
    nvcc = nvcc_path()
    os.makedirs(OBJDIR, exist_ok=True)
    flags = [*ARCH, *FLAGS, *(extra or []), *(["-Xptxas=-v"] if verbose else [])]

    def compile_one(src: str):
        obj = _object(src)
        if not force and _mtime(obj) >= max(_mtime(f) for f in _deps(src)):
            return src, None
        cmd = [nvcc, *flags, "-I", INCLUDE, "-c", "-o", obj + ".tmp", src]
        res = subprocess.run(cmd, capture_output=True, text=True)
        if res.returncode == 0:
            os.replace(obj + ".tmp", obj)
        return src, res

    srcs = sources()
    with ThreadPoolExecutor(max_workers=max(1, min(len(srcs), os.cpu_count() or 1))) as pool:
        results = list(pool.map(compile_one, srcs))
    for src, res in results:
        if res is None:
            continue
        if res.returncode != 0:
            sys.stderr.write(res.stdout + res.stderr)
            raise RuntimeError(f"nvcc failed compiling {os.path.basename(src)}")
        if verbose:
            sys.stderr.write(res.stderr)
    # --no-undefined: a symbol missing across translation units fails the build, not the import
    cmd = [nvcc, *ARCH, "-shared", "-Xlinker", "--no-undefined", "-o", LIBRARY + ".tmp",
           *[_object(s) for s in srcs]]
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        sys.stderr.write(res.stdout + res.stderr)
        raise RuntimeError("nvcc failed linking libssm_causal.so")
    os.replace(LIBRARY + ".tmp", LIBRARY)
    return LIBRARY


if __name__ == "__main__":
    build_library(force="--force" in sys.argv, verbose="-v" in sys.argv)
    print(LIBRARY)
