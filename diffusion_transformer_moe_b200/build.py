"""Builds libnmoe.so and libnmoe_debug.so (sm_100a) in the package directory with nvcc.

Usage: ``python -m diffusion_transformer_moe_b200.build`` (or ``build()`` from Python).
The debug library is the same code compiled with -DNMOE_DEBUG: its kernels check their
gathered indices, row positions and token-list spans and report a failed check through
the error word instead of touching memory outside their buffers. Objects go to
``_build/`` and ``_build_debug/`` beside this file and are rebuilt when a source or
header is newer than the object.
"""

from __future__ import annotations

import concurrent.futures as cf
import glob
import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(ROOT, "include")
BUILD = os.path.join(HERE, "_build")
LIB = os.path.join(HERE, "libnmoe.so")
BUILD_DEBUG = os.path.join(HERE, "_build_debug")
LIB_DEBUG = os.path.join(HERE, "libnmoe_debug.so")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
NVCC_FLAGS = ARCH + [
    "-O3", "-lineinfo", "-std=c++17", "--expt-relaxed-constexpr",
    "-Xcompiler", "-fPIC,-fvisibility=hidden", "-I", CSRC, "-I", INCLUDE,
]


def _nvcc() -> str:
    p = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(p):
        raise RuntimeError("nvcc not found")
    return p


def _deps() -> list[str]:
    return (glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.h"))
            + glob.glob(os.path.join(INCLUDE, "*.h")))


def _stale(obj: str, src: str, deps: list[str]) -> bool:
    if not os.path.exists(obj):
        return True
    t = os.path.getmtime(obj)
    return any(os.path.getmtime(p) > t for p in [src] + deps)


def _compile(src: str, obj: str, extra: list[str]) -> str:
    cmd = [_nvcc()] + NVCC_FLAGS + extra + ["-c", src, "-o", obj]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"nvcc failed for {os.path.basename(src)}:\n{r.stderr}")
    return r.stderr


def _build_one(build_dir: str, lib: str, extra: list[str], forced: bool,
               verbose: bool) -> str:
    os.makedirs(build_dir, exist_ok=True)
    srcs = sorted(glob.glob(os.path.join(CSRC, "*.cu")))
    deps = _deps()
    jobs = []
    objs = []
    for s in srcs:
        o = os.path.join(build_dir, os.path.basename(s)[:-3] + ".o")
        objs.append(o)
        if _stale(o, s, deps) or forced:
            jobs.append((s, o))
    if jobs:
        with cf.ThreadPoolExecutor(max_workers=min(8, len(jobs))) as ex:
            for (s, _), log in zip(jobs, ex.map(lambda j: _compile(j[0], j[1], extra), jobs)):
                if verbose and log.strip():
                    print(f"[{os.path.basename(s)}]\n{log}", file=sys.stderr)
    if jobs or not os.path.exists(lib) or any(os.path.getmtime(o) > os.path.getmtime(lib)
                                               for o in objs):
        cmd = [_nvcc()] + ARCH + ["-shared", "-o", lib] + objs
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"link failed:\n{r.stderr}")
    return lib


def build(verbose: bool = False, extra: list[str] | None = None, debug: bool = True) -> str:
    """Compile every ``csrc/*.cu`` for sm_100a and link ``libnmoe.so`` (and, with
    ``debug``, ``libnmoe_debug.so``). Returns the release library's path."""
    extra = list(extra or [])
    _build_one(BUILD, LIB, extra, bool(extra), verbose)
    if debug:
        _build_one(BUILD_DEBUG, LIB_DEBUG, ["-DNMOE_DEBUG"] + extra, bool(extra), verbose)
    return LIB


if __name__ == "__main__":
    v = "-v" in sys.argv
    extra = ["-Xptxas", "-v"] if "--ptxas-v" in sys.argv else None
    print(build(verbose=v or bool(extra), extra=extra))
