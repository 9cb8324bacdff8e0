"""Builds libtkv.so in-tree for sm_100a with nvcc (no JIT cache, no torch types).

Every source compiles to its own object in parallel (a private temporary folder per
process, so concurrent builds cannot clobber each other), then nvcc links the
shared library.  `debug=True` builds libtkv_debug.so with TKV_DEBUG defined: every
kernel then checks the indices of its table and pool accesses against the cache's
capacities and, instead of making an out-of-range access, latches TKV_ERR_INVALID
with the failing check in the device error word."""
from __future__ import annotations

import os
import shutil
import subprocess
import sys
import tempfile
from concurrent.futures import ThreadPoolExecutor
from pathlib import Path

PKG = Path(__file__).resolve().parent
ROOT = PKG.parent
CSRC = PKG / "csrc"
LIB = PKG / "libtkv.so"
LIB_DEBUG = PKG / "libtkv_debug.so"
SOURCES = ["tkv_api.cu", "append.cu", "attention.cu", "attention_i8.cu", "attention_ws.cu", "evict.cu", "noalloc.cu",
           "selftest.cu", "evict_segments.cu"]
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")

FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17", "--expt-relaxed-constexpr",
    "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
]


def _stale(lib: Path) -> bool:
    if not lib.exists():
        return True
    t = lib.stat().st_mtime
    deps = [CSRC / s for s in SOURCES] + list(CSRC.glob("*.cuh")) + [ROOT / "include" / "tkv.h"]
    return any(p.stat().st_mtime > t for p in deps if p.exists())


def build(force: bool = False, verbose: bool = False, extra: list[str] | None = None,
          debug: bool = False) -> Path:
    lib = LIB_DEBUG if debug else LIB
    if not force and not _stale(lib):
        return lib
    flags = [*FLAGS, *(["-DTKV_DEBUG=1"] if debug else []), *(extra or []),
             "-I", str(ROOT / "include"), "-I", str(CSRC)]
    tmpdir = Path(tempfile.mkdtemp(prefix="tkv_build_", dir=str(PKG)))
    try:
        def compile_one(src: str) -> Path:
            obj = tmpdir / (Path(src).stem + ".o")
            cmd = [NVCC, *flags, "-c", str(CSRC / src), "-o", str(obj)]
            if verbose:
                print(" ".join(cmd), file=sys.stderr)
            subprocess.check_call(cmd)
            return obj

        with ThreadPoolExecutor(max_workers=min(len(SOURCES), os.cpu_count() or 4)) as ex:
            objs = list(ex.map(compile_one, SOURCES))
        tmp = tmpdir / lib.name
        cmd = [NVCC, "-gencode", "arch=compute_100a,code=sm_100a", "-shared", "-cudart", "static",
               *[str(o) for o in objs], "-o", str(tmp)]
        if verbose:
            print(" ".join(cmd), file=sys.stderr)
        subprocess.check_call(cmd)
        os.replace(tmp, lib)
    finally:
        shutil.rmtree(tmpdir, ignore_errors=True)
    return lib


if __name__ == "__main__":
    args = [a for a in sys.argv[1:] if a != "--debug"]
    print(build(force=True, verbose=True, extra=args, debug="--debug" in sys.argv[1:]))
