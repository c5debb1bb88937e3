"""Build step of the CUDA library: compiles csrc/*.cu for sm_100a with nvcc and
links them, with the static CUDA runtime, into libttt_b200.so next to this file.

Object files go to ../_build (ignored by git); a source whose text and flags are
unchanged since the last build is not recompiled.
"""
from __future__ import annotations

import glob
import hashlib
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
BUILD = os.path.join(ROOT, "_build")
LIB = os.path.join(PKG, "libttt_b200.so")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
NVCC_FLAGS = ARCH + ["-lineinfo", "-O3", "-std=c++17", "-Xcompiler", "-fPIC,-O2", "--expt-relaxed-constexpr",
                     "-I", INCLUDE, "-I", CSRC]


def nvcc_path() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found: the CUDA library cannot be built")


def _digest(path: str, flags: list[str]) -> str:
    h = hashlib.sha256()
    h.update(" ".join(flags).encode())
    for f in sorted(glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(INCLUDE, "*.h")) + [path]):
        h.update(f.encode())
        with open(f, "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def build(verbose: bool = False, extra_flags: list[str] | None = None) -> str:
    """Compile every csrc/*.cu and link libttt_b200.so; returns the library path."""
    nvcc = nvcc_path()
    flags = NVCC_FLAGS + list(extra_flags or [])
    os.makedirs(BUILD, exist_ok=True)
    objs, changed = [], False
    for src in sorted(glob.glob(os.path.join(CSRC, "*.cu"))):
        name = os.path.splitext(os.path.basename(src))[0]
        obj = os.path.join(BUILD, f"{name}.{_digest(src, flags)}.o")
        if not os.path.exists(obj):
            cmd = [nvcc] + flags + ["-c", src, "-o", obj]
            if verbose:
                print(" ".join(cmd), file=sys.stderr)
            subprocess.run(cmd, check=True)
            changed = True
        objs.append(obj)
    # the objects the library was last linked from: relink whenever they differ (a
    # source reverted to an earlier version finds its old object in the cache)
    manifest = os.path.join(BUILD, "libttt_b200.objects")
    listing = "\n".join(os.path.basename(o) for o in objs)
    linked = open(manifest).read() if os.path.exists(manifest) else None
    if changed or linked != listing or not os.path.exists(LIB):
        tmp = LIB + ".tmp"
        cmd = [nvcc] + ARCH + ["-shared", "-cudart", "static", "-o", tmp] + objs
        if verbose:
            print(" ".join(cmd), file=sys.stderr)
        subprocess.run(cmd, check=True)
        os.replace(tmp, LIB)
        with open(manifest, "w") as f:
            f.write(listing)
    return LIB


if __name__ == "__main__":
    print(build(verbose="-v" in sys.argv))
