"""Builds libgs.so (the CUDA library behind include/gs.h) in-tree with nvcc
for sm_100a.  Incremental: sources are recompiled only when they or a header
changed."""
from __future__ import annotations

import concurrent.futures as cf
import glob
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
OBJ_DIR = os.path.join(PKG, "_build")
LIB = os.path.join(PKG, "libgs.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "-I", INCLUDE, "-I", CSRC]
# extra nvcc flags (e.g. -DGS_ADAM_STAGES=4 to compare tuning constants); a
# change of them is not tracked, so rebuild with --force after setting them
FLAGS += os.environ.get("GS_NVCC_FLAGS", "").split()


def _sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")) + glob.glob(os.path.join(CSRC, "*.cpp")))


def _headers():
    return glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(INCLUDE, "*.h"))


def _mtime(p):
    return os.path.getmtime(p) if os.path.exists(p) else 0.0


def _compile(src, extra):
    obj = os.path.join(OBJ_DIR, os.path.basename(src) + ".o")
    hdr = max((_mtime(h) for h in _headers()), default=0.0)
    if _mtime(obj) >= max(_mtime(src), hdr) and not extra.get("force"):
        return obj, None
    cmd = [NVCC] + ARCH + FLAGS + extra.get("flags", []) + ["-c", src, "-o", obj]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        return obj, (" ".join(cmd), r.stdout + r.stderr)
    if extra.get("verbose") and (r.stdout or r.stderr):
        sys.stderr.write(r.stdout + r.stderr)
    return obj, None


def build(force: bool = False, verbose: bool = False, ptxas_info: bool = False) -> str:
    os.makedirs(OBJ_DIR, exist_ok=True)
    extra = {"force": force or ptxas_info, "verbose": verbose or ptxas_info,
             "flags": ["-Xptxas", "-v"] if ptxas_info else []}
    srcs = _sources()
    with cf.ThreadPoolExecutor(max_workers=min(8, len(srcs))) as ex:
        results = list(ex.map(lambda s: _compile(s, extra), srcs))
    errors = [e for _, e in results if e]
    if errors:
        msg = "\n\n".join(f"$ {c}\n{o}" for c, o in errors)
        raise RuntimeError("nvcc failed:\n" + msg)
    objs = [o for o, _ in results]
    if _mtime(LIB) < max(_mtime(o) for o in objs) or force:
        tmp = LIB + ".tmp"
        cmd = [NVCC] + ARCH + ["-shared", "-o", tmp] + objs
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError("link failed:\n" + r.stdout + r.stderr)
        os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose=True, ptxas_info="--ptxas" in sys.argv))
