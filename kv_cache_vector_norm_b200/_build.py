"""Build libtq.so (the C-ABI library) in-tree with nvcc for sm_100a.

Usage: ``python -m kv_cache_vector_norm_b200._build [--force] [--verbose]``.  The library is rebuilt
when any source under csrc/ or include/ is newer than the existing .so.
"""
from __future__ import annotations

import os
import subprocess
import sys
import time

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libtq.so")

ARCH_FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a"]


def _sources():
    out = []
    for d in (CSRC, INCLUDE):
        for name in sorted(os.listdir(d)):
            if name.endswith((".cu", ".cuh", ".cpp", ".h")):
                out.append(os.path.join(d, name))
    return out


def needs_build() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    return any(os.path.getmtime(s) > t for s in _sources())


def nvcc() -> str:
    cand = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "bin", "nvcc")
    return cand if os.path.exists(cand) else "nvcc"


def build(force: bool = False, verbose: bool = False, extra=()) -> str:
    if not force and not needs_build():
        return LIB
    build_dir = os.path.join(PKG, "_build")
    os.makedirs(build_dir, exist_ok=True)
    common = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC,-O2", f"-I{INCLUDE}"]
    objs = []
    cmds = []
    for src, kind in (("tq_lib.cu", "cu"), ("tq_host.cpp", "cpp")):
        obj = os.path.join(build_dir, src + ".o")
        if kind == "cu":
            cmd = [nvcc(), *ARCH_FLAGS, *common, "-Xptxas", "-warn-spills", *extra, "-c",
                   os.path.join(CSRC, src), "-o", obj]
        else:
            cmd = ["g++", "-O2", "-std=c++17", "-fPIC", "-ffp-contract=off", f"-I{INCLUDE}",
                   "-I/usr/local/cuda/include", "-c", os.path.join(CSRC, src), "-o", obj]
        cmds.append(cmd)
        objs.append(obj)
    t0 = time.time()
    procs = [subprocess.Popen(c, stdout=subprocess.PIPE, stderr=subprocess.STDOUT, text=True) for c in cmds]
    for c, p in zip(cmds, procs):
        out, _ = p.communicate()
        if verbose or p.returncode:
            sys.stderr.write(" ".join(c) + "\n" + out)
        if p.returncode:
            raise RuntimeError(f"compilation failed: {' '.join(c[:2])} ...")
    tmp = LIB + ".tmp"
    link = [nvcc(), *ARCH_FLAGS, "-shared", "-o", tmp, *objs, "-lcudart_static", "-lrt", "-lpthread", "-ldl"]
    r = subprocess.run(link, stdout=subprocess.PIPE, stderr=subprocess.STDOUT, text=True)
    if r.returncode:
        sys.stderr.write(" ".join(link) + "\n" + r.stdout)
        raise RuntimeError("link failed")
    os.replace(tmp, LIB)
    if verbose:
        sys.stderr.write(f"built {LIB} in {time.time() - t0:.1f}s\n")
    return LIB


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose=True)
