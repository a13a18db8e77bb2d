"""Build libsol.so (CUDA, sm_100a) in-tree with nvcc.

    python -m dit_block_b200.build [--force]

Each ``csrc/*.cu`` compiles to an object under ``dit_block_b200/_build/`` (ptxas
register/spill report beside it in ``<name>.ptxas.txt``) and the objects link into
``dit_block_b200/libsol.so`` with the CUDA runtime linked statically.
"""
from __future__ import annotations

import glob
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
BUILD = os.path.join(PKG, "_build")
LIB = os.path.join(PKG, "libsol.so")

NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
CFLAGS = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC,-O2", "-Xptxas", "-v",
          f"-I{INCLUDE}", f"-I{CSRC}"] + ARCH


def _sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _deps():
    return _sources() + glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.h")) \
        + [os.path.join(INCLUDE, "sol.h")]


def up_to_date() -> bool:
    if not os.path.exists(LIB):
        return False
    t = os.path.getmtime(LIB)
    return all(os.path.getmtime(p) <= t for p in _deps())


def build(force: bool = False, verbose: bool = False) -> str:
    if not force and up_to_date():
        return LIB
    os.makedirs(BUILD, exist_ok=True)
    procs = []
    objs = []
    for src in _sources():
        name = os.path.splitext(os.path.basename(src))[0]
        obj = os.path.join(BUILD, name + ".o")
        log = open(os.path.join(BUILD, name + ".ptxas.txt"), "w")
        cmd = [NVCC, *CFLAGS, "-c", src, "-o", obj]
        if verbose:
            print(" ".join(cmd), file=sys.stderr)
        procs.append((subprocess.Popen(cmd, stdout=log, stderr=subprocess.STDOUT), log, src))
        objs.append(obj)
    failed = []
    for p, log, src in procs:
        rc = p.wait()
        log.close()
        if rc != 0:
            failed.append(src)
    if failed:
        msgs = []
        for src in failed:
            name = os.path.splitext(os.path.basename(src))[0]
            with open(os.path.join(BUILD, name + ".ptxas.txt")) as f:
                msgs.append(f.read()[-4000:])
        raise RuntimeError("nvcc failed for " + ", ".join(failed) + "\n" + "\n".join(msgs))
    tmp = LIB + f".tmp{os.getpid()}"
    subprocess.check_call([NVCC, *ARCH, "-shared", "-cudart", "static", *objs, "-o", tmp])
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose=True))
