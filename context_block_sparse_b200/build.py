"""Build libsplitkv.so in-tree with nvcc for sm_100a (B200).

    python context_block_sparse_b200/build.py [-v] [-f] [--ptxas]

(Run it as a script: importing the package itself needs the built library.)

Objects go to _build/ at the repository root; the shared library lands next
to this file so the Python binding finds it.  Only splitkv_* symbols are
exported.  Nothing here needs a GPU: nvcc cross-compiles.
"""

from __future__ import annotations

import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
BUILD = os.path.join(ROOT, "_build")
LIB = os.path.join(PKG, "libsplitkv.so")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
COMMON = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC,-O3", "-I", INCLUDE, "-I", CSRC]


def _nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def sources():
    return sorted(f for f in os.listdir(CSRC) if f.endswith((".cu", ".cpp")))


def build(verbose: bool = False, force: bool = False, ptxas_info: bool = False) -> str:
    nvcc = _nvcc()
    os.makedirs(BUILD, exist_ok=True)
    headers = [os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith((".h", ".cuh"))]
    headers.append(os.path.join(INCLUDE, "splitkv.h"))
    newest_header = max(os.path.getmtime(h) for h in headers)
    objs = []
    for src in sources():
        path = os.path.join(CSRC, src)
        obj = os.path.join(BUILD, src + ".o")
        objs.append(obj)
        if (not force and os.path.exists(obj)
                and os.path.getmtime(obj) >= max(os.path.getmtime(path), newest_header)):
            continue
        cmd = [nvcc, *ARCH, *COMMON, "-c", path, "-o", obj]
        if src.endswith(".cu"):
            cmd.insert(1, "-Xptxas=-v")
        if verbose:
            print(" ".join(cmd), flush=True)
        res = subprocess.run(cmd, capture_output=True, text=True)
        if ptxas_info or res.returncode != 0:
            sys.stderr.write(res.stderr)
        if res.returncode != 0:
            raise subprocess.CalledProcessError(res.returncode, cmd)

    link = [nvcc, *ARCH, "-shared", "-o", LIB, *objs,
            "-Xlinker", "--version-script=" + os.path.join(CSRC, "exports.map"), "-lcuda"]
    if verbose:
        print(" ".join(link), flush=True)
    subprocess.run(link, check=True)
    return LIB


if __name__ == "__main__":
    build(verbose="-v" in sys.argv, force="-f" in sys.argv, ptxas_info="--ptxas" in sys.argv)
    print(LIB)
