"""Build libtq.so in-tree with nvcc for sm_100a (B200).

Run as ``python online_vector_quantization_b200/build.py`` (not with -m: the
package import loads the library this script builds) or call build().
The shared library exports the C ABI declared in include/tq.h.
"""
from __future__ import annotations

import os
import shutil
import subprocess

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
LIB = os.path.join(PKG, "libtq.so")
SOURCES = ["tq_host.cpp", "tq_quantize.cu", "tq_attn.cu", "tq_search.cu", "tq_noalloc.cu"]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def nvcc() -> str:
    cand = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(cand):
        raise RuntimeError("nvcc not found")
    return cand


def build(verbose: bool = False, ptxas_info: bool = False) -> str:
    """Compile every source (in parallel, one nvcc per source) and link."""
    from concurrent.futures import ThreadPoolExecutor

    objdir = os.path.join(PKG, "_build")
    os.makedirs(objdir, exist_ok=True)
    cmds, objs = [], []
    for src in SOURCES:
        path = os.path.join(CSRC, src)
        obj = os.path.join(objdir, src + ".o")
        cmd = [nvcc(), "-c", path, "-o", obj, "-O3", "-std=c++17", "-Xcompiler", "-fPIC",
               "-I", os.path.join(ROOT, "include"), "-lineinfo", *ARCH]
        if src.endswith(".cu"):
            cmd += ["--expt-relaxed-constexpr"]
            if ptxas_info:
                cmd += ["-Xptxas", "-v"]
        if verbose:
            print(" ".join(cmd))
        cmds.append(cmd)
        objs.append(obj)
    with ThreadPoolExecutor(max_workers=min(len(cmds), os.cpu_count() or 1)) as pool:
        for r in list(pool.map(lambda c: subprocess.run(c, capture_output=not verbose, text=True), cmds)):
            if r.returncode != 0:
                import sys
                sys.stderr.write((r.stdout or "") + (r.stderr or ""))
                raise subprocess.CalledProcessError(r.returncode, r.args, r.stdout, r.stderr)
    link = [nvcc(), "-shared", "-o", LIB, *objs, *ARCH]
    if verbose:
        print(" ".join(link))
    subprocess.run(link, check=True)
    return LIB


if __name__ == "__main__":
    import sys
    build(verbose=True, ptxas_info="-v" in sys.argv)
