"""Build libmk.so (the C-ABI library with every CUDA kernel) in-tree for sm_100a.

    python -m hybrid_deltanet_attention_b200.build [--verbose]

nvcc cross-compiles without a GPU. The library lands next to this file so the
Python binding (and anything that travels with the source tree) finds it.
"""
from __future__ import annotations

import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libmk.so")
SOURCES = ["api.cu", "decode.cu", "noalloc.cu", "gemm.cu", "prefill.cu", "attn.cu"]
HEADERS = ["mk_internal.h", "mk_model.h", "dev.cuh", "tc.cuh"]

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC,-O2",
         "-shared", "-I" + os.path.join(ROOT, "include")]


def nvcc() -> str:
    cand = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "bin", "nvcc")
    return cand if os.path.exists(cand) else (shutil.which("nvcc") or "nvcc")


def _inputs():
    files = [os.path.join(CSRC, s) for s in SOURCES + HEADERS]
    files.append(os.path.join(ROOT, "include", "mk.h"))
    return files


def up_to_date() -> bool:
    if not os.path.exists(LIB):
        return False
    t = os.path.getmtime(LIB)
    return all(os.path.getmtime(f) <= t for f in _inputs())


def build(force: bool = False, verbose: bool = False) -> str:
    if not force and up_to_date():
        return LIB
    # one nvcc per source file in parallel (relocatable device code is not needed: the
    # files share host-side declarations only), then one link step
    import concurrent.futures as cf
    import tempfile
    tmp = tempfile.mkdtemp(prefix="mk_build_")
    compile_flags = [f for f in FLAGS if f != "-shared"]

    def one(src):
        obj = os.path.join(tmp, os.path.splitext(src)[0] + ".o")
        cmd = [nvcc(), *ARCH, *compile_flags, "-c", os.path.join(CSRC, src), "-o", obj]
        if verbose:
            cmd += ["-Xptxas", "-v"]
        r = subprocess.run(cmd, capture_output=True, text=True)
        return src, obj, cmd, r

    try:
        with cf.ThreadPoolExecutor(len(SOURCES)) as ex:
            results = list(ex.map(one, SOURCES))
        for src, obj, cmd, r in results:
            if r.returncode != 0:
                raise RuntimeError("nvcc failed:\n" + " ".join(cmd) + "\n" + r.stdout + r.stderr)
            if verbose:
                sys.stderr.write(r.stdout + r.stderr)
        link = [nvcc(), *ARCH, "-shared", "-Xcompiler", "-fPIC", *[o for _, o, _, _ in results], "-o", LIB + ".tmp"]
        r = subprocess.run(link, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError("nvcc link failed:\n" + " ".join(link) + "\n" + r.stdout + r.stderr)
    finally:
        shutil.rmtree(tmp, ignore_errors=True)
    os.replace(LIB + ".tmp", LIB)
    return LIB


if __name__ == "__main__":
    print(build(force=True, verbose="--verbose" in sys.argv))
