"""Build ``libconvrot.so`` in-tree with nvcc for sm_100a (B200).

``python -m w8a8_int8_quantized_block_b200.build [--force] [--ptxas-v]``
"""
from __future__ import annotations

import argparse
import hashlib
import os
import shutil
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
BUILD = os.path.join(ROOT, "_build")
LIB = os.path.join(PKG, "libconvrot.so")
SOURCES = ["api.cu", "rotate_quant.cu", "rotate_quant_block.cu", "igemm_tcgen05.cu", "linear_fused.cu",
           "attention.cu"]
HEADERS = ["ptx.cuh", "ptx_attn.cuh", "kernels.h", "attention.h", "quant_core.cuh", "gemm_core.cuh"]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "-Xcompiler", "-O3",
         "-I" + os.path.join(ROOT, "include")]


def _nvcc() -> str:
    cand = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "bin", "nvcc")
    return cand if os.path.exists(cand) else (shutil.which("nvcc") or "nvcc")


DIGEST = LIB + ".inputs"  # sha256 of the sources, headers and flags the library was built from


def _inputs_digest() -> str:
    """Digest of everything the library is built from (file contents, not
    times: a copied tree keeps the digest whatever its files' times)."""
    h = hashlib.sha256()
    paths = [os.path.join(CSRC, f) for f in SOURCES + HEADERS]
    paths.append(os.path.join(ROOT, "include", "convrot.h"))
    paths.append(os.path.abspath(__file__))
    for p in paths:
        h.update(os.path.relpath(p, ROOT).encode())  # where the tree sits does not matter
        with open(p, "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def is_current() -> bool:
    """Whether the built library matches the current sources."""
    try:
        with open(DIGEST) as f:
            return os.path.exists(LIB) and f.read().strip() == _inputs_digest()
    except OSError:
        return False


def build(force: bool = False, ptxas_verbose: bool = False) -> str:
    """Compile every CUDA source for sm_100a and link the shared library."""
    if not force and is_current():
        return LIB
    os.makedirs(BUILD, exist_ok=True)
    nvcc = _nvcc()
    extra = ["-Xptxas", "-v"] if ptxas_verbose else []

    def compile_one(src: str) -> str:
        obj = os.path.join(BUILD, src.replace(".cu", ".o"))
        cmd = [nvcc, *ARCH, *FLAGS, *extra, "-c", os.path.join(CSRC, src), "-o", obj]
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"nvcc failed for {src}:\n{r.stdout}\n{r.stderr}")
        if ptxas_verbose:
            sys.stderr.write(r.stdout + r.stderr)
        return obj

    with ThreadPoolExecutor(max_workers=len(SOURCES)) as ex:
        objs = list(ex.map(compile_one, SOURCES))
    tmp = LIB + ".tmp"
    cmd = [nvcc, *ARCH, "-shared", "-o", tmp, *objs, "-lcudart_static", "-ldl", "-lpthread", "-lrt"]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"link failed:\n{r.stdout}\n{r.stderr}")
    os.replace(tmp, LIB)
    with open(DIGEST, "w") as f:
        f.write(_inputs_digest() + "\n")
    return LIB


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--ptxas-v", action="store_true")
    a = ap.parse_args()
    print(build(force=a.force, ptxas_verbose=a.ptxas_v))
