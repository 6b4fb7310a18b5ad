"""Build libh3dit.so in-tree with nvcc for sm_100a (no GPU needed to build).

    python -m image_generation_b200.build [-v]            # libh3dit.so
    python -m image_generation_b200.build --stamps        # libh3dit_stamps.so (diagnostic)
"""
from __future__ import annotations

import concurrent.futures as cf
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
BUILD = os.path.join(PKG, "_build")
LIB = os.path.join(PKG, "libh3dit.so")
SOURCES = ["api.cu", "gemm.cu", "gemm_pair.cu", "gemm_mx.cu", "attention.cu", "elementwise.cu",
           "io_layers.cu", "sp.cu", "vae.cu"]

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC,-O2",
         "--expt-relaxed-constexpr", "-I", os.path.join(ROOT, "include")]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def _compile(src: str, verbose: bool, extra=(), build_dir: str = BUILD) -> str:
    obj = os.path.join(build_dir, os.path.splitext(src)[0] + ".o")
    cmd = [nvcc(), *ARCH, *FLAGS, *extra, "-c", os.path.join(CSRC, src), "-o", obj]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"nvcc failed for {src}:\n{r.stdout}\n{r.stderr}")
    if verbose and (r.stdout or r.stderr):
        print(r.stdout + r.stderr, file=sys.stderr)
    return obj


def build(verbose: bool = False, extra=(), out: str = LIB, build_dir: str = BUILD) -> str:
    """Compile and link; `extra` nvcc flags and `out` are for building
    variants of the library side by side (the default is the product)."""
    os.makedirs(build_dir, exist_ok=True)
    with cf.ThreadPoolExecutor(len(SOURCES)) as ex:
        objs = list(ex.map(lambda s: _compile(s, verbose, extra, build_dir), SOURCES))
    tmp = out + ".tmp"
    cmd = [nvcc(), *ARCH, "-shared", "-o", tmp, *objs]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"link failed:\n{r.stdout}\n{r.stderr}")
    os.replace(tmp, out)
    return out


LIB_STAMPS = os.path.join(PKG, "libh3dit_stamps.so")


def build_stamps(verbose: bool = False) -> str:
    """The diagnostic build: the product sources with the attention kernel's
    clock-stamp points compiled in (read with h3dit_attention_stamps)."""
    return build(verbose, extra=["-DH3_ATTN_STAMPS"], out=LIB_STAMPS,
                 build_dir=BUILD + "_stamps")


if __name__ == "__main__":
    if "--stamps" in sys.argv:
        print(build_stamps(verbose="-v" in sys.argv))
    else:
        print(build(verbose="-v" in sys.argv))
