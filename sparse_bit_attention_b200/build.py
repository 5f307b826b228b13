"""Builds libsagesla.so (the C-ABI library) in-tree with nvcc for sm_100a, and its
bounds-checking twin libsagesla_checks.so (the same sources compiled with SAGESLA_CHECKS=1:
kept-list entries, Top-K output positions and the attention kernels' TMA row coordinates are
checked before use, a failed check records SAGESLA_ERR_BOUNDS and skips the access).

Usage: python -m sparse_bit_attention_b200.build [--verbose-ptxas] [--force] [--checks]
"""
from __future__ import annotations

import concurrent.futures
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libsagesla.so")
BUILD_DIR = os.path.join(PKG, "_build")
LIB_CHECKS = os.path.join(PKG, "libsagesla_checks.so")
BUILD_DIR_CHECKS = os.path.join(PKG, "_build_checks")

SOURCES = ["sagesla_api.cu", "prologue.cu", "topk.cu", "linear.cu", "attention.cu",
           "attention_dense.cu", "checks.cu", "no_alloc.cu",
           "norm.cu", "w8a8.cu", "backward.cu"]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "-Xcompiler", "-O2",
         "-I" + INCLUDE, "-I" + CSRC]


def nvcc() -> str:
    path = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(path):
        raise RuntimeError("nvcc not found: the CUDA toolkit is required to build libsagesla.so")
    return path


def _compile(src: str, verbose_ptxas: bool, checks: bool) -> tuple[str, str]:
    obj = os.path.join(BUILD_DIR_CHECKS if checks else BUILD_DIR, os.path.splitext(src)[0] + ".o")
    cmd = [nvcc(), *ARCH, *FLAGS, "-c", os.path.join(CSRC, src), "-o", obj]
    if checks:
        cmd.append("-DSAGESLA_CHECKS=1")
    if verbose_ptxas:
        cmd += ["-Xptxas", "-v"]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"nvcc failed on {src}:\n{r.stdout}\n{r.stderr}")
    return obj, r.stderr


def build(verbose_ptxas: bool = False, force: bool = False, checks: bool = False) -> str:
    lib_path = LIB_CHECKS if checks else LIB
    os.makedirs(BUILD_DIR_CHECKS if checks else BUILD_DIR, exist_ok=True)
    srcs = [os.path.join(CSRC, s) for s in SOURCES] + [
        os.path.join(CSRC, h) for h in os.listdir(CSRC) if h.endswith((".cuh", ".h"))
    ] + [os.path.join(INCLUDE, "sagesla.h")]
    if not force and os.path.exists(lib_path) and not verbose_ptxas:
        lib_t = os.path.getmtime(lib_path)
        if all(os.path.getmtime(s) <= lib_t for s in srcs):
            return lib_path
    with concurrent.futures.ThreadPoolExecutor(max_workers=len(SOURCES)) as ex:
        results = list(ex.map(lambda s: _compile(s, verbose_ptxas, checks), SOURCES))
    if verbose_ptxas:
        for obj, log in results:
            print(f"== {os.path.basename(obj)}\n{log}")
    tmp = lib_path + ".tmp"
    cmd = [nvcc(), *ARCH, "-shared", "-o", tmp] + [o for o, _ in results]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"link failed:\n{r.stdout}\n{r.stderr}")
    os.replace(tmp, lib_path)
    return lib_path


if __name__ == "__main__":
    print(build(verbose_ptxas="--verbose-ptxas" in sys.argv, force="--force" in sys.argv,
                checks="--checks" in sys.argv))
