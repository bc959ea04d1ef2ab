"""Builds the CUDA library ``libsdk.so`` in-tree for sm_100a with nvcc.

Run ``python -m unet_latent_attention_b200.build`` (or ``__graft_entry__.build()``). Objects go to
``_build/`` at the repository root; the shared library lands next to this file.
"""
from __future__ import annotations

import concurrent.futures as cf
import fcntl
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
BUILD = os.path.join(ROOT, "_build")
LIB = os.path.join(PKG, "libsdk.so")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
NVCC_FLAGS = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC,-O3", "--expt-relaxed-constexpr",
              "-I" + INCLUDE, "-I" + CSRC]


def nvcc() -> str:
    exe = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(exe):
        raise RuntimeError("nvcc not found: the CUDA toolkit is required to build libsdk.so")
    return exe


def sources():
    return sorted(os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith(".cu"))


def _compile(src: str, verbose_ptxas: bool, extra=()) -> str:
    obj = os.path.join(BUILD, os.path.basename(src)[:-3] + ".o")
    cmd = [nvcc(), *ARCH, *NVCC_FLAGS, *extra, "-c", src, "-o", obj]
    if verbose_ptxas:
        cmd.insert(1, "-Xptxas=-v")
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"nvcc failed for {src}:\n{r.stdout}\n{r.stderr}")
    if verbose_ptxas and r.stderr:
        sys.stderr.write(r.stderr)
    return obj


def build(verbose_ptxas: bool = False, force: bool = False, defines=(), out: str | None = None) -> str:
    """Compile every ``csrc/*.cu`` and link ``libsdk.so``; returns the library path.

    ``defines`` (e.g. ``["SD_POLY_PAIRS=2"]``) and ``out`` build a tuning variant of the library
    under another name; the default build is the product library."""
    global BUILD
    lib_path = out or LIB
    if defines:
        tag = "_".join(d.replace("=", "") for d in defines)
        saved, BUILD = BUILD, os.path.join(BUILD, tag)
        try:
            return _build(verbose_ptxas, True, [f"-D{d}" for d in defines], lib_path)
        finally:
            BUILD = saved
    return _build(verbose_ptxas, force, [], lib_path)


def _up_to_date(lib_path: str) -> bool:
    srcs = sources()
    deps = srcs + [os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith((".h", ".cuh"))]
    deps.append(os.path.join(INCLUDE, "sd_kernels.h"))
    return os.path.exists(lib_path) and os.path.getmtime(lib_path) >= max(os.path.getmtime(d) for d in deps)


def _build(verbose_ptxas: bool, force: bool, extra, lib_path: str) -> str:
    os.makedirs(BUILD, exist_ok=True)
    if not force and not verbose_ptxas and _up_to_date(lib_path):
        return lib_path
    # Concurrent callers (one process per GPU, parallel test workers) build one at a time; whoever
    # gets the lock second finds the library fresh and returns.
    with open(os.path.join(BUILD, ".lock"), "w") as lock:
        fcntl.flock(lock, fcntl.LOCK_EX)
        if not force and not verbose_ptxas and _up_to_date(lib_path):
            return lib_path
        srcs = sources()
        with cf.ThreadPoolExecutor(max_workers=min(8, len(srcs))) as ex:
            objs = list(ex.map(lambda s: _compile(s, verbose_ptxas, extra), srcs))
        tmp = f"{lib_path}.{os.getpid()}.tmp"
        cmd = [nvcc(), *ARCH, "-shared", "-o", tmp, *objs, "-lcudart_static", "-ldl", "-lpthread", "-lrt"]
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"link failed:\n{r.stdout}\n{r.stderr}")
        os.replace(tmp, lib_path)
    return lib_path


if __name__ == "__main__":
    print(build(verbose_ptxas="-v" in sys.argv, force="-f" in sys.argv))
