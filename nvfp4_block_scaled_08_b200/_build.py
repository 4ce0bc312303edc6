"""Build libnvfp4.so (sm_100a) in-tree with nvcc.

Each ``csrc/*.cu`` file is compiled to an object in parallel, then linked into a shared
library with the CUDA runtime linked statically, so that the library loads without a GPU
(the driver is only opened on the first CUDA call).
"""
from __future__ import annotations

import os
import subprocess
import sys
import threading

PKG_DIR = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(PKG_DIR, "csrc")
ROOT = os.path.dirname(PKG_DIR)
INCLUDE = os.path.join(ROOT, "include")
LIB_PATH = os.path.join(PKG_DIR, "libnvfp4.so")
BUILD_DIR = os.path.join(ROOT, "_build")

SOURCES = ["api.cu", "gemm.cu", "quantize.cu", "moe.cu", "noalloc.cu"]
HEADERS = ["ptx.cuh", "gemm_kernel.cuh", "internal.h", "quant_core.cuh"]

NVCC_FLAGS = [
    "-std=c++17", "-O3", "-lineinfo",
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-Xcompiler", "-fPIC",
    "--expt-relaxed-constexpr",
    "-I", INCLUDE,
]

_lock = threading.Lock()


def _nvcc() -> str:
    cuda_home = os.environ.get("CUDA_HOME", "/usr/local/cuda")
    cand = os.path.join(cuda_home, "bin", "nvcc")
    return cand if os.path.exists(cand) else "nvcc"


def _inputs() -> list[str]:
    files = [os.path.join(CSRC, s) for s in SOURCES + HEADERS]
    files.append(os.path.join(INCLUDE, "nvfp4.h"))
    return files


def is_stale() -> bool:
    if not os.path.exists(LIB_PATH):
        return True
    t = os.path.getmtime(LIB_PATH)
    return any(os.path.getmtime(f) > t for f in _inputs())


def build(force: bool = False, verbose: bool = False, ptxas_verbose: bool = False) -> str:
    """Compile the library if it is missing or older than its sources; return its path."""
    with _lock:
        if not force and not is_stale():
            return LIB_PATH
        os.makedirs(BUILD_DIR, exist_ok=True)
        nvcc = _nvcc()
        extra = ["-Xptxas", "-v"] if ptxas_verbose else []
        procs = []
        objs = []
        for src in SOURCES:
            obj = os.path.join(BUILD_DIR, src.replace(".cu", ".o"))
            objs.append(obj)
            cmd = [nvcc, *NVCC_FLAGS, *extra, "-c", os.path.join(CSRC, src), "-o", obj]
            if verbose:
                print(" ".join(cmd), file=sys.stderr)
            procs.append((src, subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.STDOUT)))
        failed = []
        for src, p in procs:
            out, _ = p.communicate()
            text = out.decode(errors="replace")
            if p.returncode != 0:
                failed.append((src, text))
            elif verbose or ptxas_verbose:
                print(text, file=sys.stderr)
        if failed:
            msg = "\n".join(f"--- {s}\n{t}" for s, t in failed)
            raise RuntimeError(f"nvcc failed:\n{msg}")
        tmp = LIB_PATH + f".{os.getpid()}.tmp"
        link = [nvcc, "-shared", "-gencode", "arch=compute_100a,code=sm_100a", "--cudart", "static",
                *objs, "-o", tmp]
        subprocess.check_call(link)
        os.replace(tmp, LIB_PATH)
        return LIB_PATH


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv,
                ptxas_verbose="--ptxas" in sys.argv))
