"""Compile the sm_100a libraries in-tree with nvcc.

  libgdn.so          the mixer (C ABI declared in include/gdn.h)
  libgdn_debug.so    the same with GDN_DEBUG: every workspace access of the prefill kernels is
                     bounds-checked (an access outside is skipped and reported, error bit 64)
  libgdn_selftest.so tcgen05/UMMA layout self-test kernel used by the GPU tests
"""
from __future__ import annotations

import os
import shutil
import subprocess

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-std=c++17", "-lineinfo",
    "-shared", "-Xcompiler", "-fPIC",
    "-diag-suppress", "177",
]

_GDN_SOURCES = ["gdn_api.cu", "gdn_prefill.cu", "gdn_decode.cu", "gdn_noalloc.cu", "gdn_gemm.cu", "gdn_attention.cu"]
TARGETS = {
    "libgdn.so": _GDN_SOURCES,
    "libgdn_debug.so": _GDN_SOURCES,
    "libgdn_selftest.so": ["umma_selftest.cu", "wait_selftest.cu"],
}
EXTRA_FLAGS = {"libgdn_debug.so": ["-DGDN_DEBUG"]}


def _nvcc() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found: the gated-delta-rule CUDA library cannot be built")


def _deps(srcs):
    files = [os.path.join(CSRC, s) for s in srcs]
    files += [os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith(".cuh")]
    files.append(os.path.join(INCLUDE, "gdn.h"))
    return files


def lib_path(name: str = "libgdn.so") -> str:
    return os.path.join(PKG, name)


def build(force: bool = False, verbose: bool = False) -> list[str]:
    built = []
    for name, srcs in TARGETS.items():
        out = lib_path(name)
        stale = force or not os.path.exists(out) or any(
            os.path.getmtime(f) > os.path.getmtime(out) for f in _deps(srcs))
        if stale:
            tmp = out + f".tmp{os.getpid()}"
            cmd = [_nvcc(), *NVCC_FLAGS, *EXTRA_FLAGS.get(name, []), "-I", INCLUDE, "-o", tmp,
                   *[os.path.join(CSRC, s) for s in srcs]]
            if verbose:
                print(" ".join(cmd))
            subprocess.run(cmd, check=True)
            os.replace(tmp, out)
        built.append(out)
    return built


if __name__ == "__main__":
    for p in build(force=True, verbose=True):
        print(p)
