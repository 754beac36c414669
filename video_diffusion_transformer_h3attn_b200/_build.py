"""Build of the h3attn CUDA library (libh3attn.so) for sm_100a with nvcc.

The library is one translation unit (csrc/h3attn_api.cu pulls in the kernels),
linked against the static CUDA runtime so it loads without a GPU and does not
depend on which libcudart the host process already has.
"""
from __future__ import annotations

import glob
import os
import subprocess

PKG_DIR = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG_DIR)
CSRC = os.path.join(PKG_DIR, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIBRARY = os.path.join(PKG_DIR, "libh3attn.so")
# the same sources with H3ATTN_DEBUG_BOUNDS: every kernel checks its store indices
# against its own launch's extents and reports instead of storing out of place
DEBUG_LIBRARY = os.path.join(PKG_DIR, "libh3attn_debug.so")
MAIN_SOURCE = os.path.join(CSRC, "h3attn_api.cu")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC", "-shared",
    "-cudart", "static",
    "-diag-suppress", "177",
]


def _nvcc() -> str:
    cand = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "bin", "nvcc")
    return cand if os.path.exists(cand) else "nvcc"


def _sources():
    return sorted(glob.glob(os.path.join(CSRC, "*"))) + sorted(glob.glob(os.path.join(INCLUDE, "*.h")))


def needs_build(output: str = LIBRARY) -> bool:
    if not os.path.exists(output):
        return True
    t = os.path.getmtime(output)
    return any(os.path.getmtime(s) > t for s in _sources())


def build(force: bool = False, output: str = LIBRARY, verbose: bool = False, debug_bounds: bool = False) -> str:
    """Compile libh3attn.so (or, with debug_bounds, libh3attn_debug.so) in place;
    skipped when the library is newer than every source."""
    if debug_bounds and output == LIBRARY:
        output = DEBUG_LIBRARY
    if not force and not needs_build(output):
        return output
    tmp = output + ".tmp%d" % os.getpid()
    cmd = [_nvcc(), *NVCC_FLAGS, "-I" + INCLUDE, "-o", tmp, MAIN_SOURCE]
    if debug_bounds:
        cmd.insert(1, "-DH3ATTN_DEBUG_BOUNDS")
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
    subprocess.run(cmd, check=True)
    os.replace(tmp, output)
    return output


if __name__ == "__main__":
    print(build(force=True, verbose=True))
