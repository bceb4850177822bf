"""Builds librkl.so in-tree with nvcc for sm_100a (B200).

    python -m full_vocabulary_reverse_b200.build [--force] [--debug]

--debug builds librkl_debug.so instead: the same library compiled with
-DRKL_DEBUG, whose kernels check tile indices, TMA coordinates and row
indices at run time, skip a failing access and report its source line
through rkl_device_error (the binding loads it when RKL_LIBRARY=debug).

Cross-compiles without a GPU.  The CUDA runtime is linked statically; the
driver's cuTensorMapEncodeTiled is resolved at run time through
cudaGetDriverEntryPoint, so the library has no link-time dependency on
libcuda.
"""

from __future__ import annotations

import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
ROOT = os.path.dirname(HERE)
LIB = os.path.join(HERE, "librkl.so")
LIB_DEBUG = os.path.join(HERE, "librkl_debug.so")
SOURCES = ["api.cu", "tc_kernels.cu", "small_kernels.cu", "simt_kernels.cu", "topk_kernels.cu"]
HEADERS = ["kernels.h", "sm100.cuh", "bounds.cuh"]


def nvcc_path():
    cand = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(cand):
        raise RuntimeError("nvcc not found")
    return cand


def _stale(lib):
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    deps = [os.path.join(CSRC, f) for f in SOURCES + HEADERS] + [os.path.join(ROOT, "include", "rkl.h"), __file__]
    return any(os.path.getmtime(d) > t for d in deps if os.path.exists(d))


def build(force=False, verbose=False, debug=False):
    lib = LIB_DEBUG if debug else LIB
    if not force and not _stale(lib):
        return lib
    cmd = [nvcc_path(), "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo", "-std=c++17",
           "--cudart", "static", "-shared", "-Xcompiler", "-fPIC", "-Xcompiler", "-Wall",
           "-I", os.path.join(ROOT, "include"), "-o", lib + ".tmp"]
    if debug:
        cmd += ["-DRKL_DEBUG"]
    cmd += [os.path.join(CSRC, f) for f in SOURCES]
    if verbose:
        print(" ".join(cmd))
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        sys.stderr.write(r.stdout + r.stderr)
        raise RuntimeError("nvcc failed building %s" % os.path.basename(lib))
    os.replace(lib + ".tmp", lib)
    return lib


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose=True, debug="--debug" in sys.argv))
