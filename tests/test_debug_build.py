"""The RKL_DEBUG build (librkl_debug.so): the same library with device bounds
checks on tile indices, TMA coordinates and row indices.  On the CPU: it
builds, loads, says it is the debug build and exports every function that
include/rkl.h declares.  On the GPU: a small forward + backward through it
matches the oracle and no check fires (a failed check is reported by
rkl_device_error with its source line)."""

import ctypes
import os
import subprocess
import sys

import pytest

from full_vocabulary_reverse_b200.build import build
from tests.test_abi import declared_functions

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def debug_lib():
    return build(debug=True)


def test_debug_build_loads_and_exports_every_symbol(debug_lib):
    L = ctypes.CDLL(debug_lib)
    L.rkl_version.restype = ctypes.c_char_p
    assert b"debug bounds checks" in L.rkl_version()
    for n in declared_functions():
        assert hasattr(L, n), n


def test_binding_selects_the_debug_build(debug_lib):
    code = ("import sys; sys.path.insert(0, %r); from full_vocabulary_reverse_b200 import binding as rb; "
            "print(rb.lib().rkl_version().decode())" % ROOT)
    out = subprocess.run([sys.executable, "-c", code], env=dict(os.environ, RKL_LIBRARY="debug"),
                         capture_output=True, text=True, check=True, timeout=300).stdout
    assert "debug bounds checks" in out


GPU_CASE = r'''
import sys
sys.path.insert(0, sys.argv[1])
import numpy as np, torch
from full_vocabulary_reverse_b200 import binding as rb
from tests.gpu_cases import GRAD_RTOL, assert_tok_close, grad_rel_err, run_gpu, run_oracle, small_case
assert "debug" in rb.lib().rkl_version().decode()
for kw in (dict(B=2, Sm1=300, H=640, V=70000, payload="hidden"), dict(B=2, Sm1=200, H=128, V=2048, payload="logits"),
           dict(B=2, Sm1=64, H=40, V=300, payload="hidden", dtype="fp32")):
    inp = small_case(mask="random", seed=3, **kw)
    g = run_gpu(inp, 1)   # asserts rkl_device_error() == 0: no bounds check fired
    r = run_oracle(inp, 1)
    assert_tok_close(g["loss_tok"], r["loss_tok"])
    tol = GRAD_RTOL if kw.get("dtype", "bf16") == "bf16" else 1e-4
    assert grad_rel_err(g["dH_s"], r["dH_s"]) < tol and grad_rel_err(g["dW_s"], r["dW_s"]) < tol
print("debug build parity ok")
'''


@pytest.mark.gpu
def test_debug_build_small_parity_on_gpu(debug_lib):
    r = subprocess.run([sys.executable, "-c", GPU_CASE, ROOT], env=dict(os.environ, RKL_LIBRARY="debug"),
                       capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert r.returncode == 0, r.stdout[-2000:] + r.stderr[-4000:]
    assert "debug build parity ok" in r.stdout
