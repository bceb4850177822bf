"""Every compute entry point of librkl.so opens an NVTX range named after
itself and closes it on return (also on an argument error), so a profiler
that listens to NVTX shows each call with its kernels under it.

No GPU is needed: the calls are made with NULL arguments, which every entry
point rejects after opening its range.  The ranges are recorded by a small
NVTX injection library (tests/nvtx_recorder.c) built here with gcc.
"""

import os
import shutil
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CUDA_INC = "/usr/local/cuda/include"

ENTRY_POINTS = [
    "rkl_compact_rows", "rkl_compact_rows_multi", "rkl_forward_hidden", "rkl_forward_logits",
    "rkl_forward_hidden_ex", "rkl_forward_logits_ex", "rkl_backward", "rkl_forward_logits_pair",
    "rkl_backward_logits_pair", "rkl_forward_topk_pair", "rkl_backward_topk_pair", "rkl_forward_topk_hidden",
    "rkl_backward_topk_hidden", "rkl_forward_hidden_multi", "rkl_backward_hidden_multi",
    "rkl_forward_hidden_noalloc", "rkl_forward_topk_logits", "rkl_backward_topk_logits",
]

CALLER = r'''
import ctypes, sys
sys.path.insert(0, sys.argv[1])
from full_vocabulary_reverse_b200 import binding as rb
L = rb.lib()
for name in sys.argv[2:]:
    fn = getattr(L, name)
    args = [None if t is ctypes.c_void_p or hasattr(t, "contents") else 0 for t in fn.argtypes]
    assert fn(*args) != 0, name  # rejected: NULL pointers / empty shapes
'''


@pytest.fixture(scope="module")
def recorder(tmp_path_factory):
    gcc = shutil.which("gcc")
    if gcc is None or not os.path.exists(os.path.join(CUDA_INC, "nvtx3", "nvToolsExt.h")):
        pytest.skip("gcc or the NVTX headers are not available")
    out = str(tmp_path_factory.mktemp("nvtx") / "libnvtx_recorder.so")
    subprocess.run([gcc, "-shared", "-fPIC", "-O1", "-I", CUDA_INC, "-o", out,
                    os.path.join(ROOT, "tests", "nvtx_recorder.c")], check=True)
    return out


def test_every_entry_point_opens_and_closes_a_named_range(recorder, tmp_path):
    from full_vocabulary_reverse_b200.build import build
    build()
    log = tmp_path / "ranges.log"
    env = dict(os.environ, NVTX_INJECTION64_PATH=recorder, RKL_NVTX_LOG=str(log))
    subprocess.run([sys.executable, "-c", CALLER, ROOT] + ENTRY_POINTS, env=env, check=True, timeout=300)
    lines = log.read_text().split("\n")[:-1]
    pushes = [ln[5:] for ln in lines if ln.startswith("push ")]
    assert pushes == ENTRY_POINTS
    # each push is closed before the next call's push
    assert lines == [x for name in ENTRY_POINTS for x in ("push " + name, "pop")]
