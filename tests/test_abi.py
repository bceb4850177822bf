"""The C ABI without a GPU: the library loads, exports every function that
include/rkl.h declares, and rejects bad arguments with a status (never an
abort) before touching the device."""

import ctypes
import os
import re

import pytest

from full_vocabulary_reverse_b200 import binding
from full_vocabulary_reverse_b200.build import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "rkl.h")


@pytest.fixture(scope="module")
def L():
    build()
    return binding.lib()


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(rkl_[a-z_]+)\s*\(", src)))


def test_header_declares_the_four_hot_path_calls():
    names = declared_functions()
    for n in ("rkl_compact_rows", "rkl_forward_hidden", "rkl_forward_logits", "rkl_backward"):
        assert n in names


def test_every_declared_symbol_is_exported(L):
    names = declared_functions()
    assert len(names) >= 10
    for n in names:
        assert hasattr(L, n), n
    # and the binding declares a signature for each of them
    assert set(names) <= set(binding._SIGS)


def test_version_and_kernel_names(L):
    assert b"sm_100a" in L.rkl_version()
    n = L.rkl_kernel_count()
    names = [L.rkl_kernel_name(i).decode() for i in range(n)]
    assert "fwd_dual_tc" in names and "grad_dw_dh_tc" in names and "teacher_lse" in names
    assert L.rkl_kernel_name(n) is None


def _fake(addr):
    return ctypes.c_void_p(addr)


GOOD = 0x10000  # 16-byte aligned fake device address (never dereferenced)


def _fwd(L, **kw):
    a = dict(h_s=GOOD, h_t=GOOD, W_s=GOOD, W_t=GOOD, dtype=0, B=2, Sm1=3, H=64, V=100, row_idx=GOOD, N=4, n_dev=0,
             red=1, loss_tok=GOOD, loss=GOOD, saved=GOOD, ws=GOOD, ws_bytes=1 << 40)
    a.update(kw)
    return L.rkl_forward_hidden(_fake(a["h_s"]) if a["h_s"] else None, _fake(a["h_t"]) if a["h_t"] else None,
                                _fake(a["W_s"]), _fake(a["W_t"]), a["dtype"], a["B"], a["Sm1"], a["H"], a["V"],
                                _fake(a["row_idx"]), a["N"], _fake(a["n_dev"]) if a["n_dev"] else None, a["red"],
                                _fake(a["loss_tok"]), _fake(a["loss"]), _fake(a["saved"]), _fake(a["ws"]),
                                a["ws_bytes"], None)


def test_forward_argument_errors(L):
    assert _fwd(L, h_s=0) == 1                      # NULL
    assert b"h_s" in L.rkl_last_error()
    assert _fwd(L, dtype=7) == 3                    # dtype enum
    assert _fwd(L, red=9) == 3                      # reduction enum
    assert _fwd(L, H=100) == 2                      # bf16 needs H % 64 == 0
    assert _fwd(L, N=7) == 2                        # N > B*Sm1
    assert _fwd(L, N=-1) == 2
    assert _fwd(L, B=0) == 2
    assert _fwd(L, W_s=GOOD + 4) == 4               # misaligned
    assert _fwd(L, ws_bytes=1000) == 5              # workspace too small
    assert b"workspace" in L.rkl_last_error()
    assert _fwd(L, n_dev=GOOD + 2) == 4             # device row count not 4-byte aligned
    assert b"n_dev" in L.rkl_last_error()
    assert _fwd(L, N=7, n_dev=GOOD) == 2            # the bound is still checked against B*Sm1


def test_logits_payload_needs_v_multiple_of_8_in_bf16(L):
    st = L.rkl_forward_logits(_fake(GOOD), _fake(GOOD), _fake(GOOD), 0, 2, 3, 64, 100 + 3, _fake(GOOD), 4, None, 1,
                              _fake(GOOD), _fake(GOOD), _fake(GOOD), _fake(GOOD), 1 << 40, None)
    assert st == 2


def test_backward_argument_errors(L):
    def bwd(**kw):
        a = dict(payload=0, W_t=GOOD, dH=GOOD, dW=GOOD, saved=GOOD, gl=GOOD, N=4, ws_bytes=1 << 40)
        a.update(kw)
        return L.rkl_backward(a["payload"], _fake(GOOD), _fake(GOOD), _fake(GOOD),
                              _fake(a["W_t"]) if a["W_t"] else None, 0, 2, 3, 64, 128, _fake(GOOD), a["N"], None, 1,
                              _fake(a["saved"]) if a["saved"] else None, _fake(a["gl"]) if a["gl"] else None, None,
                              _fake(a["dH"]) if a["dH"] else None, _fake(a["dW"]), _fake(GOOD), a["ws_bytes"], None)
    assert bwd(payload=5) == 3
    assert bwd(W_t=0) == 1                           # hidden payload needs W_t
    assert bwd(dH=0) == 1
    assert bwd(saved=0) == 1
    assert bwd(gl=GOOD + 8) == 4
    assert bwd(ws_bytes=16) == 5


def test_workspace_size(L):
    sz = ctypes.c_size_t()
    assert L.rkl_workspace_size(0, 0, 4096, 4, 2048, 2048, 151936, ctypes.byref(sz)) == 0
    big = sz.value
    assert L.rkl_workspace_size(0, 0, 128, 4, 2048, 2048, 151936, ctypes.byref(sz)) == 0
    assert sz.value < big
    # one more row than the batch holds is rejected
    assert L.rkl_workspace_size(0, 0, 4 * 2048 + 1, 4, 2048, 2048, 151936, ctypes.byref(sz)) == 2
    assert L.rkl_workspace_size(0, 0, 1, 1, 1, 64, 8, None) == 1
    # logits payload keeps no teacher hidden copy
    assert L.rkl_workspace_size(1, 0, 4096, 4, 2048, 2048, 151936, ctypes.byref(sz)) == 0
    assert sz.value < big


def test_compact_rows_argument_errors(L):
    assert L.rkl_compact_rows(None, 2, 3, _fake(GOOD), _fake(GOOD), None) == 1
    assert L.rkl_compact_rows(_fake(GOOD), 0, 3, _fake(GOOD), _fake(GOOD), None) == 2
    assert L.rkl_compact_rows(_fake(GOOD), 2, 3, _fake(GOOD + 2), _fake(GOOD), None) == 4


def test_binding_raises_without_library(monkeypatch, tmp_path):
    monkeypatch.setattr(binding, "LIB_PATH", str(tmp_path / "missing.so"))
    monkeypatch.setattr(binding, "_lib", None)
    with pytest.raises(binding.RKLError):
        binding.lib()


def test_multi_teacher_argument_errors(L):
    sz = ctypes.c_size_t()
    assert L.rkl_workspace_size_multi(0, 4096, 2, 4, 2048, 2048, 151936, ctypes.byref(sz)) == 0
    two = sz.value
    assert L.rkl_workspace_size_multi(0, 4096, 1, 4, 2048, 2048, 151936, ctypes.byref(sz)) == 0
    assert sz.value < two              # one extra pair tile of rows per extra teacher, plus slot maps
    assert L.rkl_workspace_size_multi(0, 4096, 0, 4, 2048, 2048, 151936, ctypes.byref(sz)) == 2
    assert L.rkl_workspace_size_multi(0, 4096, 17, 4, 2048, 2048, 151936, ctypes.byref(sz)) == 2

    def fwd(counts, n_teachers=2, N=4, tid=GOOD):
        arr = (ctypes.c_int32 * len(counts))(*counts)
        return L.rkl_forward_hidden_multi(_fake(GOOD), _fake(GOOD), _fake(GOOD), _fake(GOOD), n_teachers,
                                          _fake(tid) if tid else None, arr, 0, 2, 3, 64, 128, _fake(GOOD), N, 1,
                                          _fake(GOOD), _fake(GOOD), _fake(GOOD), _fake(GOOD), 1 << 40, None)
    assert fwd([1, 2]) == 2            # counts add up to 3, N = 4
    assert b"counts" in L.rkl_last_error()
    assert fwd([1, -1, 4], n_teachers=3) == 2
    assert fwd([2, 2], n_teachers=20) == 2
    assert fwd([2, 2], tid=0) == 1
    assert fwd([2, 2], tid=GOOD + 4) == 4
    assert L.rkl_compact_rows_multi(_fake(GOOD), None, 2, 3, 2, _fake(GOOD), _fake(GOOD), _fake(GOOD), None) == 1
    assert L.rkl_compact_rows_multi(_fake(GOOD), _fake(GOOD), 2, 3, 0, _fake(GOOD), _fake(GOOD), _fake(GOOD),
                                    None) == 2


def test_topk_argument_errors(L):
    def fwd_pair(k=8, targets=GOOD, ws_bytes=1 << 40):
        return L.rkl_forward_topk_pair(_fake(GOOD), _fake(GOOD), 0, 2, 3, 1000, _fake(GOOD), 4, None, k,
                                       _fake(targets) if targets else None, 1, _fake(GOOD), _fake(GOOD), _fake(GOOD),
                                       _fake(GOOD), ws_bytes, None)
    assert fwd_pair(k=-1) == 2
    assert fwd_pair(targets=0) == 1
    assert fwd_pair(targets=GOOD + 4) == 4
    assert fwd_pair(ws_bytes=8) == 5

    def fwd_hidden(dtype=0, k=8, targets=GOOD, H=64):
        return L.rkl_forward_topk_hidden(_fake(GOOD), _fake(GOOD), _fake(GOOD), _fake(GOOD), dtype, 2, 3, H, 1000,
                                         _fake(GOOD), 4, None, k, _fake(targets) if targets else None, 1, _fake(GOOD),
                                         _fake(GOOD), _fake(GOOD), _fake(GOOD), 1 << 40, None)
    assert fwd_hidden(dtype=1) == 6          # fp32: unsupported on this path
    assert fwd_hidden(k=-3) == 2
    assert fwd_hidden(targets=0) == 1
    assert fwd_hidden(H=100) == 2            # bf16 needs H % 64 == 0


def test_workspace_sizes_follow_the_layout(L):
    def size(payload, n, H=2048, V=151936, B=4, Sm1=2048):
        sz = ctypes.c_size_t()
        assert L.rkl_workspace_size(payload, 0, n, B, Sm1, H, V, ctypes.byref(sz)) == 0
        return sz.value
    # grows with the rows; the top-k hidden workspace adds the logit block and row constants
    assert size(0, 1) < size(0, 1000) < size(0, 8192)
    assert size(3, 4096) > size(0, 4096) + 2 * 2048 * 151936 * 4 - 1
    # the logits-pair workspace holds only per-row constants
    assert size(2, 8192) < 1 << 20
    # rows round up to whole 256-row pair tiles
    assert size(0, 1) == size(0, 256) and size(0, 257) > size(0, 256)
