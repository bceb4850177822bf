"""rkl_forward_hidden_noalloc: the forward for callers that cannot allocate
device memory when they call (runtimes that plan all device memory up front,
code where cudaMalloc is forbidden or would stall).  Its scratch is a fixed
array inside the library instead of a caller workspace.

The GPU test drives it through the C ABI (ctypes, raw pointers) and compares
it with rkl_forward_hidden, which takes a caller workspace, on two calls in a
row with different problems, so that whatever the first call left in the
shared array cannot leak into the second.  A second test checks it against
the float64 oracle on a small bf16 and a small fp32 problem, so that a fault
shared with the workspace path would show too.  This file is collected last."""

import ctypes

import numpy as np
import pytest
import torch

from full_vocabulary_reverse_b200 import binding as rb
from full_vocabulary_reverse_b200.build import build
from full_vocabulary_reverse_b200.workloads import make_inputs

TOK_ATOL, TOK_RTOL = 1e-4, 1e-3  # per-token loss tolerance used by the parity tests


def _p(t):
    return ctypes.c_void_p(t.data_ptr())


def _problem(B, Sm1, H, V, seed, dtype="bf16"):
    inp = make_inputs(B, Sm1, H, V, dtype=dtype, payload="hidden", mask="random", weights="perturbed",
                      seed=seed, device="cuda", teacher_noise=0.05)
    return inp


def _forward(L, inp, use_static):
    B, Sm1 = inp["mask"].shape
    H = inp["h_s"].shape[1]
    V = inp["W_s"].shape[0]
    s = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    row_idx = torch.empty(B * Sm1, dtype=torch.int32, device="cuda")
    n_dev = torch.empty(1, dtype=torch.int32, device="cuda")
    assert L.rkl_compact_rows(_p(inp["mask"]), B, Sm1, _p(row_idx), _p(n_dev), s) == 0
    N = int(n_dev.item())
    loss_tok = torch.full((B, Sm1), float("nan"), device="cuda")
    loss = torch.full((1,), float("nan"), device="cuda")
    saved = torch.full((max(N, 1), 3), float("nan"), device="cuda")
    dt = 0 if inp["h_s"].dtype == torch.bfloat16 else 1
    args = (_p(inp["h_s"]), _p(inp["h_t"]), _p(inp["W_s"]), _p(inp["W_t"]), dt, B, Sm1, H, V, _p(row_idx), N, 1,
            _p(loss_tok), _p(loss), _p(saved))
    if use_static:
        st = L.rkl_forward_hidden_noalloc(*args, s)
    else:
        nbytes = ctypes.c_size_t(0)
        assert L.rkl_workspace_size(0, dt, N, B, Sm1, H, V, ctypes.byref(nbytes)) == 0
        ws = torch.empty(nbytes.value, dtype=torch.uint8, device="cuda")
        # the workspace entry point takes an optional device row count after N
        st = L.rkl_forward_hidden(*args[:11], None, *args[11:], _p(ws), nbytes.value, s)
    assert st == 0, L.rkl_last_error().decode()
    torch.cuda.synchronize()
    return loss_tok, loss, saved[:N]


@pytest.mark.gpu
def test_noalloc_forward_matches_workspace_forward_twice():
    build()
    L = rb.lib()
    # two different problems in a row (different N, H, V and vocab tails)
    for shape, seed in (((3, 700, 256, 9000), 11), ((2, 1500, 512, 20000), 12)):
        inp = _problem(*shape, seed)
        ref_tok, ref_loss, ref_saved = _forward(L, inp, use_static=False)
        tok, loss, saved = _forward(L, inp, use_static=True)
        r = ref_tok.double().cpu().numpy()
        g = tok.double().cpu().numpy()
        assert np.all(np.abs(g - r) <= TOK_ATOL + TOK_RTOL * np.abs(r))
        assert abs(float(loss) - float(ref_loss)) <= TOK_ATOL + TOK_RTOL * abs(float(ref_loss))
        assert torch.allclose(saved, ref_saved, atol=TOK_ATOL, rtol=TOK_RTOL)
    code = ctypes.c_int32(0)
    assert L.rkl_device_error(ctypes.byref(code)) == 0 and code.value == 0


@pytest.mark.gpu
@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
def test_noalloc_forward_matches_the_oracle(dtype):
    from oracle import rkl_oracle as O

    build()
    L = rb.lib()
    H = 128 if dtype == "bf16" else 40
    inp = _problem(2, 300, H, 3000, 21, dtype=dtype)
    tok, loss, saved = _forward(L, inp, use_static=True)
    f = lambda t: t.double().cpu().numpy()  # noqa: E731
    ref = O.forward(f(inp["h_s"]), f(inp["W_s"]), f(inp["h_t"]), f(inp["W_t"]), inp["mask"].cpu().numpy(), 1)
    g = tok.double().cpu().numpy()
    assert np.all(np.abs(g - ref["loss_tok"]) <= TOK_ATOL + TOK_RTOL * np.abs(ref["loss_tok"]))
    assert abs(float(loss) - ref["loss"]) <= TOK_ATOL + TOK_RTOL * abs(ref["loss"])
    code = ctypes.c_int32(0)
    assert L.rkl_device_error(ctypes.byref(code)) == 0 and code.value == 0


@pytest.mark.gpu
def test_noalloc_rejects_problems_beyond_the_static_scratch():
    build()
    L = rb.lib()
    fake = ctypes.c_void_p(0x10000)
    # 8192 rows x 2048 hidden in bf16 needs 2 x 32 MiB for the compacted rows alone
    st = L.rkl_forward_hidden_noalloc(fake, fake, fake, fake, 0, 4, 2048, 2048, 151936, fake, 8192, 1,
                                      fake, fake, fake, None)
    assert st == 5
    msg = L.rkl_last_error().decode()
    assert "static limit" in msg and "33554432" in msg
