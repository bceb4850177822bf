"""GPU parity of the teacher-per-row mode against the float64 oracle.

Rows are regrouped by teacher into whole 256-row tiles inside the library;
these cases cover several teachers per batch, a teacher with no rows, ragged
groups and vocabulary tails, more than one backward vocab chunk, the fp32
path, both reductions, bitwise agreement with the one-teacher entry points
when every head is the same, exact zeros under self-distillation, and the
full-size workload (sampled rows and whole-problem identities).
"""

import numpy as np
import pytest
import torch

from full_vocabulary_reverse_b200 import binding as rb
from full_vocabulary_reverse_b200.workloads import make_workload
from oracle import rkl_oracle as O
from tests.gpu_cases import (GRAD_RTOL, TOK_ATOL, TOK_RTOL, assert_tok_close, grad_rel_err, run_gpu, run_oracle,
                             small_case, to_np)

pytestmark = pytest.mark.gpu


def _check(inp, red, grad_rtol=GRAD_RTOL, grad_tok=None):
    g = run_gpu(inp, red, grad_tok=grad_tok)
    r = run_oracle(inp, red, grad_tok=grad_tok)
    counts, n_bad = O.count_rows_per_teacher(inp["mask"].numpy(), inp["teacher_idx"].numpy(), inp["W_t"].shape[0])
    assert n_bad == 0 and list(counts) == g["counts"]
    assert g["N"] == r["N"]
    assert np.array_equal(g["row_idx"].astype(np.int64), r["row_idx"])
    assert_tok_close(g["loss_tok"], r["loss_tok"])
    if r["loss"] is not None:
        assert abs(float(g["loss"]) - r["loss"]) <= 1e-4 + 1e-3 * abs(r["loss"])
    assert grad_rel_err(g["dH_s"], r["dH_s"]) < grad_rtol
    assert grad_rel_err(g["dW_s"], r["dW_s"]) < grad_rtol
    off = inp["mask"].reshape(-1).numpy() == 0
    assert np.all(to_np(g["loss_tok"]).reshape(-1)[off] == 0)
    assert np.all(to_np(g["dH_s"])[off] == 0)
    return g


@pytest.mark.parametrize("red", [1, 2])
def test_three_teachers_random_rows(red):
    # teachers drawn per position: three ragged groups, each padded to a tile
    inp = small_case(B=3, Sm1=300, H=192, V=1040, payload="hidden_multi", mask="random", seed=31, n_teachers=3,
                     teacher_assign="random")
    _check(inp, red)


def test_teacher_without_rows_and_several_chunks():
    # four teachers by sequence over three sequences: teacher 3 has no rows;
    # V spans two backward vocab chunks with a ragged tail
    inp = small_case(B=3, Sm1=200, H=128, V=65536 + 2072, payload="hidden_multi", mask="random", seed=32,
                     n_teachers=4, teacher_assign="sequence")
    g = _check(inp, 1)
    assert g["counts"][3] == 0


def test_per_token_upstream_gradient():
    inp = small_case(B=2, Sm1=260, H=128, V=800, payload="hidden_multi", mask="random", seed=33, n_teachers=2,
                     teacher_assign="random")
    gt = np.random.RandomState(5).normal(size=inp["mask"].shape)
    _check(inp, 0, grad_tok=gt)


def test_fp32_teachers():
    inp = small_case(B=2, Sm1=40, H=64, V=512, dtype="fp32", payload="hidden_multi", mask="random", seed=34,
                     n_teachers=3, teacher_assign="random")
    _check(inp, 2, grad_rtol=1e-4)


def test_identical_heads_match_one_teacher_bitwise():
    # every teacher head equal to W_t[0]: each row's loss, saved scalars and
    # dH row must be bitwise those of the one-teacher path (a row's results do
    # not depend on which tile it lands in); dW sums rows in another order.
    inp = small_case(B=3, Sm1=300, H=128, V=1500, payload="hidden_multi", mask="random", seed=35, n_teachers=3,
                     teacher_assign="random")
    inp["W_t"] = inp["W_t"][:1].repeat(3, 1, 1).contiguous()
    g = run_gpu(inp, 1)
    single = {k: v for k, v in inp.items() if k not in ("teacher_idx",)}
    single["W_t"] = inp["W_t"][0].contiguous()
    s = run_gpu(single, 1)
    assert torch.equal(g["loss_tok"], s["loss_tok"])
    assert torch.equal(g["saved"], s["saved"])
    assert torch.equal(g["dH_s"], s["dH_s"])
    assert grad_rel_err(g["dW_s"], to_np(s["dW_s"])) < 1e-5


def test_self_distillation_several_teachers_exact_zero():
    inp = small_case(B=3, Sm1=120, H=128, V=900, payload="hidden_multi", mask="random", seed=36, n_teachers=3,
                     teacher_assign="random")
    inp["h_t"] = inp["h_s"].clone()
    inp["W_t"] = inp["W_s"].unsqueeze(0).repeat(3, 1, 1).contiguous()
    g = run_gpu(inp, 2)
    for k in ("loss_tok", "dH_s", "dW_s"):
        assert float(torch.count_nonzero(g[k])) == 0, k
    assert float(g["loss"]) == 0.0


def test_empty_mask_several_teachers():
    inp = small_case(B=2, Sm1=50, H=64, V=300, payload="hidden_multi", mask="none", seed=37, n_teachers=2)
    g = run_gpu(inp, 1)
    assert g["N"] == 0 and float(g["loss"]) == 0.0
    for k in ("loss_tok", "dH_s", "dW_s"):
        assert float(torch.count_nonzero(g[k])) == 0, k


def test_out_of_range_teacher_index_is_rejected():
    inp = small_case(B=2, Sm1=50, H=64, V=300, payload="hidden_multi", mask="all", seed=38, n_teachers=2)
    tid = inp["teacher_idx"].clone()
    tid[1, 7] = 2
    with pytest.raises(rb.RKLError):
        rb.compact_rows_multi(inp["mask"].cuda(), tid.cuda(), 2)
    # an out-of-range index at a masked position is never read
    mask = inp["mask"].clone()
    mask[1, 7] = 0
    _, N, counts = rb.compact_rows_multi(mask.cuda(), tid.cuda(), 2)
    assert N == int(mask.sum()) and sum(counts) == N


@pytest.mark.slow
def test_multi_teacher_full_size():
    inp = make_workload("multi_teacher", device="cuda")
    red = inp["reduction"]
    mask = inp["mask"].cuda()
    B, Sm1 = mask.shape
    tid = inp["teacher_idx"]
    row_idx, N, counts = rb.compact_rows_multi(mask, tid, inp["W_t"].shape[0])
    lt, loss, saved = rb.forward_hidden_multi(inp["h_s"], inp["h_t"], inp["W_s"], inp["W_t"], tid, counts, B, Sm1,
                                              row_idx, N, red)
    gl = torch.ones(1, dtype=torch.float32, device="cuda")
    dH, dW = rb.backward_hidden_multi(inp["h_s"], inp["h_t"], inp["W_s"], inp["W_t"], tid, counts, B, Sm1, row_idx,
                                      N, red, saved, grad_loss=gl)
    torch.cuda.synchronize()
    assert rb.device_error() == 0
    assert N == int(inp["mask"].sum())
    # sampled rows, both teachers, tile edges included
    ridx = row_idx[:N].cpu().numpy()
    rs = np.random.RandomState(3)
    pick = np.unique(np.concatenate([[0, N - 1], rs.choice(N, size=12, replace=False)]))
    rows = ridx[pick]
    f = lambda t: t.float().cpu().numpy().astype(np.float64)  # noqa: E731
    rows_t = torch.as_tensor(rows, device="cuda")
    sub_mask = np.ones((1, len(rows)), np.uint8)
    sub_tid = tid.reshape(-1)[rows_t].cpu().numpy().reshape(1, -1)
    ref = O.forward_multi(f(inp["h_s"][rows_t]), f(inp["W_s"]), f(inp["h_t"][rows_t]), f(inp["W_t"]), sub_tid,
                          sub_mask, O.REDUCE_NONE)
    dH_ref, _ = O.backward_multi(f(inp["h_s"][rows_t]), f(inp["W_s"]), f(inp["h_t"][rows_t]), f(inp["W_t"]), sub_tid,
                                 sub_mask, O.REDUCE_NONE, grad_tok=np.full((1, len(rows)), 1.0 / N))
    g_tok = to_np(lt.reshape(-1)[rows_t])
    r_tok = ref["loss_tok"].reshape(-1)
    assert np.all(np.abs(g_tok - r_tok) <= TOK_ATOL + TOK_RTOL * np.abs(r_tok)), (g_tok, r_tok)
    np.testing.assert_allclose(to_np(saved[:N])[pick, 1], ref["lse_t"], atol=5e-4, rtol=0)
    g_dH = to_np(dH[rows_t])
    assert np.max(np.abs(g_dH - dH_ref)) / np.max(np.abs(dH_ref)) < GRAD_RTOL
    # whole-problem identities: sum_v dW = 0 and <dW, W_s> = <dH, h_s>
    dWd, dHd = dW.double(), dH.double()
    assert dWd.sum(dim=0).abs().max().item() <= 2e-2 * dWd.abs().sum(dim=0).max().item()
    a = (dWd * inp["W_s"].double()).sum().item()
    b = (dHd * inp["h_s"].double()).sum().item()
    assert abs(a - b) <= 1e-3 * (dWd * inp["W_s"].double()).abs().sum().item()
    off = ~inp["mask"].reshape(-1).bool()
    assert float(torch.count_nonzero(lt.reshape(-1)[off])) == 0
    assert float(torch.count_nonzero(dH[off])) == 0


def test_autograd_wrapper_several_teachers():
    inp = small_case(B=2, Sm1=100, H=128, V=700, payload="hidden_multi", mask="random", seed=39, n_teachers=3,
                     teacher_assign="random")
    h_s = inp["h_s"].cuda().requires_grad_(True)
    W_s = inp["W_s"].cuda().requires_grad_(True)
    loss, loss_tok = rb.reverse_kl_hidden_multi(h_s, inp["h_t"].cuda(), W_s, inp["W_t"].cuda(),
                                                inp["teacher_idx"].cuda(), inp["mask"].cuda(), 2)
    (loss + 0.5 * loss_tok.sum()).backward()
    gt = np.full(inp["mask"].shape, 0.5)
    r = run_oracle(inp, 2, grad_tok=gt)
    assert abs(float(loss.detach()) - r["loss"]) <= 1e-4 + 1e-3 * abs(r["loss"])
    assert grad_rel_err(h_s.grad.float(), r["dH_s"]) < GRAD_RTOL
    assert grad_rel_err(W_s.grad.float(), r["dW_s"]) < GRAD_RTOL
