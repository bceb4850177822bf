"""GPU parity of librkl.so against the float64 CPU oracle (small shapes).

The shapes span several 128-row and 128-column tiles with ragged tails, more
than one backward vocab chunk, and the degenerate cases of the method: an
empty mask, a single trainable token, all rows trainable, and teacher ==
student.  Per-token losses must agree within |dL| <= 1e-4 + 1e-3 |L|,
gradients within 2e-2 relative max-norm, compaction bit-exactly.
"""

import numpy as np
import pytest
import torch

from full_vocabulary_reverse_b200 import binding as rb
from full_vocabulary_reverse_b200.workloads import make_mask
from oracle import rkl_oracle as O
from tests.gpu_cases import (GRAD_RTOL, assert_tok_close, grad_rel_err, run_gpu, run_oracle, small_case, to_np)

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("B,Sm1,kind", [(1, 1, "all"), (3, 7, "random"), (4, 2048, "prefix"), (8, 4096, "suffix256"),
                                        (5, 3001, "random"), (2, 9000, "none"), (3, 5000, "one")])
def test_compact_rows_bit_exact(B, Sm1, kind):
    mask = make_mask(kind, B, Sm1, seed=B * 1000 + Sm1)
    row_idx, N = rb.compact_rows(torch.from_numpy(mask).cuda())
    ref, n_ref = O.compact_rows(mask)
    assert N == n_ref
    assert np.array_equal(row_idx[:N].cpu().numpy().astype(np.int64), ref)


@pytest.mark.parametrize("red", [1, 2])
def test_hidden_bf16_forward_backward(red):
    inp = small_case(B=3, Sm1=150, H=192, V=1000, mask="random", seed=11)
    g = run_gpu(inp, red)
    r = run_oracle(inp, red)
    assert g["N"] == r["N"]
    assert_tok_close(g["loss_tok"], r["loss_tok"])
    assert abs(float(g["loss"]) - r["loss"]) <= 1e-4 + 1e-3 * abs(r["loss"])
    assert grad_rel_err(g["dH_s"], r["dH_s"]) < GRAD_RTOL
    assert grad_rel_err(g["dW_s"], r["dW_s"]) < GRAD_RTOL


def test_hidden_bf16_multi_chunk_ragged():
    # V spans three backward chunks (equal widths of at most 65536 columns)
    # with a ragged last tile; N = 200ish rows: one partial 256-row pair tile.
    inp = small_case(B=2, Sm1=200, H=256, V=131072 + 1040, mask="random", seed=5)
    g = run_gpu(inp, 1)
    r = run_oracle(inp, 1)
    assert_tok_close(g["loss_tok"], r["loss_tok"])
    assert grad_rel_err(g["dH_s"], r["dH_s"]) < GRAD_RTOL
    assert grad_rel_err(g["dW_s"], r["dW_s"]) < GRAD_RTOL


def test_saved_row_scalars():
    inp = small_case(B=2, Sm1=64, H=128, V=700, mask="random", seed=3)
    g = run_gpu(inp, 1, backward=False)
    r = run_oracle(inp, 1, backward=False)
    saved = to_np(g["saved"])
    np.testing.assert_allclose(saved[:, 0], r["lse_s"], atol=2e-4, rtol=1e-5)
    np.testing.assert_allclose(saved[:, 1], r["lse_t"], atol=2e-4, rtol=1e-5)


@pytest.mark.parametrize("red", [1, 2])
def test_self_distillation_exact_zero(red):
    inp = small_case(B=3, Sm1=100, H=128, V=1500, mask="random", weights="same", seed=9)
    g = run_gpu(inp, red)
    assert float(torch.count_nonzero(g["loss_tok"])) == 0
    assert float(g["loss"]) == 0.0
    assert float(torch.count_nonzero(g["dH_s"])) == 0
    assert float(torch.count_nonzero(g["dW_s"])) == 0


@pytest.mark.parametrize("red", [1, 2])
def test_logits_payload(red):
    inp = small_case(B=2, Sm1=130, H=128, V=1200, payload="logits", mask="random", seed=21)
    g = run_gpu(inp, red)
    r = run_oracle(inp, red)
    assert_tok_close(g["loss_tok"], r["loss_tok"])
    assert grad_rel_err(g["dH_s"], r["dH_s"]) < GRAD_RTOL
    assert grad_rel_err(g["dW_s"], r["dW_s"]) < GRAD_RTOL


@pytest.mark.parametrize("H", [192, 320])
def test_logits_payload_odd_k_steps(H):
    # H / 64 odd: the logits-payload kernels stage 128 of K at a time, so
    # their last stage holds one 64-deep box of data and one zero-filled box
    # past H (whose MMAs add zeros)
    inp = small_case(B=2, Sm1=150, H=H, V=1504, payload="logits", mask="random", seed=H)
    g = run_gpu(inp, 1)
    r = run_oracle(inp, 1)
    assert_tok_close(g["loss_tok"], r["loss_tok"])
    assert abs(float(g["loss"]) - r["loss"]) <= 1e-4 + 1e-3 * abs(r["loss"])
    assert grad_rel_err(g["dH_s"], r["dH_s"]) < GRAD_RTOL
    assert grad_rel_err(g["dW_s"], r["dW_s"]) < GRAD_RTOL


def test_logits_payload_all_rows():
    inp = small_case(B=2, Sm1=128, H=64, V=520, payload="logits", mask="all", seed=22)
    g = run_gpu(inp, 1)
    r = run_oracle(inp, 1)
    assert_tok_close(g["loss_tok"], r["loss_tok"])
    assert grad_rel_err(g["dH_s"], r["dH_s"]) < GRAD_RTOL
    assert grad_rel_err(g["dW_s"], r["dW_s"]) < GRAD_RTOL


@pytest.mark.parametrize("payload", ["hidden", "logits"])
def test_fp32_tiny(payload):
    # the tiny fp32 workload shape: B=2, S-1=32, H=64, V=512, mask all ones
    inp = small_case(B=2, Sm1=32, H=64, V=512, dtype="fp32", payload=payload, mask="all",
                     weights="independent", seed=1235)
    g = run_gpu(inp, 1)
    r = run_oracle(inp, 1)
    assert_tok_close(g["loss_tok"], r["loss_tok"])
    assert grad_rel_err(g["dH_s"], r["dH_s"]) < 1e-4
    assert grad_rel_err(g["dW_s"], r["dW_s"]) < 1e-4


def test_fp32_ragged_nested():
    inp = small_case(B=3, Sm1=45, H=37, V=333, dtype="fp32", mask="random", seed=4)
    g = run_gpu(inp, 2)
    r = run_oracle(inp, 2)
    assert_tok_close(g["loss_tok"], r["loss_tok"])
    assert grad_rel_err(g["dH_s"], r["dH_s"]) < 1e-4
    assert grad_rel_err(g["dW_s"], r["dW_s"]) < 1e-4


@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
def test_empty_mask(dtype):
    inp = small_case(B=2, Sm1=50, H=64, V=300, dtype=dtype, mask="none", seed=2)
    g = run_gpu(inp, 1)
    assert g["N"] == 0
    assert float(g["loss"]) == 0.0
    for k in ("loss_tok", "dH_s", "dW_s"):
        t = g[k]
        assert bool(torch.isfinite(t).all()) and float(torch.count_nonzero(t)) == 0


def test_single_trainable_token():
    inp = small_case(B=3, Sm1=77, H=128, V=640, mask="one", seed=8)
    g = run_gpu(inp, 2)
    r = run_oracle(inp, 2)
    assert g["N"] == 1
    assert_tok_close(g["loss_tok"], r["loss_tok"])
    assert grad_rel_err(g["dH_s"], r["dH_s"]) < GRAD_RTOL
    assert grad_rel_err(g["dW_s"], r["dW_s"]) < GRAD_RTOL


def test_masked_rows_exact_zero_and_compact_equals_full():
    inp = small_case(B=2, Sm1=300, H=128, V=900, mask="random", seed=13)
    comp = run_gpu(inp, 0, grad_tok=np.ones((2, 300)))
    full_inp = dict(inp)
    full_inp["mask"] = torch.ones_like(inp["mask"])
    full = run_gpu(full_inp, 0, grad_tok=inp["mask"].numpy().astype(np.float64))
    m = inp["mask"].reshape(-1).bool().cuda()
    lc, lf = comp["loss_tok"].reshape(-1), full["loss_tok"].reshape(-1)
    assert float(torch.count_nonzero(lc[~m])) == 0
    assert float(torch.count_nonzero(comp["dH_s"][~m])) == 0
    # a row's results do not depend on which other rows are in the batch
    assert torch.equal(lc[m], lf[m])
    assert torch.equal(comp["dH_s"][m], full["dH_s"][m])
    assert grad_rel_err(comp["dW_s"], to_np(full["dW_s"])) < 1e-3


def test_grad_tok_and_grad_loss_together():
    inp = small_case(B=2, Sm1=90, H=128, V=700, mask="random", seed=17)
    rs = np.random.RandomState(0)
    gt = rs.normal(size=(2, 90))
    g = run_gpu(inp, 2, grad_loss=0.5, grad_tok=gt)
    r = run_oracle(inp, 2, grad_loss=0.5, grad_tok=gt)
    assert grad_rel_err(g["dH_s"], r["dH_s"]) < GRAD_RTOL
    assert grad_rel_err(g["dW_s"], r["dW_s"]) < GRAD_RTOL


def test_deterministic_bitwise():
    inp = small_case(B=2, Sm1=200, H=128, V=1100, mask="random", seed=30)
    a = run_gpu(inp, 1)
    b = run_gpu(inp, 1)
    for k in ("loss_tok", "loss", "dH_s", "dW_s"):
        assert torch.equal(a[k], b[k]), k


def test_autograd_wrapper():
    inp = small_case(B=2, Sm1=64, H=128, V=500, mask="random", seed=40)
    h_s = inp["h_s"].cuda().requires_grad_(True)
    W_s = inp["W_s"].cuda().requires_grad_(True)
    loss, loss_tok = rb.reverse_kl_hidden(h_s, inp["h_t"].cuda(), W_s, inp["W_t"].cuda(), inp["mask"].cuda(), 1)
    loss.backward()
    r = run_oracle(inp, 1)
    assert abs(float(loss.detach()) - r["loss"]) <= 1e-4 + 1e-3 * abs(r["loss"])
    assert grad_rel_err(h_s.grad.float(), r["dH_s"]) < GRAD_RTOL
    assert grad_rel_err(W_s.grad.float(), r["dW_s"]) < GRAD_RTOL


# ---------------------------------------------------------------- logits pair
def _pair_case(B, Sm1, V, dtype="bf16", mask="random", seed=0, same=False):
    from full_vocabulary_reverse_b200.workloads import make_inputs
    return make_inputs(B, Sm1, 0, V, dtype=dtype, payload="logits_pair", mask=mask,
                       weights="same" if same else "perturbed", seed=seed, device="cuda")


def _pair_run(inp, red, grad_tok=None):
    mask = inp["mask"]
    B, Sm1 = mask.shape
    row_idx, N = rb.compact_rows(mask)
    lt, loss, saved = rb.forward_logits_pair(inp["student_logits"], inp["teacher_logits"], B, Sm1, row_idx, N, red)
    gl = torch.ones(1, device="cuda")
    gt = None if grad_tok is None else torch.as_tensor(grad_tok, dtype=torch.float32).cuda()
    dz = rb.backward_logits_pair(inp["student_logits"], inp["teacher_logits"], B, Sm1, row_idx, N, red, saved,
                                 grad_loss=gl, grad_tok=gt)
    torch.cuda.synchronize()
    assert rb.device_error() == 0
    return lt, loss, saved[:N], dz, N


@pytest.mark.parametrize("V,dtype,red", [(1000, "bf16", 1), (1003, "bf16", 2), (777, "fp32", 1), (4096, "fp32", 2)])
def test_logits_pair_small(V, dtype, red):
    inp = _pair_case(3, 70, V, dtype=dtype, seed=V)
    lt, loss, saved, dz, N = _pair_run(inp, red)
    m = inp["mask"].cpu().numpy()
    zs, zt = to_np(inp["student_logits"]), to_np(inp["teacher_logits"])
    ref = O.forward_logits_pair(zs, zt, m, red)
    rdz = O.backward_logits_pair(zs, zt, m, red)
    assert_tok_close(lt, ref["loss_tok"])
    assert abs(float(loss) - ref["loss"]) <= 1e-4 + 1e-3 * abs(ref["loss"])
    # dz is rounded to the logits' dtype: bf16 relative error ~2^-8 per element
    tol = 2e-2 if dtype == "bf16" else 1e-4
    assert grad_rel_err(dz, rdz) < tol
    off = m.reshape(-1) == 0
    assert float(torch.count_nonzero(dz[torch.as_tensor(off).cuda()])) == 0


def test_logits_pair_self_distill_and_empty():
    inp = _pair_case(2, 50, 999, seed=3, same=True)
    lt, loss, saved, dz, N = _pair_run(inp, 2)
    assert float(torch.count_nonzero(lt)) == 0 and float(loss) == 0.0 and float(torch.count_nonzero(dz)) == 0
    inp = _pair_case(2, 50, 999, seed=4, mask="none")
    lt, loss, saved, dz, N = _pair_run(inp, 1)
    assert N == 0 and float(loss) == 0.0 and float(torch.count_nonzero(dz)) == 0
    assert bool(torch.isfinite(dz.float()).all())


def test_logits_pair_matches_logits_payload_forward():
    # the logits-pair forward and the LM-head forward agree when z_s = h_s W_s^T is given explicitly
    inp = small_case(B=2, Sm1=64, H=128, V=640, payload="logits", mask="random", seed=31)
    h_s, W_s = inp["h_s"].cuda(), inp["W_s"].cuda()
    zs = (h_s.double() @ W_s.double().t()).to(torch.bfloat16)
    mask = inp["mask"].cuda()
    row_idx, N = rb.compact_rows(mask)
    a = rb.forward_logits_pair(zs, inp["teacher_logits"].cuda(), 2, 64, row_idx, N, 1)[0]
    ref = O.forward_logits_pair(to_np(zs), to_np(inp["teacher_logits"]), inp["mask"].numpy(), 1)
    assert_tok_close(a, ref["loss_tok"])


# ---------------------------------------------------------------- student entropy / target log-prob
@pytest.mark.parametrize("payload,dtype,V", [("hidden", "bf16", 1000), ("logits", "bf16", 1200),
                                             ("hidden", "fp32", 333), ("logits", "fp32", 520)])
def test_student_entropy_and_target_logprob(payload, dtype, V):
    H = 128 if dtype == "bf16" else 40
    inp = small_case(B=3, Sm1=90, H=H, V=V, dtype=dtype, payload=payload, mask="random", seed=V + 7)
    rs = np.random.RandomState(V)
    targets = torch.from_numpy(rs.randint(0, V, size=(3, 90)).astype(np.int32))
    mask = inp["mask"].cuda()
    row_idx, N = rb.compact_rows(mask)
    teacher = inp["h_t"].cuda() if payload == "hidden" else inp["teacher_logits"].cuda()
    W_t = inp["W_t"].cuda() if payload == "hidden" else None
    lt, loss, saved, ent, tlp = rb.forward_with_stats(inp["h_s"].cuda(), teacher, inp["W_s"].cuda(), W_t, 3, 90,
                                                      row_idx, N, 1, targets=targets)
    torch.cuda.synchronize()
    assert rb.device_error() == 0
    h_s, W_s = to_np(inp["h_s"]), to_np(inp["W_s"])
    m = inp["mask"].numpy()
    r_ent, r_tlp = O.student_stats(h_s, W_s, m, targets.numpy())
    # the loss outputs are unchanged by the extra statistics
    assert_tok_close(lt, run_oracle(inp, 1, backward=False)["loss_tok"])
    assert np.max(np.abs(to_np(ent) - r_ent)) <= 1e-4 + 1e-3 * np.max(np.abs(r_ent))
    assert np.all(np.abs(to_np(tlp) - r_tlp) <= 1e-4 + 1e-3 * np.abs(r_tlp))
    off = torch.as_tensor(m.reshape(-1) == 0)
    assert float(torch.count_nonzero(ent.reshape(-1).cpu()[off])) == 0
    assert float(torch.count_nonzero(tlp.reshape(-1).cpu()[off])) == 0


@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
@pytest.mark.parametrize("B,Sm1,H,V,mask", [(1, 1, 64, 1, "all"), (1, 3, 64, 2, "all"), (2, 5, 128, 7, "all"),
                                            (3, 40, 64, 300, "one"), (1, 257, 64, 257, "all")])
def test_degenerate_shapes(dtype, B, Sm1, H, V, mask):
    # a one-token vocabulary (L = 0, zero gradients), two tokens, a single
    # trainable row, and one row past a whole pair tile
    inp = small_case(B=B, Sm1=Sm1, H=H, V=V, dtype=dtype, mask=mask, seed=B * 100 + V)
    g = run_gpu(inp, 1)
    r = run_oracle(inp, 1)
    assert g["N"] == r["N"]
    assert_tok_close(g["loss_tok"], r["loss_tok"])
    tol = GRAD_RTOL if dtype == "bf16" else 1e-4
    if V == 1:
        assert float(torch.count_nonzero(g["dH_s"])) == 0 and float(torch.count_nonzero(g["dW_s"])) == 0
    else:
        assert grad_rel_err(g["dH_s"], r["dH_s"]) < tol
        assert grad_rel_err(g["dW_s"], r["dW_s"]) < tol


@pytest.mark.parametrize("V", [1, 8, 1000])
def test_logits_pair_degenerate(V):
    inp = small_case(B=1, Sm1=3, H=0, V=V, payload="logits_pair", mask="all", seed=V)
    zs, zt = inp["student_logits"].cuda(), inp["teacher_logits"].cuda()
    mask = inp["mask"].cuda()
    row_idx, N = rb.compact_rows(mask)
    lt, loss, saved = rb.forward_logits_pair(zs, zt, 1, 3, row_idx, N, 1)
    dz = rb.backward_logits_pair(zs, zt, 1, 3, row_idx, N, 1, saved, grad_loss=torch.ones(1, device="cuda"))
    ref = O.forward_logits_pair(to_np(zs), to_np(zt), mask.cpu().numpy(), 1)
    dz_ref = O.backward_logits_pair(to_np(zs), to_np(zt), mask.cpu().numpy(), 1)
    assert_tok_close(lt, ref["loss_tok"])
    if V == 1:
        assert float(torch.count_nonzero(dz)) == 0
    else:
        assert grad_rel_err(dz, dz_ref) < GRAD_RTOL
