"""GPU parity of the top-k estimator on the teacher-logits payload (student
hidden states and LM head, shipped bf16 teacher logits) against the float64
oracle.

The support is decided on the kernels' fp32 student logits and on the
oracle's float64 ones; rows whose k-th and (k+1)-th student logits (or the
sampled token's logit and the k-th) lie within fp32 rounding of each other
may legitimately differ and are left out of the per-token comparison (they
must be rare).  Covers k from the empty support to the whole row, more than
one 2048-row logit block, two backward vocabulary chunks, both reductions, a
per-token upstream gradient, the device-resident row count, the autograd
wrapper and the full-size teacher-logits workload.
"""

import numpy as np
import pytest
import torch

from full_vocabulary_reverse_b200 import binding as rb
from full_vocabulary_reverse_b200.workloads import make_inputs, make_workload
from oracle import rkl_oracle as O
from tests.gpu_cases import GRAD_RTOL, TOK_ATOL, TOK_RTOL, grad_rel_err, to_np

pytestmark = pytest.mark.gpu


def _case(B, Sm1, H, V, seed, mask="random"):
    inp = make_inputs(B, Sm1, H, V, dtype="bf16", payload="logits", mask=mask, weights="perturbed", seed=seed,
                      device="cpu")
    y = torch.from_numpy(np.random.RandomState(seed + 5).randint(0, V, size=(B, Sm1)).astype(np.int32))
    return inp, y


def _ambiguous(h_s, W_s, y, k, mask):
    """Flattened positions whose support or tail decision is within fp32 reach."""
    z = h_s @ W_s.T
    V = z.shape[1]
    out = set()
    if k <= 0 or k >= V:
        return out
    zs = -np.sort(-z, axis=1)
    yflat = y.reshape(-1)
    trainable = mask.reshape(-1) != 0
    for r in range(z.shape[0]):
        if not trainable[r]:
            continue
        thr = zs[r, k - 1]
        tol = 2e-5 * max(1.0, abs(thr))
        if zs[r, k - 1] - zs[r, k] < tol or abs(z[r, yflat[r]] - thr) < tol:
            out.add(r)
    return out


def _run(inp, y, k, red, grad_tok=None, on_device=False):
    h_s, W_s, zt = (inp[n].cuda() for n in ("h_s", "W_s", "teacher_logits"))
    mask = inp["mask"].cuda()
    B, Sm1 = mask.shape
    row_idx, N = rb.compact_rows(mask, on_device=on_device)
    lt, loss, saved = rb.forward_topk_logits(h_s, W_s, zt, y.cuda(), k, B, Sm1, row_idx, N, red)
    gt = None if grad_tok is None else torch.as_tensor(grad_tok, dtype=torch.float32).cuda()
    dH, dW = rb.backward_topk_logits(h_s, W_s, zt, y.cuda(), B, Sm1, row_idx, N, red, saved,
                                     grad_loss=torch.ones(1, device="cuda"), grad_tok=gt)
    torch.cuda.synchronize()
    assert rb.device_error() == 0
    N = N if isinstance(N, int) else int(N.item())
    return lt, loss, dH, dW, N


def _check(inp, y, k, red, grad_tok=None, on_device=False):
    lt, loss, dH, dW, N = _run(inp, y, k, red, grad_tok, on_device)
    h_s, W_s = to_np(inp["h_s"]), to_np(inp["W_s"])
    args = (h_s, W_s, to_np(inp["teacher_logits"]), y.numpy(), k, inp["mask"].numpy(), red)
    ref = O.forward_topk_logits(*args)
    dH_ref, dW_ref = O.backward_topk_logits(*args, grad_tok=grad_tok)
    amb = _ambiguous(h_s, W_s, y.numpy(), k, inp["mask"].numpy())
    assert len(amb) <= max(2, N // 50)
    keep = np.array([r not in amb for r in range(lt.numel())])
    g = to_np(lt).reshape(-1)[keep]
    r = ref["loss_tok"].reshape(-1)[keep]
    bad = np.abs(g - r) > TOK_ATOL + TOK_RTOL * np.abs(r)
    assert not bad.any(), (np.flatnonzero(bad)[:5], g[bad][:5], r[bad][:5])
    if not amb and ref["loss"] is not None:
        assert abs(float(loss) - ref["loss"]) <= TOK_ATOL + TOK_RTOL * abs(ref["loss"])
    assert grad_rel_err(dH, dH_ref) < GRAD_RTOL
    assert grad_rel_err(dW, dW_ref) < GRAD_RTOL
    off = inp["mask"].reshape(-1).numpy() == 0
    assert np.all(to_np(lt).reshape(-1)[off] == 0) and np.all(to_np(dH)[off] == 0)
    return N


@pytest.mark.parametrize("k", [0, 1, 64, 1040])
def test_topk_logits_two_blocks(k):
    # about 2400 trainable rows: two 2048-row logit blocks, the second partial
    inp, y = _case(6, 800, 128, 1040, seed=160 + k)
    assert _check(inp, y, k, 1) > 2048


@pytest.mark.parametrize("red", [0, 2])
def test_topk_logits_reductions_and_chunks(red):
    # V spans two backward vocab chunks; per-token upstream gradient or nested mean
    inp, y = _case(2, 100, 64, 65536 + 904, seed=170 + red)
    gt = np.random.RandomState(3).normal(size=inp["mask"].shape) if red == 0 else None
    _check(inp, y, 32, red, grad_tok=gt)


def test_topk_logits_device_count_and_wide_hidden():
    # the row count read on the device; H = 1152 (gradient H blocks 512, 512, 128)
    inp, y = _case(2, 300, 1152, 3000, seed=181)
    _check(inp, y, 64, 1, on_device=True)


def test_topk_logits_odd_k_steps():
    # H = 192: the last 128-deep stage of the writer / dz kernels is half
    # zero-filled; the selection reads the shipped teacher rows directly
    inp, y = _case(2, 150, 192, 1504, seed=185)
    _check(inp, y, 40, 1)


def test_topk_logits_whole_row_equals_exact_loss():
    inp, y = _case(2, 120, 128, 776, seed=180)
    lt, loss, dH, dW, N = _run(inp, y, 776, 1)
    h_s, W_s, zt = (inp[n].cuda() for n in ("h_s", "W_s", "teacher_logits"))
    row_idx, N2 = rb.compact_rows(inp["mask"].cuda())
    lt2, _, saved = rb.forward_logits(h_s, W_s, zt, 2, 120, row_idx, N2, 1)
    dH2, dW2 = rb.backward(rb.PAYLOAD_LOGITS, h_s, zt, W_s, None, 2, 120, row_idx, N2, 1, saved,
                           grad_loss=torch.ones(1, device="cuda"))
    assert np.max(np.abs(to_np(lt) - to_np(lt2))) < 1e-4
    assert grad_rel_err(dH, to_np(dH2)) < 1e-2 and grad_rel_err(dW, to_np(dW2)) < 1e-2


def test_topk_logits_autograd_wrapper():
    inp, y = _case(2, 80, 128, 600, seed=190)
    h_s = inp["h_s"].cuda().requires_grad_(True)
    W_s = inp["W_s"].cuda().requires_grad_(True)
    loss, _ = rb.topk_estimator_logits(h_s, W_s, inp["teacher_logits"].cuda(), y.cuda(), inp["mask"].cuda(), 16, 1)
    loss.backward()
    args = (to_np(inp["h_s"]), to_np(inp["W_s"]), to_np(inp["teacher_logits"]), y.numpy(), 16, inp["mask"].numpy(),
            1)
    dH_ref, dW_ref = O.backward_topk_logits(*args)
    assert grad_rel_err(h_s.grad.float(), dH_ref) < GRAD_RTOL
    assert grad_rel_err(W_s.grad.float(), dW_ref) < GRAD_RTOL


@pytest.mark.slow
def test_topk_logits_full_size_sampled_rows():
    """The teacher-logits workload (8192 rows, V = 151936) with k = 64, in
    the launch configuration bench.py times (row count on the device).  Each
    row's estimate and dH row depend on that row alone: sampled rows are
    compared with the oracle run on just those rows."""
    inp = make_workload("topk_logits", device="cuda")
    k, red = inp["cfg"]["k"], inp["reduction"]
    y = inp["targets"]
    mask = inp["mask"]
    B, Sm1 = mask.shape
    row_idx, n_dev = rb.compact_rows(mask, on_device=True)
    lt, loss, saved = rb.forward_topk_logits(inp["h_s"], inp["W_s"], inp["teacher_logits"], y, k, B, Sm1, row_idx,
                                             n_dev, red)
    dH, dW = rb.backward_topk_logits(inp["h_s"], inp["W_s"], inp["teacher_logits"], y, B, Sm1, row_idx, n_dev, red,
                                     saved, grad_loss=torch.ones(1, device="cuda"))
    torch.cuda.synchronize()
    assert rb.device_error() == 0
    N = int(n_dev.item())
    rows = np.unique(np.concatenate([[0, 127, 128, 255, 256, 2047, 2048, N - 1],
                                     np.random.RandomState(4).choice(N, 16, replace=False)]))
    rt = torch.as_tensor(rows, device="cuda")
    f = lambda t: t.float().cpu().numpy().astype(np.float64)  # noqa: E731
    h_s, W_s, zt = f(inp["h_s"][rt]), f(inp["W_s"]), f(inp["teacher_logits"][rt])
    yy = y.reshape(-1)[rt].cpu().numpy().reshape(1, -1)
    one = np.ones((1, len(rows)), np.uint8)
    ref = O.forward_topk_logits(h_s, W_s, zt, yy, k, one, O.REDUCE_NONE)
    dH_ref, _ = O.backward_topk_logits(h_s, W_s, zt, yy, k, one, O.REDUCE_NONE,
                                       grad_tok=np.full((1, len(rows)), 1.0 / N))
    amb = _ambiguous(h_s, W_s, yy, k, one)
    keep = np.array([i not in amb for i in range(len(rows))])
    assert keep.sum() >= len(rows) - 2
    g_tok = to_np(lt.reshape(-1)[rt])
    r_tok = ref["loss_tok"].reshape(-1)
    assert np.all(np.abs(g_tok - r_tok)[keep] <= TOK_ATOL + TOK_RTOL * np.abs(r_tok)[keep])
    g_dH = to_np(dH[rt])[keep]
    assert np.max(np.abs(g_dH - dH_ref[keep])) / np.max(np.abs(dH_ref[keep])) < GRAD_RTOL
    # <dW_s, W_s> = <dH_s, h_s> ties the full dW_s to the checked dH_s rows
    a = (dW.double() * inp["W_s"].double()).sum().item()
    b = (dH.double() * inp["h_s"].double()).sum().item()
    assert abs(a - b) <= 1e-3 * (dW.double() * inp["W_s"].double()).abs().sum().item()
