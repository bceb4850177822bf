"""Shared helpers of the GPU parity tests: run one problem through the C ABI
(via the ctypes binding) and through the CPU oracle on the same inputs."""

import numpy as np
import torch

from full_vocabulary_reverse_b200 import binding as rb
from full_vocabulary_reverse_b200.workloads import make_inputs
from oracle import rkl_oracle as O

# Tolerances for bf16 inputs with fp32 accumulation:
#   per-token loss |dL| <= 1e-4 + 1e-3 |L|; gradients max-norm relative 2e-2.
TOK_ATOL, TOK_RTOL, GRAD_RTOL = 1e-4, 1e-3, 2e-2


def to_np(t):
    return t.detach().float().cpu().numpy().astype(np.float64) if t.dtype != torch.float64 else t.cpu().numpy()


def run_gpu(inp, reduction, backward=True, grad_loss=1.0, grad_tok=None):
    """Forward (+ backward) of one problem through librkl.so."""
    mask = inp["mask"].cuda()
    B, Sm1 = mask.shape
    if "teacher_idx" in inp:
        return _run_gpu_multi(inp, reduction, backward, grad_loss, grad_tok)
    row_idx, N = rb.compact_rows(mask)
    payload = rb.PAYLOAD_LOGITS if "teacher_logits" in inp else rb.PAYLOAD_HIDDEN
    h_s = inp["h_s"].cuda()
    W_s = inp["W_s"].cuda()
    if payload == rb.PAYLOAD_HIDDEN:
        teacher, W_t = inp["h_t"].cuda(), inp["W_t"].cuda()
        loss_tok, loss, saved = rb.forward_hidden(h_s, teacher, W_s, W_t, B, Sm1, row_idx, N, reduction)
    else:
        teacher, W_t = inp["teacher_logits"].cuda(), None
        loss_tok, loss, saved = rb.forward_logits(h_s, W_s, teacher, B, Sm1, row_idx, N, reduction)
    out = {"row_idx": row_idx[:N].cpu().numpy(), "N": N, "loss_tok": loss_tok, "loss": loss, "saved": saved[:N]}
    if backward:
        gl = torch.tensor([grad_loss], dtype=torch.float32, device="cuda")
        gt = None if grad_tok is None else torch.as_tensor(grad_tok, dtype=torch.float32).cuda()
        dH, dW = rb.backward(payload, h_s, teacher, W_s, W_t, B, Sm1, row_idx, N, reduction, saved,
                             grad_loss=gl, grad_tok=gt)
        out["dH_s"], out["dW_s"] = dH, dW
    torch.cuda.synchronize()
    assert rb.device_error() == 0
    return out


def _run_gpu_multi(inp, reduction, backward, grad_loss, grad_tok):
    mask = inp["mask"].cuda()
    B, Sm1 = mask.shape
    h_s, h_t, W_s, W_t = (inp[k].cuda() for k in ("h_s", "h_t", "W_s", "W_t"))
    tid = inp["teacher_idx"].cuda()
    row_idx, N, counts = rb.compact_rows_multi(mask, tid, W_t.shape[0])
    loss_tok, loss, saved = rb.forward_hidden_multi(h_s, h_t, W_s, W_t, tid, counts, B, Sm1, row_idx, N, reduction)
    out = {"row_idx": row_idx[:N].cpu().numpy(), "N": N, "counts": counts, "loss_tok": loss_tok, "loss": loss,
           "saved": saved[:N]}
    if backward:
        gl = torch.tensor([grad_loss], dtype=torch.float32, device="cuda")
        gt = None if grad_tok is None else torch.as_tensor(grad_tok, dtype=torch.float32).cuda()
        out["dH_s"], out["dW_s"] = rb.backward_hidden_multi(h_s, h_t, W_s, W_t, tid, counts, B, Sm1, row_idx, N,
                                                            reduction, saved, grad_loss=gl, grad_tok=gt)
    torch.cuda.synchronize()
    assert rb.device_error() == 0
    return out


def run_oracle(inp, reduction, backward=True, grad_loss=1.0, grad_tok=None):
    h_s = to_np(inp["h_s"])
    W_s = to_np(inp["W_s"])
    mask = inp["mask"].cpu().numpy()
    if "teacher_idx" in inp:
        h_t, W_t = to_np(inp["h_t"]), to_np(inp["W_t"])
        tid = inp["teacher_idx"].cpu().numpy()
        out = O.forward_multi(h_s, W_s, h_t, W_t, tid, mask, reduction)
        if backward:
            out["dH_s"], out["dW_s"] = O.backward_multi(h_s, W_s, h_t, W_t, tid, mask, reduction,
                                                        grad_loss=grad_loss, grad_tok=grad_tok)
        return out
    if "teacher_logits" in inp:
        teacher, W_t = to_np(inp["teacher_logits"]), None
    else:
        teacher, W_t = to_np(inp["h_t"]), to_np(inp["W_t"])
    out = O.forward(h_s, W_s, teacher, W_t, mask, reduction)
    if backward:
        out["dH_s"], out["dW_s"] = O.backward(h_s, W_s, teacher, W_t, mask, reduction,
                                              grad_loss=grad_loss, grad_tok=grad_tok)
    return out


def assert_tok_close(gpu_tok, ref_tok):
    g = to_np(gpu_tok).reshape(-1)
    r = np.asarray(ref_tok).reshape(-1)
    err = np.abs(g - r)
    bound = TOK_ATOL + TOK_RTOL * np.abs(r)
    bad = np.flatnonzero(err > bound)
    assert bad.size == 0, "per-token loss: %d of %d outside tolerance, worst |d|=%.3e at %d (ref %.6f gpu %.6f)" % (
        bad.size, g.size, err.max(), int(np.argmax(err)), r[np.argmax(err)], g[np.argmax(err)])


def grad_rel_err(gpu, ref):
    g = to_np(gpu)
    r = np.asarray(ref)
    scale = np.max(np.abs(r))
    if scale == 0.0:
        return float(np.max(np.abs(g)))
    return float(np.max(np.abs(g - r)) / scale)


def small_case(B=2, Sm1=100, H=128, V=1000, dtype="bf16", payload="hidden", mask="random", weights="perturbed",
               seed=0, teacher_noise=0.05, n_teachers=1, teacher_assign="sequence"):
    return make_inputs(B, Sm1, H, V, dtype=dtype, payload=payload, mask=mask, weights=weights, seed=seed,
                       device="cpu", teacher_noise=teacher_noise, n_teachers=n_teachers,
                       teacher_assign=teacher_assign)
