"""The library's calls can be captured in a CUDA graph: every step is
enqueued on the caller's stream with no host synchronisation and no device
allocation, so a captured forward + backward replays to bitwise the same
results as the eager calls (the kernels are deterministic)."""

import pytest
import torch

from full_vocabulary_reverse_b200 import binding as rb
from tests.gpu_cases import small_case

pytestmark = pytest.mark.gpu


def test_hidden_forward_backward_in_cuda_graph():
    inp = small_case(B=2, Sm1=300, H=256, V=70000, mask="random", seed=51)
    h_s, h_t, W_s, W_t = (inp[k].cuda() for k in ("h_s", "h_t", "W_s", "W_t"))
    mask = inp["mask"].cuda()
    B, Sm1 = mask.shape
    row_idx, N = rb.compact_rows(mask)
    ws = rb._workspace(rb.PAYLOAD_HIDDEN, rb.DT_BF16, N, B, Sm1, 256, 70000, "cuda")
    gl = torch.ones(1, device="cuda")
    dH = torch.empty((B * Sm1, 256), device="cuda")
    dW = torch.empty((70000, 256), device="cuda")

    def step():
        lt, loss, saved = rb.forward_hidden(h_s, h_t, W_s, W_t, B, Sm1, row_idx, N, 1, workspace=ws)
        rb.backward(rb.PAYLOAD_HIDDEN, h_s, h_t, W_s, W_t, B, Sm1, row_idx, N, 1, saved, grad_loss=gl,
                    workspace=ws, dH_s=dH, dW_s=dW)
        return lt, loss

    lt0, loss0 = step()
    torch.cuda.synchronize()
    ref = (lt0.clone(), loss0.clone(), dH.clone(), dW.clone())
    dH.zero_()
    dW.zero_()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        step()  # warm-up on the capture stream
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        lt1, loss1 = step()
    dH.zero_()
    dW.zero_()
    for _ in range(2):
        g.replay()
    torch.cuda.synchronize()
    assert rb.device_error() == 0
    assert torch.equal(lt1, ref[0]) and torch.equal(loss1, ref[1])
    assert torch.equal(dH, ref[2]) and torch.equal(dW, ref[3])


def test_logits_pair_in_cuda_graph():
    inp = small_case(B=2, Sm1=64, H=0, V=5000, payload="logits_pair", mask="random", seed=52)
    zs, zt, mask = inp["student_logits"].cuda(), inp["teacher_logits"].cuda(), inp["mask"].cuda()
    B, Sm1 = mask.shape
    row_idx, N = rb.compact_rows(mask)
    gl = torch.ones(1, device="cuda")
    dz = torch.empty_like(zs)

    def step():
        lt, loss, saved = rb.forward_logits_pair(zs, zt, B, Sm1, row_idx, N, 2)
        rb.backward_logits_pair(zs, zt, B, Sm1, row_idx, N, 2, saved, grad_loss=gl, dz=dz)
        return lt

    ref_lt = step().clone()
    torch.cuda.synchronize()
    ref_dz = dz.clone()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        step()
    torch.cuda.current_stream().wait_stream(side)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        lt = step()
    dz.zero_()
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(lt, ref_lt) and torch.equal(dz, ref_dz)
