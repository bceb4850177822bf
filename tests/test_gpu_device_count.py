"""The trainable-row count kept on the device.

rkl_compact_rows leaves N in device memory.  When the forward and backward
entry points get that pointer (n_dev), the kernels read N themselves, so a
whole step is enqueued without any host read of N.  These tests:

- change the mask between consecutive steps without reading anything back,
  and compare every step with the float64 oracle;
- check that the device-count and host-count modes give bitwise-identical
  results;
- cover an empty mask, which gives the gradient kernel zero-depth dW tiles;
- capture a whole step, compaction included, in one CUDA graph and replay it
  on different masks.
"""

import numpy as np
import pytest
import torch

from full_vocabulary_reverse_b200 import binding as rb
from full_vocabulary_reverse_b200.workloads import make_mask
from oracle import rkl_oracle as O
from tests.gpu_cases import GRAD_RTOL, assert_tok_close, grad_rel_err, small_case, to_np

pytestmark = pytest.mark.gpu


def _masks(B, Sm1, seed):
    """Three different masks of one shape: random, prefix-masked, and all rows."""
    return [torch.from_numpy(make_mask(k, B, Sm1, seed + i)) for i, k in enumerate(("random", "prefix", "all"))]


def _oracle(inp, mask, red):
    f = to_np
    teacher = f(inp["teacher_logits"]) if "teacher_logits" in inp else f(inp["h_t"])
    W_t = None if "teacher_logits" in inp else f(inp["W_t"])
    m = mask.numpy()
    fw = O.forward(f(inp["h_s"]), f(inp["W_s"]), teacher, W_t, m, red)
    dH, dW = O.backward(f(inp["h_s"]), f(inp["W_s"]), teacher, W_t, m, red)
    return fw, dH, dW


def _step(inp, mask_buf, row_idx, n_dev, red, ws, dH, dW, logits):
    """Compaction + forward + backward with the count on the device; returns
    the outputs as fresh device tensors (no host synchronisation)."""
    B, Sm1 = mask_buf.shape
    h_s, W_s = inp["h_s_d"], inp["W_s_d"]
    rb._check(rb.lib().rkl_compact_rows(rb._ptr(mask_buf), B, Sm1, rb._ptr(row_idx), rb._ptr(n_dev),
                                        rb._stream(mask_buf.device)))
    gl = torch.ones(1, device="cuda")
    if logits:
        teacher, W_t = inp["teacher_d"], None
        lt, loss, saved = rb.forward_logits(h_s, W_s, teacher, B, Sm1, row_idx, n_dev, red, workspace=ws)
        payload = rb.PAYLOAD_LOGITS
    else:
        teacher, W_t = inp["teacher_d"], inp["W_t_d"]
        lt, loss, saved = rb.forward_hidden(h_s, teacher, W_s, W_t, B, Sm1, row_idx, n_dev, red, workspace=ws)
        payload = rb.PAYLOAD_HIDDEN
    rb.backward(payload, h_s, teacher, W_s, W_t, B, Sm1, row_idx, n_dev, red, saved, grad_loss=gl, workspace=ws,
                dH_s=dH, dW_s=dW)
    return lt.clone(), loss.clone(), dH.clone(), dW.clone()


def _to_device(inp):
    inp = dict(inp)
    inp["h_s_d"], inp["W_s_d"] = inp["h_s"].cuda(), inp["W_s"].cuda()
    if "teacher_logits" in inp:
        inp["teacher_d"] = inp["teacher_logits"].cuda()
    else:
        inp["teacher_d"], inp["W_t_d"] = inp["h_t"].cuda(), inp["W_t"].cuda()
    return inp


@pytest.mark.parametrize("payload,dtype,H,V,red", [("hidden", "bf16", 128, 70000, 1), ("logits", "bf16", 128, 3000, 2),
                                                   ("hidden", "fp32", 40, 700, 2), ("logits", "fp32", 40, 600, 1)])
def test_mask_changes_between_steps_without_host_read(payload, dtype, H, V, red):
    B, Sm1 = 3, 200
    inp = _to_device(small_case(B=B, Sm1=Sm1, H=H, V=V, dtype=dtype, payload=payload, mask="all", seed=V + H))
    T = B * Sm1
    mask_buf = torch.empty((B, Sm1), dtype=torch.uint8, device="cuda")
    row_idx = torch.empty(T, dtype=torch.int32, device="cuda")
    n_dev = torch.empty(1, dtype=torch.int32, device="cuda")
    ws = rb._workspace(rb.PAYLOAD_LOGITS if payload == "logits" else rb.PAYLOAD_HIDDEN,
                       rb.DT_BF16 if dtype == "bf16" else rb.DT_FP32, T, B, Sm1, H, V, "cuda")
    dH = torch.empty((T, H), device="cuda")
    dW = torch.empty((V, H), device="cuda")
    masks = _masks(B, Sm1, seed=V)
    outs = []
    for m in masks:
        mask_buf.copy_(m, non_blocking=True)
        outs.append(_step(inp, mask_buf, row_idx, n_dev, red, ws, dH, dW, payload == "logits"))
    torch.cuda.synchronize()
    assert rb.device_error() == 0
    tol = GRAD_RTOL if dtype == "bf16" else 1e-4
    for m, (lt, loss, g_dH, g_dW) in zip(masks, outs):
        fw, r_dH, r_dW = _oracle(inp, m, red)
        assert_tok_close(lt, fw["loss_tok"])
        assert abs(float(loss) - fw["loss"]) <= 1e-4 + 1e-3 * abs(fw["loss"])
        assert grad_rel_err(g_dH, r_dH) < tol
        assert grad_rel_err(g_dW, r_dW) < tol
        off = torch.as_tensor(m.reshape(-1) == 0).cuda()
        assert float(torch.count_nonzero(lt.reshape(-1)[off])) == 0
        assert float(torch.count_nonzero(g_dH[off])) == 0


@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
@pytest.mark.parametrize("payload", ["hidden", "logits"])
def test_empty_mask_with_device_count(dtype, payload):
    B, Sm1, H = 2, 150, (128 if dtype == "bf16" else 40)
    V = 70000 if dtype == "bf16" else 500
    inp = _to_device(small_case(B=B, Sm1=Sm1, H=H, V=V, dtype=dtype, payload=payload, mask="all", seed=3))
    T = B * Sm1
    mask_buf = torch.zeros((B, Sm1), dtype=torch.uint8, device="cuda")
    row_idx = torch.empty(T, dtype=torch.int32, device="cuda")
    n_dev = torch.empty(1, dtype=torch.int32, device="cuda")
    ws = rb._workspace(rb.PAYLOAD_LOGITS if payload == "logits" else rb.PAYLOAD_HIDDEN,
                       rb.DT_BF16 if dtype == "bf16" else rb.DT_FP32, T, B, Sm1, H, V, "cuda")
    # outputs start as NaN so that anything left unwritten shows
    dH = torch.full((T, H), float("nan"), device="cuda")
    dW = torch.full((V, H), float("nan"), device="cuda")
    lt, loss, g_dH, g_dW = _step(inp, mask_buf, row_idx, n_dev, 1, ws, dH, dW, payload == "logits")
    torch.cuda.synchronize()
    assert rb.device_error() == 0
    assert int(n_dev.item()) == 0
    assert float(loss) == 0.0
    for t in (lt, g_dH, g_dW):
        assert bool(torch.isfinite(t).all()) and float(torch.count_nonzero(t)) == 0


@pytest.mark.parametrize("payload,mask,V", [("hidden", "random", 70000), ("logits", "all", 4096),
                                            ("hidden", "one", 1000)])
def test_device_count_bitwise_equals_host_count(payload, mask, V):
    B, Sm1, H = 2, 300, 256
    inp = small_case(B=B, Sm1=Sm1, H=H, V=V, payload=payload, mask=mask, seed=77)
    h_s, W_s = inp["h_s"].cuda(), inp["W_s"].cuda()
    logits = payload == "logits"
    teacher = inp["teacher_logits"].cuda() if logits else inp["h_t"].cuda()
    W_t = None if logits else inp["W_t"].cuda()
    pl = rb.PAYLOAD_LOGITS if logits else rb.PAYLOAD_HIDDEN
    maskd = inp["mask"].cuda()
    res = []
    for on_device in (False, True):
        row_idx, N = rb.compact_rows(maskd, on_device=on_device)
        if logits:
            lt, loss, saved = rb.forward_logits(h_s, W_s, teacher, B, Sm1, row_idx, N, 1)
        else:
            lt, loss, saved = rb.forward_hidden(h_s, teacher, W_s, W_t, B, Sm1, row_idx, N, 1)
        dH, dW = rb.backward(pl, h_s, teacher, W_s, W_t, B, Sm1, row_idx, N, 1, saved,
                             grad_loss=torch.ones(1, device="cuda"))
        n = N if isinstance(N, int) else int(N.item())
        res.append((lt, loss, saved[:n], dH, dW))
    torch.cuda.synchronize()
    assert rb.device_error() == 0
    for a, b in zip(*res):
        assert torch.equal(a, b)


def test_whole_step_in_one_cuda_graph_on_changing_masks():
    """Compaction, forward and backward captured together: the graph reads the
    mask buffer, so new masks need only a copy before each replay."""
    B, Sm1, H, V = 2, 300, 256, 70000
    inp = _to_device(small_case(B=B, Sm1=Sm1, H=H, V=V, mask="all", seed=91))
    T = B * Sm1
    masks = _masks(B, Sm1, seed=5)
    mask_buf = masks[0].cuda()
    row_idx = torch.empty(T, dtype=torch.int32, device="cuda")
    n_dev = torch.empty(1, dtype=torch.int32, device="cuda")
    ws = rb._workspace(rb.PAYLOAD_HIDDEN, rb.DT_BF16, T, B, Sm1, H, V, "cuda")
    dH = torch.empty((T, H), device="cuda")
    dW = torch.empty((V, H), device="cuda")
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        _step(inp, mask_buf, row_idx, n_dev, 1, ws, dH, dW, False)  # warm-up on the capture stream
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        lt, loss, g_dH, g_dW = _step(inp, mask_buf, row_idx, n_dev, 1, ws, dH, dW, False)
    for m in masks[::-1]:
        mask_buf.copy_(m)
        g.replay()
        torch.cuda.synchronize()
        assert rb.device_error() == 0
        fw, r_dH, r_dW = _oracle(inp, m, 1)
        assert int(n_dev.item()) == int(m.sum())
        assert_tok_close(lt, fw["loss_tok"])
        assert abs(float(loss) - fw["loss"]) <= 1e-4 + 1e-3 * abs(fw["loss"])
        assert grad_rel_err(g_dH, r_dH) < GRAD_RTOL
        assert grad_rel_err(g_dW, r_dW) < GRAD_RTOL


def test_logits_pair_and_topk_pair_with_device_count():
    B, Sm1, V = 3, 70, 3000
    inp = small_case(B=B, Sm1=Sm1, H=0, V=V, payload="logits_pair", mask="all", seed=13)
    zs, zt = inp["student_logits"].cuda(), inp["teacher_logits"].cuda()
    y = torch.from_numpy(np.random.RandomState(2).randint(0, V, size=(B, Sm1)).astype(np.int32))
    masks = _masks(B, Sm1, seed=21)
    mask_buf = torch.empty((B, Sm1), dtype=torch.uint8, device="cuda")
    row_idx = torch.empty(B * Sm1, dtype=torch.int32, device="cuda")
    n_dev = torch.empty(1, dtype=torch.int32, device="cuda")
    gl = torch.ones(1, device="cuda")
    outs = []
    for m in masks:
        mask_buf.copy_(m, non_blocking=True)
        rb._check(rb.lib().rkl_compact_rows(rb._ptr(mask_buf), B, Sm1, rb._ptr(row_idx), rb._ptr(n_dev),
                                            rb._stream(mask_buf.device)))
        lt, loss, saved = rb.forward_logits_pair(zs, zt, B, Sm1, row_idx, n_dev, 2)
        dz = rb.backward_logits_pair(zs, zt, B, Sm1, row_idx, n_dev, 2, saved, grad_loss=gl)
        lk, lossk, savedk = rb.forward_topk_pair(zs, zt, y, 16, B, Sm1, row_idx, n_dev, 1)
        dzk = rb.backward_topk_pair(zs, zt, y, B, Sm1, row_idx, n_dev, 1, savedk, grad_loss=gl)
        outs.append((lt.clone(), loss.clone(), dz.clone(), lk.clone(), lossk.clone(), dzk.clone()))
    torch.cuda.synchronize()
    assert rb.device_error() == 0
    z_s, z_t = to_np(zs), to_np(zt)
    for m, (lt, loss, dz, lk, lossk, dzk) in zip(masks, outs):
        mm = m.numpy()
        ref = O.forward_logits_pair(z_s, z_t, mm, 2)
        assert_tok_close(lt, ref["loss_tok"])
        assert abs(float(loss) - ref["loss"]) <= 1e-4 + 1e-3 * abs(ref["loss"])
        assert grad_rel_err(dz, O.backward_logits_pair(z_s, z_t, mm, 2)) < GRAD_RTOL
        refk = O.forward_topk_pair(z_s, z_t, y.numpy(), 16, mm, 1)
        assert_tok_close(lk, refk["loss_tok"])
        assert grad_rel_err(dzk, O.backward_topk_pair(z_s, z_t, y.numpy(), 16, mm, 1)) < GRAD_RTOL


@pytest.mark.parametrize("mask", ["random", "all"])
def test_topk_hidden_device_count_bitwise_equals_host_count(mask):
    # T = 3000 rows: two logit blocks of 2048 rows in the forward; with the
    # random mask the second block has no live row in the device mode
    B, Sm1, H, V = 2, 1500, 128, 3000
    inp = small_case(B=B, Sm1=Sm1, H=H, V=V, mask=mask, seed=17)
    h_s, h_t, W_s, W_t = (inp[k].cuda() for k in ("h_s", "h_t", "W_s", "W_t"))
    y = torch.from_numpy(np.random.RandomState(5).randint(0, V, size=(B, Sm1)).astype(np.int32)).cuda()
    maskd = inp["mask"].cuda()
    res = []
    for on_device in (False, True):
        row_idx, N = rb.compact_rows(maskd, on_device=on_device)
        lt, loss, saved = rb.forward_topk_hidden(h_s, h_t, W_s, W_t, y, 32, B, Sm1, row_idx, N, 1)
        dH, dW = rb.backward_topk_hidden(h_s, h_t, W_s, W_t, y, B, Sm1, row_idx, N, 1, saved,
                                         grad_loss=torch.ones(1, device="cuda"))
        res.append((lt, loss, dH, dW))
    torch.cuda.synchronize()
    assert rb.device_error() == 0
    for a, b in zip(*res):
        assert torch.equal(a, b)
