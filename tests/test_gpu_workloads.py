"""GPU parity at the full sizes of the pages' workloads, in the launch
configuration bench.py times.

The oracle cannot afford every row of these shapes, so each test checks
(a) sampled trainable rows one by one against the oracle (per-token loss,
saved scalars, dH rows -- a row's results depend only on that row), and
(b) identities that hold at any size: sum_v dW_s[v, :] = sum_k (sum_v dz[k, v]) hc_s[k] = 0,
and <dW_s, W_s> = sum_k sum_v dz[k, v] z_s[k, v] = <dH_s, h_s>, which ties the
full dW_s to the sampled-checked dH_s.
"""

import numpy as np
import pytest
import torch

from full_vocabulary_reverse_b200 import binding as rb
from full_vocabulary_reverse_b200.workloads import make_workload
from oracle import rkl_oracle as O
from tests.gpu_cases import GRAD_RTOL, TOK_ATOL, TOK_RTOL, to_np

pytestmark = [pytest.mark.gpu, pytest.mark.slow]

SAMPLE = 24

# vocabulary rows of dW_s at the edges of the three backward chunks of V = 151936
# (50688 columns each), of 256-row gradient tiles, and the ragged last tile
VOCAB_EDGES = np.array([0, 1, 255, 256, 50687, 50688, 101375, 101376, 151807, 151808, 151935])


def _run(inp, reduction, mask=None, grad_tok=None, grad_loss=1.0, on_device=True):
    """One step as bench.py times it: the row count stays on the device
    (on_device=False: read back to the host first)."""
    mask = inp["mask"] if mask is None else mask
    B, Sm1 = mask.shape
    row_idx, N = rb.compact_rows(mask.cuda(), on_device=on_device)
    logits = "teacher_logits" in inp
    if logits:
        lt, loss, saved = rb.forward_logits(inp["h_s"], inp["W_s"], inp["teacher_logits"], B, Sm1, row_idx, N,
                                            reduction)
        teacher, W_t, payload = inp["teacher_logits"], None, rb.PAYLOAD_LOGITS
    else:
        lt, loss, saved = rb.forward_hidden(inp["h_s"], inp["h_t"], inp["W_s"], inp["W_t"], B, Sm1, row_idx, N,
                                            reduction)
        teacher, W_t, payload = inp["h_t"], inp["W_t"], rb.PAYLOAD_HIDDEN
    gl = torch.tensor([grad_loss], dtype=torch.float32, device="cuda")
    gt = None if grad_tok is None else grad_tok.cuda().float()
    dH, dW = rb.backward(payload, inp["h_s"], teacher, inp["W_s"], W_t, B, Sm1, row_idx, N, reduction, saved,
                         grad_loss=gl, grad_tok=gt)
    torch.cuda.synchronize()
    assert rb.device_error() == 0
    N = N if isinstance(N, int) else int(N.item())
    return {"N": N, "row_idx": row_idx[:N], "loss_tok": lt, "loss": loss, "saved": saved[:N], "dH": dH, "dW": dW}


def _oracle_rows(inp, rows, weights):
    """Oracle per-token loss, lse and dH for the given flattened rows, with
    row weights g (the full problem's dLoss/dL of those rows).  Each row's
    results depend on that row alone, so the oracle gets a one-sequence
    problem made of just these rows; outputs are returned indexed like the
    full problem's rows."""
    B, Sm1 = inp["mask"].shape
    rows_t = torch.as_tensor(rows, device=inp["h_s"].device)
    f = lambda t: t.float().cpu().numpy().astype(np.float64)  # noqa: E731
    h_s, W_s = f(inp["h_s"][rows_t]), f(inp["W_s"])
    if "teacher_logits" in inp:
        teacher, W_t = f(inp["teacher_logits"][rows_t]), None
    else:
        teacher, W_t = f(inp["h_t"][rows_t]), f(inp["W_t"])
    n = len(rows)
    sub = np.ones((1, n), np.uint8)
    fw_small = O.forward(h_s, W_s, teacher, W_t, sub, O.REDUCE_NONE)
    dH_small, _ = O.backward(h_s, W_s, teacher, W_t, sub, O.REDUCE_NONE,
                             grad_tok=np.asarray(weights, dtype=np.float64).reshape(1, n))
    loss_tok = np.zeros(B * Sm1)
    loss_tok[rows] = fw_small["loss_tok"].reshape(-1)
    dH = {int(r): dH_small[i] for i, r in enumerate(rows)}
    fw = {"loss_tok": loss_tok, "lse_s": fw_small["lse_s"], "lse_t": fw_small["lse_t"]}
    return fw, dH


def _row_weights(out, inp, reduction, rows):
    N = out["N"]
    if reduction == O.REDUCE_TOKEN_MEAN:
        return np.full(len(rows), 1.0 / N)
    Sm1 = inp["mask"].shape[1]
    ridx = out["row_idx"].cpu().numpy()
    seq = ridx // Sm1
    counts = np.bincount(seq, minlength=inp["mask"].shape[0])
    b_eff = np.count_nonzero(counts)
    return np.array([1.0 / (b_eff * counts[r // Sm1]) for r in rows])


def _tile_edges(n):
    """Compact-row indices at the edges of 128-row CTA tiles and 256-row pair
    tiles, and the last row."""
    e = [0, 127, 128, 255, 256, 511, 512, n - 1]
    return np.array([k for k in e if 0 <= k < n])


def _check_sampled(inp, out, reduction, seed):
    rs = np.random.RandomState(seed)
    ridx = out["row_idx"].cpu().numpy()
    pick = np.sort(rs.choice(len(ridx), size=min(SAMPLE, len(ridx)), replace=False))
    # always include the rows at tile edges and the last trainable row
    pick = np.unique(np.concatenate([_tile_edges(len(ridx)), pick]))
    rows = ridx[pick]
    fw, dH_ref = _oracle_rows(inp, rows, _row_weights(out, inp, reduction, rows))
    g_tok = to_np(out["loss_tok"].reshape(-1)[torch.as_tensor(rows, device=out["loss_tok"].device)])
    r_tok = fw["loss_tok"].reshape(-1)[rows]
    assert np.all(np.abs(g_tok - r_tok) <= TOK_ATOL + TOK_RTOL * np.abs(r_tok)), (g_tok, r_tok)
    saved = to_np(out["saved"])[pick]
    np.testing.assert_allclose(saved[:, 0], fw["lse_s"], atol=5e-4, rtol=0)
    np.testing.assert_allclose(saved[:, 1], fw["lse_t"], atol=5e-4, rtol=0)
    g_dH = to_np(out["dH"][torch.as_tensor(rows, device=out["dH"].device)])
    r_dH = np.stack([dH_ref[int(r)] for r in rows])
    assert np.max(np.abs(g_dH - r_dH)) / np.max(np.abs(r_dH)) < GRAD_RTOL


def _check_dw_rows(inp, out, reduction, seed, grad_tok=None):
    """Sampled vocabulary rows of the full dW_s against the oracle, whose dz
    comes from its own forward statistics over every trainable row."""
    V = inp["W_s"].shape[0]
    rs = np.random.RandomState(seed)
    ids = np.unique(np.concatenate([VOCAB_EDGES[VOCAB_EDGES < V], rs.choice(V, 8, replace=False)]))
    f = lambda t: None if t is None else t.float().cpu().numpy()  # noqa: E731
    if "teacher_logits" in inp:
        teacher, W_t = f(inp["teacher_logits"]), None
    else:
        teacher, W_t = f(inp["h_t"]), f(inp["W_t"])
    ref = O.backward_dw_rows(f(inp["h_s"]), f(inp["W_s"]), teacher, W_t, inp["mask"].cpu().numpy(), reduction, ids,
                             grad_tok=None if grad_tok is None else grad_tok.cpu().numpy())
    got = to_np(out["dW"][torch.as_tensor(ids, device=out["dW"].device)])
    err = np.max(np.abs(got - ref)) / np.max(np.abs(ref))
    assert err < GRAD_RTOL, (err, ids)
    # and row by row, each on its own scale
    for i, v in enumerate(ids):
        e = np.max(np.abs(got[i] - ref[i])) / np.max(np.abs(ref[i]))
        assert e < GRAD_RTOL, (int(v), e)


def _check_identities(inp, out):
    dW = out["dW"].double()
    dH = out["dH"].double()
    W_s = inp["W_s"].double()
    h_s = inp["h_s"].double()
    # sum over the vocabulary of dW_s vanishes (sum_v dz = 0 for every row)
    col = dW.sum(dim=0).abs().max().item()
    scale = dW.abs().sum(dim=0).max().item()
    assert col <= 2e-2 * scale
    # <dW_s, W_s> == <dH_s, h_s>  (both equal sum_k sum_v dz[k, v] z_s[k, v])
    a = (dW * W_s).sum().item()
    b = (dH * h_s).sum().item()
    scale = (dW * W_s).abs().sum().item()
    assert abs(a - b) <= 1e-3 * scale


def test_qwen_hidden_full_size():
    inp = make_workload("qwen_hidden", device="cuda")
    red = inp["reduction"]
    out = _run(inp, red)
    assert out["N"] == int(inp["mask"].sum())
    _check_sampled(inp, out, red, seed=1)
    _check_identities(inp, out)
    _check_dw_rows(inp, out, red, seed=11)
    lt = out["loss_tok"].reshape(-1)
    off = ~inp["mask"].reshape(-1).bool()
    assert float(torch.count_nonzero(lt[off])) == 0
    assert float(torch.count_nonzero(out["dH"][off])) == 0
    # the host-count mode gives bitwise the same results
    host = _run(inp, red, on_device=False)
    for k in ("loss_tok", "loss", "saved", "dH", "dW"):
        assert torch.equal(out[k], host[k]), k


def test_self_distill_full_size_exact_zero():
    inp = make_workload("self_distill", device="cuda")
    out = _run(inp, inp["reduction"])
    assert out["N"] > 0
    for k in ("loss_tok", "dH", "dW"):
        assert float(torch.count_nonzero(out[k])) == 0, k
    assert float(out["loss"]) == 0.0


def test_teacher_logits_full_size():
    inp = make_workload("teacher_logits", device="cuda")
    red = inp["reduction"]
    out = _run(inp, red)
    assert out["N"] == 8192
    _check_sampled(inp, out, red, seed=2)
    _check_identities(inp, out)
    _check_dw_rows(inp, out, red, seed=12)


def test_long_prompt_compact_equals_full():
    inp = make_workload("long_prompt", device="cuda")
    mask = inp["mask"]
    comp = _run(inp, 0, grad_tok=torch.full(mask.shape, 1.0 / 2048))
    assert comp["N"] == 2048
    # full path: every row projected, masked rows weighted 0
    full = _run(inp, 0, mask=torch.ones_like(mask), grad_tok=mask.float() / 2048)
    m = mask.reshape(-1).bool().cuda()
    lc, lf = comp["loss_tok"].reshape(-1), full["loss_tok"].reshape(-1)
    assert float(torch.count_nonzero(lc[~m])) == 0
    assert float(torch.count_nonzero(comp["dH"][~m])) == 0
    assert torch.equal(lc[m], lf[m])
    assert torch.equal(comp["dH"][m], full["dH"][m])
    rel = ((comp["dW"] - full["dW"]).abs().max() / full["dW"].abs().max()).item()
    assert rel < 1e-3
    del full
    # sampled vocabulary rows of dW_s (H = 4096: eight 512-column blocks)
    _check_dw_rows(inp, comp, 0, seed=13, grad_tok=torch.full(mask.shape, 1.0 / 2048, dtype=torch.float64))
    # sampled rows against the oracle (row weights 1/2048 on the compact run)
    out = dict(comp)
    rs = np.random.RandomState(5)
    ridx = out["row_idx"].cpu().numpy()
    pick = np.unique(np.concatenate([[0, len(ridx) - 1], rs.choice(len(ridx), size=6, replace=False)]))
    rows = ridx[pick]
    fw, dH_ref = _oracle_rows(inp, rows, np.full(len(rows), 1.0 / 2048))
    g_tok = to_np(out["loss_tok"].reshape(-1)[torch.as_tensor(rows, device=out["loss_tok"].device)])
    r_tok = fw["loss_tok"].reshape(-1)[rows]
    assert np.all(np.abs(g_tok - r_tok) <= TOK_ATOL + TOK_RTOL * np.abs(r_tok))
    g_dH = to_np(out["dH"][torch.as_tensor(rows, device=out["dH"].device)])
    r_dH = np.stack([dH_ref[int(r)] for r in rows])
    assert np.max(np.abs(g_dH - r_dH)) / np.max(np.abs(r_dH)) < GRAD_RTOL


def test_logits_pair_full_size():
    inp = make_workload("logits_pair", device="cuda")
    mask = inp["mask"]
    B, Sm1 = mask.shape
    row_idx, N = rb.compact_rows(mask)
    lt, loss, saved = rb.forward_logits_pair(inp["student_logits"], inp["teacher_logits"], B, Sm1, row_idx, N, 1)
    dz = rb.backward_logits_pair(inp["student_logits"], inp["teacher_logits"], B, Sm1, row_idx, N, 1, saved,
                                 grad_loss=torch.ones(1, device="cuda"))
    torch.cuda.synchronize()
    assert rb.device_error() == 0 and N == B * Sm1
    rows = np.unique(np.concatenate([[0, N - 1], np.random.RandomState(9).choice(N, 10, replace=False)]))
    rt = torch.as_tensor(rows, device="cuda")
    zs = to_np(inp["student_logits"][rt])
    zt = to_np(inp["teacher_logits"][rt])
    one = np.ones((1, len(rows)), np.uint8)
    ref = O.forward_logits_pair(zs, zt, one, O.REDUCE_NONE)
    rdz = O.backward_logits_pair(zs, zt, one, O.REDUCE_NONE, grad_tok=np.full((1, len(rows)), 1.0 / N))
    g_tok = to_np(lt.reshape(-1)[rt])
    assert np.all(np.abs(g_tok - ref["L"]) <= TOK_ATOL + TOK_RTOL * np.abs(ref["L"]))
    assert np.max(np.abs(to_np(dz[rt]) - rdz)) / np.max(np.abs(rdz)) < 2e-2
    # every dz row sums to ~0 (sum_v p_s (w - L) = 0), at every size
    s = dz.float().sum(dim=1).abs()
    a = dz.float().abs().sum(dim=1)
    assert float((s / a.clamp_min(1e-30)).max()) < 2e-2
