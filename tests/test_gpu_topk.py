"""GPU parity of the top-k estimator (both sides as logits) against the
float64 oracle: several k from the empty support to the whole row, tied
bf16 logits, rows whose length is not a multiple of the vector width, fp32,
masked rows, and the estimator's defining property checked on the GPU
output itself -- averaged over the sampled token y ~ p_s it gives the exact
loss and gradient."""

import numpy as np
import pytest
import torch

from full_vocabulary_reverse_b200 import binding as rb
from full_vocabulary_reverse_b200.workloads import make_inputs
from oracle import rkl_oracle as O
from tests.gpu_cases import GRAD_RTOL, assert_tok_close, grad_rel_err, to_np

pytestmark = pytest.mark.gpu


def _case(T_B, Sm1, V, dtype="bf16", mask="random", seed=0):
    inp = make_inputs(T_B, Sm1, 0, V, dtype=dtype, payload="logits_pair", mask=mask, seed=seed, device="cpu")
    y = torch.from_numpy(np.random.RandomState(seed + 99).randint(0, V, size=(T_B, Sm1)).astype(np.int32))
    return inp, y


def _run(inp, y, k, red, grad_tok=None):
    zs, zt, mask = inp["student_logits"].cuda(), inp["teacher_logits"].cuda(), inp["mask"].cuda()
    B, Sm1 = mask.shape
    row_idx, N = rb.compact_rows(mask)
    lt, loss, saved = rb.forward_topk_pair(zs, zt, y.cuda(), k, B, Sm1, row_idx, N, red)
    gl = torch.ones(1, device="cuda")
    gt = None if grad_tok is None else torch.as_tensor(grad_tok, dtype=torch.float32).cuda()
    dz = rb.backward_topk_pair(zs, zt, y.cuda(), B, Sm1, row_idx, N, red, saved, grad_loss=gl, grad_tok=gt)
    torch.cuda.synchronize()
    return lt, loss, dz, N


def _ref(inp, y, k, red, grad_tok=None):
    zs, zt = to_np(inp["student_logits"]), to_np(inp["teacher_logits"])
    mask = inp["mask"].numpy()
    out = O.forward_topk_pair(zs, zt, y.numpy(), k, mask, red)
    dz = O.backward_topk_pair(zs, zt, y.numpy(), k, mask, red, grad_tok=grad_tok)
    return out, dz


@pytest.mark.parametrize("k", [0, 1, 7, 64, 1023, 1024, 5000])
@pytest.mark.parametrize("V", [1024, 1037])
def test_topk_bf16(k, V):
    inp, y = _case(2, 60, V, seed=k + V)
    lt, loss, dz, N = _run(inp, y, k, 1)
    ref, dz_ref = _ref(inp, y, k, 1)
    assert N == ref["N"]
    assert_tok_close(lt, ref["loss_tok"])
    assert abs(float(loss) - ref["loss"]) <= 1e-4 + 1e-3 * abs(ref["loss"])
    assert grad_rel_err(dz, dz_ref) < GRAD_RTOL


@pytest.mark.parametrize("k", [0, 3, 50, 333])
def test_topk_fp32_nested(k):
    inp, y = _case(3, 20, 333, dtype="fp32", seed=k)
    lt, loss, dz, N = _run(inp, y, k, 2)
    ref, dz_ref = _ref(inp, y, k, 2)
    assert_tok_close(lt, ref["loss_tok"])
    assert grad_rel_err(dz, dz_ref) < 1e-4


def test_topk_per_token_grad_and_masked_rows():
    inp, y = _case(2, 40, 700, seed=3)
    gt = np.random.RandomState(4).normal(size=inp["mask"].shape)
    lt, loss, dz, N = _run(inp, y, 16, 0, grad_tok=gt)
    ref, dz_ref = _ref(inp, y, 16, 0, grad_tok=gt)
    assert_tok_close(lt, ref["loss_tok"])
    assert grad_rel_err(dz, dz_ref) < GRAD_RTOL
    off = inp["mask"].reshape(-1) == 0
    assert float(torch.count_nonzero(lt.reshape(-1).cpu()[off])) == 0
    assert float(torch.count_nonzero(dz.cpu()[off])) == 0


def test_topk_unbiased_on_gpu_outputs():
    # one logit row repeated V times with sampled token y = 0 .. V-1: the
    # p_s-weighted mean of the GPU estimates (and gradients) over y is the
    # exact loss (and gradient) of that row
    V = 256
    rs = np.random.RandomState(7)
    z_s = (rs.normal(size=V) * 2).astype(np.float32)
    z_t = (rs.normal(size=V) * 2).astype(np.float32)
    zs = torch.from_numpy(np.tile(z_s, (V, 1))).cuda()
    zt = torch.from_numpy(np.tile(z_t, (V, 1))).cuda()
    y = torch.arange(V, dtype=torch.int32).reshape(1, V).cuda()
    mask = torch.ones((1, V), dtype=torch.uint8).cuda()
    row_idx, N = rb.compact_rows(mask)
    p = torch.softmax(torch.from_numpy(z_s).double(), 0).numpy()
    L, _, _ = O.per_row_kl(z_s[None].astype(np.float64), z_t[None].astype(np.float64))
    dz_exact = O.dz_rows(z_s[None].astype(np.float64), z_t[None].astype(np.float64), np.ones(1))[0]
    for k in (1, 10, 100):
        lt, _, saved = rb.forward_topk_pair(zs, zt, y, k, 1, V, row_idx, N, 0)
        dz = rb.backward_topk_pair(zs, zt, y, 1, V, row_idx, N, 0, saved,
                                   grad_tok=torch.ones((1, V), device="cuda"))
        est = lt.double().cpu().numpy().reshape(-1)
        assert abs(np.dot(p, est) - L[0]) < 1e-5 * max(1.0, abs(L[0]))
        Edz = p @ dz.double().cpu().numpy()
        assert np.max(np.abs(Edz - dz_exact)) < 1e-5 * max(1.0, np.max(np.abs(dz_exact)))


def test_topk_whole_row_equals_logits_pair():
    inp, y = _case(2, 50, 900, seed=9)
    zs, zt, mask = inp["student_logits"].cuda(), inp["teacher_logits"].cuda(), inp["mask"].cuda()
    B, Sm1 = mask.shape
    row_idx, N = rb.compact_rows(mask)
    a, _, _ = rb.forward_topk_pair(zs, zt, y.cuda(), 900, B, Sm1, row_idx, N, 1)
    b, _, _ = rb.forward_logits_pair(zs, zt, B, Sm1, row_idx, N, 1)
    assert np.max(np.abs(to_np(a) - to_np(b))) < 1e-4


def test_topk_empty_mask():
    inp, y = _case(2, 30, 500, mask="none", seed=11)
    lt, loss, dz, N = _run(inp, y, 8, 1)
    assert N == 0 and float(loss) == 0.0
    assert float(torch.count_nonzero(lt)) == 0 and float(torch.count_nonzero(dz)) == 0


@pytest.mark.slow
def test_topk_full_size():
    # logits_pair_topk: [8192, 151936] bf16 on each side, k = 64, sampled
    # tokens drawn from the student; sampled rows against the oracle, and
    # sum_v dz = 0 on every row (the estimator's gradient keeps the softmax
    # normalisation: sum_v p_s([v in S](w+1) - C) + a = 0)
    from full_vocabulary_reverse_b200.workloads import make_workload
    inp = make_workload("logits_pair_topk", device="cuda")
    k = inp["cfg"]["k"]
    zs, zt, mask, y = inp["student_logits"], inp["teacher_logits"], inp["mask"], inp["targets"]
    B, Sm1 = mask.shape
    row_idx, N = rb.compact_rows(mask)
    lt, loss, saved = rb.forward_topk_pair(zs, zt, y, k, B, Sm1, row_idx, N, inp["reduction"])
    dz = rb.backward_topk_pair(zs, zt, y, B, Sm1, row_idx, N, inp["reduction"], saved,
                               grad_loss=torch.ones(1, device="cuda"))
    torch.cuda.synchronize()
    rows = np.unique(np.concatenate([[0, N - 1], np.random.RandomState(5).choice(N, 14, replace=False)]))
    rt = torch.as_tensor(rows, device="cuda")
    z_s = to_np(zs[rt])
    z_t = to_np(zt[rt])
    L_ref, dz_ref = O.topk_rows(z_s, z_t, y.reshape(-1)[rt].cpu().numpy(), k, np.full(len(rows), 1.0 / N))
    g_tok = to_np(lt.reshape(-1)[rt])
    assert np.all(np.abs(g_tok - L_ref) <= 1e-4 + 1e-3 * np.abs(L_ref)), (g_tok, L_ref)
    g_dz = to_np(dz[rt])
    assert np.max(np.abs(g_dz - dz_ref)) / np.max(np.abs(dz_ref)) < GRAD_RTOL
    rs_ = dz.double().sum(dim=1).abs()
    assert float((rs_ / dz.double().abs().sum(dim=1)).max()) < 1e-2


@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
@pytest.mark.parametrize("k,probs", [(100, [0.2, 0.5, 0.3]), (3000, [0.2, 0.5, 0.3]), (8999, [0.2, 0.5, 0.3]),
                                     (1, [0.2, 0.3, 0.5]), (100, [0.2, 0.3, 0.5]), (256, [0.2, 0.3, 0.5])])
def test_topk_many_ties_take_the_exact_path(dtype, k, probs):
    # student logits drawn from three values: the bin of the k-th logit (or,
    # for k <= 256, the bound from the threads' maxima) admits thousands of
    # tied entries; above 4096, more than the shared-memory candidate list,
    # the selection finishes with the exact radix / index-order path
    inp, y = _case(2, 20, 9000, dtype=dtype, seed=k)
    rs = np.random.RandomState(k)
    vals = rs.choice([-1.0, 0.5, 2.0], size=inp["student_logits"].shape, p=probs)
    inp["student_logits"] = torch.from_numpy(vals).to(inp["student_logits"].dtype)
    lt, loss, dz, N = _run(inp, y, k, 1)
    ref, dz_ref = _ref(inp, y, k, 1)
    assert_tok_close(lt, ref["loss_tok"])
    assert grad_rel_err(dz, dz_ref) < (GRAD_RTOL if dtype == "bf16" else 1e-4)


def _key(x, dtype):
    # order-preserving integer key of a logit, -0 and +0 sharing one key; a
    # bf16 logit keeps only its 16 significant bits
    u = np.float32(x).view(np.uint32) if x != 0 else np.uint32(0)
    k = (~u if u & np.uint32(0x80000000) else u | np.uint32(0x80000000)) & np.uint32(0xFFFFFFFF)
    return int(k) & (0xFFFF0000 if dtype == "bf16" else 0xFFFFFFFF)


# logit values: -1, -0, +0, 1e-39, -1e-39, 3e-39 (subnormal), 0.5
_ZERO_MIXES = [
    # k-th logit inside a run of ~1600 zeros (candidate list, histogram path)
    (4103, [0.25, 0.2, 0.2, 0.05, 0.05, 0.05, 0.2], 2051),
    # a run of ~4900 keys in the bin of zero: more than the list holds (exact path)
    (9000, [0.25, 0.25, 0.25, 0.05, 0.05, 0.05, 0.1], 4050),
    # k <= 256: the bound from the threads' maxima is zero, ~3760 candidates
    (9000, [0.55, 0.2, 0.2, 0.01, 0.03, 0.005, 0.005], 250),
    # k <= 256 with ~5570 logits at or above the bound (exact path from the top)
    (9000, [0.35, 0.3, 0.3, 0.01, 0.03, 0.005, 0.005], 250),
    # small k: the bound comes from the first slice of the row only, the rest
    # is listed as it streams (~3650 candidates)
    (9000, [0.556, 0.2, 0.2, 0.002, 0.038, 0.001, 0.003], 90),
    # the same with ~4570 logits at or above the bound (exact path from the top)
    (9000, [0.456, 0.25, 0.25, 0.002, 0.036, 0.001, 0.005], 110),
]


@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
@pytest.mark.parametrize("V,probs,k", _ZERO_MIXES)
def test_topk_signed_zeros_and_subnormals(dtype, V, probs, k):
    # -0 and +0 are one logit value (ties ranked by token id) and subnormal
    # logits keep their order, with the k-th logit of every row a zero
    inp, y = _case(2, 10, V, dtype=dtype, seed=V + k)
    rs = np.random.RandomState(V + k + 1)
    vals = np.array([-1.0, -0.0, 0.0, 1e-39, -1e-39, 3e-39, 0.5])
    inp["student_logits"] = torch.from_numpy(rs.choice(vals, size=inp["student_logits"].shape, p=probs)).to(
        inp["student_logits"].dtype)
    zs, zt, mask = inp["student_logits"].cuda(), inp["teacher_logits"].cuda(), inp["mask"].cuda()
    B, Sm1 = mask.shape
    row_idx, N = rb.compact_rows(mask)
    lt, loss, saved = rb.forward_topk_pair(zs, zt, y.cuda(), k, B, Sm1, row_idx, N, 1)
    dz = rb.backward_topk_pair(zs, zt, y.cuda(), B, Sm1, row_idx, N, 1, saved, grad_loss=torch.ones(1, device="cuda"))
    torch.cuda.synchronize()
    ref, dz_ref = _ref(inp, y, k, 1)
    assert_tok_close(lt, ref["loss_tok"])
    assert grad_rel_err(dz, dz_ref) < (GRAD_RTOL if dtype == "bf16" else 1e-4)
    # the k-th key K* and the last token id taken at it, exactly
    z = to_np(inp["student_logits"].reshape(-1, V))
    rows = row_idx[:N].cpu().numpy()
    S = O.topk_support(z[rows], k)
    tk = saved[3 * N:].reshape(N, 4).cpu().numpy()
    for i in range(N):
        zmin = z[rows[i]][S[i]].min()
        assert zmin == 0.0  # the boundary falls in the zero run
        assert int(tk[i, 2:3].view(np.uint32)[0]) == _key(zmin, dtype)
        assert int(tk[i, 3:4].view(np.int32)[0]) == int(np.flatnonzero(S[i] & (z[rows[i]] == zmin)).max())


def test_topk_autograd_wrapper():
    inp, y = _case(2, 50, 1024, seed=21)
    zs = inp["student_logits"].cuda().requires_grad_(True)
    loss, loss_tok = rb.topk_estimator_logits_pair(zs, inp["teacher_logits"].cuda(), y.cuda(), inp["mask"].cuda(),
                                                   32, 1)
    loss.backward()
    ref, dz_ref = _ref(inp, y, 32, 1)
    assert abs(float(loss.detach()) - ref["loss"]) <= 1e-4 + 1e-3 * abs(ref["loss"])
    assert grad_rel_err(zs.grad.float(), dz_ref) < GRAD_RTOL
