"""Checks that pin the CPU oracle to facts fixed outside it.

Each function takes the oracle module (so that the mutation tests can hand in
a copy with a planted mistake) and returns the worst violation it found; the
pin tests assert it is below a bound, the mutation tests assert that a planted
mistake pushes it above.  The facts come from the mathematics of the objective
in NeMo RL PR #3978 ("feat(mopd): add full-vocabulary on-policy distillation",
description and first implementation note) and the masking rules of slime
PR #2310 ("fix(megatron): compact actor logits before projection", Summary).
"""

import math

import numpy as np
import scipy.special
import scipy.stats

from oracle import brute


def rand_problem(rs, B=2, Sm1=3, H=4, V=7, scale=1.0, mask=None, payload="hidden"):
    T = B * Sm1
    h_s = rs.normal(size=(T, H)) * scale
    W_s = rs.normal(size=(V, H)) * scale
    if payload == "hidden":
        teacher = rs.normal(size=(T, H)) * scale
        W_t = rs.normal(size=(V, H)) * scale
    else:
        teacher = rs.normal(size=(T, V)) * 2.0
        W_t = None
    if mask is None:
        mask = (rs.uniform(size=(B, Sm1)) < 0.7).astype(np.uint8)
        mask[0, -1] = 1
    return h_s, W_s, teacher, W_t, mask


def kl_vs_scipy(O, rs):
    """L equals scipy.stats.entropy(p_s, p_t) = sum p_s log(p_s / p_t).

    This is the Kullback-Leibler divergence of p_s from p_t, so a swapped
    direction (forward KL) or a wrong log-softmax fails here."""
    worst = 0.0
    for V in (2, 5, 33, 1000):
        z_s = rs.normal(size=(4, V)) * 3
        z_t = rs.normal(size=(4, V)) * 3
        L, _, _ = O.per_row_kl(z_s, z_t)
        ref = scipy.stats.entropy(scipy.special.softmax(z_s, axis=1),
                                  scipy.special.softmax(z_t, axis=1), axis=1)
        worst = max(worst, float(np.max(np.abs(L - ref) / (1e-12 + np.abs(ref)))))
    return worst


def lse_vs_scipy(O, rs):
    worst = 0.0
    for V in (1, 3, 1000):
        z = rs.normal(size=(5, V)) * 10 + 50
        _, lse_s, lse_t = O.per_row_kl(z, z + 1.0)
        ref = scipy.special.logsumexp(z, axis=1)
        worst = max(worst, float(np.max(np.abs(lse_s - ref))), float(np.max(np.abs(lse_t - 1.0 - ref))))
    return worst


def uniform_teacher(O, rs):
    """W_t = 0 -> p_t uniform -> L = log V - H(p_s), H from scipy.stats.entropy."""
    worst = 0.0
    for V in (3, 17, 512):
        h_s, W_s, h_t, _, mask = rand_problem(rs, B=1, Sm1=4, H=5, V=V, mask=np.ones((1, 4), np.uint8))
        W_t = np.zeros_like(W_s)
        out = O.forward(h_s, W_s, h_t, W_t, mask, O.REDUCE_NONE)
        p_s = scipy.special.softmax(h_s @ W_s.T, axis=1)
        ref = math.log(V) - scipy.stats.entropy(p_s, axis=1)
        worst = max(worst, float(np.max(np.abs(out["L"] - ref))))
    return worst


def one_logit_bump(O, rs):
    """z_t = z_s + delta e_k -> L = -delta p_s(k) + log(1 + p_s(k)(e^delta - 1))."""
    worst = 0.0
    for delta in (-3.0, -0.5, 0.25, 2.0):
        z_s = rs.normal(size=(3, 11)) * 2
        k = 4
        z_t = z_s.copy()
        z_t[:, k] += delta
        L, _, _ = O.per_row_kl(z_s, z_t)
        p = scipy.special.softmax(z_s, axis=1)[:, k]
        ref = -delta * p + np.log1p(p * math.expm1(delta))
        worst = max(worst, float(np.max(np.abs(L - ref))))
    return worst


def binary_kl(O, rs):
    """Two-token vocabulary: L = p log(p/q) + (1-p) log((1-p)/(1-q)), p = sigmoid."""
    z_s = rs.normal(size=(6, 2)) * 2
    z_t = rs.normal(size=(6, 2)) * 2
    L, _, _ = O.per_row_kl(z_s, z_t)
    p = scipy.special.expit(z_s[:, 1] - z_s[:, 0])
    q = scipy.special.expit(z_t[:, 1] - z_t[:, 0])
    ref = p * np.log(p / q) + (1 - p) * np.log((1 - p) / (1 - q))
    return float(np.max(np.abs(L - ref)))


def brute_force(O, rs):
    """Per-token loss and both reductions against the pure-Python loops."""
    worst = 0.0
    for payload_seed in range(3):
        h_s, W_s, h_t, W_t, mask = rand_problem(rs, B=3, Sm1=4, H=3, V=9)
        ref_tok = np.array(brute.loss_tokens(h_s.tolist(), W_s.tolist(), h_t.tolist(), W_t.tolist(), mask.tolist()))
        for red, ref_fn in ((O.REDUCE_TOKEN_MEAN, brute.token_mean), (O.REDUCE_SEQ_MEAN_NESTED, brute.nested_mean)):
            out = O.forward(h_s, W_s, h_t, W_t, mask, red)
            worst = max(worst, float(np.max(np.abs(out["loss_tok"] - ref_tok))))
            worst = max(worst, abs(out["loss"] - ref_fn(ref_tok.tolist(), mask.tolist())))
    return worst


def compact_rows_brute(O, rs):
    bad = 0
    for kind in range(5):
        mask = (rs.uniform(size=(3, 7)) < [0.0, 0.2, 0.5, 0.9, 1.0][kind]).astype(np.uint8)
        idx, n = O.compact_rows(mask)
        ref = brute.compact_rows(mask.tolist())
        bad += int(n != len(ref) or list(idx) != ref)
    return bad


def _loss_fn(O, h_s, W_s, teacher, W_t, mask, red, grad_tok):
    out = O.forward(h_s, W_s, teacher, W_t, mask, red)
    val = 0.0 if out["loss"] is None else out["loss"]
    if grad_tok is not None:
        val += float(np.sum(grad_tok * out["loss_tok"]))
    return val


def finite_differences(O, rs, payload="hidden", red=None, with_grad_tok=False, grad_loss=1.0):
    """Central differences of the scalar objective w.r.t. h_s and W_s.

    Objective = grad_loss * loss + sum(grad_tok * loss_tok); backward must
    return its gradient.  Returns the worst relative error."""
    red = 1 if red is None else red
    # unequal per-sequence counts and one empty sequence, so that the token
    # mean and the nested mean have different row weights
    mask = np.array([[1, 1, 1], [0, 1, 0], [0, 0, 0]], dtype=np.uint8)
    h_s, W_s, teacher, W_t, mask = rand_problem(rs, B=3, Sm1=3, H=4, V=7, payload=payload, mask=mask)
    grad_tok = rs.normal(size=mask.shape) if with_grad_tok else None

    def f(hs, ws):
        out = O.forward(hs, ws, teacher, W_t, mask, red)
        val = 0.0 if out["loss"] is None else grad_loss * out["loss"]
        if grad_tok is not None:
            val += float(np.sum(grad_tok * out["loss_tok"]))
        return val

    dH, dW = O.backward(h_s, W_s, teacher, W_t, mask, red, grad_loss=grad_loss, grad_tok=grad_tok)
    eps = 1e-6
    num_H = np.zeros_like(h_s)
    for i in range(h_s.shape[0]):
        for j in range(h_s.shape[1]):
            hp = h_s.copy(); hp[i, j] += eps
            hm = h_s.copy(); hm[i, j] -= eps
            num_H[i, j] = (f(hp, W_s) - f(hm, W_s)) / (2 * eps)
    num_W = np.zeros_like(W_s)
    for i in range(W_s.shape[0]):
        for j in range(W_s.shape[1]):
            wp = W_s.copy(); wp[i, j] += eps
            wm = W_s.copy(); wm[i, j] -= eps
            num_W[i, j] = (f(h_s, wp) - f(h_s, wm)) / (2 * eps)
    scale_H = max(1e-12, float(np.max(np.abs(num_H))))
    scale_W = max(1e-12, float(np.max(np.abs(num_W))))
    return max(float(np.max(np.abs(dH - num_H))) / scale_H, float(np.max(np.abs(dW - num_W))) / scale_W)


def self_distillation(O, rs):
    """Teacher == student: L and every gradient exactly 0 (PR #3978 recipe)."""
    h_s, W_s, _, _, mask = rand_problem(rs, B=2, Sm1=5, H=6, V=40)
    out = O.forward(h_s, W_s, h_s.copy(), W_s.copy(), mask, O.REDUCE_SEQ_MEAN_NESTED)
    dH, dW = O.backward(h_s, W_s, h_s.copy(), W_s.copy(), mask, O.REDUCE_SEQ_MEAN_NESTED)
    return max(float(np.max(np.abs(out["loss_tok"]))), abs(out["loss"]),
               float(np.max(np.abs(dH))), float(np.max(np.abs(dW))))


def dz_sums_to_zero(O, rs):
    """sum_v dL/dz_s = 0 per row (sum_v p_s (w - L) = L - L)."""
    z_s = rs.normal(size=(8, 300)) * 3
    z_t = z_s + rs.normal(size=(8, 300)) * 0.5
    dz = O.dz_rows(z_s, z_t, np.ones(8))
    return float(np.max(np.abs(dz.sum(axis=1)) / np.abs(dz).sum(axis=1)))


def shift_invariance(O, rs):
    """Adding a per-row constant to the teacher logits changes nothing."""
    h_s, W_s, logits, _, mask = rand_problem(rs, B=2, Sm1=4, H=5, V=30, payload="logits")
    shift = rs.uniform(-20, 20, size=(logits.shape[0], 1))
    a = O.forward(h_s, W_s, logits, None, mask, 1)
    b = O.forward(h_s, W_s, logits + shift, None, mask, 1)
    dHa, dWa = O.backward(h_s, W_s, logits, None, mask, 1)
    dHb, dWb = O.backward(h_s, W_s, logits + shift, None, mask, 1)
    return max(float(np.max(np.abs(a["loss_tok"] - b["loss_tok"]))),
               float(np.max(np.abs(dHa - dHb))), float(np.max(np.abs(dWa - dWb))))


def masked_rows_exact_zero(O, rs):
    """Masked positions: loss exactly 0 and dH row exactly 0 (slime PR #2310)."""
    h_s, W_s, h_t, W_t, mask = rand_problem(rs, B=3, Sm1=5, H=4, V=9)
    out = O.forward(h_s, W_s, h_t, W_t, mask, 1)
    dH, _ = O.backward(h_s, W_s, h_t, W_t, mask, 1)
    off = mask.reshape(-1) == 0
    return float(np.max(np.abs(out["loss_tok"].reshape(-1)[off]), initial=0.0)) + \
        float(np.max(np.abs(dH[off]), initial=0.0))


def compact_equals_full(O, rs):
    """Compact rows vs all rows then select (slime PR #2310 compact/full parity)."""
    h_s, W_s, h_t, W_t, mask = rand_problem(rs, B=3, Sm1=6, H=5, V=21)
    comp = O.forward(h_s, W_s, h_t, W_t, mask, 0)
    full = O.forward(h_s, W_s, h_t, W_t, np.ones_like(mask), 0)
    sel = mask.reshape(-1) != 0
    return float(np.max(np.abs(comp["loss_tok"].reshape(-1)[sel] - full["loss_tok"].reshape(-1)[sel])))


def empty_mask(O, rs):
    """N = 0: loss 0, gradients 0, nothing NaN (slime PR #2310: empty masks)."""
    h_s, W_s, h_t, W_t, _ = rand_problem(rs, B=2, Sm1=3, H=4, V=7)
    mask = np.zeros((2, 3), np.uint8)
    worst = 0.0
    for red in (1, 2):
        out = O.forward(h_s, W_s, h_t, W_t, mask, red)
        dH, dW = O.backward(h_s, W_s, h_t, W_t, mask, red)
        vals = np.concatenate([out["loss_tok"].ravel(), [out["loss"]], dH.ravel(), dW.ravel()])
        if not np.all(np.isfinite(vals)):
            return float("inf")
        worst = max(worst, float(np.max(np.abs(vals))))
    return worst


def nested_vs_token_mean_equal_counts(O, rs):
    """With equal per-sequence counts, the nested mean equals the token mean."""
    h_s, W_s, h_t, W_t, _ = rand_problem(rs, B=3, Sm1=4, H=4, V=7)
    mask = np.zeros((3, 4), np.uint8)
    mask[0, [0, 2]] = 1
    mask[1, [1, 3]] = 1
    mask[2, [2, 3]] = 1
    a = O.forward(h_s, W_s, h_t, W_t, mask, 1)["loss"]
    b = O.forward(h_s, W_s, h_t, W_t, mask, 2)["loss"]
    return abs(a - b)


def nested_mean_by_hand(O, rs):
    """Nested mean of a 2-sequence batch with an empty third sequence."""
    h_s, W_s, h_t, W_t, _ = rand_problem(rs, B=3, Sm1=4, H=4, V=7)
    mask = np.zeros((3, 4), np.uint8)
    mask[0, [1]] = 1
    mask[2, [0, 1, 3]] = 1
    out = O.forward(h_s, W_s, h_t, W_t, mask, 2)
    lt = out["loss_tok"]
    ref = 0.5 * (lt[0, 1] + (lt[2, 0] + lt[2, 1] + lt[2, 3]) / 3.0)
    return abs(out["loss"] - ref)


def logits_pair_finite_differences(O, rs, red=1, with_grad_tok=False):
    """Central differences of the objective w.r.t. the student logits."""
    mask = np.array([[1, 1, 0], [0, 1, 0], [0, 0, 0]], dtype=np.uint8)
    z_s = rs.normal(size=(9, 6)) * 2
    z_t = rs.normal(size=(9, 6)) * 2
    grad_tok = rs.normal(size=mask.shape) if with_grad_tok else None

    def f(zs):
        out = O.forward_logits_pair(zs, z_t, mask, red)
        val = 0.0 if out["loss"] is None else out["loss"]
        if grad_tok is not None:
            val += float(np.sum(grad_tok * out["loss_tok"]))
        return val

    dz = O.backward_logits_pair(z_s, z_t, mask, red, grad_tok=grad_tok)
    eps = 1e-6
    num = np.zeros_like(z_s)
    for i in range(z_s.shape[0]):
        for j in range(z_s.shape[1]):
            zp = z_s.copy(); zp[i, j] += eps
            zm = z_s.copy(); zm[i, j] -= eps
            num[i, j] = (f(zp) - f(zm)) / (2 * eps)
    return float(np.max(np.abs(dz - num)) / max(1e-12, np.max(np.abs(num))))


def logits_pair_matches_hidden_chain_rule(O, rs):
    """With z_s = h_s W_s^T and z_t = h_t W_t^T, the logits-pair loss equals the
    hidden-payload loss and dH_s = dz W_s, dW_s = dz^T h_s (chain rule)."""
    h_s, W_s, h_t, W_t, mask = rand_problem(rs, B=2, Sm1=4, H=3, V=8)
    z_s, z_t = h_s @ W_s.T, h_t @ W_t.T
    a = O.forward(h_s, W_s, h_t, W_t, mask, 2)
    b = O.forward_logits_pair(z_s, z_t, mask, 2)
    dH, dW = O.backward(h_s, W_s, h_t, W_t, mask, 2)
    dz = O.backward_logits_pair(z_s, z_t, mask, 2)
    return max(float(np.max(np.abs(a["loss_tok"] - b["loss_tok"]))), abs(a["loss"] - b["loss"]),
               float(np.max(np.abs(dH - dz @ W_s))), float(np.max(np.abs(dW - dz.T @ h_s))))


# ----------------------------------------------------------------- several teachers

def rand_multi_problem(rs, B=3, Sm1=4, H=3, V=9, n_teachers=3):
    T = B * Sm1
    h_s = rs.normal(size=(T, H))
    W_s = rs.normal(size=(V, H))
    h_t = rs.normal(size=(T, H))
    W_t = rs.normal(size=(n_teachers, V, H))
    tid = rs.randint(0, n_teachers, size=(B, Sm1))
    mask = (rs.uniform(size=(B, Sm1)) < 0.7).astype(np.uint8)
    mask[0, -1] = 1
    return h_s, W_s, h_t, W_t, tid, mask


def multi_teacher_brute_force(O, rs):
    """Per-token loss and both reductions with a teacher per row, against the
    pure-Python loops that pick each position's teacher head."""
    worst = 0.0
    for _ in range(3):
        h_s, W_s, h_t, W_t, tid, mask = rand_multi_problem(rs)
        ref_tok = np.array(brute.loss_tokens_multi(h_s.tolist(), W_s.tolist(), h_t.tolist(),
                                                   [w.tolist() for w in W_t], tid.tolist(), mask.tolist()))
        for red, ref_fn in ((O.REDUCE_TOKEN_MEAN, brute.token_mean), (O.REDUCE_SEQ_MEAN_NESTED, brute.nested_mean)):
            out = O.forward_multi(h_s, W_s, h_t, W_t, tid, mask, red)
            worst = max(worst, float(np.max(np.abs(out["loss_tok"] - ref_tok))))
            worst = max(worst, abs(out["loss"] - ref_fn(ref_tok.tolist(), mask.tolist())))
    return worst


def multi_teacher_kl_vs_scipy(O, rs):
    """Each row's loss is scipy's KL of softmax(z_s) from softmax(z_t) with
    z_t built from that row's own teacher head."""
    h_s, W_s, h_t, W_t, tid, mask = rand_multi_problem(rs, B=4, Sm1=5, H=6, V=50, n_teachers=4)
    out = O.forward_multi(h_s, W_s, h_t, W_t, tid, mask, O.REDUCE_NONE)
    worst = 0.0
    for r in np.flatnonzero(mask.reshape(-1)):
        z_s = h_s[r] @ W_s.T
        z_t = h_t[r] @ W_t[tid.reshape(-1)[r]].T
        ref = scipy.stats.entropy(scipy.special.softmax(z_s), scipy.special.softmax(z_t))
        worst = max(worst, abs(out["loss_tok"].reshape(-1)[r] - ref))
    return worst


def multi_teacher_finite_differences(O, rs, red=1):
    """Central differences of the objective w.r.t. h_s and W_s, teacher per row."""
    mask = np.array([[1, 1, 1], [0, 1, 0], [0, 0, 0]], dtype=np.uint8)
    h_s, W_s, h_t, W_t, tid, _ = rand_multi_problem(rs, B=3, Sm1=3, H=4, V=7, n_teachers=2)
    tid[0] = [0, 1, 1]

    def f(hs, ws):
        return O.forward_multi(hs, ws, h_t, W_t, tid, mask, red)["loss"]

    dH, dW = O.backward_multi(h_s, W_s, h_t, W_t, tid, mask, red)
    eps = 1e-6
    num_H = np.zeros_like(h_s)
    for i in range(h_s.shape[0]):
        for j in range(h_s.shape[1]):
            hp = h_s.copy(); hp[i, j] += eps
            hm = h_s.copy(); hm[i, j] -= eps
            num_H[i, j] = (f(hp, W_s) - f(hm, W_s)) / (2 * eps)
    num_W = np.zeros_like(W_s)
    for i in range(W_s.shape[0]):
        for j in range(W_s.shape[1]):
            wp = W_s.copy(); wp[i, j] += eps
            wm = W_s.copy(); wm[i, j] -= eps
            num_W[i, j] = (f(h_s, wp) - f(h_s, wm)) / (2 * eps)
    return max(float(np.max(np.abs(dH - num_H))) / max(1e-12, float(np.max(np.abs(num_H)))),
               float(np.max(np.abs(dW - num_W))) / max(1e-12, float(np.max(np.abs(num_W)))))


def multi_teacher_counts_brute(O, rs):
    """Rows per teacher and out-of-range indices, against loops.  Masked
    positions may hold any index (never read)."""
    bad = 0
    for _ in range(5):
        mask = (rs.uniform(size=(3, 8)) < 0.6).astype(np.uint8)
        tid = rs.randint(-1, 5, size=(3, 8))
        counts, n_bad = O.count_rows_per_teacher(mask, tid, 4)
        ref_counts, ref_bad = brute.count_rows_per_teacher(mask.tolist(), tid.tolist(), 4)
        bad += int(list(counts) != ref_counts or n_bad != ref_bad)
    return bad


# ----------------------------------------------------------------- top-k estimator

def topk_limits(O, rs):
    """k >= V: the exact loss and dL/dz = p_s (w - L).  k = 0: the
    sampled-token gap log p_s(y) - log p_t(y) (scipy) and its score-function
    gradient (w(y) + 1)(e_y - p_s)."""
    worst = 0.0
    n, V = 5, 23
    z_s = rs.normal(size=(n, V)) * 3
    z_t = rs.normal(size=(n, V)) * 3
    y = rs.randint(0, V, size=n)
    g = rs.uniform(0.5, 2.0, size=n)
    L, _, _ = O.per_row_kl(z_s, z_t)
    for k in (V, V + 7):
        Lk, dz = O.topk_rows(z_s, z_t, y, k, g)
        worst = max(worst, float(np.max(np.abs(Lk - L))), float(np.max(np.abs(dz - O.dz_rows(z_s, z_t, g)))))
    L0, dz0 = O.topk_rows(z_s, z_t, y, 0, g)
    ls = scipy.special.log_softmax(z_s, axis=1)
    lt = scipy.special.log_softmax(z_t, axis=1)
    wy = ls[np.arange(n), y] - lt[np.arange(n), y]
    ref = -np.exp(ls) * (wy + 1.0)[:, None]
    ref[np.arange(n), y] += wy + 1.0
    worst = max(worst, float(np.max(np.abs(L0 - wy))), float(np.max(np.abs(dz0 - g[:, None] * ref))))
    return worst


def topk_unbiased(O, rs):
    """Averaging the estimate and its gradient over the sampled token
    y ~ p_s gives the exact loss and the exact gradient, for every k."""
    worst = 0.0
    V = 17
    z_s = rs.normal(size=(1, V)) * 2
    z_t = rs.normal(size=(1, V)) * 2
    p = scipy.special.softmax(z_s[0])
    L, _, _ = O.per_row_kl(z_s, z_t)
    dz_exact = O.dz_rows(z_s, z_t, np.ones(1))
    for k in (1, 2, 5, 11, 16):
        EL = 0.0
        Edz = np.zeros(V)
        for yy in range(V):
            Lk, dz = O.topk_rows(z_s, z_t, np.array([yy]), k, np.ones(1))
            EL += p[yy] * Lk[0]
            Edz += p[yy] * dz[0]
        worst = max(worst, abs(EL - L[0]), float(np.max(np.abs(Edz - dz_exact[0]))))
    return worst


def topk_brute(O, rs):
    """Estimate against the pure-Python loop, on rows with tied logits."""
    worst = 0.0
    for _ in range(4):
        V = 9
        z_s = rs.randint(-2, 3, size=(3, V)).astype(float)  # many ties
        z_t = rs.normal(size=(3, V))
        y = rs.randint(0, V, size=3)
        for k in (0, 1, 3, 4, 8, 9):
            Lk, _ = O.topk_rows(z_s, z_t, y, k)
            for i in range(3):
                ref = brute.topk_estimate_row(z_s[i].tolist(), z_t[i].tolist(), int(y[i]), k)
                worst = max(worst, abs(Lk[i] - ref))
    return worst


def topk_support_ties(O, rs):
    """The support takes the k largest student logits, lower token id first
    among equal logits (compared with a sort by (-z, id))."""
    bad = 0
    for _ in range(5):
        z = rs.randint(-1, 2, size=(2, 12)).astype(float)
        for k in (0, 1, 4, 7, 12):
            S = O.topk_support(z, k)
            for i in range(2):
                ranked = sorted(range(12), key=lambda v: (-z[i, v], v))
                bad += int(sorted(np.flatnonzero(S[i]).tolist()) != sorted(ranked[:k]))
    return bad


def topk_finite_differences(O, rs):
    """With the sampled token inside the support, the estimate is the exact
    reverse-KL sum over S; its gradient (S held fixed) against central
    differences (logits well separated, so S does not move)."""
    V, k = 10, 4
    z_s = np.sort(rs.uniform(-3, 3, size=V))[::-1].copy() + np.arange(V)[::-1] * 0.3
    z_s = z_s[rs.permutation(V)][None, :]
    z_t = rs.normal(size=(1, V))
    S = O.topk_support(z_s, k)[0]
    y = np.array([int(np.flatnonzero(S)[0])])
    _, dz = O.topk_rows(z_s, z_t, y, k, np.ones(1))
    eps = 1e-6
    num = np.zeros(V)
    for j in range(V):
        zp = z_s.copy(); zp[0, j] += eps
        zm = z_s.copy(); zm[0, j] -= eps
        num[j] = (O.topk_rows(zp, z_t, y, k)[0][0] - O.topk_rows(zm, z_t, y, k)[0][0]) / (2 * eps)
    return float(np.max(np.abs(dz[0] - num)) / np.max(np.abs(num)))


def topk_hidden_chain_rule(O, rs):
    """The hidden-payload top-k estimate equals the logits-pair one on
    z = h W^T, and its gradients are dz W_s and dz^T h_s (chain rule)."""
    h_s, W_s, h_t, W_t, mask = rand_problem(rs, B=2, Sm1=4, H=3, V=11)
    y = rs.randint(0, 11, size=mask.shape)
    z_s, z_t = h_s @ W_s.T, h_t @ W_t.T
    worst = 0.0
    for k in (0, 3, 11):
        a = O.forward_topk_hidden(h_s, W_s, h_t, W_t, y, k, mask, 2)
        b = O.forward_topk_pair(z_s, z_t, y, k, mask, 2)
        dH, dW = O.backward_topk_hidden(h_s, W_s, h_t, W_t, y, k, mask, 2)
        dz = O.backward_topk_pair(z_s, z_t, y, k, mask, 2)
        worst = max(worst, float(np.max(np.abs(a["loss_tok"] - b["loss_tok"]))), abs(a["loss"] - b["loss"]),
                    float(np.max(np.abs(dH - dz @ W_s))), float(np.max(np.abs(dW - dz.T @ h_s))))
    return worst


def topk_hidden_finite_differences(O, rs):
    """Central differences of the top-k objective w.r.t. h_s and W_s when the
    sampled tokens lie in the support (no score-function term) and the
    support does not move under the perturbation."""
    B, Sm1, H, V, k = 1, 3, 3, 9, 4
    h_s = rs.normal(size=(3, H))
    W_s = rs.normal(size=(V, H)) * 2
    h_t = rs.normal(size=(3, H))
    W_t = rs.normal(size=(V, H))
    mask = np.ones((B, Sm1), np.uint8)
    S = O.topk_support(h_s @ W_s.T, k)
    y = np.array([[int(np.flatnonzero(S[i])[0]) for i in range(3)]])
    f = lambda hs, ws: O.forward_topk_hidden(hs, ws, h_t, W_t, y, k, mask, 1)["loss"]  # noqa: E731
    dH, dW = O.backward_topk_hidden(h_s, W_s, h_t, W_t, y, k, mask, 1)
    eps = 1e-6
    num_H = np.zeros_like(h_s)
    for i in range(h_s.shape[0]):
        for j in range(H):
            hp = h_s.copy(); hp[i, j] += eps
            hm = h_s.copy(); hm[i, j] -= eps
            num_H[i, j] = (f(hp, W_s) - f(hm, W_s)) / (2 * eps)
    num_W = np.zeros_like(W_s)
    for i in range(V):
        for j in range(H):
            wp = W_s.copy(); wp[i, j] += eps
            wm = W_s.copy(); wm[i, j] -= eps
            num_W[i, j] = (f(h_s, wp) - f(h_s, wm)) / (2 * eps)
    return max(float(np.max(np.abs(dH - num_H))) / float(np.max(np.abs(num_H))),
               float(np.max(np.abs(dW - num_W))) / float(np.max(np.abs(num_W))))


def dw_rows_vs_backward(O, rs):
    """The selected-vocabulary-rows gradient equals those rows of the full
    dW_s of `backward` (itself pinned by finite differences), on both
    payloads, both reductions and with a per-token upstream gradient, for
    sorted, unsorted and repeated vocabulary ids."""
    worst = 0.0
    for payload in ("hidden", "logits"):
        for red in (1, 2):
            h_s, W_s, teacher, W_t, mask = rand_problem(rs, B=3, Sm1=5, H=6, V=19, payload=payload)
            gt = rs.normal(size=mask.shape)
            ids = np.array([0, 18, 7, 7, 3, 12])
            _, dW = O.backward(h_s, W_s, teacher, W_t, mask, red, grad_loss=0.8, grad_tok=gt)
            sel = O.backward_dw_rows(h_s, W_s, teacher, W_t, mask, red, ids, grad_loss=0.8, grad_tok=gt)
            worst = max(worst, float(np.max(np.abs(sel - dW[ids]))) / float(np.max(np.abs(dW))))
    return worst


def topk_logits_chain_rule(O, rs):
    """The logits-payload top-k estimate equals the logits-pair one on
    z_s = h_s W_s^T and the shipped teacher rows, and its gradients are
    dz W_s and dz^T h_s (chain rule)."""
    h_s, W_s, teacher, _, mask = rand_problem(rs, B=2, Sm1=4, H=3, V=11, payload="logits")
    y = rs.randint(0, 11, size=mask.shape)
    z_s = h_s @ W_s.T
    worst = 0.0
    for k in (0, 3, 11):
        a = O.forward_topk_logits(h_s, W_s, teacher, y, k, mask, 2)
        b = O.forward_topk_pair(z_s, teacher, y, k, mask, 2)
        dH, dW = O.backward_topk_logits(h_s, W_s, teacher, y, k, mask, 2)
        dz = O.backward_topk_pair(z_s, teacher, y, k, mask, 2)
        worst = max(worst, float(np.max(np.abs(a["loss_tok"] - b["loss_tok"]))), abs(a["loss"] - b["loss"]),
                    float(np.max(np.abs(dH - dz @ W_s))), float(np.max(np.abs(dW - dz.T @ h_s))))
    return worst


def topk_logits_exact_limit(O, rs):
    """k >= V on the logits payload gives the exact objective of `forward` /
    `backward` with shipped teacher logits (pinned by scipy and finite
    differences)."""
    h_s, W_s, teacher, _, mask = rand_problem(rs, B=2, Sm1=5, H=4, V=13, payload="logits")
    y = rs.randint(0, 13, size=mask.shape)
    a = O.forward_topk_logits(h_s, W_s, teacher, y, 13, mask, 1)
    b = O.forward(h_s, W_s, teacher, None, mask, 1)
    dHa, dWa = O.backward_topk_logits(h_s, W_s, teacher, y, 20, mask, 1)
    dHb, dWb = O.backward(h_s, W_s, teacher, None, mask, 1)
    return max(float(np.max(np.abs(a["loss_tok"] - b["loss_tok"]))), abs(a["loss"] - b["loss"]),
               float(np.max(np.abs(dHa - dHb))), float(np.max(np.abs(dWa - dWb))))


def topk_logits_finite_differences(O, rs):
    """Central differences of the logits-payload top-k objective w.r.t. h_s
    and W_s, with sampled tokens inside the support and a support that does
    not move under the perturbation."""
    H, V, k = 3, 9, 4
    h_s = rs.normal(size=(3, H))
    W_s = rs.normal(size=(V, H)) * 2
    zt = rs.normal(size=(3, V)) * 2
    mask = np.ones((1, 3), np.uint8)
    S = O.topk_support(h_s @ W_s.T, k)
    y = np.array([[int(np.flatnonzero(S[i])[-1]) for i in range(3)]])
    f = lambda hs, ws: O.forward_topk_logits(hs, ws, zt, y, k, mask, 1)["loss"]  # noqa: E731
    dH, dW = O.backward_topk_logits(h_s, W_s, zt, y, k, mask, 1)
    eps = 1e-6
    num_H = np.zeros_like(h_s)
    for i in range(h_s.shape[0]):
        for j in range(H):
            hp = h_s.copy(); hp[i, j] += eps
            hm = h_s.copy(); hm[i, j] -= eps
            num_H[i, j] = (f(hp, W_s) - f(hm, W_s)) / (2 * eps)
    num_W = np.zeros_like(W_s)
    for i in range(V):
        for j in range(H):
            wp = W_s.copy(); wp[i, j] += eps
            wm = W_s.copy(); wm[i, j] -= eps
            num_W[i, j] = (f(h_s, wp) - f(h_s, wm)) / (2 * eps)
    return max(float(np.max(np.abs(dH - num_H))) / float(np.max(np.abs(num_H))),
               float(np.max(np.abs(dW - num_W))) / float(np.max(np.abs(num_W))))
