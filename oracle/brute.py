"""Pure-Python loop restatement of the reverse-KL loss for tiny shapes.

TEST INFRASTRUCTURE, like the rest of ``oracle/``: only tests may call it.
It shares no code with ``rkl_oracle`` (no NumPy vector ops, only ``math`` and
plain loops) so that it can pin that module on small inputs.

Objective: NeMo RL PR #3978 ("feat(mopd): add full-vocabulary on-policy
distillation"), description: L_t = sum_v p_s(v)(log p_s(v) - log p_t(v)),
with p = softmax(z), z_s = h_s . W_s[v], z_t = h_t . W_t[v].
"""

import math


def _dot(a, b):
    s = 0.0
    for x, y in zip(a, b):
        s += float(x) * float(y)
    return s


def _softmax(z):
    m = max(z)
    e = [math.exp(v - m) for v in z]
    s = sum(e)
    return [v / s for v in e]


def kl_row(z_s, z_t):
    """sum_v p_s(v) (log p_s(v) - log p_t(v)) for one row of logits."""
    p_s = _softmax(z_s)
    p_t = _softmax(z_t)
    total = 0.0
    for a, b in zip(p_s, p_t):
        if a > 0.0:
            total += a * (math.log(a) - math.log(b))
    return total


def logits_row(h, W):
    return [_dot(h, W[v]) for v in range(len(W))]


def loss_tokens(h_s, W_s, h_t, W_t, mask):
    """Per-position loss [B][S-1] by loops; masked positions are 0."""
    B = len(mask)
    Sm1 = len(mask[0])
    out = [[0.0] * Sm1 for _ in range(B)]
    for b in range(B):
        for t in range(Sm1):
            if mask[b][t]:
                r = b * Sm1 + t
                out[b][t] = kl_row(logits_row(h_s[r], W_s), logits_row(h_t[r], W_t))
    return out


def nested_mean(loss_tok, mask):
    """Mean over non-empty sequences of the per-sequence mean of trainable positions."""
    means = []
    for row, mrow in zip(loss_tok, mask):
        vals = [v for v, m in zip(row, mrow) if m]
        if vals:
            means.append(sum(vals) / len(vals))
    return sum(means) / len(means) if means else 0.0


def token_mean(loss_tok, mask):
    vals = [v for row, mrow in zip(loss_tok, mask) for v, m in zip(row, mrow) if m]
    return sum(vals) / len(vals) if vals else 0.0


def compact_rows(mask):
    """Ascending flattened indices of the nonzero mask positions, by a loop."""
    out = []
    k = 0
    for row in mask:
        for m in row:
            if m:
                out.append(k)
            k += 1
    return out


def loss_tokens_multi(h_s, W_s, h_t, W_t_list, teacher_idx, mask):
    """Per-position loss [B][S-1] with the teacher head W_t_list[k] chosen by
    the position's teacher index k; masked positions are 0."""
    B = len(mask)
    Sm1 = len(mask[0])
    out = [[0.0] * Sm1 for _ in range(B)]
    for b in range(B):
        for t in range(Sm1):
            if mask[b][t]:
                r = b * Sm1 + t
                W_t = W_t_list[teacher_idx[b][t]]
                out[b][t] = kl_row(logits_row(h_s[r], W_s), logits_row(h_t[r], W_t))
    return out


def count_rows_per_teacher(mask, teacher_idx, n_teachers):
    counts = [0] * n_teachers
    bad = 0
    for mrow, trow in zip(mask, teacher_idx):
        for m, k in zip(mrow, trow):
            if m:
                if 0 <= k < n_teachers:
                    counts[k] += 1
                else:
                    bad += 1
    return counts, bad


def topk_estimate_row(z_s, z_t, y, k):
    """Top-k estimate of one row by loops: the exact reverse-KL terms of the k
    largest student logits (ties: lower token id first) plus w(y) when the
    sampled token y is outside them."""
    p_s = _softmax(z_s)
    p_t = _softmax(z_t)
    ranked = sorted(range(len(z_s)), key=lambda v: (-z_s[v], v))
    S = set(ranked[:max(0, min(k, len(z_s)))])
    total = 0.0
    for v in S:
        total += p_s[v] * (math.log(p_s[v]) - math.log(p_t[v]))
    if y not in S:
        total += math.log(p_s[y]) - math.log(p_t[y])
    return total
