"""Pins of the float64 CPU oracle (no GPU).

Every check compares the oracle with something outside it: a library routine
for a special case (scipy KL / entropy / logsumexp), a closed form, an
invariant of the objective, a pure-Python brute force, or finite differences.
The mutation tests plant plausible mistakes in a private copy of the oracle
and show that at least one pin catches each.
"""

import json
import os
import types

import numpy as np
import pytest

from oracle import brute
from oracle import rkl_oracle as O
from tests import pins

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


@pytest.fixture
def rs():
    return np.random.RandomState(20261202)


def test_kl_matches_scipy_entropy(rs):
    assert pins.kl_vs_scipy(O, rs) < 1e-10


def test_lse_matches_scipy(rs):
    assert pins.lse_vs_scipy(O, rs) < 1e-10


def test_kl_nonnegative(rs):
    for V in (2, 10, 5000):
        z_s = rs.normal(size=(16, V)) * 4
        z_t = rs.normal(size=(16, V)) * 4
        L, _, _ = O.per_row_kl(z_s, z_t)
        assert np.all(L >= -1e-12)


def test_uniform_teacher_closed_form(rs):
    assert pins.uniform_teacher(O, rs) < 1e-10


def test_one_logit_bump_closed_form(rs):
    assert pins.one_logit_bump(O, rs) < 1e-12


def test_binary_vocabulary_closed_form(rs):
    assert pins.binary_kl(O, rs) < 1e-12


def test_brute_force_loops(rs):
    assert pins.brute_force(O, rs) < 1e-12


def test_compact_rows_brute(rs):
    assert pins.compact_rows_brute(O, rs) == 0


@pytest.mark.parametrize("payload", ["hidden", "logits"])
@pytest.mark.parametrize("red", [1, 2])
def test_finite_differences(rs, payload, red):
    assert pins.finite_differences(O, rs, payload=payload, red=red) < 1e-6


def test_finite_differences_grad_tok(rs):
    # reduction NONE: only the per-token upstream gradient drives backward
    assert pins.finite_differences(O, rs, red=0, with_grad_tok=True) < 1e-6
    # both a reduced-loss gradient and a per-token gradient at once
    assert pins.finite_differences(O, rs, red=2, with_grad_tok=True, grad_loss=0.7) < 1e-6


def test_self_distillation_exact_zero(rs):
    assert pins.self_distillation(O, rs) == 0.0


def test_dz_rows_sum_to_zero(rs):
    assert pins.dz_sums_to_zero(O, rs) < 1e-13


def test_teacher_shift_invariance(rs):
    assert pins.shift_invariance(O, rs) < 1e-10


def test_masked_rows_exact_zero(rs):
    assert pins.masked_rows_exact_zero(O, rs) == 0.0


def test_compact_equals_full(rs):
    assert pins.compact_equals_full(O, rs) < 1e-12


def test_empty_mask(rs):
    assert pins.empty_mask(O, rs) == 0.0


def test_nested_equals_token_mean_for_equal_counts(rs):
    assert pins.nested_vs_token_mean_equal_counts(O, rs) < 1e-14


def test_nested_mean_skips_empty_sequences(rs):
    assert pins.nested_mean_by_hand(O, rs) < 1e-14


def test_payload_ratio_golden():
    """The logits payload is ~74x the hidden payload at 2k hidden / 152k vocab."""
    with open(os.path.join(GOLDEN, "payload_ratio.json")) as f:
        g = json.load(f)
    ratio = g["V"] / g["H"]
    assert round(ratio) == g["quoted_ratio"]
    from full_vocabulary_reverse_b200.workloads import WORKLOADS
    w = WORKLOADS["qwen_hidden"]
    assert (w["H"], w["V"]) == (g["H"], g["V"])


def test_golden_tiny_case():
    """Stored oracle outputs of a tiny case (written by tests/golden/make_golden.py)."""
    with open(os.path.join(GOLDEN, "tiny_case.json")) as f:
        g = json.load(f)
    a = {k: np.array(v) for k, v in g["inputs"].items()}
    out = O.forward(a["h_s"], a["W_s"], a["h_t"], a["W_t"], a["mask"].astype(np.uint8), g["reduction"])
    dH, dW = O.backward(a["h_s"], a["W_s"], a["h_t"], a["W_t"], a["mask"].astype(np.uint8), g["reduction"])
    np.testing.assert_allclose(out["loss_tok"], np.array(g["loss_tok"]), rtol=1e-12, atol=1e-15)
    np.testing.assert_allclose(out["loss"], g["loss"], rtol=1e-12)
    np.testing.assert_allclose(dH, np.array(g["dH_s"]), rtol=1e-10, atol=1e-15)
    np.testing.assert_allclose(dW, np.array(g["dW_s"]), rtol=1e-10, atol=1e-15)


# --------------------------------------------------------------------------
# Mutation tests: plant a mistake in a private copy of the oracle and check
# that the pins notice.  The planted copy is built from the source text; the
# real module is untouched.
# --------------------------------------------------------------------------

def _mutant(old, new):
    src = open(O.__file__).read()
    assert src.count(old) >= 1, old
    mod = types.ModuleType("oracle_mutant")
    exec(compile(src.replace(old, new), "oracle_mutant", "exec"), mod.__dict__)
    return mod


MUTATIONS = [
    # dropped -L term in the shared backward
    ("dz = g[c0:c0 + len(rows), None] * p_s * (w - L[:, None])",
     "dz = g[c0:c0 + len(rows), None] * p_s * (w)", "fd"),
    # forward KL instead of reverse KL
    ("    p_s = np.exp(lp_s)\n    L = np.sum(p_s * (lp_s - lp_t), axis=1)",
     "    p_s = np.exp(lp_t)\n    L = np.sum(p_s * (lp_t - lp_s), axis=1)", "kl"),
    # wrong sign in the log-sum-exp
    ("return z - (m + np.log(", "return z - (m - np.log(", "kl"),
    # transposed / wrong operand in dW_s
    ("dW += dz.T @ _f64(h_s[rows])", "dW += dz.T @ _f64(teacher[rows])", "fd"),
    # wrong nested-mean weight
    ("g += grad_loss / (b_eff * counts[seq])", "g += grad_loss / N", "fd_nested"),
    # scatter to the wrong positions
    ("loss_tok[row_idx] = L", "loss_tok[:N] = L", "masked"),
    # off-by-one in compaction
    ("row_idx = np.flatnonzero(flat).astype(np.int64)",
     "row_idx = (np.flatnonzero(flat) + 1).astype(np.int64) % flat.size", "compact"),
    # teacher max-shift applied to student lse in saved scalars
    ("return m + np.log(np.sum(np.exp(z - m[:, None]), axis=1))",
     "return m + np.log(np.sum(np.exp(z - m[:, None]), axis=1)) + 1e-3", "lse"),
    # dH rows scattered to compact positions
    ("dH[rows] = dz @ W_s64", "dH[c0:c0 + len(rows)] = dz @ W_s64", "masked"),
]


@pytest.mark.parametrize("old,new,kind", MUTATIONS)
def test_pins_catch_planted_mistakes(old, new, kind):
    M = _mutant(old, new)
    rs = np.random.RandomState(7)
    caught = {
        "fd": lambda: pins.finite_differences(M, rs) > 1e-4,
        "fd_nested": lambda: pins.finite_differences(M, rs, red=2) > 1e-4,
        "kl": lambda: pins.kl_vs_scipy(M, rs) > 1e-6 or pins.brute_force(M, rs) > 1e-6,
        "masked": lambda: pins.masked_rows_exact_zero(M, rs) > 0 or pins.brute_force(M, rs) > 1e-6,
        "compact": lambda: pins.compact_rows_brute(M, rs) > 0,
        "lse": lambda: pins.lse_vs_scipy(M, rs) > 1e-6,
    }[kind]()
    assert caught


@pytest.mark.parametrize("red", [1, 2])
def test_logits_pair_finite_differences(rs, red):
    assert pins.logits_pair_finite_differences(O, rs, red=red) < 1e-6
    assert pins.logits_pair_finite_differences(O, rs, red=0, with_grad_tok=True) < 1e-6


def test_logits_pair_kl_matches_scipy(rs):
    import scipy.special
    import scipy.stats
    z_s = rs.normal(size=(6, 50)) * 3
    z_t = rs.normal(size=(6, 50)) * 3
    out = O.forward_logits_pair(z_s, z_t, np.ones((2, 3), np.uint8), 0)
    ref = scipy.stats.entropy(scipy.special.softmax(z_s, axis=1), scipy.special.softmax(z_t, axis=1), axis=1)
    assert np.max(np.abs(out["L"] - ref)) < 1e-10


def test_logits_pair_chain_rule_to_hidden_payload(rs):
    assert pins.logits_pair_matches_hidden_chain_rule(O, rs) < 1e-12


def test_logits_pair_masked_rows_zero_and_self_distill(rs):
    z = rs.normal(size=(6, 40)) * 3
    mask = np.array([[1, 0, 1], [0, 0, 1]], np.uint8)
    dz = O.backward_logits_pair(z, rs.normal(size=(6, 40)), mask, 1)
    assert np.all(dz[mask.reshape(-1) == 0] == 0)
    assert np.all(O.backward_logits_pair(z, z.copy(), mask, 1) == 0)
    assert O.forward_logits_pair(z, z.copy(), mask, 1)["loss"] == 0.0


def test_student_entropy_and_logprob_match_scipy(rs):
    import scipy.special
    import scipy.stats
    h_s, W_s, _, _, mask = rand_problem_for_stats(rs)
    targets = rs.randint(0, W_s.shape[0], size=mask.shape)
    ent, tlp = O.student_stats(h_s, W_s, mask, targets)
    z = h_s @ W_s.T
    ref_ent = scipy.stats.entropy(scipy.special.softmax(z, axis=1), axis=1)
    ref_lp = scipy.special.log_softmax(z, axis=1)[np.arange(z.shape[0]), targets.reshape(-1)]
    on = mask.reshape(-1) != 0
    assert np.max(np.abs(ent.reshape(-1)[on] - ref_ent[on])) < 1e-10
    assert np.max(np.abs(tlp.reshape(-1)[on] - ref_lp[on])) < 1e-10
    assert np.all(ent.reshape(-1)[~on] == 0) and np.all(tlp.reshape(-1)[~on] == 0)


def test_student_entropy_closed_forms(rs):
    # uniform student logits: entropy = log V; one-hot limit: entropy -> 0
    ent, _ = O.student_stats_rows(np.zeros((2, 37)))
    assert np.max(np.abs(ent - np.log(37))) < 1e-12
    z = np.full((1, 10), -1e3)
    z[0, 3] = 0.0
    ent, tlp = O.student_stats_rows(z, [3])
    assert abs(ent[0]) < 1e-12 and abs(tlp[0]) < 1e-12


def test_student_stats_from_logits_equal_hidden(rs):
    h_s, W_s, _, _, mask = rand_problem_for_stats(rs)
    targets = rs.randint(0, W_s.shape[0], size=mask.shape)
    a = O.student_stats(h_s, W_s, mask, targets)
    b = O.student_stats(None, None, mask, targets, student_logits=h_s @ W_s.T)
    assert np.max(np.abs(a[0] - b[0])) < 1e-12 and np.max(np.abs(a[1] - b[1])) < 1e-12


def rand_problem_for_stats(rs):
    return pins.rand_problem(rs, B=3, Sm1=5, H=4, V=23)


# ------------------------------------------------------------ several teachers

def test_multi_teacher_brute_force(rs):
    assert pins.multi_teacher_brute_force(O, rs) < 1e-12


def test_multi_teacher_kl_vs_scipy(rs):
    assert pins.multi_teacher_kl_vs_scipy(O, rs) < 1e-10


@pytest.mark.parametrize("red", [1, 2])
def test_multi_teacher_finite_differences(rs, red):
    assert pins.multi_teacher_finite_differences(O, rs, red=red) < 1e-6


def test_multi_teacher_counts_brute(rs):
    assert pins.multi_teacher_counts_brute(O, rs) == 0


def test_multi_teacher_single_teacher_reduces(rs):
    # every row on teacher g: the single-teacher forward/backward with W_t[g]
    h_s, W_s, h_t, W_t, _, mask = pins.rand_multi_problem(rs)
    for g in range(W_t.shape[0]):
        tid = np.full(mask.shape, g)
        a = O.forward_multi(h_s, W_s, h_t, W_t, tid, mask, 2)
        b = O.forward(h_s, W_s, h_t, W_t[g], mask, 2)
        assert np.max(np.abs(a["loss_tok"] - b["loss_tok"])) < 1e-14 and abs(a["loss"] - b["loss"]) < 1e-14
        dHa, dWa = O.backward_multi(h_s, W_s, h_t, W_t, tid, mask, 2)
        dHb, dWb = O.backward(h_s, W_s, h_t, W_t[g], mask, 2)
        assert np.max(np.abs(dHa - dHb)) < 1e-14 and np.max(np.abs(dWa - dWb)) < 1e-14


MULTI_MUTATIONS = [
    # every row projected with the first teacher's head
    ("z_t[sel] = _f64(h_t[rows[sel]]) @ W_t64[g].T", "z_t[sel] = _f64(h_t[rows[sel]]) @ W_t64[0].T", "brute"),
    # teacher index read at the compact position instead of the token position
    ("    k = tid_flat[rows]\n", "    k = tid_flat[np.arange(len(rows))]\n", "brute"),
    # teacher indices off by one
    ("z_t[sel] = _f64(h_t[rows[sel]]) @ W_t64[g].T",
     "z_t[sel] = _f64(h_t[rows[sel]]) @ W_t64[(g + 1) % W_t64.shape[0]].T", "brute"),
    # masked rows counted per teacher
    ("    tid = np.asarray(teacher_idx).reshape(-1)[flat]\n", "    tid = np.asarray(teacher_idx).reshape(-1)\n",
     "counts"),
]


@pytest.mark.parametrize("old,new,kind", MULTI_MUTATIONS)
def test_multi_teacher_pins_catch_planted_mistakes(old, new, kind):
    M = _mutant(old, new)
    rs = np.random.RandomState(11)
    if kind == "brute":
        assert pins.multi_teacher_brute_force(M, rs) > 1e-6
    else:
        assert pins.multi_teacher_counts_brute(M, rs) > 0


# ------------------------------------------------------------ top-k estimator

def test_topk_limits(rs):
    assert pins.topk_limits(O, rs) < 1e-12


def test_topk_unbiased_over_sampled_token(rs):
    assert pins.topk_unbiased(O, rs) < 1e-12


def test_topk_brute_force_with_ties(rs):
    assert pins.topk_brute(O, rs) < 1e-12


def test_topk_support_ties(rs):
    assert pins.topk_support_ties(O, rs) == 0


def test_topk_finite_differences(rs):
    assert pins.topk_finite_differences(O, rs) < 1e-6


def test_topk_pair_masked_rows_and_reduction(rs):
    z_s = rs.normal(size=(6, 30)) * 2
    z_t = rs.normal(size=(6, 30)) * 2
    y = rs.randint(0, 30, size=(2, 3))
    mask = np.array([[1, 0, 1], [0, 1, 1]], np.uint8)
    out = O.forward_topk_pair(z_s, z_t, y, 5, mask, 2)
    assert np.all(out["loss_tok"][mask == 0] == 0)
    assert abs(out["loss"] - brute.nested_mean(out["loss_tok"].tolist(), mask.tolist())) < 1e-14
    dz = O.backward_topk_pair(z_s, z_t, y, 5, mask, 2)
    assert np.all(dz[mask.reshape(-1) == 0] == 0)
    # k = V reduces to the logits-pair path
    a = O.forward_topk_pair(z_s, z_t, y, 30, mask, 1)
    b = O.forward_logits_pair(z_s, z_t, mask, 1)
    assert np.max(np.abs(a["loss_tok"] - b["loss_tok"])) < 1e-12
    assert np.max(np.abs(O.backward_topk_pair(z_s, z_t, y, 30, mask, 1) - O.backward_logits_pair(z_s, z_t, mask, 1))) < 1e-12


TOPK_MUTATIONS = [
    # ties broken by higher id
    ("order = np.argsort(-z_s[i], kind=\"stable\")", "order = V - 1 - np.argsort(-z_s[i][::-1], kind=\"stable\")", "support"),
    # score-function term without the +1
    ("a = np.where(out_y, w_y + 1.0, 0.0)", "a = np.where(out_y, w_y, 0.0)", "unbiased"),
    # tail estimate applied even when y is inside the support
    ("L_hat = L_S + np.where(out_y, w_y, 0.0)", "L_hat = L_S + w_y", "brute"),
    # support mass missing from the gradient constant
    ("- (L_S + P_S)[:, None])", "- (L_S)[:, None])", "limits"),
]


@pytest.mark.parametrize("old,new,kind", TOPK_MUTATIONS)
def test_topk_pins_catch_planted_mistakes(old, new, kind):
    M = _mutant(old, new)
    rs = np.random.RandomState(13)
    caught = {
        "support": lambda: pins.topk_support_ties(M, rs) > 0 or pins.topk_brute(M, rs) > 1e-6,
        "unbiased": lambda: pins.topk_unbiased(M, rs) > 1e-6,
        "brute": lambda: pins.topk_brute(M, rs) > 1e-6,
        "limits": lambda: pins.topk_limits(M, rs) > 1e-6,
    }[kind]()
    assert caught


def test_topk_hidden_chain_rule(rs):
    assert pins.topk_hidden_chain_rule(O, rs) < 1e-12


def test_topk_hidden_finite_differences(rs):
    assert pins.topk_hidden_finite_differences(O, rs) < 1e-6


# ------------------------------------------------------------ selected dW rows

def test_backward_dw_rows_equal_full_backward(rs):
    assert pins.dw_rows_vs_backward(O, rs) < 1e-12


@pytest.mark.parametrize("old,new", [
    # dz columns taken from the wrong vocabulary ids
    ("p_s[:, vocab_ids] * (w[:, vocab_ids] - L[:, None])", "p_s[:, vocab_ids] * (w[:, vocab_ids - 1] - L[:, None])"),
    # the -L term dropped in the selected columns
    ("p_s[:, vocab_ids] * (w[:, vocab_ids] - L[:, None])", "p_s[:, vocab_ids] * (w[:, vocab_ids])"),
])
def test_dw_rows_pin_catches_planted_mistakes(old, new):
    M = _mutant(old, new)
    assert pins.dw_rows_vs_backward(M, np.random.RandomState(3)) > 1e-6


# ------------------------------------------------------------ top-k on the logits payload

def test_topk_logits_chain_rule(rs):
    assert pins.topk_logits_chain_rule(O, rs) < 1e-12


def test_topk_logits_exact_limit(rs):
    assert pins.topk_logits_exact_limit(O, rs) < 1e-12


def test_topk_logits_finite_differences(rs):
    assert pins.topk_logits_finite_differences(O, rs) < 1e-6


@pytest.mark.parametrize("old,new", [
    # the student's logits taken for the teacher's as well
    ("        z_s, z_t = _student_teacher_logits(rows, h_s, W_s64, teacher_logits, None)\n"
     "        L[c0:c0 + len(rows)], _ = topk_rows(z_s, z_t, yflat[rows], k)",
     "        z_s, z_t = _student_teacher_logits(rows, h_s, W_s64, teacher_logits, None)\n"
     "        L[c0:c0 + len(rows)], _ = topk_rows(z_s, z_s, yflat[rows], k)"),
    # dW from the teacher's logits instead of the student's hidden rows
    ("        _, dz = topk_rows(z_s, z_t, yflat[rows], k, g[c0:c0 + len(rows)])\n"
     "        dH[rows] = dz @ W_s64\n        dW += dz.T @ _f64(h_s[rows])\n    return dH, dW\n",
     "        _, dz = topk_rows(z_s, z_t, yflat[rows], k, g[c0:c0 + len(rows)])\n"
     "        dH[rows] = dz @ W_s64\n        dW += dz.T @ _f64(h_s[rows][::-1])\n    return dH, dW\n"),
])
def test_topk_logits_pins_catch_planted_mistakes(old, new):
    M = _mutant(old, new)
    rs = np.random.RandomState(17)
    assert (pins.topk_logits_chain_rule(M, rs) > 1e-6 or pins.topk_logits_exact_limit(M, rs) > 1e-6
            or pins.topk_logits_finite_differences(M, rs) > 1e-4)
