"""Seeded synthetic inputs shaped like the pages' workloads.

This module only draws random numbers; it holds none of the loss arithmetic.
Both the CUDA path and the CPU oracle are fed from it.

Shapes (NeMo RL PR #3978 quotes a 2k-hidden / 152k-vocab model and a
Qwen3-1.7B self-distillation recipe; slime PR #2310 motivates long masked
prompts).  No dataset or trained weights are used anywhere.

Named workloads:
  tiny_fp32       fp32, B=2, S-1=32, H=64, V=512, W_s and W_t independent
                  N(0,1/H)*3, mask all ones, token mean.
  qwen_hidden     bf16, B=4, S-1=2048, H=2048, V=151936, h ~ N(0,1),
                  W_s ~ N(0,1)*3/sqrt(H) (logit std ~3), W_t = W_s + N(0,0.004^2),
                  per sequence a U[0.25,0.75] prompt prefix masked, token mean.
  self_distill    qwen_hidden shapes with h_t = h_s, W_t = W_s, nested mean.
  teacher_logits  bf16 teacher logits [8192, 151936] ~ N(0,9) plus a per-row
                  shift U(-20,20); h_s [8192, 2048]; W_s as qwen_hidden; all
                  rows trainable; token mean.
  long_prompt     bf16, B=8, S-1=4096 (T=32768), H=4096, V=151936, W as
                  qwen_hidden at H=4096, last 256 positions of each sequence
                  trainable (N=2048), token mean.
  logits_pair     both sides as bf16 logits [8192, 151936]: student ~ N(0,9),
                  teacher = student + N(0, 0.5^2) + per-row shift U(-20,20);
                  all rows trainable; token mean.
  logits_pair_topk  logits_pair inputs, top-k estimator with k = 64 and the
                  sampled token of each position drawn from the student's
                  softmax (on-policy sample).
  topk_hidden     qwen_hidden inputs, top-k estimator with k = 64 and a
                  sampled token per position drawn uniformly (the estimator's
                  cost does not depend on how the tokens were drawn).
  topk_logits     teacher_logits inputs, top-k estimator with k = 64 on the
                  teacher-logits payload and a sampled token per position
                  drawn uniformly.
  qwen_hidden_stats  qwen_hidden inputs, the forward also returning the
                  student's per-token entropy and the log-probability of a
                  target token per position (drawn uniformly).
  multi_teacher   qwen_hidden shapes and mask with two teacher heads
                  W_t[g] = W_s + N(0, 0.004^2) (independent draws), teacher
                  of sequence b = b mod 2; token mean.
"""

from __future__ import annotations

import math

import numpy as np
import torch

REDUCE_NONE = 0
REDUCE_TOKEN_MEAN = 1
REDUCE_SEQ_MEAN_NESTED = 2

WORKLOADS = {
    "tiny_fp32": dict(dtype="fp32", B=2, Sm1=32, H=64, V=512, payload="hidden",
                      reduction=REDUCE_TOKEN_MEAN, mask="all", weights="independent", seed=1235),
    "qwen_hidden": dict(dtype="bf16", B=4, Sm1=2048, H=2048, V=151936, payload="hidden",
                        reduction=REDUCE_TOKEN_MEAN, mask="prefix", weights="perturbed", seed=1236),
    "self_distill": dict(dtype="bf16", B=4, Sm1=2048, H=2048, V=151936, payload="hidden",
                         reduction=REDUCE_SEQ_MEAN_NESTED, mask="prefix", weights="same", seed=1237,
                         mask_seed=1236),
    "teacher_logits": dict(dtype="bf16", B=4, Sm1=2048, H=2048, V=151936, payload="logits",
                           reduction=REDUCE_TOKEN_MEAN, mask="all", weights="perturbed", seed=1238),
    "long_prompt": dict(dtype="bf16", B=8, Sm1=4096, H=4096, V=151936, payload="hidden",
                        reduction=REDUCE_TOKEN_MEAN, mask="suffix256", weights="perturbed", seed=1239),
    "logits_pair": dict(dtype="bf16", B=4, Sm1=2048, H=0, V=151936, payload="logits_pair",
                        reduction=REDUCE_TOKEN_MEAN, mask="all", weights="perturbed", seed=1240),
    "logits_pair_topk": dict(dtype="bf16", B=4, Sm1=2048, H=0, V=151936, payload="logits_pair",
                             reduction=REDUCE_TOKEN_MEAN, mask="all", weights="perturbed", seed=1242,
                             targets="sampled", k=64),
    "topk_hidden": dict(dtype="bf16", B=4, Sm1=2048, H=2048, V=151936, payload="hidden",
                        reduction=REDUCE_TOKEN_MEAN, mask="prefix", weights="perturbed", seed=1236,
                        targets="uniform", k=64),
    "topk_logits": dict(dtype="bf16", B=4, Sm1=2048, H=2048, V=151936, payload="logits",
                        reduction=REDUCE_TOKEN_MEAN, mask="all", weights="perturbed", seed=1238,
                        targets="uniform", k=64),
    "qwen_hidden_stats": dict(dtype="bf16", B=4, Sm1=2048, H=2048, V=151936, payload="hidden",
                              reduction=REDUCE_TOKEN_MEAN, mask="prefix", weights="perturbed", seed=1236,
                              targets="uniform", stats=True),
    "multi_teacher": dict(dtype="bf16", B=4, Sm1=2048, H=2048, V=151936, payload="hidden_multi",
                          reduction=REDUCE_TOKEN_MEAN, mask="prefix", weights="perturbed", seed=1241,
                          mask_seed=1236, n_teachers=2, teacher_assign="sequence"),
}

TORCH_DTYPES = {"bf16": torch.bfloat16, "fp32": torch.float32}


def make_mask(kind, B, Sm1, seed):
    """uint8 mask [B, Sm1]; nonzero = trainable position."""
    rs = np.random.RandomState(seed)
    m = np.zeros((B, Sm1), dtype=np.uint8)
    if kind == "all":
        m[:] = 1
    elif kind == "none":
        pass
    elif kind == "prefix":
        # a random prompt prefix of 25-75% of each sequence is masked out
        for b in range(B):
            p = int(round(rs.uniform(0.25, 0.75) * Sm1))
            m[b, p:] = 1
    elif kind.startswith("suffix"):
        n = int(kind[len("suffix"):])
        m[:, max(0, Sm1 - n):] = 1
    elif kind == "random":
        m[:] = (rs.uniform(size=(B, Sm1)) < 0.5).astype(np.uint8)
    elif kind == "one":
        m[rs.randint(B), rs.randint(Sm1)] = 1
    else:
        raise ValueError(kind)
    return m


def _randn(shape, gen, device, scale=1.0, chunk_rows=8192):
    out = torch.empty(shape, dtype=torch.float32, device=device)
    rows = shape[0]
    for r0 in range(0, rows, chunk_rows):
        r1 = min(rows, r0 + chunk_rows)
        out[r0:r1] = torch.randn((r1 - r0,) + tuple(shape[1:]), generator=gen, device=device) * scale
    return out


def make_teacher_idx(assign, B, Sm1, n_teachers, seed):
    """int32 [B, Sm1] teacher index of every position: per sequence
    (b mod n_teachers) or drawn uniformly per position."""
    if assign == "sequence":
        idx = np.repeat((np.arange(B) % n_teachers)[:, None], Sm1, axis=1)
    elif assign == "random":
        idx = np.random.RandomState(seed + 7).randint(0, n_teachers, size=(B, Sm1))
    else:
        raise ValueError(assign)
    return torch.from_numpy(idx.astype(np.int32))


def make_inputs(B, Sm1, H, V, dtype="bf16", payload="hidden", mask="prefix",
                weights="perturbed", seed=0, device="cpu", mask_seed=None,
                logit_std=3.0, teacher_noise=0.004, n_teachers=1, teacher_assign="sequence", targets=None):
    """Draw one problem.  Returns a dict of torch tensors on `device`:
    h_s [T,H], W_s [V,H], mask uint8 [B,Sm1], and h_t [T,H] + W_t [V,H]
    (hidden payload) or teacher_logits [T,V] (logits payload).  The
    hidden_multi payload gives W_t [n_teachers, V, H] and teacher_idx
    [B, Sm1] int32 instead."""
    T = B * Sm1
    tdt = TORCH_DTYPES[dtype]
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    out = {}
    if payload == "logits_pair":
        zs = torch.empty((T, V), dtype=tdt, device=device)
        zt = torch.empty((T, V), dtype=tdt, device=device)
        shift = torch.rand((T, 1), generator=gen, device=device) * 40.0 - 20.0
        for r0 in range(0, T, 512):
            r1 = min(T, r0 + 512)
            a = torch.randn((r1 - r0, V), generator=gen, device=device) * logit_std
            zs[r0:r1] = a.to(tdt)
            b = a + torch.randn((r1 - r0, V), generator=gen, device=device) * 0.5 + shift[r0:r1]
            zt[r0:r1] = (b if weights != "same" else a).to(tdt)
        out["student_logits"], out["teacher_logits"] = zs, zt
        if targets == "sampled":
            # the sampled token of each position, drawn from the student's softmax
            y = torch.empty(T, dtype=torch.int64, device=device)
            for r0 in range(0, T, 512):
                r1 = min(T, r0 + 512)
                p = torch.softmax(zs[r0:r1].float(), dim=1)
                y[r0:r1] = torch.multinomial(p, 1, generator=gen).reshape(-1)
            out["targets"] = y.to(torch.int32).reshape(B, Sm1)
        out["mask"] = torch.from_numpy(make_mask(mask, B, Sm1, seed if mask_seed is None else mask_seed)).to(device)
        return out
    out["h_s"] = _randn((T, H), gen, device).to(tdt)
    w_scale = logit_std / math.sqrt(H)
    W_s32 = _randn((V, H), gen, device, scale=w_scale)
    out["W_s"] = W_s32.to(tdt)
    if payload == "hidden_multi":
        out["h_t"] = _randn((T, H), gen, device).to(tdt)
        W_t = torch.empty((n_teachers, V, H), dtype=tdt, device=device)
        for g in range(n_teachers):
            W_t[g] = (W_s32 + _randn((V, H), gen, device, scale=teacher_noise)).to(tdt)
        out["W_t"] = W_t
        out["teacher_idx"] = make_teacher_idx(teacher_assign, B, Sm1, n_teachers, seed).to(device)
        del W_s32
        out["mask"] = torch.from_numpy(make_mask(mask, B, Sm1, seed if mask_seed is None else mask_seed)).to(device)
        return out
    if payload == "hidden":
        if weights == "same":
            out["h_t"] = out["h_s"].clone()
            out["W_t"] = out["W_s"].clone()
        elif weights == "independent":
            out["h_t"] = _randn((T, H), gen, device).to(tdt)
            out["W_t"] = _randn((V, H), gen, device, scale=w_scale).to(tdt)
        elif weights == "perturbed":
            out["h_t"] = _randn((T, H), gen, device).to(tdt)
            W_s32 += _randn((V, H), gen, device, scale=teacher_noise)
            out["W_t"] = W_s32.to(tdt)
        elif weights == "uniform_teacher":
            out["h_t"] = _randn((T, H), gen, device).to(tdt)
            out["W_t"] = torch.zeros((V, H), dtype=tdt, device=device)
        else:
            raise ValueError(weights)
    elif payload == "logits":
        logits = torch.empty((T, V), dtype=tdt, device=device)
        shift = torch.rand((T, 1), generator=gen, device=device) * 40.0 - 20.0
        for r0 in range(0, T, 512):
            r1 = min(T, r0 + 512)
            blk = torch.randn((r1 - r0, V), generator=gen, device=device) * logit_std
            logits[r0:r1] = (blk + shift[r0:r1]).to(tdt)
        out["teacher_logits"] = logits
    else:
        raise ValueError(payload)
    del W_s32
    if targets == "uniform":
        y = np.random.RandomState(seed + 11).randint(0, V, size=(B, Sm1)).astype(np.int32)
        out["targets"] = torch.from_numpy(y).to(device)
    out["mask"] = torch.from_numpy(make_mask(mask, B, Sm1, seed if mask_seed is None else mask_seed)).to(device)
    return out


def make_workload(name, device="cpu", **overrides):
    """Inputs of a named workload (see module docstring)."""
    cfg = dict(WORKLOADS[name])
    cfg.update(overrides)
    red = cfg.pop("reduction")
    inp = make_inputs(cfg["B"], cfg["Sm1"], cfg["H"], cfg["V"], dtype=cfg["dtype"],
                      payload=cfg["payload"], mask=cfg["mask"], weights=cfg["weights"],
                      seed=cfg["seed"], device=device, mask_seed=cfg.get("mask_seed"),
                      n_teachers=cfg.get("n_teachers", 1), teacher_assign=cfg.get("teacher_assign", "sequence"),
                      targets=cfg.get("targets"))
    inp["reduction"] = red
    inp["cfg"] = cfg
    return inp
