"""Benchmark of the exact full-vocabulary reverse-KL loss, forward + backward.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl reference]

One step = S1 compaction + S2-S4 forward + S5-S7 backward (dH_s and dW_s) of
one batch through librkl.so, upstream gradient 1.0.  The default workload is
the Qwen3-1.7B-shaped hidden-state problem (B=4, S-1=2048, H=2048,
V=151936, bf16, ~4096 trainable rows).  The metric is trainable tokens per
second.  With torchrun (N > 1) each rank runs an independent replica of the
problem (no collective on the data path); the elapsed time is the max over
ranks.

Rank 0 prints one JSON line.  `--impl reference` times the float64 CPU
oracle (the reference arm) on a bounded sample of the same workload instead.
"""

from __future__ import annotations

import argparse
import ctypes
import hashlib
import json
import math
import os
import statistics
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from full_vocabulary_reverse_b200 import binding as rb  # noqa: E402
from full_vocabulary_reverse_b200.workloads import WORKLOADS, make_workload  # noqa: E402

METRIC = "tokens/s fused full-vocab reverse-KL fwd+bwd (H2048,V151936); % of TC peak"
UNIT = "tokens/s"
L2_BYTES = 126 * 2 ** 20
CPU_SAMPLE_ROWS = 192
# nominal dense B200 figures, printed beside the measured roofline
DATASHEET_BF16_TFLOPS = 2250.0
DATASHEET_HBM_GBS = 8000.0


# ----------------------------------------------------------------- helpers
def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return {"hbm_gbs": p["hbm_gbs"], "bf16_tflops": p["bf16_tflops"],
                "bf16_tflops_sustained": p.get("bf16_tflops_sustained", p["bf16_tflops"]),
                "sm_max_mhz": p.get("sm_max_mhz"), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "sm_max_mhz": 1965.0,
            "source": "fallback"}


class ClockSampler:
    """Samples SM clock and throttle reasons with NVML while the timed region runs."""

    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
               0x80: "hw_power_brake_slowdown"}

    def __init__(self, device_index):
        self.samples, self.reasons, self.ok = [], set(), False
        self.max_mhz = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            self.ok = False
        self._stop = threading.Event()

    def _run(self):
        while not self._stop.is_set():
            try:
                self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
                fn = getattr(self.nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                    self.nv.nvmlDeviceGetCurrentClocksThrottleReasons
                bits = fn(self.h)
                for b, name in self.REASONS.items():
                    if bits & b:
                        self.reasons.add(name)
            except Exception:
                pass
            self._stop.wait(0.05)

    def __enter__(self):
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *a):
        if self.ok:
            self._stop.set()
            self.t.join()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons), "samples": 0}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


PATHS = ("hidden", "stats", "topk_hidden", "multi", "logits", "topk_logits", "pair", "topk_pair")


def path_of(cfg):
    """The entry points a workload's step goes through, from its config:
    hidden (rkl_forward_hidden), stats (rkl_forward_hidden_ex with targets),
    topk_hidden, multi (a teacher per row), logits (shipped teacher logits),
    topk_logits, pair (both sides as logits) or topk_pair."""
    payload = cfg["payload"]
    if payload == "logits_pair":
        return "topk_pair" if cfg.get("k") is not None else "pair"
    if payload == "logits":
        return "topk_logits" if cfg.get("k") is not None else "logits"
    if payload == "hidden_multi":
        return "multi"
    if cfg.get("k") is not None:
        return "topk_hidden"
    return "stats" if cfg.get("stats") else "hidden"


class Problem:
    """One batch of a workload, resident on the device, driven through the C ABI."""

    def __init__(self, name, device, seed_offset=0, overrides=None):
        cfg = dict(WORKLOADS[name])
        self.name = name
        inp = make_workload(name, device=device, seed=cfg["seed"] + seed_offset, **(overrides or {}))
        self.cfg = inp.pop("cfg")
        self.reduction = inp.pop("reduction")
        self.inp = inp
        self.dev = device
        self.B, self.Sm1 = inp["mask"].shape
        self.T = self.B * self.Sm1
        path = path_of(self.cfg)
        self.pair = path in ("pair", "topk_pair")
        self.topk_logits = path == "topk_logits"
        self.logits = path in ("logits", "topk_logits")
        self.multi = path == "multi"
        self.n_teachers = inp["W_t"].shape[0] if self.multi else 1
        self.topk = path == "topk_pair"
        # per-token student entropy and target log-prob from the same forward
        self.stats = path == "stats"
        self.topk_hidden = path == "topk_hidden"
        self.k = int(self.cfg.get("k", 0)) if (self.topk or self.topk_hidden or self.topk_logits) else None
        self.student = inp["student_logits"] if self.pair else inp["h_s"]
        self.H = 0 if self.pair else inp["h_s"].shape[1]
        self.V = inp["student_logits"].shape[1] if self.pair else inp["W_s"].shape[0]
        self.payload = rb.PAYLOAD_LOGITS_PAIR if self.pair else (rb.PAYLOAD_LOGITS if self.logits else
                                                                 rb.PAYLOAD_HIDDEN)
        self.dt = rb._dtype_code(self.student)
        self.teacher = inp["teacher_logits"] if (self.logits or self.pair) else inp["h_t"]
        self.W_t = None if (self.logits or self.pair) else inp["W_t"]
        L = rb.lib()
        self.L = L
        self.row_idx = torch.empty(self.T, dtype=torch.int32, device=device)
        self.n_dev = torch.empty(1, dtype=torch.int32, device=device)
        self.n_host = torch.empty(1, dtype=torch.int32).pin_memory()
        if self.multi:
            nbytes = rb.workspace_size_multi(self.dt, self.T, self.n_teachers, self.B, self.Sm1, self.H, self.V)
            self.counts_dev = torch.empty(self.n_teachers + 1, dtype=torch.int32, device=device)
            self.counts_host = torch.empty(self.n_teachers + 1, dtype=torch.int32).pin_memory()
        elif self.topk_hidden:
            nbytes = rb.workspace_size(rb.PAYLOAD_TOPK_HIDDEN, self.dt, self.T, self.B, self.Sm1, self.H, self.V)
        elif self.topk_logits:
            nbytes = rb.workspace_size(rb.PAYLOAD_TOPK_LOGITS, self.dt, self.T, self.B, self.Sm1, self.H, self.V)
        else:
            nbytes = rb.workspace_size(self.payload, self.dt, self.T, self.B, self.Sm1, max(self.H, 64), self.V)
        self.ws = torch.empty(nbytes, dtype=torch.uint8, device=device)
        self.loss_tok = torch.empty((self.B, self.Sm1), dtype=torch.float32, device=device)
        self.loss = torch.empty(1, dtype=torch.float32, device=device)
        self.saved = torch.empty(7 * self.T, dtype=torch.float32, device=device)
        if self.stats:
            self.entropy = torch.empty((self.B, self.Sm1), dtype=torch.float32, device=device)
            self.target_logprob = torch.empty((self.B, self.Sm1), dtype=torch.float32, device=device)
        if self.pair:
            self.dz = torch.empty_like(self.student)
        else:
            self.dH = torch.empty((self.T, self.H), dtype=torch.float32, device=device)
            self.dW = torch.empty((self.V, self.H), dtype=torch.float32, device=device)
        self.grad_loss = torch.ones(1, dtype=torch.float32, device=device)
        self.N = None

    def _p(self, t):
        return None if t is None else ctypes.c_void_p(t.data_ptr())

    def trainable_rows(self):
        """N of the last step's batch (a host read of the device count; only
        outside the timed regions)."""
        torch.cuda.synchronize()
        return self.N if self.multi else int(self.n_dev.item())

    def inputs(self):
        """The per-batch input tensors (what a data loader would deliver each step)."""
        out = [self.student, self.teacher, self.inp["mask"]]
        if self.multi:
            out.append(self.inp["teacher_idx"])
        if self.topk or self.topk_hidden or self.topk_logits or self.stats:
            out.append(self.inp["targets"])
        return out

    def step(self, h_s=None, teacher=None, mask=None, extra=None):
        """S1..S7 for one batch.  Inputs default to the resident ones.  The
        trainable-row count stays on the device (the kernels read it), so the
        step is enqueued without any host synchronisation; the teacher-per-row
        path reads N and the per-teacher counts back to plan its row layout."""
        L, p = self.L, self._p
        h_s = self.student if h_s is None else h_s
        teacher = self.teacher if teacher is None else teacher
        mask = self.inp["mask"] if mask is None else mask
        s = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
        if self.multi:
            tid = self.inp["teacher_idx"] if extra is None else extra
            return self._step_multi(h_s, teacher, mask, tid, s)
        rb._check(L.rkl_compact_rows(p(mask), self.B, self.Sm1, p(self.row_idx), p(self.n_dev), s))
        N, nd = self.T, p(self.n_dev)  # bound and device count
        if self.topk:
            tg = self.inp["targets"] if extra is None else extra
            rb._check(L.rkl_forward_topk_pair(p(h_s), p(teacher), self.dt, self.B, self.Sm1, self.V, p(self.row_idx), N, nd,
                                              self.k, p(tg), self.reduction, p(self.loss_tok), p(self.loss),
                                              p(self.saved), p(self.ws), self.ws.numel(), s))
            rb._check(L.rkl_backward_topk_pair(p(h_s), p(teacher), self.dt, self.B, self.Sm1, self.V, p(self.row_idx),
                                               N, nd, p(tg), self.reduction, p(self.saved), p(self.grad_loss), None,
                                               p(self.dz), p(self.ws), self.ws.numel(), s))
            return None
        if self.pair:
            rb._check(L.rkl_forward_logits_pair(p(h_s), p(teacher), self.dt, self.B, self.Sm1, self.V,
                                                p(self.row_idx), N, nd, self.reduction, p(self.loss_tok), p(self.loss),
                                                p(self.saved), p(self.ws), self.ws.numel(), s))
            rb._check(L.rkl_backward_logits_pair(p(h_s), p(teacher), self.dt, self.B, self.Sm1, self.V,
                                                 p(self.row_idx), N, nd, self.reduction, p(self.saved),
                                                 p(self.grad_loss), None, p(self.dz), p(self.ws), self.ws.numel(), s))
            return None
        if self.topk_hidden:
            tg = self.inp["targets"] if extra is None else extra
            rb._check(L.rkl_forward_topk_hidden(p(h_s), p(teacher), p(self.inp["W_s"]), p(self.W_t), self.dt, self.B,
                                                self.Sm1, self.H, self.V, p(self.row_idx), N, nd, self.k, p(tg),
                                                self.reduction, p(self.loss_tok), p(self.loss), p(self.saved),
                                                p(self.ws), self.ws.numel(), s))
            rb._check(L.rkl_backward_topk_hidden(p(h_s), p(teacher), p(self.inp["W_s"]), p(self.W_t), self.dt,
                                                 self.B, self.Sm1, self.H, self.V, p(self.row_idx), N, nd, p(tg),
                                                 self.reduction, p(self.saved), p(self.grad_loss), None, p(self.dH),
                                                 p(self.dW), p(self.ws), self.ws.numel(), s))
            return None
        if self.topk_logits:
            tg = self.inp["targets"] if extra is None else extra
            rb._check(L.rkl_forward_topk_logits(p(h_s), p(self.inp["W_s"]), p(teacher), self.dt, self.B, self.Sm1,
                                                self.H, self.V, p(self.row_idx), N, nd, self.k, p(tg),
                                                self.reduction, p(self.loss_tok), p(self.loss), p(self.saved),
                                                p(self.ws), self.ws.numel(), s))
            rb._check(L.rkl_backward_topk_logits(p(h_s), p(self.inp["W_s"]), p(teacher), self.dt, self.B, self.Sm1,
                                                 self.H, self.V, p(self.row_idx), N, nd, p(tg), self.reduction,
                                                 p(self.saved), p(self.grad_loss), None, p(self.dH), p(self.dW),
                                                 p(self.ws), self.ws.numel(), s))
            return None
        if self.logits:
            rb._check(L.rkl_forward_logits(p(h_s), p(self.inp["W_s"]), p(teacher), self.dt, self.B, self.Sm1, self.H,
                                           self.V, p(self.row_idx), N, nd, self.reduction, p(self.loss_tok), p(self.loss),
                                           p(self.saved), p(self.ws), self.ws.numel(), s))
        elif self.stats:
            tg = self.inp["targets"] if extra is None else extra
            rb._check(L.rkl_forward_hidden_ex(p(h_s), p(teacher), p(self.inp["W_s"]), p(self.W_t), self.dt, self.B,
                                              self.Sm1, self.H, self.V, p(self.row_idx), N, nd, self.reduction,
                                              p(self.loss_tok), p(self.loss), p(self.saved), p(tg),
                                              p(self.entropy), p(self.target_logprob), p(self.ws),
                                              self.ws.numel(), s))
        else:
            rb._check(L.rkl_forward_hidden(p(h_s), p(teacher), p(self.inp["W_s"]), p(self.W_t), self.dt, self.B,
                                           self.Sm1, self.H, self.V, p(self.row_idx), N, nd, self.reduction,
                                           p(self.loss_tok), p(self.loss), p(self.saved), p(self.ws),
                                           self.ws.numel(), s))
        rb._check(L.rkl_backward(self.payload, p(h_s), p(teacher), p(self.inp["W_s"]), p(self.W_t), self.dt, self.B,
                                 self.Sm1, self.H, self.V, p(self.row_idx), N, nd, self.reduction, p(self.saved),
                                 p(self.grad_loss), None, p(self.dH), p(self.dW), p(self.ws), self.ws.numel(), s))
        return None

    def _step_multi(self, h_s, h_t, mask, tid, s):
        L, p = self.L, self._p
        nt = self.n_teachers
        rb._check(L.rkl_compact_rows_multi(p(mask), p(tid), self.B, self.Sm1, nt, p(self.row_idx), p(self.n_dev),
                                           p(self.counts_dev), s))
        self.n_host.copy_(self.n_dev, non_blocking=True)
        self.counts_host.copy_(self.counts_dev, non_blocking=True)
        torch.cuda.current_stream().synchronize()
        N = int(self.n_host[0])
        counts = (ctypes.c_int32 * nt)(*self.counts_host[:nt].tolist())
        rb._check(L.rkl_forward_hidden_multi(p(h_s), p(h_t), p(self.inp["W_s"]), p(self.W_t), nt, p(tid), counts,
                                             self.dt, self.B, self.Sm1, self.H, self.V, p(self.row_idx), N,
                                             self.reduction, p(self.loss_tok), p(self.loss), p(self.saved),
                                             p(self.ws), self.ws.numel(), s))
        rb._check(L.rkl_backward_hidden_multi(p(h_s), p(h_t), p(self.inp["W_s"]), p(self.W_t), nt, p(tid), counts,
                                              self.dt, self.B, self.Sm1, self.H, self.V, p(self.row_idx), N,
                                              self.reduction, p(self.saved), p(self.grad_loss), None, p(self.dH),
                                              p(self.dW), p(self.ws), self.ws.numel(), s))
        self.N = N
        return N


def reduce_over_ranks(ms, tokens, dist, device):
    """(max over ranks of the device-timed milliseconds, sum over ranks of the tokens)."""
    t = torch.tensor([float(ms)], dtype=torch.float64, device=device)
    n = torch.tensor([float(tokens)], dtype=torch.float64, device=device)
    if dist is not None:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        dist.all_reduce(n, op=dist.ReduceOp.SUM)
    return float(t[0]), float(n[0])


def kernel_profile():
    L = rb.lib()
    out = {}
    for i in range(L.rkl_kernel_count()):
        ms, n = ctypes.c_double(0), ctypes.c_int64(0)
        rb._check(L.rkl_profile_read(i, ctypes.byref(ms), ctypes.byref(n)))
        if n.value:
            out[L.rkl_kernel_name(i).decode()] = {"ms": ms.value, "launches": n.value}
    return out


def algorithmic_work(prob, N):
    """Per-kernel algorithmic flops (tensor kernels) or bytes (bandwidth kernels) of one step."""
    H, V = prob.H, prob.V
    if prob.dt != 0:
        # fp32 inputs: the FFMA (SIMT) kernels, bound by the FP32 pipe
        w = {"fwd_simt_fp32": ("alu", (2.0 if prob.logits else 4.0) * N * H * V),
             "dz_simt_fp32": ("alu", (2.0 if prob.logits else 4.0) * N * H * V),
             "grad_simt_fp32": ("alu", 4.0 * N * H * V)}
        if prob.logits:
            w["teacher_lse"] = ("hbm", 4.0 * N * V + 4.0 * N)
        return w
    if prob.topk:
        # the estimator must read both logit rows once and write dz once
        return {"topk_fwd": ("hbm", 4.0 * N * V + 28.0 * N),
                "topk_bwd": ("hbm", 4.0 * N * V + 2.0 * prob.T * V)}
    if prob.pair:
        return {"pair_fwd": ("hbm", 4.0 * N * V + 16.0 * N),
                "pair_bwd": ("hbm", 4.0 * N * V + 2.0 * prob.T * V)}
    if prob.topk_logits:
        # writer 2 N H V (z_s), selection / estimate over the written fp32 z_s
        # block beside the shipped bf16 teacher rows (4 N V + 2 N V bytes),
        # dz recompute 2 N H V (+ the teacher rows again), grad 4 N H V
        return {"zw_single_tc": ("tensor", 2.0 * N * H * V), "topk_fwd": ("hbm", 6.0 * N * V),
                "dz_topk_single_tc": ("tensor", 2.0 * N * H * V), "grad_dw_dh_tc": ("tensor", 4.0 * N * H * V)}
    if prob.topk_hidden:
        # writer 4 N H V (z_s and z_t), selection/estimate over the written fp32
        # logits (read 2 x 4 N V bytes once), dz recompute 4 N H V, grad 4 N H V
        return {"zw_dual_tc": ("tensor", 4.0 * N * H * V), "topk_fwd": ("hbm", 8.0 * N * V),
                "dz_topk_tc": ("tensor", 4.0 * N * H * V), "grad_dw_dh_tc": ("tensor", 4.0 * N * H * V)}
    if prob.logits:
        return {"fwd_single_tc": ("tensor", 2.0 * N * H * V), "dz_single_tc": ("tensor", 2.0 * N * H * V),
                "grad_dw_dh_tc": ("tensor", 4.0 * N * H * V), "teacher_lse": ("hbm", 2.0 * N * V + 4.0 * N)}
    return {"fwd_dual_tc": ("tensor", 4.0 * N * H * V), "dz_dual_tc": ("tensor", 4.0 * N * H * V),
            "grad_dw_dh_tc": ("tensor", 4.0 * N * H * V)}


# the sources each kernel family is built from: a family's stored DRAM traffic
# stays valid while these files are unchanged
SOURCE_GROUPS = {
    "tc": ("tc_kernels.cu", "sm100.cuh", "kernels.h", "api.cu"),
    "small": ("small_kernels.cu", "kernels.h", "api.cu"),
    "topk": ("topk_kernels.cu", "sm100.cuh", "kernels.h", "api.cu"),
}


def kernel_group(kernel):
    if kernel.startswith("topk_"):
        return "topk"
    return "tc" if kernel.endswith("_tc") else "small"


def source_sha(group):
    h = hashlib.sha256()
    for f in SOURCE_GROUPS[group]:
        with open(os.path.join(ROOT, "full_vocabulary_reverse_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def traffic_for(kernel, workload):
    """DRAM bytes per launch of `kernel` on `workload` from the committed ncu
    summary, or None if there is none or the kernel's sources changed since."""
    path = os.path.join(ROOT, "profiles", "dram_traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        d = json.load(f)
    group = kernel_group(kernel)
    if d.get("source_sha", {}).get(group) != source_sha(group):
        return None
    k = d.get("kernels", {}).get("%s@%s" % (kernel, workload))
    return None if k is None else k.get("dram_bytes_per_launch")


# ----------------------------------------------------------------- arms
def cpu_oracle_sample(inp, reduction, name, rows=CPU_SAMPLE_ROWS, k=None):
    """Time the float64 oracle (as it stands) on the first `rows` trainable
    rows, with the BLAS thread pools set to the host cores this process may
    run on."""
    from threadpoolctl import threadpool_info, threadpool_limits
    from oracle import rkl_oracle as O

    cores = len(os.sched_getaffinity(0))
    with threadpool_limits(limits=cores):
        out = _cpu_oracle_sample(O, inp, reduction, name, rows, k)
        blas = max([d.get("num_threads", 1) for d in threadpool_info()] or [1])
    out["cores"] = cores
    out["blas_threads"] = blas
    return out


def _cpu_oracle_sample(O, inp, reduction, name, rows, k):
    mask = inp["mask"].cpu().numpy()
    flat = np.flatnonzero(mask.reshape(-1))[:rows]
    sub = np.zeros(mask.size, np.uint8)
    sub[flat] = 1
    sub = sub.reshape(mask.shape)
    f64 = lambda t: None if t is None else t.float().cpu().numpy()  # noqa: E731
    path = path_of(WORKLOADS[name])
    if path in ("pair", "topk_pair"):
        zs, zt = f64(inp["student_logits"]), f64(inp["teacher_logits"])
        t0 = time.perf_counter()
        if path == "topk_pair":
            y = inp["targets"].cpu().numpy()
            O.forward_topk_pair(zs, zt, y, k, sub, reduction)
            O.backward_topk_pair(zs, zt, y, k, sub, reduction)
        else:
            O.forward_logits_pair(zs, zt, sub, reduction)
            O.backward_logits_pair(zs, zt, sub, reduction)
        dt = time.perf_counter() - t0
    else:
        h_s, W_s = f64(inp["h_s"]), f64(inp["W_s"])
        if path in ("logits", "topk_logits"):
            teacher, W_t = f64(inp["teacher_logits"]), None
        else:
            teacher, W_t = f64(inp["h_t"]), f64(inp["W_t"])
        t0 = time.perf_counter()
        if path == "topk_logits":
            y = inp["targets"].cpu().numpy()
            O.forward_topk_logits(h_s, W_s, teacher, y, k, sub, reduction)
            O.backward_topk_logits(h_s, W_s, teacher, y, k, sub, reduction)
        elif path == "multi":
            tid = inp["teacher_idx"].cpu().numpy()
            O.forward_multi(h_s, W_s, teacher, W_t, tid, sub, reduction)
            O.backward_multi(h_s, W_s, teacher, W_t, tid, sub, reduction)
        elif path == "topk_hidden":
            y = inp["targets"].cpu().numpy()
            O.forward_topk_hidden(h_s, W_s, teacher, W_t, y, k, sub, reduction)
            O.backward_topk_hidden(h_s, W_s, teacher, W_t, y, k, sub, reduction)
        elif path == "stats":  # the loss plus the student's per-token statistics
            O.forward(h_s, W_s, teacher, W_t, sub, reduction)
            O.student_stats(h_s, W_s, sub, targets=inp["targets"].cpu().numpy())
            O.backward(h_s, W_s, teacher, W_t, sub, reduction)
        else:
            O.forward(h_s, W_s, teacher, W_t, sub, reduction)
            O.backward(h_s, W_s, teacher, W_t, sub, reduction)
        dt = time.perf_counter() - t0
    return {"value": len(flat) / dt, "unit": UNIT, "kind": "oracle",
            "sample": "%d trainable rows of the %s workload (float64 NumPy forward+backward incl. weight upcast), "
                      "%.1f s" % (len(flat), name, dt),
            "seconds": dt, "rows": int(len(flat))}


def run_reference(args, rank, world):
    """Reference arm: the CPU oracle timed on bounded samples of the same workload."""
    if rank != 0:
        return
    inp = make_workload(args.workload, device="cpu", **shape_overrides(args))
    cfg = inp.pop("cfg")
    red = inp.pop("reduction")
    vals = []
    for i in range(args.warmup + args.steps):
        r = cpu_oracle_sample(inp, red, args.workload, rows=args.ref_rows, k=cfg.get("k"))
        if i >= args.warmup:
            vals.append(r)
    v = statistics.median([x["value"] for x in vals])
    secs = sum(x["seconds"] for x in vals)
    B, Sm1 = inp["mask"].shape
    out = {"impl": "reference", "metric": METRIC, "value": v, "unit": UNIT, "n_gpus": world, "steps": len(vals),
           "warmup": args.warmup, "ms_per_step": 1000.0 * secs / max(1, len(vals)), "higher_is_better": True,
           "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
           "config": {"workload": args.workload, "B": B, "Sm1": Sm1,
                      "H": inp["h_s"].shape[1] if "h_s" in inp else 0,
                      "V": inp["W_s"].shape[0] if "W_s" in inp else inp["student_logits"].shape[1],
                      "sample_rows": vals[-1]["rows"]},
           "cpu_baseline": {"value": v, "unit": UNIT, "cores": vals[-1]["cores"],
                            "blas_threads": vals[-1]["blas_threads"], "kind": "oracle",
                            "sample": vals[-1]["sample"]},
           "e2e": {"value": v, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(out), flush=True)


def run_gpu(args, rank, world, dist):
    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", 0)))
    torch.cuda.set_device(dev)
    prob = Problem(args.workload, dev, seed_offset=rank, overrides=shape_overrides(args))
    L = rb.lib()
    stream = torch.cuda.current_stream()

    def barrier():
        if dist is not None:
            dist.barrier()

    for _ in range(args.warmup):
        prob.step()
    N = prob.trainable_rows()

    # ---- device-timed region: inputs resident in HBM, no per-launch
    # instrumentation (the headline value)
    rb._check(L.rkl_profile_enable(0))
    launches0 = L.rkl_launch_count()
    barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(dev.index) as clk:
        e0.record(stream)
        for _ in range(args.steps):
            prob.step()
        e1.record(stream)
        torch.cuda.synchronize()
    barrier()
    launches = L.rkl_launch_count() - launches0
    ms = e0.elapsed_time(e1)
    ms_max, n_tot = reduce_over_ranks(ms, N * args.steps, dist, dev)
    value = n_tot / (ms_max / 1000.0)

    # ---- per-kernel split: the same steps again with a CUDA event pair
    # around every launch of the library (on the launching stream)
    rb._check(L.rkl_profile_reset())
    rb._check(L.rkl_profile_enable(1))
    barrier()
    torch.cuda.synchronize()
    p0, p1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    p0.record(stream)
    for _ in range(args.steps):
        prob.step()
    p1.record(stream)
    torch.cuda.synchronize()
    barrier()
    rb._check(L.rkl_profile_enable(0))
    prof = kernel_profile()
    ms_prof = p0.elapsed_time(p1)

    # ---- end to end through the C ABI with host buffers.  Every step's inputs
    # (hidden rows, teacher payload, mask) are copied from pinned host memory
    # and the loss is read back; the copy of step i+1's inputs runs on a side
    # stream while step i computes (two device buffers), as a training loop
    # with a prefetching data loader would do.  All copies are inside the
    # timed region.
    pins = [t.cpu().pin_memory() for t in prob.inputs()]
    loss_host = torch.empty(1, dtype=torch.float32).pin_memory()
    loss_tok_host = torch.empty(prob.loss_tok.shape, dtype=torch.float32).pin_memory()
    bufs = [[torch.empty_like(t) for t in prob.inputs()] for _ in range(2)]
    copy_stream = torch.cuda.Stream(dev)
    ready = [torch.cuda.Event(), torch.cuda.Event()]
    consumed = [torch.cuda.Event(), torch.cuda.Event()]

    def issue_copy(i):
        b = bufs[i % 2]
        with torch.cuda.stream(copy_stream):
            copy_stream.wait_event(consumed[i % 2])
            for dst, src in zip(b, pins):
                dst.copy_(src, non_blocking=True)
            ready[i % 2].record(copy_stream)

    def e2e_run(n):
        for e in consumed:
            e.record(stream)
        issue_copy(0)
        for i in range(n):
            if i + 1 < n:
                issue_copy(i + 1)
            stream.wait_event(ready[i % 2])
            prob.step(*bufs[i % 2])
            consumed[i % 2].record(stream)
            loss_host.copy_(prob.loss, non_blocking=True)
            loss_tok_host.copy_(prob.loss_tok, non_blocking=True)

    e2e_run(2)
    torch.cuda.synchronize()
    barrier()
    f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    f0.record(stream)
    e2e_run(args.steps)
    f1.record(stream)
    torch.cuda.synchronize()
    ms_e2e, _ = reduce_over_ranks(f0.elapsed_time(f1), 0, dist, dev)
    e2e_value = n_tot / (ms_e2e / 1000.0)
    h2d = sum(t.numel() * t.element_size() for t in pins)
    # loss scalar + per-token losses [B, S-1], plus N and the per-teacher row
    # counts in the teacher-per-row mode (read back to plan its row layout;
    # the other paths keep N on the device).  The gradients stay on the
    # device, where the optimizer step would consume them.
    d2h = 4 + 4 * prob.T + (4 * (prob.n_teachers + 2) if prob.multi else 0)

    if rank != 0:
        return
    pk = peaks()
    work = algorithmic_work(prob, N)
    # dominant kernel = the one with the largest share of device time
    dom = max((k for k in prof if k in work), key=lambda k: prof[k]["ms"])
    bound, per_step = work[dom]
    per_launch = per_step * args.steps / prof[dom]["launches"]
    avg_launch_s = prof[dom]["ms"] / prof[dom]["launches"] / 1000.0
    if bound == "tensor":
        achieved = per_launch / avg_launch_s / 1e12
        # the timed region is well under a second: the burst GEMM rate is the
        # roofline (the sustained one is for seconds-long runs)
        peak = pk["bf16_tflops"]
        unit = "TFLOP/s"
    elif bound == "alu":
        # FP32 FMA pipe: 148 SMs x 128 lanes x 2 flop per cycle at the max SM clock
        achieved = per_launch / avg_launch_s / 1e12
        peak = 148 * 128 * 2 * (pk.get("sm_max_mhz") or 1965.0) * 1e6 / 1e12
        unit = "TFLOP/s"
    else:
        achieved = per_launch / avg_launch_s / 1e9
        peak = pk["hbm_gbs"]
        unit = "GB/s"
    extra, extra_tc = {}, {}
    for k, (b, w) in work.items():
        if k not in prof:
            continue
        per_l = w * args.steps / prof[k]["launches"]
        avg_s = prof[k]["ms"] / prof[k]["launches"] / 1000.0
        if b == "hbm":
            ach = per_l / avg_s / 1e9
            extra[k] = {"bound": "hbm", "achieved": ach, "peak": pk["hbm_gbs"], "unit": "GB/s",
                        "frac": ach / pk["hbm_gbs"], "traffic": traffic_for(k, prob.name)}
        elif b == "tensor":
            # every tensor-core kernel of the step against the same burst peak
            ach = per_l / avg_s / 1e12
            extra_tc[k] = {"bound": "tensor", "achieved": ach, "peak": pk["bf16_tflops"], "unit": "TFLOP/s",
                           "frac": ach / pk["bf16_tflops"], "traffic": traffic_for(k, prob.name)}
    step_flops = sum(w for b, w in work.values() if b in ("tensor", "alu"))
    step_tflops = step_flops * args.steps / (ms / 1000.0) / 1e12
    csum = clk.summary()
    clock_ratio = (csum["sm_mhz"] / csum["sm_max_mhz"]) if (csum.get("sm_mhz") and csum.get("sm_max_mhz")) else None
    step_bytes = sum(w for b, w in work.values() if b == "hbm")
    total_ms = sum(v["ms"] for v in prof.values())
    out = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_max / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16" if prob.dt == 0 else "fp32", "data": "synthetic",
        "config": {"workload": args.workload, "B": prob.B, "Sm1": prob.Sm1, "H": prob.H, "V": prob.V,
                   "trainable_rows": N, "tokens_T": prob.T,
                   "payload": ("logits_pair, top-k estimator k=%d" % prob.k if prob.topk else "logits_pair")
                   if prob.pair else ("hidden, top-k estimator k=%d" % prob.k if prob.topk_hidden else
                                      "hidden, with student entropy and target log-prob" if prob.stats else
                                      "logits, top-k estimator k=%d" % prob.k if prob.topk_logits else
                                      "logits" if prob.logits else
                                                                 ("hidden, %d teachers" % prob.n_teachers
                                                                  if prob.multi else "hidden")),
                   "parallelism": "replicas" if world > 1 else "single",
                   "l2": "inputs larger than L2 (%.2f GB streamed per pass > 126 MB); no flush" % (
                       (2 * prob.T * prob.V * 2 if prob.pair else
                        ((1 + prob.n_teachers) if not prob.logits else 1) * prob.V * prob.H * 2)
                       / 1e9)},
        "roofline": {"kernel": dom, "bound": bound, "achieved": achieved, "peak": peak, "unit": unit,
                     "frac": achieved / peak, "traffic": traffic_for(dom, prob.name),
                     "peak_source": "%s %s" % (pk["source"], {"tensor": "bf16 burst", "hbm": "hbm copy"}.get(
                         bound, "fp32 FMA pipe at the max SM clock")),
                     "frac_of_sustained": achieved / pk["bf16_tflops_sustained"] if bound == "tensor" else None,
                     "frac_of_datasheet": (achieved / (DATASHEET_BF16_TFLOPS if bound == "tensor"
                                                       else DATASHEET_HBM_GBS)) if bound != "alu" else None,
                     "sm_clock_ratio": clock_ratio,
                     "split_pass_ms_per_step": ms_prof / args.steps},
        "roofline_hbm_kernels": extra or None,
        "roofline_tc_kernels": extra_tc or None,
        "step_tflops": step_tflops, "step_tc_frac_burst": step_tflops / pk["bf16_tflops"],
        "step_tc_frac_sustained": step_tflops / pk["bf16_tflops_sustained"],
        "step_tc_frac_datasheet": step_tflops / DATASHEET_BF16_TFLOPS,
        "step_hbm_gbs": step_bytes * args.steps / (ms / 1000.0) / 1e9,
        "tokens_T_per_s": value * prob.T / N,
        "kernels": {k: {"ms_per_step": v["ms"] / args.steps, "launches_per_step": v["launches"] / args.steps,
                        "share": v["ms"] / total_ms} for k, v in sorted(prof.items(), key=lambda x: -x[1]["ms"])},
        "clocks": csum,
        "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "read_back": "loss, loss_tok [B, S-1]%s; gradients stay on the device for the optimizer" % (
                    ", N and per-teacher counts" if prob.multi else "")},
        "gpu_launches": int(launches),
    }
    if world == 1 and not args.no_cpu_baseline:
        inp = dict(prob.inp)
        out["cpu_baseline"] = {k: v for k, v in cpu_oracle_sample(inp, prob.reduction, prob.name, k=prob.k).items()
                               if k not in ("seconds", "rows")}
    print(json.dumps(out), flush=True)


def shape_overrides(args):
    """Smaller shapes of the same workload (profiling captures use these)."""
    return {k: getattr(args, k) for k in ("B", "Sm1", "H", "V") if getattr(args, k) is not None}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--B", type=int, default=None)
    ap.add_argument("--Sm1", type=int, default=None)
    ap.add_argument("--H", type=int, default=None)
    ap.add_argument("--V", type=int, default=None)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default="qwen_hidden", choices=sorted(WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--ref-rows", type=int, default=32)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if args.impl == "reference":
        # each reference step is a bounded CPU sample (~5 s); keep the whole run to minutes
        args.steps = max(1, min(args.steps, 10))
        args.warmup = min(args.warmup, 1)
        return run_reference(args, rank, world)
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as tdist
        torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", 0)))
        tdist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
        dist = tdist
    try:
        run_gpu(args, rank, world, dist)
    finally:
        if dist is not None:
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
