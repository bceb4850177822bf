"""ctypes binding of librkl.so (argument marshalling only).

Every step of the loss runs in the CUDA library; this module allocates the
caller-side tensors with PyTorch, passes raw device pointers and the current
stream, and raises ``RKLError`` on any non-OK status.  There is no fallback:
if ``librkl.so`` is missing or fails to load, every call raises.
"""

from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
# RKL_LIBRARY=debug selects the RKL_DEBUG build (device bounds checks)
LIB_PATH = os.path.join(_HERE, "librkl_debug.so" if os.environ.get("RKL_LIBRARY") == "debug" else "librkl.so")

REDUCE_NONE = 0
REDUCE_TOKEN_MEAN = 1
REDUCE_SEQ_MEAN_NESTED = 2
PAYLOAD_HIDDEN = 0
PAYLOAD_LOGITS = 1
PAYLOAD_LOGITS_PAIR = 2
DT_BF16 = 0
DT_FP32 = 1

_STATUS = {0: "RKL_OK", 1: "RKL_ERR_NULL", 2: "RKL_ERR_SHAPE", 3: "RKL_ERR_DTYPE",
           4: "RKL_ERR_ALIGN", 5: "RKL_ERR_WORKSPACE", 6: "RKL_ERR_UNSUPPORTED",
           7: "RKL_ERR_CUDA", 8: "RKL_ERR_DEVICE"}


class RKLError(RuntimeError):
    def __init__(self, status, msg):
        super().__init__("%s: %s" % (_STATUS.get(status, status), msg))
        self.status = status


_lib = None

_vp = ctypes.c_void_p
_i64 = ctypes.c_int64
_i32 = ctypes.c_int32
_sz = ctypes.c_size_t

_SIGS = {
    "rkl_version": ([], ctypes.c_char_p),
    "rkl_last_error": ([], ctypes.c_char_p),
    "rkl_workspace_size": ([_i32, _i32, _i64, _i64, _i64, _i64, _i64, ctypes.POINTER(_sz)], _i32),
    "rkl_compact_rows": ([_vp, _i64, _i64, _vp, _vp, _vp], _i32),
    "rkl_forward_hidden": ([_vp, _vp, _vp, _vp, _i32, _i64, _i64, _i64, _i64, _vp, _i32, _vp, _i32,
                            _vp, _vp, _vp, _vp, _sz, _vp], _i32),
    "rkl_forward_logits": ([_vp, _vp, _vp, _i32, _i64, _i64, _i64, _i64, _vp, _i32, _vp, _i32,
                            _vp, _vp, _vp, _vp, _sz, _vp], _i32),
    "rkl_backward": ([_i32, _vp, _vp, _vp, _vp, _i32, _i64, _i64, _i64, _i64, _vp, _i32, _vp, _i32,
                      _vp, _vp, _vp, _vp, _vp, _vp, _sz, _vp], _i32),
    "rkl_forward_hidden_ex": ([_vp, _vp, _vp, _vp, _i32, _i64, _i64, _i64, _i64, _vp, _i32, _vp, _i32,
                               _vp, _vp, _vp, _vp, _vp, _vp, _vp, _sz, _vp], _i32),
    "rkl_forward_logits_ex": ([_vp, _vp, _vp, _i32, _i64, _i64, _i64, _i64, _vp, _i32, _vp, _i32,
                               _vp, _vp, _vp, _vp, _vp, _vp, _vp, _sz, _vp], _i32),
    "rkl_forward_logits_pair": ([_vp, _vp, _i32, _i64, _i64, _i64, _vp, _i32, _vp, _i32, _vp, _vp, _vp, _vp, _sz,
                                 _vp], _i32),
    "rkl_backward_logits_pair": ([_vp, _vp, _i32, _i64, _i64, _i64, _vp, _i32, _vp, _i32, _vp, _vp, _vp, _vp, _vp,
                                  _sz, _vp], _i32),
    "rkl_forward_hidden_noalloc": ([_vp, _vp, _vp, _vp, _i32, _i64, _i64, _i64, _i64, _vp, _i32, _i32,
                                    _vp, _vp, _vp, _vp], _i32),
    "rkl_compact_rows_multi": ([_vp, _vp, _i64, _i64, _i32, _vp, _vp, _vp, _vp], _i32),
    "rkl_workspace_size_multi": ([_i32, _i64, _i32, _i64, _i64, _i64, _i64, ctypes.POINTER(_sz)], _i32),
    "rkl_forward_hidden_multi": ([_vp, _vp, _vp, _vp, _i32, _vp, _vp, _i32, _i64, _i64, _i64, _i64, _vp, _i32, _i32,
                                  _vp, _vp, _vp, _vp, _sz, _vp], _i32),
    "rkl_backward_hidden_multi": ([_vp, _vp, _vp, _vp, _i32, _vp, _vp, _i32, _i64, _i64, _i64, _i64, _vp, _i32, _i32,
                                   _vp, _vp, _vp, _vp, _vp, _vp, _sz, _vp], _i32),
    "rkl_forward_topk_pair": ([_vp, _vp, _i32, _i64, _i64, _i64, _vp, _i32, _vp, _i64, _vp, _i32, _vp, _vp, _vp, _vp,
                               _sz, _vp], _i32),
    "rkl_backward_topk_pair": ([_vp, _vp, _i32, _i64, _i64, _i64, _vp, _i32, _vp, _vp, _i32, _vp, _vp, _vp, _vp, _vp,
                                _sz, _vp], _i32),
    "rkl_forward_topk_hidden": ([_vp, _vp, _vp, _vp, _i32, _i64, _i64, _i64, _i64, _vp, _i32, _vp, _i64, _vp, _i32,
                                 _vp, _vp, _vp, _vp, _sz, _vp], _i32),
    "rkl_backward_topk_hidden": ([_vp, _vp, _vp, _vp, _i32, _i64, _i64, _i64, _i64, _vp, _i32, _vp, _vp, _i32, _vp,
                                  _vp, _vp, _vp, _vp, _vp, _sz, _vp], _i32),
    "rkl_forward_topk_logits": ([_vp, _vp, _vp, _i32, _i64, _i64, _i64, _i64, _vp, _i32, _vp, _i64, _vp, _i32,
                                 _vp, _vp, _vp, _vp, _sz, _vp], _i32),
    "rkl_backward_topk_logits": ([_vp, _vp, _vp, _i32, _i64, _i64, _i64, _i64, _vp, _i32, _vp, _vp, _i32, _vp,
                                  _vp, _vp, _vp, _vp, _vp, _sz, _vp], _i32),
    "rkl_device_error": ([ctypes.POINTER(_i32)], _i32),
    "rkl_kernel_count": ([], _i32),
    "rkl_kernel_name": ([_i32], ctypes.c_char_p),
    "rkl_profile_enable": ([_i32], _i32),
    "rkl_profile_reset": ([], _i32),
    "rkl_profile_read": ([_i32, ctypes.POINTER(ctypes.c_double), ctypes.POINTER(_i64)], _i32),
    "rkl_launch_count": ([], _i64),
}


def lib():
    """The loaded librkl.so (raises if it was not built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RKLError(7, "%s is not built (python -m full_vocabulary_reverse_b200.build)" %
                           os.path.basename(LIB_PATH))
        L = ctypes.CDLL(LIB_PATH)
        for name, (args, res) in _SIGS.items():
            fn = getattr(L, name)
            fn.argtypes = args
            fn.restype = res
        _lib = L
    return _lib


def _check(status):
    if status != 0:
        raise RKLError(status, lib().rkl_last_error().decode())


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(device):
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _dtype_code(t):
    if t.dtype == torch.bfloat16:
        return DT_BF16
    if t.dtype == torch.float32:
        return DT_FP32
    raise RKLError(3, "unsupported dtype %s" % (t.dtype,))


def workspace_size(payload, dtype_code, n_max, B, Sm1, H, V):
    out = ctypes.c_size_t(0)
    _check(lib().rkl_workspace_size(payload, dtype_code, n_max, B, Sm1, H, V, ctypes.byref(out)))
    return out.value


def _workspace(payload, dtype_code, n_max, B, Sm1, H, V, device):
    nbytes = workspace_size(payload, dtype_code, n_max, B, Sm1, H, V)
    return torch.empty(max(nbytes, 256), dtype=torch.uint8, device=device)


def compact_rows(mask, on_device=False):
    """S1: (row_idx int32 [B*Sm1] device, N).  N is a host int (read back
    with one synchronising copy), or with on_device=True the 1-element int32
    device tensor the kernels read themselves (no host synchronisation).
    Every entry point below takes either form of N."""
    B, Sm1 = mask.shape
    mask = mask.contiguous()
    if mask.dtype != torch.uint8:
        mask = (mask != 0).to(torch.uint8)
    row_idx = torch.empty(B * Sm1, dtype=torch.int32, device=mask.device)
    n_dev = torch.empty(1, dtype=torch.int32, device=mask.device)
    _check(lib().rkl_compact_rows(_ptr(mask), B, Sm1, _ptr(row_idx), _ptr(n_dev), _stream(mask.device)))
    if on_device:
        return row_idx, n_dev
    return row_idx, int(n_dev.item())


def _count(N, B, Sm1):
    """(N argument, n_dev pointer) of a C call: a host count is exact; a
    device count passes the capacity B*Sm1 as the bound."""
    if isinstance(N, torch.Tensor):
        if N.dtype != torch.int32 or N.numel() != 1 or not N.is_cuda:
            raise RKLError(2, "a device row count must be a 1-element int32 CUDA tensor")
        return B * Sm1, _ptr(N)
    return int(N), None


def forward_hidden(h_s, h_t, W_s, W_t, B, Sm1, row_idx, N, reduction, workspace=None):
    """S2-S4 on the hidden payload.  Returns (loss_tok [B,Sm1], loss [1], saved [N,3])."""
    Nc, nd = _count(N, B, Sm1)
    dev = h_s.device
    T, H = h_s.shape
    V = W_s.shape[0]
    dt = _dtype_code(h_s)
    loss_tok = torch.empty((B, Sm1), dtype=torch.float32, device=dev)
    loss = torch.empty(1, dtype=torch.float32, device=dev)
    saved = torch.empty((max(Nc, 1), 3), dtype=torch.float32, device=dev)
    ws = workspace if workspace is not None else _workspace(PAYLOAD_HIDDEN, dt, max(Nc, 1), B, Sm1, H, V, dev)
    _check(lib().rkl_forward_hidden(_ptr(h_s), _ptr(h_t), _ptr(W_s), _ptr(W_t), dt, B, Sm1, H, V,
                                    _ptr(row_idx), Nc, nd, reduction, _ptr(loss_tok), _ptr(loss), _ptr(saved),
                                    _ptr(ws), ws.numel(), _stream(dev)))
    return loss_tok, loss, saved


def forward_with_stats(h_s, teacher, W_s, W_t, B, Sm1, row_idx, N, reduction, targets=None, workspace=None):
    """Forward of the hidden payload (W_t given) or the logits payload (W_t None)
    plus the student's per-token entropy and target log-prob.
    Returns (loss_tok, loss, saved, entropy [B,Sm1], target_logprob [B,Sm1] or None)."""
    Nc, nd = _count(N, B, Sm1)
    dev = h_s.device
    T, H = h_s.shape
    V = W_s.shape[0]
    dt = _dtype_code(h_s)
    payload = PAYLOAD_HIDDEN if W_t is not None else PAYLOAD_LOGITS
    loss_tok = torch.empty((B, Sm1), dtype=torch.float32, device=dev)
    loss = torch.empty(1, dtype=torch.float32, device=dev)
    saved = torch.empty((max(Nc, 1), 3), dtype=torch.float32, device=dev)
    ent = torch.empty((B, Sm1), dtype=torch.float32, device=dev)
    tlp = torch.empty((B, Sm1), dtype=torch.float32, device=dev) if targets is not None else None
    if targets is not None:
        targets = targets.to(device=dev, dtype=torch.int32).contiguous()
    ws = workspace if workspace is not None else _workspace(payload, dt, max(Nc, 1), B, Sm1, H, V, dev)
    if payload == PAYLOAD_HIDDEN:
        st = lib().rkl_forward_hidden_ex(_ptr(h_s), _ptr(teacher), _ptr(W_s), _ptr(W_t), dt, B, Sm1, H, V,
                                         _ptr(row_idx), Nc, nd, reduction, _ptr(loss_tok), _ptr(loss), _ptr(saved),
                                         _ptr(targets), _ptr(ent), _ptr(tlp), _ptr(ws), ws.numel(), _stream(dev))
    else:
        st = lib().rkl_forward_logits_ex(_ptr(h_s), _ptr(W_s), _ptr(teacher), dt, B, Sm1, H, V, _ptr(row_idx), Nc, nd,
                                         reduction, _ptr(loss_tok), _ptr(loss), _ptr(saved), _ptr(targets),
                                         _ptr(ent), _ptr(tlp), _ptr(ws), ws.numel(), _stream(dev))
    _check(st)
    return loss_tok, loss, saved, ent, tlp


def forward_logits(h_s, W_s, teacher_logits, B, Sm1, row_idx, N, reduction, workspace=None):
    """S2-S4 + S8 on the logits payload.  Returns (loss_tok, loss, saved)."""
    Nc, nd = _count(N, B, Sm1)
    dev = h_s.device
    T, H = h_s.shape
    V = W_s.shape[0]
    dt = _dtype_code(h_s)
    loss_tok = torch.empty((B, Sm1), dtype=torch.float32, device=dev)
    loss = torch.empty(1, dtype=torch.float32, device=dev)
    saved = torch.empty((max(Nc, 1), 3), dtype=torch.float32, device=dev)
    ws = workspace if workspace is not None else _workspace(PAYLOAD_LOGITS, dt, max(Nc, 1), B, Sm1, H, V, dev)
    _check(lib().rkl_forward_logits(_ptr(h_s), _ptr(W_s), _ptr(teacher_logits), dt, B, Sm1, H, V,
                                    _ptr(row_idx), Nc, nd, reduction, _ptr(loss_tok), _ptr(loss), _ptr(saved),
                                    _ptr(ws), ws.numel(), _stream(dev)))
    return loss_tok, loss, saved


def backward(payload, h_s, teacher, W_s, W_t, B, Sm1, row_idx, N, reduction, saved,
             grad_loss=None, grad_tok=None, workspace=None, dH_s=None, dW_s=None):
    """S5-S7.  Returns (dH_s [T,H] fp32, dW_s [V,H] fp32)."""
    Nc, nd = _count(N, B, Sm1)
    dev = h_s.device
    T, H = h_s.shape
    V = W_s.shape[0]
    dt = _dtype_code(h_s)
    if dH_s is None:
        dH_s = torch.empty((T, H), dtype=torch.float32, device=dev)
    if dW_s is None:
        dW_s = torch.empty((V, H), dtype=torch.float32, device=dev)
    if grad_loss is not None:
        grad_loss = grad_loss.reshape(1).to(device=dev, dtype=torch.float32).contiguous()
    if grad_tok is not None:
        grad_tok = grad_tok.to(device=dev, dtype=torch.float32).contiguous()
    ws = workspace if workspace is not None else _workspace(payload, dt, max(Nc, 1), B, Sm1, H, V, dev)
    _check(lib().rkl_backward(payload, _ptr(h_s), _ptr(teacher), _ptr(W_s), _ptr(W_t), dt, B, Sm1, H, V,
                              _ptr(row_idx), Nc, nd, reduction, _ptr(saved), _ptr(grad_loss), _ptr(grad_tok),
                              _ptr(dH_s), _ptr(dW_s), _ptr(ws), ws.numel(), _stream(dev)))
    return dH_s, dW_s


def forward_logits_pair(student_logits, teacher_logits, B, Sm1, row_idx, N, reduction, workspace=None):
    """Both sides as logits.  Returns (loss_tok [B,Sm1], loss [1], saved [N,3])."""
    Nc, nd = _count(N, B, Sm1)
    dev = student_logits.device
    V = student_logits.shape[1]
    dt = _dtype_code(student_logits)
    loss_tok = torch.empty((B, Sm1), dtype=torch.float32, device=dev)
    loss = torch.empty(1, dtype=torch.float32, device=dev)
    saved = torch.empty((max(Nc, 1), 3), dtype=torch.float32, device=dev)
    ws = workspace if workspace is not None else _workspace(PAYLOAD_LOGITS_PAIR, dt, max(Nc, 1), B, Sm1, 64, V, dev)
    _check(lib().rkl_forward_logits_pair(_ptr(student_logits), _ptr(teacher_logits), dt, B, Sm1, V, _ptr(row_idx), Nc, nd,
                                         reduction, _ptr(loss_tok), _ptr(loss), _ptr(saved), _ptr(ws), ws.numel(),
                                         _stream(dev)))
    return loss_tok, loss, saved


def backward_logits_pair(student_logits, teacher_logits, B, Sm1, row_idx, N, reduction, saved, grad_loss=None,
                         grad_tok=None, workspace=None, dz=None):
    """dLoss/dz_s [T, V] in the dtype of the logits."""
    Nc, nd = _count(N, B, Sm1)
    dev = student_logits.device
    V = student_logits.shape[1]
    dt = _dtype_code(student_logits)
    if dz is None:
        dz = torch.empty_like(student_logits)
    if grad_loss is not None:
        grad_loss = grad_loss.reshape(1).to(device=dev, dtype=torch.float32).contiguous()
    if grad_tok is not None:
        grad_tok = grad_tok.to(device=dev, dtype=torch.float32).contiguous()
    ws = workspace if workspace is not None else _workspace(PAYLOAD_LOGITS_PAIR, dt, max(Nc, 1), B, Sm1, 64, V, dev)
    _check(lib().rkl_backward_logits_pair(_ptr(student_logits), _ptr(teacher_logits), dt, B, Sm1, V, _ptr(row_idx),
                                          Nc, nd, reduction, _ptr(saved), _ptr(grad_loss), _ptr(grad_tok), _ptr(dz),
                                          _ptr(ws), ws.numel(), _stream(dev)))
    return dz


# ------------------------------------------------------------ top-k estimator

def forward_topk_pair(student_logits, teacher_logits, targets, k, B, Sm1, row_idx, N, reduction, workspace=None):
    """Top-k estimator with both sides as logits; targets [B, Sm1] are the
    sampled tokens.  Returns (loss_tok [B,Sm1], loss [1], saved [7N])."""
    Nc, nd = _count(N, B, Sm1)
    dev = student_logits.device
    V = student_logits.shape[1]
    dt = _dtype_code(student_logits)
    tg = targets.to(device=dev, dtype=torch.int32).contiguous()
    loss_tok = torch.empty((B, Sm1), dtype=torch.float32, device=dev)
    loss = torch.empty(1, dtype=torch.float32, device=dev)
    saved = torch.empty(7 * max(Nc, 1), dtype=torch.float32, device=dev)
    ws = workspace if workspace is not None else _workspace(PAYLOAD_LOGITS_PAIR, dt, max(Nc, 1), B, Sm1, 64, V, dev)
    _check(lib().rkl_forward_topk_pair(_ptr(student_logits), _ptr(teacher_logits), dt, B, Sm1, V, _ptr(row_idx), Nc, nd,
                                       int(k), _ptr(tg), reduction, _ptr(loss_tok), _ptr(loss), _ptr(saved),
                                       _ptr(ws), ws.numel(), _stream(dev)))
    return loss_tok, loss, saved


def backward_topk_pair(student_logits, teacher_logits, targets, B, Sm1, row_idx, N, reduction, saved,
                       grad_loss=None, grad_tok=None, workspace=None, dz=None):
    """Gradient estimate dLoss/dz_s [T, V] of the top-k estimator."""
    Nc, nd = _count(N, B, Sm1)
    dev = student_logits.device
    V = student_logits.shape[1]
    dt = _dtype_code(student_logits)
    tg = targets.to(device=dev, dtype=torch.int32).contiguous()
    if dz is None:
        dz = torch.empty_like(student_logits)
    if grad_loss is not None:
        grad_loss = grad_loss.reshape(1).to(device=dev, dtype=torch.float32).contiguous()
    if grad_tok is not None:
        grad_tok = grad_tok.to(device=dev, dtype=torch.float32).contiguous()
    ws = workspace if workspace is not None else _workspace(PAYLOAD_LOGITS_PAIR, dt, max(Nc, 1), B, Sm1, 64, V, dev)
    _check(lib().rkl_backward_topk_pair(_ptr(student_logits), _ptr(teacher_logits), dt, B, Sm1, V, _ptr(row_idx), Nc, nd,
                                        _ptr(tg), reduction, _ptr(saved), _ptr(grad_loss), _ptr(grad_tok), _ptr(dz),
                                        _ptr(ws), ws.numel(), _stream(dev)))
    return dz


class _RKLTopkPair(torch.autograd.Function):
    @staticmethod
    def forward(ctx, student_logits, teacher_logits, targets, mask, k, reduction):
        B, Sm1 = mask.shape
        row_idx, N = compact_rows(mask, on_device=True)  # no host synchronisation
        loss_tok, loss, saved = forward_topk_pair(student_logits, teacher_logits, targets, k, B, Sm1, row_idx, N,
                                                  reduction)
        tg = targets.to(device=student_logits.device, dtype=torch.int32).contiguous()
        ctx.save_for_backward(student_logits, teacher_logits, tg, row_idx, saved)
        ctx.meta = (B, Sm1, N, reduction)
        return loss.reshape(()), loss_tok

    @staticmethod
    def backward(ctx, g_loss, g_tok):
        zs, zt, tg, row_idx, saved = ctx.saved_tensors
        B, Sm1, N, reduction = ctx.meta
        dz = backward_topk_pair(zs, zt, tg, B, Sm1, row_idx, N, reduction, saved, grad_loss=g_loss, grad_tok=g_tok)
        return dz, None, None, None, None, None


def topk_estimator_logits_pair(student_logits, teacher_logits, targets, mask, k, reduction=REDUCE_TOKEN_MEAN):
    """Differentiable (loss, loss_tok) of the top-k estimator (both sides as
    [T, V] logits, targets = sampled tokens); grad to the student logits."""
    return _RKLTopkPair.apply(student_logits.contiguous(), teacher_logits.contiguous(), targets, mask, int(k),
                              reduction)


PAYLOAD_TOPK_HIDDEN = 3


def forward_topk_hidden(h_s, h_t, W_s, W_t, targets, k, B, Sm1, row_idx, N, reduction, workspace=None):
    """Top-k estimator on the hidden payload.  Returns (loss_tok, loss, saved [7N])."""
    Nc, nd = _count(N, B, Sm1)
    dev = h_s.device
    T, H = h_s.shape
    V = W_s.shape[0]
    dt = _dtype_code(h_s)
    tg = targets.to(device=dev, dtype=torch.int32).contiguous()
    loss_tok = torch.empty((B, Sm1), dtype=torch.float32, device=dev)
    loss = torch.empty(1, dtype=torch.float32, device=dev)
    saved = torch.empty(7 * max(Nc, 1), dtype=torch.float32, device=dev)
    ws = workspace if workspace is not None else _workspace(PAYLOAD_TOPK_HIDDEN, dt, max(Nc, 1), B, Sm1, H, V, dev)
    _check(lib().rkl_forward_topk_hidden(_ptr(h_s), _ptr(h_t), _ptr(W_s), _ptr(W_t), dt, B, Sm1, H, V,
                                         _ptr(row_idx), Nc, nd, int(k), _ptr(tg), reduction, _ptr(loss_tok), _ptr(loss),
                                         _ptr(saved), _ptr(ws), ws.numel(), _stream(dev)))
    return loss_tok, loss, saved


def backward_topk_hidden(h_s, h_t, W_s, W_t, targets, B, Sm1, row_idx, N, reduction, saved, grad_loss=None,
                         grad_tok=None, workspace=None, dH_s=None, dW_s=None):
    """(dH_s [T,H] fp32, dW_s [V,H] fp32) of the top-k estimator on the hidden payload."""
    Nc, nd = _count(N, B, Sm1)
    dev = h_s.device
    T, H = h_s.shape
    V = W_s.shape[0]
    dt = _dtype_code(h_s)
    tg = targets.to(device=dev, dtype=torch.int32).contiguous()
    if dH_s is None:
        dH_s = torch.empty((T, H), dtype=torch.float32, device=dev)
    if dW_s is None:
        dW_s = torch.empty((V, H), dtype=torch.float32, device=dev)
    if grad_loss is not None:
        grad_loss = grad_loss.reshape(1).to(device=dev, dtype=torch.float32).contiguous()
    if grad_tok is not None:
        grad_tok = grad_tok.to(device=dev, dtype=torch.float32).contiguous()
    ws = workspace if workspace is not None else _workspace(PAYLOAD_TOPK_HIDDEN, dt, max(Nc, 1), B, Sm1, H, V, dev)
    _check(lib().rkl_backward_topk_hidden(_ptr(h_s), _ptr(h_t), _ptr(W_s), _ptr(W_t), dt, B, Sm1, H, V,
                                          _ptr(row_idx), Nc, nd, _ptr(tg), reduction, _ptr(saved), _ptr(grad_loss),
                                          _ptr(grad_tok), _ptr(dH_s), _ptr(dW_s), _ptr(ws), ws.numel(),
                                          _stream(dev)))
    return dH_s, dW_s


class _RKLTopkHidden(torch.autograd.Function):
    @staticmethod
    def forward(ctx, h_s, h_t, W_s, W_t, targets, mask, k, reduction):
        B, Sm1 = mask.shape
        row_idx, N = compact_rows(mask, on_device=True)  # no host synchronisation
        tg = targets.to(device=h_s.device, dtype=torch.int32).contiguous()
        loss_tok, loss, saved = forward_topk_hidden(h_s, h_t, W_s, W_t, tg, k, B, Sm1, row_idx, N, reduction)
        ctx.save_for_backward(h_s, h_t, W_s, W_t, tg, row_idx, saved)
        ctx.meta = (B, Sm1, N, reduction)
        return loss.reshape(()), loss_tok

    @staticmethod
    def backward(ctx, g_loss, g_tok):
        h_s, h_t, W_s, W_t, tg, row_idx, saved = ctx.saved_tensors
        B, Sm1, N, reduction = ctx.meta
        dH, dW = backward_topk_hidden(h_s, h_t, W_s, W_t, tg, B, Sm1, row_idx, N, reduction, saved,
                                      grad_loss=g_loss, grad_tok=g_tok)
        return dH.to(h_s.dtype), None, dW.to(W_s.dtype), None, None, None, None, None


def topk_estimator_hidden(h_s, h_t, W_s, W_t, targets, mask, k, reduction=REDUCE_TOKEN_MEAN):
    """Differentiable (loss, loss_tok) of the top-k estimator on the hidden
    payload (targets = sampled tokens); grads to h_s and W_s."""
    return _RKLTopkHidden.apply(h_s.contiguous(), h_t.contiguous(), W_s.contiguous(), W_t.contiguous(), targets,
                                mask, int(k), reduction)


# ------------------------------------------------------------ top-k on the logits payload
PAYLOAD_TOPK_LOGITS = 4


def forward_topk_logits(h_s, W_s, teacher_logits, targets, k, B, Sm1, row_idx, N, reduction, workspace=None):
    """Top-k estimator on the logits payload (student hidden states and LM
    head, shipped bf16 teacher logits).  Returns (loss_tok, loss, saved [7N])."""
    Nc, nd = _count(N, B, Sm1)
    dev = h_s.device
    T, H = h_s.shape
    V = W_s.shape[0]
    dt = _dtype_code(h_s)
    tg = targets.to(device=dev, dtype=torch.int32).contiguous()
    loss_tok = torch.empty((B, Sm1), dtype=torch.float32, device=dev)
    loss = torch.empty(1, dtype=torch.float32, device=dev)
    saved = torch.empty(7 * max(Nc, 1), dtype=torch.float32, device=dev)
    ws = workspace if workspace is not None else _workspace(PAYLOAD_TOPK_LOGITS, dt, max(Nc, 1), B, Sm1, H, V, dev)
    _check(lib().rkl_forward_topk_logits(_ptr(h_s), _ptr(W_s), _ptr(teacher_logits), dt, B, Sm1, H, V,
                                         _ptr(row_idx), Nc, nd, int(k), _ptr(tg), reduction, _ptr(loss_tok),
                                         _ptr(loss), _ptr(saved), _ptr(ws), ws.numel(), _stream(dev)))
    return loss_tok, loss, saved


def backward_topk_logits(h_s, W_s, teacher_logits, targets, B, Sm1, row_idx, N, reduction, saved, grad_loss=None,
                         grad_tok=None, workspace=None, dH_s=None, dW_s=None):
    """(dH_s [T,H] fp32, dW_s [V,H] fp32) of the top-k estimator on the logits payload."""
    Nc, nd = _count(N, B, Sm1)
    dev = h_s.device
    T, H = h_s.shape
    V = W_s.shape[0]
    dt = _dtype_code(h_s)
    tg = targets.to(device=dev, dtype=torch.int32).contiguous()
    if dH_s is None:
        dH_s = torch.empty((T, H), dtype=torch.float32, device=dev)
    if dW_s is None:
        dW_s = torch.empty((V, H), dtype=torch.float32, device=dev)
    if grad_loss is not None:
        grad_loss = grad_loss.reshape(1).to(device=dev, dtype=torch.float32).contiguous()
    if grad_tok is not None:
        grad_tok = grad_tok.to(device=dev, dtype=torch.float32).contiguous()
    ws = workspace if workspace is not None else _workspace(PAYLOAD_TOPK_LOGITS, dt, max(Nc, 1), B, Sm1, H, V, dev)
    _check(lib().rkl_backward_topk_logits(_ptr(h_s), _ptr(W_s), _ptr(teacher_logits), dt, B, Sm1, H, V,
                                          _ptr(row_idx), Nc, nd, _ptr(tg), reduction, _ptr(saved), _ptr(grad_loss),
                                          _ptr(grad_tok), _ptr(dH_s), _ptr(dW_s), _ptr(ws), ws.numel(),
                                          _stream(dev)))
    return dH_s, dW_s


class _RKLTopkLogits(torch.autograd.Function):
    @staticmethod
    def forward(ctx, h_s, W_s, teacher_logits, targets, mask, k, reduction):
        B, Sm1 = mask.shape
        row_idx, N = compact_rows(mask, on_device=True)  # no host synchronisation
        tg = targets.to(device=h_s.device, dtype=torch.int32).contiguous()
        loss_tok, loss, saved = forward_topk_logits(h_s, W_s, teacher_logits, tg, k, B, Sm1, row_idx, N, reduction)
        ctx.save_for_backward(h_s, W_s, teacher_logits, tg, row_idx, saved)
        ctx.meta = (B, Sm1, N, reduction)
        return loss.reshape(()), loss_tok

    @staticmethod
    def backward(ctx, g_loss, g_tok):
        h_s, W_s, logits, tg, row_idx, saved = ctx.saved_tensors
        B, Sm1, N, reduction = ctx.meta
        dH, dW = backward_topk_logits(h_s, W_s, logits, tg, B, Sm1, row_idx, N, reduction, saved,
                                      grad_loss=g_loss, grad_tok=g_tok)
        return dH.to(h_s.dtype), dW.to(W_s.dtype), None, None, None, None, None


def topk_estimator_logits(h_s, W_s, teacher_logits, targets, mask, k, reduction=REDUCE_TOKEN_MEAN):
    """Differentiable (loss, loss_tok) of the top-k estimator on the logits
    payload (targets = sampled tokens); grads to h_s and W_s."""
    return _RKLTopkLogits.apply(h_s.contiguous(), W_s.contiguous(), teacher_logits.contiguous(), targets, mask,
                                int(k), reduction)


# ------------------------------------------------------------ teacher per row

def compact_rows_multi(mask, teacher_idx, n_teachers):
    """S1 with per-teacher counts: (row_idx int32 [B*Sm1] device, N, counts list
    of n_teachers ints).  Raises if a trainable row's teacher index is out of
    range."""
    B, Sm1 = mask.shape
    mask = mask.contiguous()
    if mask.dtype != torch.uint8:
        mask = (mask != 0).to(torch.uint8)
    tid = teacher_idx.to(device=mask.device, dtype=torch.int32).contiguous()
    row_idx = torch.empty(B * Sm1, dtype=torch.int32, device=mask.device)
    n_dev = torch.empty(1, dtype=torch.int32, device=mask.device)
    counts = torch.empty(n_teachers + 1, dtype=torch.int32, device=mask.device)
    _check(lib().rkl_compact_rows_multi(_ptr(mask), _ptr(tid), B, Sm1, n_teachers, _ptr(row_idx), _ptr(n_dev),
                                        _ptr(counts), _stream(mask.device)))
    host = counts.cpu().tolist()
    if host[n_teachers] != 0:
        raise RKLError(2, "%d trainable rows have a teacher index outside [0, %d)" % (host[n_teachers], n_teachers))
    return row_idx, int(n_dev.item()), host[:n_teachers]


def workspace_size_multi(dtype_code, n_max, n_teachers, B, Sm1, H, V):
    out = ctypes.c_size_t(0)
    _check(lib().rkl_workspace_size_multi(dtype_code, n_max, n_teachers, B, Sm1, H, V, ctypes.byref(out)))
    return out.value


def _counts_host(counts):
    arr = (ctypes.c_int32 * len(counts))(*[int(c) for c in counts])
    return arr


def forward_hidden_multi(h_s, h_t, W_s, W_t, teacher_idx, counts, B, Sm1, row_idx, N, reduction, workspace=None):
    """Forward with a teacher per row.  W_t [n_teachers, V, H]; teacher_idx
    [B, Sm1] int32 device; counts from compact_rows_multi.
    Returns (loss_tok [B,Sm1], loss [1], saved [N,3])."""
    dev = h_s.device
    T, H = h_s.shape
    V = W_s.shape[0]
    nt = W_t.shape[0]
    dt = _dtype_code(h_s)
    tid = teacher_idx.to(device=dev, dtype=torch.int32).contiguous()
    loss_tok = torch.empty((B, Sm1), dtype=torch.float32, device=dev)
    loss = torch.empty(1, dtype=torch.float32, device=dev)
    saved = torch.empty((max(N, 1), 3), dtype=torch.float32, device=dev)
    if workspace is None:
        nbytes = workspace_size_multi(dt, max(N, 1), nt, B, Sm1, H, V)
        workspace = torch.empty(max(nbytes, 256), dtype=torch.uint8, device=dev)
    _check(lib().rkl_forward_hidden_multi(_ptr(h_s), _ptr(h_t), _ptr(W_s), _ptr(W_t), nt, _ptr(tid),
                                          _counts_host(counts), dt, B, Sm1, H, V, _ptr(row_idx), N, reduction,
                                          _ptr(loss_tok), _ptr(loss), _ptr(saved), _ptr(workspace), workspace.numel(),
                                          _stream(dev)))
    return loss_tok, loss, saved


def backward_hidden_multi(h_s, h_t, W_s, W_t, teacher_idx, counts, B, Sm1, row_idx, N, reduction, saved,
                          grad_loss=None, grad_tok=None, workspace=None, dH_s=None, dW_s=None):
    """Backward with a teacher per row.  Returns (dH_s [T,H] fp32, dW_s [V,H] fp32)."""
    dev = h_s.device
    T, H = h_s.shape
    V = W_s.shape[0]
    nt = W_t.shape[0]
    dt = _dtype_code(h_s)
    tid = teacher_idx.to(device=dev, dtype=torch.int32).contiguous()
    if dH_s is None:
        dH_s = torch.empty((T, H), dtype=torch.float32, device=dev)
    if dW_s is None:
        dW_s = torch.empty((V, H), dtype=torch.float32, device=dev)
    if grad_loss is not None:
        grad_loss = grad_loss.reshape(1).to(device=dev, dtype=torch.float32).contiguous()
    if grad_tok is not None:
        grad_tok = grad_tok.to(device=dev, dtype=torch.float32).contiguous()
    if workspace is None:
        nbytes = workspace_size_multi(dt, max(N, 1), nt, B, Sm1, H, V)
        workspace = torch.empty(max(nbytes, 256), dtype=torch.uint8, device=dev)
    _check(lib().rkl_backward_hidden_multi(_ptr(h_s), _ptr(h_t), _ptr(W_s), _ptr(W_t), nt, _ptr(tid),
                                           _counts_host(counts), dt, B, Sm1, H, V, _ptr(row_idx), N, reduction,
                                           _ptr(saved), _ptr(grad_loss), _ptr(grad_tok), _ptr(dH_s), _ptr(dW_s),
                                           _ptr(workspace), workspace.numel(), _stream(dev)))
    return dH_s, dW_s


class _RKLHiddenMulti(torch.autograd.Function):
    @staticmethod
    def forward(ctx, h_s, h_t, W_s, W_t, teacher_idx, mask, reduction):
        B, Sm1 = mask.shape
        row_idx, N, counts = compact_rows_multi(mask, teacher_idx, W_t.shape[0])
        tid = teacher_idx.to(device=h_s.device, dtype=torch.int32).contiguous()
        loss_tok, loss, saved = forward_hidden_multi(h_s, h_t, W_s, W_t, tid, counts, B, Sm1, row_idx, N, reduction)
        ctx.save_for_backward(h_s, h_t, W_s, W_t, tid, row_idx, saved)
        ctx.meta = (B, Sm1, N, reduction, counts)
        return loss.reshape(()), loss_tok

    @staticmethod
    def backward(ctx, g_loss, g_tok):
        h_s, h_t, W_s, W_t, tid, row_idx, saved = ctx.saved_tensors
        B, Sm1, N, reduction, counts = ctx.meta
        dH, dW = backward_hidden_multi(h_s, h_t, W_s, W_t, tid, counts, B, Sm1, row_idx, N, reduction, saved,
                                       grad_loss=g_loss, grad_tok=g_tok)
        return dH.to(h_s.dtype), None, dW.to(W_s.dtype), None, None, None, None


def reverse_kl_hidden_multi(h_s, h_t, W_s, W_t, teacher_idx, mask, reduction=REDUCE_TOKEN_MEAN):
    """Differentiable (loss, loss_tok) with a teacher per row: W_t [n_teachers, V, H]
    stacked heads, teacher_idx [B, S-1]; grads to h_s and W_s."""
    return _RKLHiddenMulti.apply(h_s.contiguous(), h_t.contiguous(), W_s.contiguous(), W_t.contiguous(),
                                 teacher_idx, mask, reduction)


def device_error():
    code = ctypes.c_int32(0)
    lib().rkl_device_error(ctypes.byref(code))
    return code.value


class _RKLHidden(torch.autograd.Function):
    @staticmethod
    def forward(ctx, h_s, h_t, W_s, W_t, mask, reduction):
        B, Sm1 = mask.shape
        row_idx, N = compact_rows(mask, on_device=True)  # no host synchronisation
        loss_tok, loss, saved = forward_hidden(h_s, h_t, W_s, W_t, B, Sm1, row_idx, N, reduction)
        ctx.save_for_backward(h_s, h_t, W_s, W_t, row_idx, saved)
        ctx.meta = (B, Sm1, N, reduction)
        return loss.reshape(()), loss_tok

    @staticmethod
    def backward(ctx, g_loss, g_tok):
        h_s, h_t, W_s, W_t, row_idx, saved = ctx.saved_tensors
        B, Sm1, N, reduction = ctx.meta
        dH, dW = backward(PAYLOAD_HIDDEN, h_s, h_t, W_s, W_t, B, Sm1, row_idx, N, reduction, saved,
                          grad_loss=g_loss, grad_tok=g_tok)
        return dH.to(h_s.dtype), None, dW.to(W_s.dtype), None, None, None


class _RKLLogits(torch.autograd.Function):
    @staticmethod
    def forward(ctx, h_s, W_s, teacher_logits, mask, reduction):
        B, Sm1 = mask.shape
        row_idx, N = compact_rows(mask, on_device=True)  # no host synchronisation
        loss_tok, loss, saved = forward_logits(h_s, W_s, teacher_logits, B, Sm1, row_idx, N, reduction)
        ctx.save_for_backward(h_s, W_s, teacher_logits, row_idx, saved)
        ctx.meta = (B, Sm1, N, reduction)
        return loss.reshape(()), loss_tok

    @staticmethod
    def backward(ctx, g_loss, g_tok):
        h_s, W_s, logits, row_idx, saved = ctx.saved_tensors
        B, Sm1, N, reduction = ctx.meta
        dH, dW = backward(PAYLOAD_LOGITS, h_s, logits, W_s, None, B, Sm1, row_idx, N, reduction, saved,
                          grad_loss=g_loss, grad_tok=g_tok)
        return dH.to(h_s.dtype), dW.to(W_s.dtype), None, None, None


class _RKLLogitsPair(torch.autograd.Function):
    @staticmethod
    def forward(ctx, student_logits, teacher_logits, mask, reduction):
        B, Sm1 = mask.shape
        row_idx, N = compact_rows(mask, on_device=True)  # no host synchronisation
        loss_tok, loss, saved = forward_logits_pair(student_logits, teacher_logits, B, Sm1, row_idx, N, reduction)
        ctx.save_for_backward(student_logits, teacher_logits, row_idx, saved)
        ctx.meta = (B, Sm1, N, reduction)
        return loss.reshape(()), loss_tok

    @staticmethod
    def backward(ctx, g_loss, g_tok):
        zs, zt, row_idx, saved = ctx.saved_tensors
        B, Sm1, N, reduction = ctx.meta
        dz = backward_logits_pair(zs, zt, B, Sm1, row_idx, N, reduction, saved, grad_loss=g_loss, grad_tok=g_tok)
        return dz, None, None, None


def reverse_kl_logits_pair(student_logits, teacher_logits, mask, reduction=REDUCE_TOKEN_MEAN):
    """Differentiable (loss, loss_tok) with both sides given as [T, V] logits; grad to the student logits."""
    return _RKLLogitsPair.apply(student_logits.contiguous(), teacher_logits.contiguous(), mask, reduction)


def reverse_kl_hidden(h_s, h_t, W_s, W_t, mask, reduction=REDUCE_TOKEN_MEAN):
    """Differentiable (loss, loss_tok) of the hidden-state payload; grads to h_s and W_s."""
    return _RKLHidden.apply(h_s.contiguous(), h_t.contiguous(), W_s.contiguous(), W_t.contiguous(),
                            mask, reduction)


def reverse_kl_logits(h_s, W_s, teacher_logits, mask, reduction=REDUCE_TOKEN_MEAN):
    """Differentiable (loss, loss_tok) of the logits payload; grads to h_s and W_s."""
    return _RKLLogits.apply(h_s.contiguous(), W_s.contiguous(), teacher_logits.contiguous(), mask, reduction)
