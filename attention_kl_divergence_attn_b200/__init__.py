"""Fused attention-distillation KL divergence for B200 (sm_100a).

Thin ctypes binding over the C ABI in ``include/streamkl.h`` (library
``libstreamkl.so`` next to this file).  Every step of the computation runs in
the library's CUDA kernels; this module only checks tensors, allocates outputs
with torch and passes raw pointers.  There is no CPU fallback: if the library
is missing or the device is not an sm_100 GPU, calls raise.

Functions keep the C names:
  streamkl_fwd(q_t, k_t, q_s, k_s, ...) -> (kl, lse_t, lse_s, loss_mean)
  streamkl_bwd(q_t, k_t, q_s, k_s, kl, lse_t, lse_s, ...) -> (dq_s, dk_s, dq_t, dk_t)
Keys may have fewer heads than the queries (grouped key heads: k_t
[B, H_kt, N_K, d_t], k_s [B, H_ks, N_K, d_s], each count dividing H), and
``kv_len`` (int32 [B] on the device) marks the keys at and past each batch
element's length as padding; either routes the call to the C ABI's
``streamkl_fwd_ex`` / ``streamkl_bwd_ex``.
The autograd wrapper with temperature scaling is in ``.autograd``
(``streamkl_loss``).
"""
from __future__ import annotations

import ctypes
import math
import os
import threading

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libstreamkl.so")

STATUS = {0: "ok", 1: "invalid argument", 2: "unsupported", 3: "CUDA error", 4: "device wait timeout",
          5: "workspace", 6: "access outside a tensor (bounds-checked build)"}


class StreamKLError(RuntimeError):
    def __init__(self, fn, code):
        super().__init__(f"{fn} failed: {STATUS.get(code, code)} (status {code})")
        self.code = code


_lib = None
_lock = threading.Lock()
_VP = ctypes.c_void_p
_I = ctypes.c_int
_F = ctypes.c_float


def lib():
    """The loaded C library (raises if it has not been built)."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise RuntimeError(f"{LIB_PATH} is missing: run `python -m attention_kl_divergence_attn_b200.build`")
            L = ctypes.CDLL(LIB_PATH)
            shape = [_I] * 6 + [_F, _F, _I]
            L.streamkl_fwd.argtypes = [_VP] * 4 + shape + [_VP] * 4 + [_VP, ctypes.c_size_t, _VP]
            L.streamkl_fwd.restype = _I
            L.streamkl_bwd.argtypes = ([_VP] * 4 + shape + [_VP] * 3 + [_VP, _F] + [_VP] * 4
                                       + [_VP, ctypes.c_size_t, _VP])
            L.streamkl_bwd.restype = _I
            L.streamkl_bwd_dk.argtypes = ([_VP] * 4 + shape + [_VP] * 3 + [_VP, _F] + [_VP] * 2
                                          + [_VP, ctypes.c_size_t, _VP])
            L.streamkl_bwd_dk.restype = _I
            L.streamkl_bwd_dq.argtypes = L.streamkl_bwd_dk.argtypes
            L.streamkl_bwd_dq.restype = _I
            L.streamkl_bwd_dloss_device.argtypes = ([_VP] * 4 + shape + [_VP] * 3 + [_VP, _VP, _F] + [_VP] * 4
                                                    + [_VP, ctypes.c_size_t, _VP])
            L.streamkl_bwd_dloss_device.restype = _I
            L.streamkl_loss_mean.argtypes = [_VP, ctypes.c_longlong, _VP, _VP]
            L.streamkl_loss_mean.restype = _I
            L.streamkl_loss_reduce.argtypes = [_VP, ctypes.c_longlong, ctypes.c_double, _VP, _VP]
            L.streamkl_loss_reduce.restype = _I
            shape_ex = [_I] * 8 + [_F, _F, _I, _VP]            # B, H, H_kt, H_ks, N_Q, N_K, d_t, d_s, ..., kv_len
            L.streamkl_fwd_ex.argtypes = [_VP] * 4 + shape_ex + [_VP] * 4 + [_VP, ctypes.c_size_t, _VP]
            L.streamkl_fwd_ex.restype = _I
            L.streamkl_bwd_ex.argtypes = ([_VP] * 4 + shape_ex + [_VP] * 3 + [_VP, _F, _VP] + [_VP] * 4 + [_I]
                                          + [_VP, ctypes.c_size_t, _VP])
            L.streamkl_bwd_ex.restype = _I
            L.streamkl_workspace_size_ex.argtypes = [_I] * 10
            L.streamkl_workspace_size_ex.restype = ctypes.c_size_t
            L.streamkl_fwd_noalloc.argtypes = ([_VP] * 4 + shape + [_VP] * 4 + [_VP, ctypes.POINTER(ctypes.c_uint)])
            L.streamkl_fwd_noalloc.restype = _I
            L.streamkl_workspace_size.argtypes = [_I] * 7
            L.streamkl_workspace_size.restype = ctypes.c_size_t
            L.streamkl_workspace_init.argtypes = [_VP, ctypes.c_size_t, _VP]
            L.streamkl_workspace_init.restype = _I
            L.streamkl_check.argtypes = [_VP, _VP, ctypes.POINTER(ctypes.c_uint)]
            L.streamkl_check.restype = _I
            L.streamkl_selftest_timeout.argtypes = [_VP, ctypes.c_size_t, ctypes.c_ulonglong, _VP]
            L.streamkl_selftest_timeout.restype = _I
            L.streamkl_strerror.argtypes = [_I]
            L.streamkl_strerror.restype = ctypes.c_char_p
            L.streamkl_version.argtypes = []
            L.streamkl_version.restype = _I
            _lib = L
    return _lib


_workspaces: dict = {}
_ws_sizes: dict = {}
_STATUS_BYTES = 256


def workspace(device=None, nbytes=None) -> torch.Tensor:
    """This device's workspace, created and cleared on first use.

    Its first 256 bytes are the library's device status word.  ``nbytes``
    (from ``workspace_size``) grows it for problems whose kernels split key
    ranges; growing keeps the status word.  Calls through this module run on
    the current stream, so they are ordered and may share it.
    """
    dev = torch.device("cuda", torch.cuda.current_device() if device is None else torch.device(device).index)
    need = max(int(nbytes or 0), _STATUS_BYTES)
    ws = _workspaces.get(dev.index)
    if ws is None or ws.numel() < need:
        new = torch.zeros(need, dtype=torch.uint8, device=dev)
        if ws is not None:
            new[:_STATUS_BYTES].copy_(ws[:_STATUS_BYTES])
        ws = new
        _workspaces[dev.index] = ws
    return ws


def workspace_size(B, H, N_Q, N_K, d_t, d_s, causal, H_kt=None, H_ks=None, teacher_grads=False) -> int:
    """streamkl_workspace_size(_ex) for this problem on the current device (cached)."""
    H_kt = H if H_kt is None else H_kt
    H_ks = H if H_ks is None else H_ks
    key = (torch.cuda.current_device(), B, H, H_kt, H_ks, N_Q, N_K, d_t, d_s, int(bool(causal)),
           int(bool(teacher_grads)))
    n = _ws_sizes.get(key)
    if n is None:
        if H_kt == H and H_ks == H:
            n = int(lib().streamkl_workspace_size(B, H, N_Q, N_K, d_t, d_s, int(bool(causal))))
        else:
            n = int(lib().streamkl_workspace_size_ex(B, H, H_kt, H_ks, N_Q, N_K, d_t, d_s, int(bool(causal)),
                                                     int(bool(teacher_grads))))
        _ws_sizes[key] = n
    return n


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _check_inputs(q_t, k_t, q_s, k_s):
    for name, t in (("q_t", q_t), ("k_t", k_t), ("q_s", q_s), ("k_s", k_s)):
        if not isinstance(t, torch.Tensor) or t.dtype != torch.bfloat16 or not t.is_cuda:
            raise TypeError(f"{name} must be a CUDA bf16 tensor")
        if t.dim() != 4 or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous [B, H, N, d] tensor")
    B, H, N_Q, d_t = q_t.shape
    H_kt, N_K = k_t.shape[1], k_t.shape[2]
    d_s = q_s.shape[3]
    H_ks = k_s.shape[1]
    if k_t.shape != (B, H_kt, N_K, d_t) or q_s.shape != (B, H, N_Q, d_s) or k_s.shape != (B, H_ks, N_K, d_s):
        raise ValueError("inconsistent shapes of q_t, k_t, q_s, k_s")
    if H_kt < 1 or H_ks < 1 or H % H_kt or H % H_ks:
        raise ValueError("the key heads of k_t and k_s must each divide the query heads")
    return B, H, N_Q, N_K, d_t, d_s, H_kt, H_ks


def _check_lengths(kv_len, B, device):
    if kv_len is None:
        return None
    if (not isinstance(kv_len, torch.Tensor) or kv_len.dtype != torch.int32 or kv_len.device != device
            or kv_len.numel() != B or not kv_len.is_contiguous()):
        raise ValueError("kv_len must be a contiguous int32 tensor of B lengths on the inputs' device")
    return kv_len


def streamkl_fwd(q_t, k_t, q_s, k_s, scale_t=None, scale_s=None, causal=False, *, loss_mean=True,
                 out=None, stream=None, kv_len=None):
    """Per-row KL(P_teacher || Q_student), both log-sum-exps and the mean loss.

    Returns (kl, lse_t, lse_s, loss) with kl/lse_* fp32 [B, H, N_Q] and loss a
    0-d fp32 device tensor (None if loss_mean=False).  ``out`` may supply the
    three per-row buffers (and optionally a 4th, the loss scalar).  A row with
    no visible key (all keys padding) gets KL = 0 and LSE = -inf.
    """
    B, H, N_Q, N_K, d_t, d_s, H_kt, H_ks = _check_inputs(q_t, k_t, q_s, k_s)
    kv_len = _check_lengths(kv_len, B, q_t.device)
    scale_t = 1.0 / math.sqrt(d_t) if scale_t is None else float(scale_t)
    scale_s = 1.0 / math.sqrt(d_s) if scale_s is None else float(scale_s)
    dev = q_t.device
    if out is None:
        kl = torch.empty(B, H, N_Q, dtype=torch.float32, device=dev)
        lse_t = torch.empty_like(kl)
        lse_s = torch.empty_like(kl)
        loss = torch.empty((), dtype=torch.float32, device=dev) if loss_mean else None
    else:
        kl, lse_t, lse_s = out[:3]
        loss = (out[3] if len(out) > 3 else torch.empty((), dtype=torch.float32, device=dev)) if loss_mean else None
    ws = workspace(dev, workspace_size(B, H, N_Q, N_K, d_t, d_s, causal))
    if H_kt == H and H_ks == H and kv_len is None:
        rc = lib().streamkl_fwd(_ptr(q_t), _ptr(k_t), _ptr(q_s), _ptr(k_s), B, H, N_Q, N_K, d_t, d_s,
                                scale_t, scale_s, int(bool(causal)), _ptr(kl), _ptr(lse_t), _ptr(lse_s),
                                _ptr(loss), _ptr(ws), ws.numel(), _stream(stream))
        if rc:
            raise StreamKLError("streamkl_fwd", rc)
        return kl, lse_t, lse_s, loss
    rc = lib().streamkl_fwd_ex(_ptr(q_t), _ptr(k_t), _ptr(q_s), _ptr(k_s), B, H, H_kt, H_ks, N_Q, N_K, d_t, d_s,
                               scale_t, scale_s, int(bool(causal)), _ptr(kv_len), _ptr(kl), _ptr(lse_t),
                               _ptr(lse_s), _ptr(loss), _ptr(ws), ws.numel(), _stream(stream))
    if rc:
        raise StreamKLError("streamkl_fwd_ex", rc)
    return kl, lse_t, lse_s, loss


_PART_DK, _PART_DQ = 1, 2


def _bwd_ex(parts, q_t, k_t, q_s, k_s, kl, lse_t, lse_s, shape, scale_t, scale_s, causal, kv_len, dkl,
            dloss, dloss_scale, grads, stream):
    """streamkl_bwd_ex: grouped key heads and/or padding (grads = dq_s, dk_s, dq_t, dk_t)."""
    B, H, N_Q, N_K, d_t, d_s, H_kt, H_ks = shape
    teacher = grads[2] is not None or grads[3] is not None
    ws = workspace(q_t.device, workspace_size(B, H, N_Q, N_K, d_t, d_s, causal, H_kt, H_ks, teacher))
    if isinstance(dloss, torch.Tensor):
        if dloss.dtype != torch.float32 or dloss.numel() != 1 or dloss.device != q_t.device:
            raise ValueError("a tensor dloss must be a one-element fp32 tensor on the inputs' device")
        scale, dev_ptr = (1.0 / (B * H * N_Q) if dloss_scale is None else float(dloss_scale)), _ptr(dloss)
    else:
        if dloss_scale is not None:
            raise ValueError("dloss_scale applies to a device-tensor dloss only")
        scale, dev_ptr = float(dloss), None
    rc = lib().streamkl_bwd_ex(_ptr(q_t), _ptr(k_t), _ptr(q_s), _ptr(k_s), B, H, H_kt, H_ks, N_Q, N_K, d_t, d_s,
                               scale_t, scale_s, int(bool(causal)), _ptr(kv_len), _ptr(kl), _ptr(lse_t),
                               _ptr(lse_s), _ptr(dkl), scale, dev_ptr, *[_ptr(g) for g in grads], parts,
                               _ptr(ws), ws.numel(), _stream(stream))
    if rc:
        raise StreamKLError("streamkl_bwd_ex", rc)


def streamkl_bwd(q_t, k_t, q_s, k_s, kl, lse_t, lse_s, scale_t=None, scale_s=None, causal=False, *,
                 dkl=None, dloss=1.0, dloss_scale=None, teacher_grads=False, out=None, stream=None, kv_len=None):
    """Gradients of sum_i g_i KL_i with g = dkl, or of dloss * mean(KL) if dkl is None.

    ``dloss`` is a number or a 0-d CUDA fp32 tensor; a tensor stays on the
    device (streamkl_bwd_dloss_device) and then g = dloss_scale * dloss, with
    dloss_scale defaulting to 1 / (B*H*N_Q).  Returns (dq_s, dk_s, dq_t,
    dk_t), fp32, the teacher pair None unless teacher_grads.  ``out`` may
    supply the four buffers.  With grouped key heads dk_s, dk_t have the key
    tensors' shapes (each key head's gradient sums over its query heads).
    """
    shape = _check_inputs(q_t, k_t, q_s, k_s)
    B, H, N_Q, N_K, d_t, d_s, H_kt, H_ks = shape
    kv_len = _check_lengths(kv_len, B, q_t.device)
    scale_t = 1.0 / math.sqrt(d_t) if scale_t is None else float(scale_t)
    scale_s = 1.0 / math.sqrt(d_s) if scale_s is None else float(scale_s)
    for name, t in (("kl", kl), ("lse_t", lse_t), ("lse_s", lse_s)) + ((("dkl", dkl),) if dkl is not None else ()):
        if t.dtype != torch.float32 or t.numel() != B * H * N_Q or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous fp32 [B, H, N_Q] tensor")
    dev = q_t.device
    if out is None:
        dq_s = torch.empty(B, H, N_Q, d_s, dtype=torch.float32, device=dev)
        dk_s = torch.empty(B, H_ks, N_K, d_s, dtype=torch.float32, device=dev)
        dq_t = torch.empty(B, H, N_Q, d_t, dtype=torch.float32, device=dev) if teacher_grads else None
        dk_t = torch.empty(B, H_kt, N_K, d_t, dtype=torch.float32, device=dev) if teacher_grads else None
    else:
        dq_s, dk_s, dq_t, dk_t = out
    if H_kt != H or H_ks != H or kv_len is not None:
        _bwd_ex(_PART_DK | _PART_DQ, q_t, k_t, q_s, k_s, kl, lse_t, lse_s, shape, scale_t, scale_s, causal, kv_len,
                dkl, dloss, dloss_scale, (dq_s, dk_s, dq_t, dk_t), stream)
        return dq_s, dk_s, dq_t, dk_t
    ws = workspace(dev, workspace_size(B, H, N_Q, N_K, d_t, d_s, causal))
    if isinstance(dloss, torch.Tensor):
        if dloss.dtype != torch.float32 or dloss.numel() != 1 or dloss.device != dev:
            raise ValueError("a tensor dloss must be a one-element fp32 tensor on the inputs' device")
        scale = 1.0 / (B * H * N_Q) if dloss_scale is None else float(dloss_scale)
        rc = lib().streamkl_bwd_dloss_device(
            _ptr(q_t), _ptr(k_t), _ptr(q_s), _ptr(k_s), B, H, N_Q, N_K, d_t, d_s, scale_t, scale_s,
            int(bool(causal)), _ptr(kl), _ptr(lse_t), _ptr(lse_s), _ptr(dkl), _ptr(dloss), scale,
            _ptr(dq_s), _ptr(dk_s), _ptr(dq_t), _ptr(dk_t), _ptr(ws), ws.numel(), _stream(stream))
        if rc:
            raise StreamKLError("streamkl_bwd_dloss_device", rc)
        return dq_s, dk_s, dq_t, dk_t
    if dloss_scale is not None:
        raise ValueError("dloss_scale applies to a device-tensor dloss only")
    rc = lib().streamkl_bwd(_ptr(q_t), _ptr(k_t), _ptr(q_s), _ptr(k_s), B, H, N_Q, N_K, d_t, d_s,
                            scale_t, scale_s, int(bool(causal)), _ptr(kl), _ptr(lse_t), _ptr(lse_s),
                            _ptr(dkl), float(dloss), _ptr(dq_s), _ptr(dk_s), _ptr(dq_t), _ptr(dk_t),
                            _ptr(ws), ws.numel(), _stream(stream))
    if rc:
        raise StreamKLError("streamkl_bwd", rc)
    return dq_s, dk_s, dq_t, dk_t


def _bwd_part(fn, which, q_t, k_t, q_s, k_s, kl, lse_t, lse_s, scale_t, scale_s, causal, dkl, dloss,
              teacher_grads, out, stream, kv_len=None):
    shape = _check_inputs(q_t, k_t, q_s, k_s)
    B, H, N_Q, N_K, d_t, d_s, H_kt, H_ks = shape
    kv_len = _check_lengths(kv_len, B, q_t.device)
    scale_t = 1.0 / math.sqrt(d_t) if scale_t is None else float(scale_t)
    scale_s = 1.0 / math.sqrt(d_s) if scale_s is None else float(scale_s)
    dev = q_t.device
    if out is None:
        n_s, n_t = (H_ks, H_kt) if which == "k" else (H, H)
        n = N_K if which == "k" else N_Q
        g_s = torch.empty(B, n_s, n, d_s, dtype=torch.float32, device=dev)
        g_t = torch.empty(B, n_t, n, d_t, dtype=torch.float32, device=dev) if teacher_grads else None
    else:
        g_s, g_t = out
    if H_kt != H or H_ks != H or kv_len is not None:
        grads = (None, g_s, None, g_t) if which == "k" else (g_s, None, g_t, None)
        _bwd_ex(_PART_DK if which == "k" else _PART_DQ, q_t, k_t, q_s, k_s, kl, lse_t, lse_s, shape, scale_t,
                scale_s, causal, kv_len, dkl, dloss, None, grads, stream)
        return g_s, g_t
    ws = workspace(dev, workspace_size(B, H, N_Q, N_K, d_t, d_s, causal))
    rc = getattr(lib(), fn)(_ptr(q_t), _ptr(k_t), _ptr(q_s), _ptr(k_s), B, H, N_Q, N_K, d_t, d_s,
                            scale_t, scale_s, int(bool(causal)), _ptr(kl), _ptr(lse_t), _ptr(lse_s),
                            _ptr(dkl), float(dloss), _ptr(g_s), _ptr(g_t), _ptr(ws), ws.numel(), _stream(stream))
    if rc:
        raise StreamKLError(fn, rc)
    return g_s, g_t


def streamkl_bwd_dk(q_t, k_t, q_s, k_s, kl, lse_t, lse_s, scale_t=None, scale_s=None, causal=False, *,
                    dkl=None, dloss=1.0, teacher_grads=False, out=None, stream=None, kv_len=None):
    """Key gradients only: (dk_s, dk_t), the teacher one None unless teacher_grads."""
    return _bwd_part("streamkl_bwd_dk", "k", q_t, k_t, q_s, k_s, kl, lse_t, lse_s, scale_t, scale_s, causal,
                     dkl, dloss, teacher_grads, out, stream, kv_len)


def streamkl_bwd_dq(q_t, k_t, q_s, k_s, kl, lse_t, lse_s, scale_t=None, scale_s=None, causal=False, *,
                    dkl=None, dloss=1.0, teacher_grads=False, out=None, stream=None, kv_len=None):
    """Query gradients only: (dq_s, dq_t), the teacher one None unless teacher_grads."""
    return _bwd_part("streamkl_bwd_dq", "q", q_t, k_t, q_s, k_s, kl, lse_t, lse_s, scale_t, scale_s, causal,
                     dkl, dloss, teacher_grads, out, stream, kv_len)


def streamkl_loss_mean(kl, out=None, stream=None):
    """Deterministic mean of a contiguous fp32 per-row KL tensor, as a 0-d device tensor."""
    if kl.dtype != torch.float32 or not kl.is_cuda or not kl.is_contiguous():
        raise TypeError("kl must be a contiguous CUDA fp32 tensor")
    out = torch.empty((), dtype=torch.float32, device=kl.device) if out is None else out
    rc = lib().streamkl_loss_mean(_ptr(kl), kl.numel(), _ptr(out), _stream(stream))
    if rc:
        raise StreamKLError("streamkl_loss_mean", rc)
    return out


def streamkl_loss_reduce(kl, factor, out=None, stream=None):
    """factor * sum(kl) (fixed order, fp64 accumulation) as a 0-d device tensor."""
    if kl.dtype != torch.float32 or not kl.is_cuda or not kl.is_contiguous():
        raise TypeError("kl must be a contiguous CUDA fp32 tensor")
    out = torch.empty((), dtype=torch.float32, device=kl.device) if out is None else out
    rc = lib().streamkl_loss_reduce(_ptr(kl), kl.numel(), float(factor), _ptr(out), _stream(stream))
    if rc:
        raise StreamKLError("streamkl_loss_reduce", rc)
    return out


def streamkl_check(stream=None, device=None) -> int:
    """Synchronises and raises if a kernel gave up on a bounded wait; returns the status word."""
    ws = workspace(device)
    code = ctypes.c_uint(0)
    rc = lib().streamkl_check(_ptr(ws), _stream(stream), ctypes.byref(code))
    if rc:
        raise StreamKLError("streamkl_check", rc)
    return code.value
