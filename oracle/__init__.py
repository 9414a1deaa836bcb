"""Python front of the fp64 attention-KL oracle (test infrastructure only).

Only ``tests/``, ``__graft_entry__.smoke()`` and the bench's CPU-baseline leg
may import this package.  The product path never does: it has no CPU fallback.

The arithmetic lives in ``streamkl_oracle.c`` (plain C, fp64, one materialised
row at a time); this file only builds it with gcc, marshals numpy arrays and
regenerates sampled heads.  Nothing here imports the CUDA package except its
seeded input generator module, which holds no arithmetic of the method.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "streamkl_oracle.c")
_LIB = os.path.join(_HERE, "libstreamkl_oracle.so")
_lock = threading.Lock()
_lib = None

_D = ctypes.POINTER(ctypes.c_double)
_I64 = ctypes.POINTER(ctypes.c_int64)
_I32 = ctypes.POINTER(ctypes.c_int32)


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (no fast-math, no FMA contraction)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".{os.getpid()}.tmp"
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-pthread",
                               "-ffp-contract=off", "-fno-fast-math", _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def lib():
    global _lib
    with _lock:
        if _lib is None:
            build()
            L = ctypes.CDLL(_LIB)
            shape = [ctypes.c_int] * 6 + [ctypes.c_double, ctypes.c_double, ctypes.c_int,
                                          ctypes.c_int, ctypes.c_int, _I32]
            L.streamkl_oracle_fwd.argtypes = [_D] * 4 + shape + [_D] * 3 + [ctypes.c_int]
            L.streamkl_oracle_fwd.restype = ctypes.c_int
            L.streamkl_oracle_bwd.argtypes = [_D] * 4 + shape + [_D] + [_D] * 4 + [ctypes.c_int]
            L.streamkl_oracle_bwd.restype = ctypes.c_int
            L.streamkl_oracle_rows.argtypes = ([_D] * 4 + shape + [_I64, ctypes.c_int64, _D]
                                               + [_D] * 5 + [ctypes.c_int])
            L.streamkl_oracle_rows.restype = ctypes.c_int
            L.streamkl_oracle_bwd_rows.argtypes = ([_D] * 4 + shape + [_D, _I64, ctypes.c_int64]
                                                   + [_D] * 4 + [ctypes.c_int])
            L.streamkl_oracle_bwd_rows.restype = ctypes.c_int
            L.streamkl_oracle_mean.argtypes = [_D, ctypes.c_int64]
            L.streamkl_oracle_mean.restype = ctypes.c_double
            _lib = L
    return _lib


def _f64(a) -> np.ndarray:
    """Exact upcast of a torch/numpy array (bf16 included) to C-contiguous fp64."""
    if hasattr(a, "detach"):                      # torch tensor
        a = a.detach().cpu().double().numpy()
    return np.ascontiguousarray(a, dtype=np.float64)


def _p(a):
    return None if a is None else a.ctypes.data_as(_D)


def _shape(qt, kt, qs, ks):
    """(B, H, N_Q, N_K, d_t, d_s, H_kt, H_ks): queries [B, H, N_Q, d], keys [B, H_k, N_K, d]."""
    B, H, N_Q, d_t = qt.shape
    H_kt, N_K = kt.shape[1], kt.shape[2]
    d_s = qs.shape[3]
    H_ks = ks.shape[1]
    assert kt.shape == (B, H_kt, N_K, d_t) and qs.shape == (B, H, N_Q, d_s) and ks.shape == (B, H_ks, N_K, d_s)
    return B, H, N_Q, N_K, d_t, d_s, H_kt, H_ks


def _lens(kv_len, B):
    """Per-batch key lengths as a C int32 array (or None for no padding)."""
    if kv_len is None:
        return None
    a = np.ascontiguousarray(np.asarray(kv_len, dtype=np.int32).ravel())
    assert a.size == B, "one key length per batch element"
    return a


def _pi(a):
    return None if a is None else a.ctypes.data_as(_I32)


def fwd(qt, kt, qs, ks, scale_t, scale_s, causal, nthreads=0, kv_len=None):
    """Per-row (KL, LSE_t, LSE_s), each [B,H,N_Q] fp64.

    Keys may have fewer heads than queries (grouped key heads: query head h
    reads key head h / (H / H_k)); ``kv_len`` (one length per batch element)
    hides the keys at and past it.
    """
    qt, kt, qs, ks = map(_f64, (qt, kt, qs, ks))
    B, H, N_Q, N_K, d_t, d_s, H_kt, H_ks = _shape(qt, kt, qs, ks)
    lens = _lens(kv_len, B)
    kl = np.zeros((B, H, N_Q)); lt = np.zeros_like(kl); ls = np.zeros_like(kl)
    rc = lib().streamkl_oracle_fwd(_p(qt), _p(kt), _p(qs), _p(ks), B, H, N_Q, N_K, d_t, d_s,
                                   float(scale_t), float(scale_s), int(bool(causal)), H_kt, H_ks, _pi(lens),
                                   _p(kl), _p(lt), _p(ls), int(nthreads))
    if rc:
        raise ValueError(f"oracle fwd rejected the arguments (rc={rc})")
    return kl, lt, ls


def bwd(qt, kt, qs, ks, scale_t, scale_s, causal, g, teacher=True, nthreads=0, kv_len=None):
    """Gradients (dQ_s, dK_s, dQ_t, dK_t) for per-row upstream gradient g.

    ``g`` is a [B,H,N_Q] array or a scalar applied to every row.  With
    ``teacher=False`` the teacher gradients come back as None.
    """
    qt, kt, qs, ks = map(_f64, (qt, kt, qs, ks))
    B, H, N_Q, N_K, d_t, d_s, H_kt, H_ks = _shape(qt, kt, qs, ks)
    lens = _lens(kv_len, B)
    g = np.ascontiguousarray(np.broadcast_to(np.asarray(g, dtype=np.float64), (B, H, N_Q)))
    dqs = np.zeros_like(qs); dks = np.zeros_like(ks)
    dqt = np.zeros_like(qt) if teacher else None
    dkt = np.zeros_like(kt) if teacher else None
    rc = lib().streamkl_oracle_bwd(_p(qt), _p(kt), _p(qs), _p(ks), B, H, N_Q, N_K, d_t, d_s,
                                   float(scale_t), float(scale_s), int(bool(causal)), H_kt, H_ks, _pi(lens), _p(g),
                                   _p(dqs), _p(dks), _p(dqt), _p(dkt), int(nthreads))
    if rc:
        raise ValueError(f"oracle bwd rejected the arguments (rc={rc})")
    return dqs, dks, dqt, dkt


def rows(qt, kt, qs, ks, scale_t, scale_s, causal, row_ids, g=None, teacher=False, nthreads=0, kv_len=None):
    """KL, LSE_t, LSE_s (and dQ_s, dQ_t when g is given) for the listed flat rows.

    Returns a dict of arrays with one entry per listed row.
    """
    qt, kt, qs, ks = map(_f64, (qt, kt, qs, ks))
    B, H, N_Q, N_K, d_t, d_s, H_kt, H_ks = _shape(qt, kt, qs, ks)
    lens = _lens(kv_len, B)
    r = np.ascontiguousarray(np.asarray(row_ids, dtype=np.int64))
    kl = np.zeros(B * H * N_Q); lt = np.zeros_like(kl); ls = np.zeros_like(kl)
    gg = None
    dqs = dqt = None
    if g is not None:
        gg = np.ascontiguousarray(np.broadcast_to(np.asarray(g, dtype=np.float64), (B * H * N_Q,)))
        dqs = np.zeros_like(qs)
        dqt = np.zeros_like(qt) if teacher else None
    rc = lib().streamkl_oracle_rows(_p(qt), _p(kt), _p(qs), _p(ks), B, H, N_Q, N_K, d_t, d_s,
                                    float(scale_t), float(scale_s), int(bool(causal)), H_kt, H_ks, _pi(lens),
                                    r.ctypes.data_as(_I64), int(r.size), _p(gg),
                                    _p(kl), _p(lt), _p(ls), _p(dqs), _p(dqt), int(nthreads))
    if rc:
        raise ValueError(f"oracle rows rejected the arguments (rc={rc})")
    out = {"kl": kl[r], "lse_t": lt[r], "lse_s": ls[r]}
    if g is not None:
        out["dq_s"] = dqs.reshape(B * H * N_Q, d_s)[r]
        if teacher:
            out["dq_t"] = dqt.reshape(B * H * N_Q, d_t)[r]
    return out


def bwd_rows(qt, kt, qs, ks, scale_t, scale_s, causal, g, row_ids, teacher=True, nthreads=0, kv_len=None):
    """Backward over the listed flat rows only: their dQ rows and their dK contributions."""
    qt, kt, qs, ks = map(_f64, (qt, kt, qs, ks))
    B, H, N_Q, N_K, d_t, d_s, H_kt, H_ks = _shape(qt, kt, qs, ks)
    lens = _lens(kv_len, B)
    g = np.ascontiguousarray(np.broadcast_to(np.asarray(g, dtype=np.float64), (B, H, N_Q)))
    r = np.ascontiguousarray(np.asarray(row_ids, dtype=np.int64))
    dqs = np.zeros_like(qs); dks = np.zeros_like(ks)
    dqt = np.zeros_like(qt) if teacher else None
    dkt = np.zeros_like(kt) if teacher else None
    rc = lib().streamkl_oracle_bwd_rows(_p(qt), _p(kt), _p(qs), _p(ks), B, H, N_Q, N_K, d_t, d_s,
                                        float(scale_t), float(scale_s), int(bool(causal)), H_kt, H_ks, _pi(lens), _p(g),
                                        r.ctypes.data_as(_I64), int(r.size),
                                        _p(dqs), _p(dks), _p(dqt), _p(dkt), int(nthreads))
    if rc:
        raise ValueError(f"oracle bwd_rows rejected the arguments (rc={rc})")
    return dqs, dks, dqt, dkt


def mean(kl) -> float:
    kl = np.ascontiguousarray(np.asarray(kl, dtype=np.float64)).ravel()
    return float(lib().streamkl_oracle_mean(_p(kl), int(kl.size)))


def sampled_rows(w, row_ids, g=None, teacher=False, nthreads=0):
    """Oracle values for flat rows of a workload, regenerating only their heads.

    ``w`` is an ``inputs.Workload``; each listed row's head is redrawn with the
    shared seeded generator and evaluated as a B=H=1 problem.  Returns a dict of
    arrays in the order of ``row_ids``.
    """
    from attention_kl_divergence_attn_b200 import inputs as _inputs

    row_ids = np.asarray(row_ids, dtype=np.int64)
    by_head = {}
    for k, r in enumerate(row_ids.tolist()):
        bh, i = divmod(r, w.N_Q)
        by_head.setdefault(bh, []).append((k, i))
    n = row_ids.size
    out = {"kl": np.zeros(n), "lse_t": np.zeros(n), "lse_s": np.zeros(n)}
    if g is not None:
        out["dq_s"] = np.zeros((n, w.d_s))
        if teacher:
            out["dq_t"] = np.zeros((n, w.d_t))
    for bh, items in by_head.items():
        b, h = divmod(bh, w.H)
        qt, kt, qs, ks = (t[None, None] for t in _inputs.head_inputs(w, b, h))
        idx = [i for _, i in items]
        gr = None
        if g is not None:
            gr = np.zeros(w.N_Q)
            gr[idx] = np.asarray(g, dtype=np.float64).ravel()[[bh * w.N_Q + i for i in idx]] \
                if np.ndim(g) else float(g)
        lens = [w.kv_lens[b]] if w.kv_lens else None
        res = rows(qt, kt, qs, ks, w.scale_t, w.scale_s, w.causal, idx, g=gr,
                   teacher=teacher, nthreads=nthreads, kv_len=lens)
        for key in res:
            out[key][[k for k, _ in items]] = res[key]
    return out
