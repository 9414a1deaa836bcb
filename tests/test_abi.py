"""The C-ABI library loads on a machine without a GPU, exports every function
declared in include/streamkl.h, and rejects bad arguments before touching the
device (no compute call is made here)."""
import ctypes
import os
import re

import pytest

from attention_kl_divergence_attn_b200 import build as kbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    kbuild.build()
    import attention_kl_divergence_attn_b200 as skl
    return skl.lib()


def declared_functions():
    names = []
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            text = open(os.path.join(ROOT, "include", fn)).read()
            text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
            names += re.findall(r"\b(streamkl_[a-z0-9_]+)\s*\(", text)
    return sorted(set(names))


def test_every_declared_symbol_is_exported(L):
    names = declared_functions()
    assert "streamkl_fwd" in names and "streamkl_bwd" in names
    for n in names:
        assert hasattr(L, n), n


def test_version_and_strerror(L):
    assert L.streamkl_version() >= 100
    for code in range(7):
        assert L.streamkl_strerror(code)
    assert b"unknown" not in L.streamkl_strerror(6)
    assert L.streamkl_workspace_size(1, 1, 128, 128, 64, 64, 0) >= 4


def _fwd(L, **kw):
    a = dict(B=1, H=1, N_Q=128, N_K=128, d_t=64, d_s=64, st=0.125, ss=0.125, causal=0, ws=16, wsb=256)
    a.update(kw)
    p = ctypes.c_void_p(16)
    return L.streamkl_fwd(p, p, p, p, a["B"], a["H"], a["N_Q"], a["N_K"], a["d_t"], a["d_s"], a["st"], a["ss"],
                          a["causal"], p, p, p, None, ctypes.c_void_p(a["ws"]) if a["ws"] else None, a["wsb"], None)


def _bwd(L, dq_t=None, dk_t=None, **kw):
    a = dict(B=1, H=1, N_Q=128, N_K=128, d_t=64, d_s=64, st=0.125, ss=0.125, causal=0, ws=16, wsb=256)
    a.update(kw)
    p = ctypes.c_void_p(16)
    return L.streamkl_bwd(p, p, p, p, a["B"], a["H"], a["N_Q"], a["N_K"], a["d_t"], a["d_s"], a["st"], a["ss"],
                          a["causal"], p, p, p, None, 1.0, p, p, dq_t, dk_t,
                          ctypes.c_void_p(a["ws"]) if a["ws"] else None, a["wsb"], None)


@pytest.mark.parametrize("fn", [_fwd, _bwd])
def test_argument_errors(L, fn):
    assert fn(L, d_t=96) == 2                       # unsupported head dim
    assert fn(L, d_s=256) == 2
    assert fn(L, causal=1, N_Q=200, N_K=100) == 1   # causal rows without a key
    assert fn(L, causal=2) == 1
    assert fn(L, N_Q=-1) == 1
    assert fn(L, st=0.0) == 1
    assert fn(L, ss=float("nan")) == 1
    assert fn(L, ws=0) == 5                          # no workspace
    assert fn(L, wsb=3) == 5                         # too small


def test_bwd_teacher_pair_must_match(L):
    assert _bwd(L, dq_t=ctypes.c_void_p(16), dk_t=None) == 1


def test_misaligned_pointer_rejected(L):
    p = ctypes.c_void_p(16)
    bad = ctypes.c_void_p(18)
    rc = L.streamkl_fwd(bad, p, p, p, 1, 1, 128, 128, 64, 64, 0.125, 0.125, 0, p, p, p, None, p, 256, None)
    assert rc == 1


def test_device_scalar_backward_needs_a_gradient(L):
    p = ctypes.c_void_p(16)
    rc = L.streamkl_bwd_dloss_device(p, p, p, p, 1, 1, 128, 128, 64, 64, 0.125, 0.125, 0, p, p, p, None, None, 1.0,
                                     p, p, None, None, ctypes.c_void_p(16), 256, None)
    assert rc == 1


def test_loss_reduce_argument_errors(L):
    p = ctypes.c_void_p(16)
    assert L.streamkl_loss_reduce(p, 10, float("nan"), p, None) == 1
    assert L.streamkl_loss_reduce(p, -1, 1.0, p, None) == 1
    assert L.streamkl_loss_reduce(p, 10, 1.0, None, None) == 1


@pytest.mark.skipif(__import__("torch").cuda.is_available(), reason="checks the no-device answer")
def test_workspace_size_minimum_without_gpu(L):
    # no device: no key splitting is planned, so the minimum is reported
    assert L.streamkl_workspace_size(4, 8, 1024, 65536, 128, 64, 0) == 256
    assert L.streamkl_workspace_size(0, 0, 0, 0, 0, 0, 0) == 256


def test_selftest_argument_errors(L):
    assert L.streamkl_selftest_timeout(None, 256, 10000000, None) == 5
    assert L.streamkl_selftest_timeout(ctypes.c_void_p(16), 256, 10, None) == 1            # budget too short
    assert L.streamkl_selftest_timeout(ctypes.c_void_p(16), 256, 10 ** 10, None) == 1      # above 2 s


@pytest.mark.skipif(__import__("torch").cuda.is_available(), reason="checks the no-device answer")
def test_noalloc_checks_arguments_before_any_cuda_call(L):
    # Without a GPU every CUDA call fails, so a rejected call that answers with
    # its argument error (not STREAMKL_ERR_CUDA) made no CUDA call first: it
    # neither resolved nor cleared the library's status array.
    p = ctypes.c_void_p(16)
    bad = ctypes.c_void_p(18)
    fwd = L.streamkl_fwd_noalloc
    assert fwd(p, p, p, p, 1, 1, 128, 128, 96, 64, 0.1, 0.1, 0, p, p, p, None, None, None) == 2
    assert fwd(p, p, p, p, 1, 1, 200, 100, 64, 64, 0.1, 0.1, 1, p, p, p, None, None, None) == 1
    assert fwd(bad, p, p, p, 1, 1, 128, 128, 64, 64, 0.1, 0.1, 0, p, p, p, None, None, None) == 1
    assert fwd(p, p, p, p, 1, 1, 128, 128, 64, 64, 0.1, 0.1, 0, None, p, p, None, None, None) == 1
    # a valid call reaches the device check, which fails here
    assert fwd(p, p, p, p, 1, 1, 128, 128, 64, 64, 0.1, 0.1, 0, p, p, p, None, None, None) == 3
