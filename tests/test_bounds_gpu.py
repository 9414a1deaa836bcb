"""The bounds-checked debug build on the GPU.

libstreamkl_checked.so is the library built with STREAMKL_CHECK_BOUNDS: every
TMA coordinate (innermost coordinate a multiple of 64 inside the row, first
row and head inside the tensor), every raw global load and every output store
the kernels compute is checked against its tensor, and a violation skips the
access and sets a bit in the status word (streamkl_check ->
STREAMKL_ERR_BOUNDS) instead of faulting.  It stands in for a memory checker
on a pool where none may run.  These tests drive every kernel form through it
on shapes with ragged tails, causal masks with N_Q < N_K, key splits, padding
and grouped key heads, and require a clean status word and the same results
as the regular library (and as the oracle).
"""
import contextlib

import numpy as np
import pytest
import torch

import oracle
import attention_kl_divergence_attn_b200 as skl
from attention_kl_divergence_attn_b200 import build as kbuild, inputs
from gpu_util import assert_kl, assert_grad, to_np, cuda, rel_l2

pytestmark = pytest.mark.gpu


@contextlib.contextmanager
def library(path):
    """Runs the binding's calls against another build of the C ABI."""
    saved = (skl._lib, skl.LIB_PATH)
    skl._lib, skl.LIB_PATH = None, path
    try:
        yield skl.lib()
    finally:
        skl._lib, skl.LIB_PATH = saved


def run(w, x, teacher, lens):
    out = skl.streamkl_fwd(*x, w.scale_t, w.scale_s, w.causal, kv_len=lens)
    grads = skl.streamkl_bwd(*x, *out[:3], w.scale_t, w.scale_s, w.causal, teacher_grads=teacher, kv_len=lens)
    return [t for t in out[:3]] + [g for g in grads if g is not None]


CASES = [
    # (B, H, H_kt, H_ks, N_Q, N_K, d_t, d_s, causal, teacher, kv_lens)
    (1, 2, 2, 2, 300, 300, 64, 64, True, True, ()),            # persistent key-owner, ragged tail
    (2, 1, 1, 1, 200, 517, 128, 128, False, True, ()),         # one-item key-owner (teacher, d = 128)
    (1, 3, 3, 3, 257, 700, 128, 64, True, True, ()),           # N_Q < N_K causal, mixed heads
    (1, 1, 1, 1, 1, 1, 64, 64, False, True, ()),               # one query, one key
    (1, 2, 2, 2, 64, 1000, 128, 128, True, False, ()),         # persistent, student-only d = 128
    (1, 2, 2, 2, 256, 20000, 128, 64, False, False, ()),       # key splits (forward and query-owner)
    (3, 4, 2, 1, 190, 410, 128, 128, True, True, (410, 77, 0)),  # padding and grouped heads, one-item padded
    (2, 4, 4, 2, 130, 300, 64, 128, False, False, (299, 5)),   # padding, grouped student heads, persistent
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "x".join(map(str, c[:10])) + "_" + "-".join(map(str, c[10])))
def test_checked_build_finds_every_access_in_bounds(case):
    B, H, H_kt, H_ks, N_Q, N_K, d_t, d_s, causal, teacher, lens = case
    w = inputs.custom(B=B, H=H, N_Q=N_Q, N_K=N_K, d_t=d_t, d_s=d_s, causal=causal, student="independent",
                      seed=31 * N_Q + N_K, h_kt=H_kt, h_ks=H_ks, kv_lens=lens)
    host = inputs.make_inputs(w)
    x = cuda(*host)
    lens_dev = None if not lens else inputs.key_lengths(w).cuda()
    ref = run(w, x, teacher, lens_dev)
    assert skl.streamkl_check() == 0
    with library(kbuild.build(checked=True)):
        got = run(w, x, teacher, lens_dev)
        code = skl.streamkl_check()          # raises on STREAMKL_ERR_BOUNDS (status 6)
    assert code == 0
    for a, b in zip(ref, got):
        fa, fb = a.double(), b.double()
        same_inf = torch.equal(torch.isinf(fa), torch.isinf(fb))
        assert same_inf
        fin = torch.isfinite(fa)
        assert rel_l2(fb[fin].cpu().numpy(), fa[fin].cpu().numpy()) <= 1e-6
    # and the checked build against the oracle
    rkl, _, _ = oracle.fwd(*host, w.scale_t, w.scale_s, causal, kv_len=list(lens) if lens else None)
    k = to_np(got[0])
    fin = np.isfinite(to_np(got[1]))
    assert_kl(k[fin], rkl[fin], "checked build")
    r = oracle.bwd(*host, w.scale_t, w.scale_s, causal, g=1.0 / w.rows, teacher=teacher,
                   kv_len=list(lens) if lens else None)
    assert_grad(to_np(got[3]), r[0], "checked dq_s")
    assert_grad(to_np(got[4]), r[1], "checked dk_s")


def test_checked_build_is_a_separate_library():
    # the regular library must not carry the checks (they cost registers in the
    # tile loops): the two files differ and the regular one is the one loaded
    regular = kbuild.build()
    checked = kbuild.build(checked=True)
    assert regular != checked
    assert open(regular, "rb").read() != open(checked, "rb").read()
    assert skl.LIB_PATH == regular
