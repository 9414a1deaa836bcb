"""A seeded sweep of random problem shapes on the GPU, each against the fp64 oracle.

The other GPU tests pick their shapes by hand (tile edges, the five workloads,
the variants).  This one draws 36 problems from a fixed seed across everything
the entry points accept at once: batch and head counts, query and key lengths
from 1 to a few tiles past a multiple of the tile sizes, N_Q < N_K and (not
causal) N_Q > N_K, both head dimensions for either model, causal or not, teacher gradients
or not, grouped key heads, padding lengths and a per-row upstream gradient.
Every draw runs the forward and the full backward through the binding and is
compared element by element with the oracle (per-row KL and log-sum-exps,
whole-tensor relative L2 of every gradient), so that a kernel form, a tile
count or a hand-off schedule that only some shapes reach (one or two key tiles,
a key-owner item with a single query tile, the last ragged tile of a tail)
cannot go unchecked.
"""
import random

import numpy as np
import pytest
import torch

import oracle
from attention_kl_divergence_attn_b200 import inputs, streamkl_fwd, streamkl_bwd, streamkl_check
from gpu_util import assert_kl, assert_lse, assert_grad, to_np, cuda

pytestmark = pytest.mark.gpu


def draw(i):
    r = random.Random(5150 + i)
    B = r.choice([1, 1, 2, 3])
    H = r.choice([1, 2, 4])
    group_t = r.choice([d for d in (1, 2, 4) if H % d == 0])
    group_s = r.choice([d for d in (1, 2, 4) if H % d == 0])
    lengths = [1, 2, 63, 64, 65, 127, 128, 129, 191, 200, 257, 300, 383, 511]
    N_Q = r.choice(lengths)
    N_K = r.choice(lengths + [640, 1000])
    causal = r.random() < 0.5
    if causal and N_Q > N_K:            # the entry points reject it (rows with no key)
        N_Q, N_K = N_K, N_Q
    kv = ()
    if r.random() < 0.3:
        kv = tuple(r.choice([0, 1, N_K // 2, N_K - 1, N_K]) for _ in range(B))
    d_t, d_s = r.choice([64, 128]), r.choice([64, 128])
    h_kt, h_ks = H // group_t, H // group_s
    # a student drawn as the teacher plus noise needs the teacher's shapes
    student = r.choice(["noise", "independent"]) if (d_t, h_kt) == (d_s, h_ks) else "independent"
    return inputs.custom(f"sweep{i}", B=B, H=H, N_Q=N_Q, N_K=N_K, d_t=d_t, d_s=d_s, causal=causal,
                         student=student, teacher_grads=r.random() < 0.5, seed=7000 + i, h_kt=h_kt, h_ks=h_ks,
                         kv_lens=kv), r.random() < 0.5


@pytest.mark.parametrize("i", range(36))
def test_random_problem_matches_oracle(i):
    w, per_row_g = draw(i)
    host = inputs.make_inputs(w)
    x = cuda(*host)
    lens = list(w.kv_lens) if w.kv_lens else None
    lens_dev = inputs.key_lengths(w).cuda() if w.kv_lens else None
    kl, lt, ls, loss = streamkl_fwd(*x, w.scale_t, w.scale_s, w.causal, kv_len=lens_dev)
    assert streamkl_check() == 0
    rkl, rlt, rls = oracle.fwd(*host, w.scale_t, w.scale_s, w.causal, kv_len=lens)
    k, t, s = to_np(kl), to_np(lt), to_np(ls)
    empty = np.isneginf(rlt)                      # rows with no visible key
    assert np.array_equal(np.isneginf(t), empty)
    assert np.all(k[empty] == 0)
    assert_kl(k[~empty], rkl[~empty], w.name)
    assert_lse(t[~empty], rlt[~empty], w.name + " lse_t")
    assert_lse(s[~empty], rls[~empty], w.name + " lse_s")
    assert abs(float(loss) - rkl.mean()) <= 1e-4 + 1e-3 * abs(rkl.mean())

    if per_row_g:
        g = torch.randn(w.B, w.H, w.N_Q, generator=torch.Generator().manual_seed(w.seed)) / w.rows
        dkl, dloss, g_ref = g.cuda(), 0.0, g.double().numpy()
    else:
        dkl, dloss, g_ref = None, 1.0, 1.0 / w.rows
    dqs, dks, dqt, dkt = streamkl_bwd(*x, kl, lt, ls, w.scale_t, w.scale_s, w.causal, dkl=dkl, dloss=dloss,
                                      teacher_grads=w.teacher_grads, kv_len=lens_dev)
    assert streamkl_check() == 0
    r = oracle.bwd(*host, w.scale_t, w.scale_s, w.causal, g=g_ref, teacher=w.teacher_grads, kv_len=lens)
    assert_grad(to_np(dqs), r[0], w.name + " dq_s")
    assert_grad(to_np(dks), r[1], w.name + " dk_s")
    if w.teacher_grads:
        assert_grad(to_np(dqt), r[2], w.name + " dq_t")
        assert_grad(to_np(dkt), r[3], w.name + " dk_t")
