"""GPU forward vs the fp64 oracle, element by element, on seeded inputs.

Covers several 128-row/128-key tiles with ragged tails, causal and
non-causal masks, every supported (d_t, d_s) pair, the degenerate cases
(one key, one query row, N_Q < N_K causal), and the five named workloads
(full for the small ones, sampled rows for the large ones).
"""
import numpy as np
import pytest
import torch

import oracle
from attention_kl_divergence_attn_b200 import inputs, streamkl_fwd, streamkl_check
from gpu_util import assert_kl, assert_lse, to_np, cuda

pytestmark = pytest.mark.gpu


def run_and_compare(w):
    qt, kt, qs, ks = inputs.make_inputs(w)
    kl, lt, ls, loss = streamkl_fwd(*cuda(qt, kt, qs, ks), w.scale_t, w.scale_s, w.causal)
    assert streamkl_check() == 0
    rkl, rlt, rls = oracle.fwd(qt, kt, qs, ks, w.scale_t, w.scale_s, w.causal)
    assert_kl(to_np(kl), rkl, w.name)
    assert_lse(to_np(lt), rlt, w.name + " lse_t")
    assert_lse(to_np(ls), rls, w.name + " lse_s")
    assert abs(float(loss) - rkl.mean()) <= 1e-4 + 1e-3 * abs(rkl.mean())
    return kl


SHAPES = [
    # (B, H, N_Q, N_K, d_t, d_s, causal, student)
    (1, 1, 128, 128, 64, 64, False, "noise"),
    (1, 2, 300, 300, 64, 64, True, "noise"),
    (2, 1, 200, 517, 128, 128, False, "independent"),
    (1, 3, 257, 700, 128, 64, True, "independent"),
    (1, 1, 130, 390, 64, 128, False, "independent"),
    (1, 1, 1, 1, 64, 64, False, "independent"),
    (1, 1, 1, 513, 128, 128, True, "independent"),
    (1, 1, 129, 129, 64, 64, True, "noise"),
    (1, 2, 64, 1000, 64, 64, True, "independent"),
]


@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: "x".join(map(str, s)))
def test_fwd_small_shapes(shape):
    B, H, N_Q, N_K, d_t, d_s, causal, student = shape
    w = inputs.custom(B=B, H=H, N_Q=N_Q, N_K=N_K, d_t=d_t, d_s=d_s, causal=causal,
                      student=student, teacher_std=1.5, student_std=1.5, noise_std=0.3, seed=N_Q + N_K)
    run_and_compare(w)


def test_fwd_self_kl_is_zero():
    w = inputs.custom(B=1, H=2, N_Q=384, N_K=384, d_t=128, d_s=128, causal=True, seed=3)
    qt, kt = cuda(*inputs.make_inputs(w)[:2])
    kl, lt, ls, _ = streamkl_fwd(qt, kt, qt, kt, 0.1, 0.1, True)
    assert float(kl.abs().max()) < 1e-5
    assert torch.equal(lt, ls)           # teacher and student take identical paths


def test_fwd_deterministic():
    w = inputs.custom(B=1, H=4, N_Q=640, N_K=640, d_t=64, d_s=64, causal=True, student="independent", seed=5)
    t = cuda(*inputs.make_inputs(w))
    a = streamkl_fwd(*t, w.scale_t, w.scale_s, True)
    b = streamkl_fwd(*t, w.scale_t, w.scale_s, True)
    for x, y in zip(a, b):
        assert torch.equal(x, y)


def test_fwd_tiny_workload():
    run_and_compare(inputs.WORKLOADS["tiny_128"])


def test_fwd_causal_2k_workload():
    run_and_compare(inputs.WORKLOADS["causal_2k_d64"])


# Sampling of the large workloads: every row of 2 whole heads (8k, cross) or 1
# (32k), plus 256 seeded rows across all heads and the first and last rows.
@pytest.mark.parametrize("name,head_sample", [("causal_8k_d128", 2), ("causal_32k_d128", 1), ("cross_1k_64k", 2)])
def test_fwd_large_workload_sampled_rows(name, head_sample):
    w = inputs.WORKLOADS[name]
    qt, kt, qs, ks = inputs.make_inputs(w)
    kl, lt, ls, loss = streamkl_fwd(*cuda(qt, kt, qs, ks), w.scale_t, w.scale_s, w.causal)
    assert streamkl_check() == 0
    rows = inputs.sample_rows(w, 256).numpy()
    # include the first and last row of the first head and of the last head
    rows = np.unique(np.concatenate([rows, [0, w.N_Q - 1, w.rows - w.N_Q, w.rows - 1]]))
    ref = oracle.sampled_rows(w, rows)
    assert_kl(to_np(kl).ravel()[rows], ref["kl"], name)
    assert_lse(to_np(lt).ravel()[rows], ref["lse_t"], name + " lse_t")
    assert_lse(to_np(ls).ravel()[rows], ref["lse_s"], name + " lse_s")
    for (b, h) in inputs.sample_heads(w, head_sample):
        hq = [x[None, None] for x in inputs.head_inputs(w, b, h)]
        rkl, rlt, rls = oracle.fwd(*hq, w.scale_t, w.scale_s, w.causal)
        assert_kl(to_np(kl[b, h]), rkl, f"{name} head {b},{h}")
        assert_lse(to_np(lt[b, h]), rlt, f"{name} head {b},{h} lse_t")
        assert_lse(to_np(ls[b, h]), rls, f"{name} head {b},{h} lse_s")
    k = to_np(kl)
    assert np.isfinite(k).all() and k.min() > -1e-3
    assert abs(float(loss) - k.mean()) <= 1e-5 * max(1.0, abs(k.mean()))
