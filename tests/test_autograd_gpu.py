"""The autograd wrapper (temperature, T^2 scaling, reductions) vs the oracle.

At temperature T the wrapper's loss is T^2 times the reduced KL of the
distributions softened by T ("Lecture 05 - Where It All Lands ...", section
3.3), so the oracle is run with scales divided by T and its results are
scaled by T^2 (loss) and by T^2 times the upstream gradient (gradients).
"""
import numpy as np
import pytest
import torch

import oracle
from attention_kl_divergence_attn_b200 import inputs, streamkl_check, streamkl_fwd
from attention_kl_divergence_attn_b200.autograd import streamkl_loss
from gpu_util import assert_grad, assert_kl, to_np

pytestmark = pytest.mark.gpu

CASES = [
    # (B, H, N_Q, N_K, d_t, d_s, causal, T, teacher)
    (1, 2, 200, 200, 64, 64, True, 2.0, True),
    (2, 1, 130, 333, 128, 64, False, 0.5, False),
    (1, 1, 257, 257, 128, 128, True, 1.0, True),
]


def _setup(case, requires_teacher):
    B, H, N_Q, N_K, d_t, d_s, causal, T, _ = case
    w = inputs.custom(B=B, H=H, N_Q=N_Q, N_K=N_K, d_t=d_t, d_s=d_s, causal=causal,
                      student="noise" if d_t == d_s else "independent",
                      teacher_std=1.5, student_std=1.5, noise_std=0.4, seed=N_Q + 11 * N_K)
    qt, kt, qs, ks = inputs.make_inputs(w)
    g = [x.cuda().requires_grad_(i >= 2 or requires_teacher) for i, x in enumerate((qt, kt, qs, ks))]
    st, ss = w.scale_t / T, w.scale_s / T
    return w, (qt, kt, qs, ks), g, st, ss


@pytest.mark.parametrize("reduction", ["mean", "sum", "none"])
@pytest.mark.parametrize("case", CASES, ids=lambda c: "x".join(map(str, c)))
def test_autograd_matches_oracle(case, reduction):
    B, H, N_Q, N_K, d_t, d_s, causal, T, teacher = case
    w, (qt, kt, qs, ks), (gqt, gkt, gqs, gks), st, ss = _setup(case, teacher)
    n = B * H * N_Q
    r_kl, _, _ = oracle.fwd(qt, kt, qs, ks, st, ss, causal)
    out = streamkl_loss(gqt, gkt, gqs, gks, causal=causal, temperature=T, reduction=reduction)
    if reduction == "none":
        assert_kl(to_np(out), r_kl, "per-row kl")
        wts = torch.randn(B, H, N_Q, generator=torch.Generator().manual_seed(5))
        (out * wts.cuda()).sum().backward()
        g_ref = wts.double().numpy()
    else:
        ref = T * T * (np.mean(r_kl) if reduction == "mean" else np.sum(r_kl))
        assert abs(float(out.detach()) - ref) <= 1e-4 * (n if reduction == "sum" else 1) + 1e-3 * abs(ref)
        up = 0.75
        out.backward(torch.tensor(up, device="cuda"))
        g_ref = np.full((B, H, N_Q), up * T * T / (n if reduction == "mean" else 1.0))
    assert streamkl_check() == 0
    r = oracle.bwd(qt, kt, qs, ks, st, ss, causal, g=g_ref, teacher=teacher)
    assert gqs.grad.dtype == torch.bfloat16
    assert_grad(to_np(gqs.grad), r[0], "dq_s")
    assert_grad(to_np(gks.grad), r[1], "dk_s")
    if teacher:
        assert_grad(to_np(gqt.grad), r[2], "dq_t")
        assert_grad(to_np(gkt.grad), r[3], "dk_t")
    else:
        assert gqt.grad is None and gkt.grad is None


def test_mean_loss_equals_forward_loss_at_t1():
    w = inputs.custom(B=1, H=2, N_Q=256, N_K=256, d_t=64, d_s=64, causal=True, student="noise", seed=4)
    t = [x.cuda() for x in inputs.make_inputs(w)]
    loss = streamkl_loss(*t, causal=True)
    _, _, _, ref = streamkl_fwd(*t, w.scale_t, w.scale_s, True)
    assert torch.equal(loss, ref)     # same kernel, same fixed summation order, factor 1/n vs mean
