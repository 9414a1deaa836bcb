"""The materialised baseline of the bench (torch eager, both N_Q x N_K
distributions in fp32, autograd for the gradients) against the fp64 oracle.

This is the computation the fused method replaces ("StreamKL: Fast and
Memory-Efficient KL Divergence for Boosting Attention Distillation",
abstract: existing approaches materialise both attention distributions, then
reduce).  Its speed is only a fair comparison if it computes the same thing,
so its per-row KL, mean loss and gradients meet the same tolerances as the
fused path on the two workloads it runs in seconds.
"""
import pytest
import torch

import bench
import oracle
from attention_kl_divergence_attn_b200 import inputs
from gpu_util import assert_kl, assert_grad, to_np

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("name", ["tiny_128", "causal_2k_d64"])
def test_materialised_step_matches_oracle(name):
    w = inputs.WORKLOADS[name]
    host = inputs.make_inputs(w)
    x = [t.cuda() for t in host]
    for i, t in enumerate(x):
        t.requires_grad_(i >= 2 or w.teacher_grads)
    kl, loss = bench.materialised_step(x, w, bench.materialised_mask(w, x[0].device))
    rkl, _, _ = oracle.fwd(*host, w.scale_t, w.scale_s, w.causal)
    assert_kl(to_np(kl), rkl, name + " materialised")
    assert abs(float(loss) - rkl.mean()) <= 1e-4 + 1e-3 * abs(rkl.mean())
    r = oracle.bwd(*host, w.scale_t, w.scale_s, w.causal, g=1.0 / w.rows, teacher=w.teacher_grads)
    assert_grad(to_np(x[2].grad), r[0], name + " materialised dq_s")
    assert_grad(to_np(x[3].grad), r[1], name + " materialised dk_s")
