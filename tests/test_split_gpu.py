"""Key-split path (few query tiles, long key ranges) vs the fp64 oracle.

When a problem has too few 128-row query tiles to fill the GPU, the forward
and the query-side backward cut each tile's key range into pieces that run as
separate CTAs and are combined afterwards (the associative merge of the
online row states; a fixed-order sum of dQ partials).  These tests pick shapes
that split, check them against the oracle, check that the split and unsplit
forward agree to rounding, and that split results repeat bit for bit.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from attention_kl_divergence_attn_b200 import (inputs, lib, streamkl_bwd, streamkl_check, streamkl_fwd,
                                               workspace_size)
from gpu_util import assert_grad, assert_kl, assert_lse, cuda, to_np

pytestmark = pytest.mark.gpu

SPLIT_SHAPES = [
    # (B, H, N_Q, N_K, d_t, d_s, causal)
    (1, 2, 200, 12000, 64, 64, False),
    (2, 1, 130, 9000, 128, 64, True),
    (1, 1, 1, 5000, 64, 128, False),
    (1, 3, 384, 7000, 128, 128, False),
]


def _unsplit_fwd(t, w):
    """streamkl_fwd with the 256-byte minimum workspace, which never splits."""
    B, H, N_Q, _ = t[0].shape
    N_K = t[1].shape[2]
    kl = torch.empty(B, H, N_Q, device="cuda")
    lt, ls = torch.empty_like(kl), torch.empty_like(kl)
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    P = lambda x: ctypes.c_void_p(x.data_ptr())
    rc = lib().streamkl_fwd(P(t[0]), P(t[1]), P(t[2]), P(t[3]), B, H, N_Q, N_K, t[0].shape[3], t[2].shape[3],
                            w.scale_t, w.scale_s, int(w.causal), P(kl), P(lt), P(ls), None, P(ws), 256,
                            ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == 0
    torch.cuda.synchronize()
    assert int(ws[:4].view(torch.int32).item()) == 0
    return kl, lt, ls


@pytest.mark.parametrize("shape", SPLIT_SHAPES, ids=lambda s: "x".join(map(str, s)))
def test_split_forward_and_backward(shape):
    B, H, N_Q, N_K, d_t, d_s, causal = shape
    assert workspace_size(B, H, N_Q, N_K, d_t, d_s, causal) > 256, "shape does not split on this GPU"
    w = inputs.custom(B=B, H=H, N_Q=N_Q, N_K=N_K, d_t=d_t, d_s=d_s, causal=causal, student="independent",
                      teacher_std=2.0, student_std=2.0, seed=N_K + N_Q)
    qt, kt, qs, ks = inputs.make_inputs(w)
    t = cuda(qt, kt, qs, ks)
    kl, lt, ls, loss = streamkl_fwd(*t, w.scale_t, w.scale_s, causal)
    kl2, lt2, ls2, _ = streamkl_fwd(*t, w.scale_t, w.scale_s, causal)
    assert streamkl_check() == 0
    assert torch.equal(kl, kl2) and torch.equal(lt, lt2) and torch.equal(ls, ls2)
    r_kl, r_lt, r_ls = oracle.fwd(qt, kt, qs, ks, w.scale_t, w.scale_s, causal)
    assert_kl(to_np(kl), r_kl, "split kl")
    assert_lse(to_np(lt), r_lt, "split lse_t")
    assert_lse(to_np(ls), r_ls, "split lse_s")
    assert abs(float(loss) - float(np.mean(r_kl))) <= 1e-4 + 1e-3 * abs(float(np.mean(r_kl)))
    # the unsplit forward on the same inputs: same values up to the order of rounding
    u_kl, u_lt, u_ls = _unsplit_fwd(t, w)
    assert torch.allclose(kl, u_kl, rtol=1e-4, atol=1e-5)
    assert torch.allclose(lt, u_lt, rtol=1e-6, atol=1e-5) and torch.allclose(ls, u_ls, rtol=1e-6, atol=1e-5)

    g = torch.randn(B, H, N_Q, generator=torch.Generator().manual_seed(3)) / (B * H * N_Q)
    dqs, dks, dqt, dkt = streamkl_bwd(*t, kl, lt, ls, w.scale_t, w.scale_s, causal, dkl=g.cuda(),
                                      teacher_grads=True)
    dqs2, _, dqt2, _ = streamkl_bwd(*t, kl, lt, ls, w.scale_t, w.scale_s, causal, dkl=g.cuda(),
                                    teacher_grads=True)
    assert streamkl_check() == 0
    assert torch.equal(dqs, dqs2) and torch.equal(dqt, dqt2)
    r = oracle.bwd(qt, kt, qs, ks, w.scale_t, w.scale_s, causal, g=g.double().numpy(), teacher=True)
    assert_grad(to_np(dqs), r[0], "split dq_s")
    assert_grad(to_np(dks), r[1], "split dk_s")
    assert_grad(to_np(dqt), r[2], "split dq_t")
    assert_grad(to_np(dkt), r[3], "split dk_t")
