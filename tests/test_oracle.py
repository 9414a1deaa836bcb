"""Pins of the fp64 oracle against facts fixed outside the oracle itself.

Every check here compares the oracle with something it does not contain:
closed forms (the two-key Bernoulli case, uniform rows, a single visible key),
invariants of the KL divergence (Gibbs' inequality, KL(P||P) = 0, shift
invariance of softmax), a library routine (torch's kl_div over log_softmax and
torch autograd, in fp64), brute force (central finite differences) and an
independent re-statement of the streaming recurrence of the fused method.

Sources: "StreamKL: Fast and Memory-Efficient KL Divergence for Boosting
Attention Distillation" (abstract: fused one-pass online formulation of the
coupled two-distribution KL; tile-by-tile recompute in the backward), and
"Lecture 05 - Where It All Lands ..." section 1 (H(p,q) = H(p) + D_KL(p||q),
D_KL >= 0) and section 3.1 (forward KL, teacher in the first slot).
"""
import math

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
from attention_kl_divergence_attn_b200 import inputs


def rand(shape, seed, std=1.0):
    g = np.random.default_rng(seed)
    return g.standard_normal(shape) * std


def problem(B=1, H=2, N_Q=24, N_K=24, d_t=8, d_s=8, seed=0, std=1.0):
    return (rand((B, H, N_Q, d_t), seed, std), rand((B, H, N_K, d_t), seed + 1, std),
            rand((B, H, N_Q, d_s), seed + 2, std), rand((B, H, N_K, d_s), seed + 3, std))


def visible(N_Q, N_K, causal):
    i = np.arange(N_Q)[:, None]
    j = np.arange(N_K)[None, :]
    return (j <= i + (N_K - N_Q)) if causal else np.ones((N_Q, N_K), bool)


# ---------------------------------------------------------------- invariants

@pytest.mark.parametrize("causal", [False, True])
def test_self_kl_is_zero_and_grads_vanish(causal):
    qt, kt, _, _ = problem(seed=3)
    kl, lt, ls = oracle.fwd(qt, kt, qt, kt, 0.35, 0.35, causal)
    assert np.abs(kl).max() < 1e-13
    np.testing.assert_allclose(lt, ls, rtol=0, atol=1e-13)
    grads = oracle.bwd(qt, kt, qt, kt, 0.35, 0.35, causal, g=1.0)
    for gr in grads:
        assert np.abs(gr).max() < 1e-12


@pytest.mark.parametrize("causal", [False, True])
def test_gibbs_nonnegative(causal):
    qt, kt, qs, ks = problem(seed=5, std=2.0)
    kl, _, _ = oracle.fwd(qt, kt, qs, ks, 0.5, 0.4, causal)
    assert kl.min() > -1e-12
    assert kl.max() > 1e-3          # genuinely different distributions


def test_identical_keys_give_uniform_rows():
    # every key equal -> every logit of a row equal -> both softmaxes uniform
    qt, kt, qs, ks = problem(seed=7)
    kt[:] = kt[:, :, :1, :]
    ks[:] = ks[:, :, :1, :]
    for causal in (False, True):
        kl, lt, _ = oracle.fwd(qt, kt, qs, ks, 0.3, 0.3, causal)
        assert np.abs(kl).max() < 1e-13
        n_vis = visible(24, 24, causal).sum(1)
        s_row = 0.3 * np.einsum("bhid,bhd->bhi", qt, kt[:, :, 0, :])
        np.testing.assert_allclose(lt, s_row + np.log(n_vis), rtol=0, atol=1e-12)
        dqs, dks, dqt, dkt = oracle.bwd(qt, kt, qs, ks, 0.3, 0.3, causal, g=0.7)
        assert np.abs(dqs).max() < 1e-13 and np.abs(dqt).max() < 1e-13


def test_single_visible_key_row():
    # causal row 0 of a square problem sees only key 0: P = Q = [1], KL = 0
    qt, kt, qs, ks = problem(N_Q=9, N_K=9, seed=9)
    kl, lt, ls = oracle.fwd(qt, kt, qs, ks, 0.6, 0.45, True)
    assert np.abs(kl[..., 0]).max() < 1e-15
    np.testing.assert_allclose(lt[..., 0], 0.6 * np.einsum("bhd,bhd->bh", qt[:, :, 0], kt[:, :, 0]), atol=1e-14)
    np.testing.assert_allclose(ls[..., 0], 0.45 * np.einsum("bhd,bhd->bh", qs[:, :, 0], ks[:, :, 0]), atol=1e-14)


def test_key_shift_invariance():
    # adding one vector c to every key adds q.c to a whole logit row
    qt, kt, qs, ks = problem(seed=11)
    kl0, _, _ = oracle.fwd(qt, kt, qs, ks, 0.4, 0.4, False)
    c_t, c_s = rand(8, 100), rand(8, 101)
    kl1, _, _ = oracle.fwd(qt, kt + c_t, qs, ks + c_s, 0.4, 0.4, False)
    np.testing.assert_allclose(kl1, kl0, rtol=1e-9, atol=1e-12)


def test_dk_columns_sum_to_zero():
    # every row of dS sums to zero, so the dK rows of a head sum to zero
    qt, kt, qs, ks = problem(seed=13)
    for causal in (False, True):
        g = rand((1, 2, 24), 14)
        _, dks, _, dkt = oracle.bwd(qt, kt, qs, ks, 0.4, 0.3, causal, g=g)
        assert np.abs(dks.sum(axis=2)).max() < 1e-12
        assert np.abs(dkt.sum(axis=2)).max() < 1e-12


# ---------------------------------------------------------------- closed forms

def test_two_keys_bernoulli_closed_form():
    # N_K = 2: P = (1-p, p) with p = sigmoid(s_t1 - s_t0), same for Q; the KL of
    # two Bernoulli distributions is p ln(p/q) + (1-p) ln((1-p)/(1-q)).
    qt, kt, qs, ks = problem(N_Q=6, N_K=2, d_t=3, d_s=5, seed=17, std=1.5)
    kl, lt, ls = oracle.fwd(qt, kt, qs, ks, 0.8, 0.6, False)
    for h in range(2):
        for i in range(6):
            a = 0.8 * (qt[0, h, i] @ kt[0, h, 1] - qt[0, h, i] @ kt[0, h, 0])
            b = 0.6 * (qs[0, h, i] @ ks[0, h, 1] - qs[0, h, i] @ ks[0, h, 0])
            p, q = 1 / (1 + math.exp(-a)), 1 / (1 + math.exp(-b))
            ref = p * math.log(p / q) + (1 - p) * math.log((1 - p) / (1 - q))
            assert abs(kl[0, h, i] - ref) < 1e-13 * max(1, abs(ref))
            s0 = 0.8 * (qt[0, h, i] @ kt[0, h, 0])
            assert abs(lt[0, h, i] - (s0 + math.log1p(math.exp(a)))) < 1e-12


def test_cross_entropy_minus_entropy():
    # D_KL(P||Q) = H(P,Q) - H(P), both entropies formed from explicit
    # probability vectors (softmax by division, logs of probabilities).
    qt, kt, qs, ks = problem(N_Q=10, N_K=13, d_t=6, d_s=4, seed=19)
    kl, _, _ = oracle.fwd(qt, kt, qs, ks, 0.5, 0.7, False)
    for h in range(2):
        st = 0.5 * qt[0, h] @ kt[0, h].T
        ss = 0.7 * qs[0, h] @ ks[0, h].T
        P = np.exp(st) / np.exp(st).sum(1, keepdims=True)
        Q = np.exp(ss) / np.exp(ss).sum(1, keepdims=True)
        H_pq = -(P * np.log(Q)).sum(1)
        H_p = -(P * np.log(P)).sum(1)
        np.testing.assert_allclose(kl[0, h], H_pq - H_p, rtol=1e-10, atol=1e-13)


# ---------------------------------------------------------------- library routine

@pytest.mark.parametrize("causal,N_Q,N_K,d_t,d_s", [(False, 33, 47, 16, 8), (True, 40, 40, 8, 8),
                                                    (True, 17, 50, 12, 16)])
def test_matches_torch_kl_div_and_autograd(causal, N_Q, N_K, d_t, d_s):
    qt, kt, qs, ks = problem(B=2, H=2, N_Q=N_Q, N_K=N_K, d_t=d_t, d_s=d_s, seed=23)
    st_scale, ss_scale = 1 / math.sqrt(d_t), 1 / math.sqrt(d_s)
    g = rand((2, 2, N_Q), 24)
    T = [torch.tensor(a, dtype=torch.float64, requires_grad=True) for a in (qt, kt, qs, ks)]
    mask = torch.tensor(visible(N_Q, N_K, causal))
    S_t = st_scale * T[0] @ T[1].transpose(-1, -2)
    S_s = ss_scale * T[2] @ T[3].transpose(-1, -2)
    neg = torch.finfo(torch.float64).min
    lp = F.log_softmax(S_t.masked_fill(~mask, neg), -1)
    lq = F.log_softmax(S_s.masked_fill(~mask, neg), -1)
    kl_t = F.kl_div(lq, lp, log_target=True, reduction="none").masked_fill(~mask, 0).sum(-1)
    (kl_t * torch.tensor(g)).sum().backward()

    kl, lt, ls = oracle.fwd(qt, kt, qs, ks, st_scale, ss_scale, causal)
    np.testing.assert_allclose(kl, kl_t.detach().numpy(), rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(lt, torch.logsumexp(S_t.masked_fill(~mask, -math.inf), -1).detach().numpy(),
                               rtol=1e-12, atol=1e-12)
    dqs, dks, dqt, dkt = oracle.bwd(qt, kt, qs, ks, st_scale, ss_scale, causal, g=g)
    for mine, leaf in ((dqt, T[0]), (dkt, T[1]), (dqs, T[2]), (dks, T[3])):
        ref = leaf.grad.numpy()
        assert np.linalg.norm(mine - ref) <= 1e-10 * np.linalg.norm(ref) + 1e-14


# ---------------------------------------------------------------- brute force

@pytest.mark.parametrize("causal", [False, True])
def test_central_finite_differences(causal):
    qt, kt, qs, ks = problem(B=1, H=1, N_Q=8, N_K=8, d_t=4, d_s=4, seed=29)
    g = rand((1, 1, 8), 30)
    sc_t, sc_s = 0.7, 0.45

    def loss(a, b, c, d):
        kl, _, _ = oracle.fwd(a, b, c, d, sc_t, sc_s, causal)
        return float((kl * g).sum())

    grads = oracle.bwd(qt, kt, qs, ks, sc_t, sc_s, causal, g=g)
    base = [qt, kt, qs, ks]
    order = {0: 2, 1: 3, 2: 0, 3: 1}       # bwd returns (dQ_s, dK_s, dQ_t, dK_t)
    h = 1e-6
    for which in range(4):
        an = grads[order[which]]
        fd = np.zeros_like(base[which])
        for idx in np.ndindex(*base[which].shape):
            plus = [x.copy() for x in base]
            minus = [x.copy() for x in base]
            plus[which][idx] += h
            minus[which][idx] -= h
            fd[idx] = (loss(*plus) - loss(*minus)) / (2 * h)
        assert np.linalg.norm(an - fd) <= 1e-6 * np.linalg.norm(fd) + 1e-9, which


# ---------------------------------------------------------------- streaming identity

def streaming_kl(st, ss, widths, order):
    """Online coupled recurrence of the fused method, on one logit row pair.

    Per tile: new maxima, rescale factors, then l_t, l_s and the teacher-weighted
    logit-difference accumulator A = sum e^{s_t - m_t} (s_t - s_s).  Tiles are
    visited in ``order`` and partial states merged with the same rule, so the
    check also covers any tile order.  Returns (KL, LSE_t, LSE_s).
    """
    cuts = np.cumsum([0] + list(widths))
    tiles = [(cuts[k], cuts[k + 1]) for k in range(len(widths))]
    m_t = m_s = -math.inf
    l_t = l_s = A = 0.0
    for k in order:
        a, b = tiles[k]
        xt, xs = st[a:b], ss[a:b]
        nm_t, nm_s = max(m_t, xt.max()), max(m_s, xs.max())
        alpha_t = math.exp(m_t - nm_t) if m_t > -math.inf else 0.0
        alpha_s = math.exp(m_s - nm_s) if m_s > -math.inf else 0.0
        e_t, e_s = np.exp(xt - nm_t), np.exp(xs - nm_s)
        l_t = alpha_t * l_t + e_t.sum()
        A = alpha_t * A + (e_t * (xt - xs)).sum()
        l_s = alpha_s * l_s + e_s.sum()
        m_t, m_s = nm_t, nm_s
    lse_t, lse_s = m_t + math.log(l_t), m_s + math.log(l_s)
    return A / l_t - lse_t + lse_s, lse_t, lse_s


def test_streaming_recurrence_matches_materialised_definition():
    rng = np.random.default_rng(31)
    qt, kt, qs, ks = problem(B=1, H=1, N_Q=12, N_K=301, d_t=16, d_s=16, seed=31, std=2.5)
    kl, lt, ls = oracle.fwd(qt, kt, qs, ks, 0.25, 0.25, False)
    st = 0.25 * qt[0, 0] @ kt[0, 0].T
    ss = 0.25 * qs[0, 0] @ ks[0, 0].T
    for i in range(12):
        widths = []
        left = 301
        while left:
            w = int(min(left, rng.integers(1, 80)))
            widths.append(w)
            left -= w
        order = rng.permutation(len(widths))
        k2, l2t, l2s = streaming_kl(st[i], ss[i], widths, order)
        assert abs(k2 - kl[0, 0, i]) < 1e-11 * max(1, abs(kl[0, 0, i]))
        assert abs(l2t - lt[0, 0, i]) < 1e-11 and abs(l2s - ls[0, 0, i]) < 1e-11


# ---------------------------------------------------------------- plumbing

def test_rows_and_sampled_rows_match_full():
    w = inputs.custom(B=2, H=3, N_Q=70, N_K=90, d_t=16, d_s=8, causal=True,
                      student="independent", seed=41)
    qt, kt, qs, ks = inputs.make_inputs(w)
    g = rand((2, 3, 70), 42)
    kl, lt, ls = oracle.fwd(qt, kt, qs, ks, w.scale_t, w.scale_s, True)
    dqs, dks, dqt, dkt = oracle.bwd(qt, kt, qs, ks, w.scale_t, w.scale_s, True, g=g)
    r = np.array([0, 5, 69, 70, 211, 419])
    res = oracle.sampled_rows(w, r, g=g, teacher=True)
    np.testing.assert_allclose(res["kl"], kl.ravel()[r], rtol=1e-13, atol=1e-15)
    np.testing.assert_allclose(res["lse_s"], ls.ravel()[r], rtol=1e-13)
    np.testing.assert_allclose(res["dq_s"], dqs.reshape(-1, 8)[r], rtol=1e-12, atol=1e-15)
    np.testing.assert_allclose(res["dq_t"], dqt.reshape(-1, 16)[r], rtol=1e-12, atol=1e-15)
    assert abs(oracle.mean(kl) - kl.mean()) < 1e-14


def test_rejects_bad_shapes():
    qt, kt, qs, ks = problem(N_Q=10, N_K=8)
    with pytest.raises(ValueError):
        oracle.fwd(qt, kt, qs, ks, 1.0, 1.0, True)     # causal with N_Q > N_K


def test_thread_count_does_not_change_results():
    qt, kt, qs, ks = problem(N_Q=31, N_K=31, seed=43)
    a = oracle.bwd(qt, kt, qs, ks, 0.3, 0.3, True, g=1.0, nthreads=1)
    b = oracle.bwd(qt, kt, qs, ks, 0.3, 0.3, True, g=1.0, nthreads=5)
    for x, y in zip(a, b):
        np.testing.assert_allclose(x, y, rtol=1e-13, atol=1e-16)


def test_golden_tiny_regression():
    # fixture written by tests/golden/make_golden.py (oracle only)
    import json
    import os
    path = os.path.join(os.path.dirname(__file__), "golden", "tiny_128.json")
    ref = json.load(open(path))
    w = inputs.WORKLOADS["tiny_128"]
    qt, kt, qs, ks = inputs.make_inputs(w)
    kl, lt, _ = oracle.fwd(qt, kt, qs, ks, w.scale_t, w.scale_s, w.causal)
    assert abs(oracle.mean(kl) - ref["loss_mean"]) < 1e-13
    np.testing.assert_allclose(kl.ravel()[:8], ref["kl_rows_0_8"], rtol=1e-12)
    np.testing.assert_allclose(lt.ravel()[:8], ref["lse_t_rows_0_8"], rtol=1e-13)
    dqs, dks, _, _ = oracle.bwd(qt, kt, qs, ks, w.scale_t, w.scale_s, w.causal, g=ref["g"], teacher=False)
    np.testing.assert_allclose(dqs.reshape(-1, 64)[0], ref["dq_s_row0"], rtol=1e-10, atol=1e-18)
    assert abs(np.linalg.norm(dks) - ref["norms"]["dk_s"]) < 1e-10 * ref["norms"]["dk_s"]


def test_bwd_rows_partition_sums_to_full():
    # the backward over two disjoint row sets adds up to the full backward
    qt, kt, qs, ks = problem(N_Q=20, N_K=25, seed=47)
    g = rand((1, 2, 20), 48)
    full = oracle.bwd(qt, kt, qs, ks, 0.4, 0.3, True, g=g)
    a = oracle.bwd_rows(qt, kt, qs, ks, 0.4, 0.3, True, g, np.arange(0, 40, 2))
    b = oracle.bwd_rows(qt, kt, qs, ks, 0.4, 0.3, True, g, np.arange(1, 40, 2))
    for f, x, y in zip(full, a, b):
        np.testing.assert_allclose(x + y, f, rtol=1e-12, atol=1e-15)
