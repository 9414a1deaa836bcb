"""Pins of the oracle's two variants: padded batches and grouped key heads.

The abstract of "StreamKL: Fast and Memory-Efficient KL Divergence for
Boosting Attention Distillation" names sparse-attention training and
long-context distillation as uses; both need batches whose sequences are
padded to a common key length and models whose keys have fewer heads than
their queries.  The pages give no formula for either, so the oracle takes the
plain readings:

  padding:  key j is visible to row i of batch b iff it is visible under the
            causal rule (if any) and j < kv_len[b]; a row with no visible key
            has KL = 0, LSE = -inf and no gradient;
  grouped key heads: query head h reads key head h / (H / H_k); a key head's
            gradient is the sum over the query heads that read it.

Each pin compares the variant with something it does not contain: the same
problem with the padding cut off (a smaller problem of the pinned base
case), with the key heads repeated explicitly, or torch autograd in fp64 over
an explicit boolean mask.
"""
import math

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle


def rand(shape, seed, std=1.0):
    return np.random.default_rng(seed).standard_normal(shape) * std


def close(a, b, rtol=1e-12, atol=1e-14):
    np.testing.assert_allclose(a, b, rtol=rtol, atol=atol)


# ---------------------------------------------------------------- padding

def test_padded_keys_equal_the_truncated_problem():
    B, H, N_Q, N_K, d_t, d_s = 3, 2, 20, 37, 8, 6
    lens = [N_K, 17, 1]
    qt, kt = rand((B, H, N_Q, d_t), 1), rand((B, H, N_K, d_t), 2)
    qs, ks = rand((B, H, N_Q, d_s), 3), rand((B, H, N_K, d_s), 4)
    g = rand((B, H, N_Q), 5)
    kl, lt, ls = oracle.fwd(qt, kt, qs, ks, 0.4, 0.5, False, kv_len=lens)
    dqs, dks, dqt, dkt = oracle.bwd(qt, kt, qs, ks, 0.4, 0.5, False, g=g, kv_len=lens)
    for b, L in enumerate(lens):
        sl = slice(b, b + 1)
        k2, t2, s2 = oracle.fwd(qt[sl], kt[sl, :, :L], qs[sl], ks[sl, :, :L], 0.4, 0.5, False)
        close(kl[sl], k2)
        close(lt[sl], t2)
        close(ls[sl], s2)
        r = oracle.bwd(qt[sl], kt[sl, :, :L], qs[sl], ks[sl, :, :L], 0.4, 0.5, False, g=g[sl])
        close(dqs[sl], r[0])
        close(dqt[sl], r[2])
        close(dks[sl, :, :L], r[1])
        close(dkt[sl, :, :L], r[3])
        assert not dks[sl, :, L:].any() and not dkt[sl, :, L:].any()


def test_causal_padding_splits_into_a_causal_head_and_a_full_tail():
    # N_Q = N_K = 30 with 12 keys: rows i < 12 see keys 0..i (the causal
    # problem on the first 12 rows and keys); rows i >= 12 see all 12 keys (the
    # unmasked problem of those rows against the first 12 keys); the key
    # gradients are the sum of the two parts
    N, L, d = 30, 12, 8
    qt, kt, qs, ks = (rand((1, 1, N, d), s) for s in (11, 12, 13, 14))
    g = rand((1, 1, N), 15)
    kl, lt, ls = oracle.fwd(qt, kt, qs, ks, 0.45, 0.35, True, kv_len=[L])
    grads = oracle.bwd(qt, kt, qs, ks, 0.45, 0.35, True, g=g, kv_len=[L])
    head = [x[:, :, :L] for x in (qt, kt, qs, ks)]
    tail = [qt[:, :, L:], kt[:, :, :L], qs[:, :, L:], ks[:, :, :L]]
    k1, t1, s1 = oracle.fwd(*head, 0.45, 0.35, True)
    k2, t2, s2 = oracle.fwd(*tail, 0.45, 0.35, False)
    close(kl, np.concatenate([k1, k2], axis=2))
    close(lt, np.concatenate([t1, t2], axis=2))
    close(ls, np.concatenate([s1, s2], axis=2))
    r1 = oracle.bwd(*head, 0.45, 0.35, True, g=g[:, :, :L])
    r2 = oracle.bwd(*tail, 0.45, 0.35, False, g=g[:, :, L:])
    for q_idx in (0, 2):                                    # dQ_s, dQ_t: rows split
        close(grads[q_idx], np.concatenate([r1[q_idx], r2[q_idx]], axis=2))
    for k_idx in (1, 3):                                    # dK_s, dK_t: parts add up
        close(grads[k_idx][:, :, :L], r1[k_idx] + r2[k_idx], rtol=1e-11, atol=1e-13)
        assert not grads[k_idx][:, :, L:].any()


def test_rows_without_a_visible_key():
    # a batch element with no keys: every row is the empty sum
    qt, kt, qs, ks = (rand((2, 2, 9, 4), s) for s in (21, 22, 23, 24))
    kl, lt, ls = oracle.fwd(qt, kt, qs, ks, 0.5, 0.5, False, kv_len=[0, 5])
    assert np.all(kl[0] == 0) and np.all(np.isneginf(lt[0])) and np.all(np.isneginf(ls[0]))
    assert np.all(np.isfinite(kl[1])) and np.all(np.isfinite(lt[1]))
    grads = oracle.bwd(qt, kt, qs, ks, 0.5, 0.5, False, g=1.0, kv_len=[0, 5])
    for gr in grads:
        assert not gr[0].any()


def test_lengths_outside_the_key_range_are_clamped():
    qt, kt, qs, ks = (rand((2, 1, 6, 4), s) for s in (31, 32, 33, 34))
    a = oracle.fwd(qt, kt, qs, ks, 0.5, 0.5, False, kv_len=[-3, 99])
    b = oracle.fwd(qt, kt, qs, ks, 0.5, 0.5, False, kv_len=[0, 6])
    for x, y in zip(a, b):
        np.testing.assert_array_equal(x, y)


# ---------------------------------------------------------------- grouped key heads

@pytest.mark.parametrize("causal", [False, True])
def test_grouped_key_heads_equal_repeated_heads(causal):
    B, H, H_kt, H_ks, N_Q, N_K, d_t, d_s = 2, 6, 2, 3, 14, 19, 8, 4
    qt, qs = rand((B, H, N_Q, d_t), 41), rand((B, H, N_Q, d_s), 42)
    kt, ks = rand((B, H_kt, N_K, d_t), 43), rand((B, H_ks, N_K, d_s), 44)
    g = rand((B, H, N_Q), 45)
    Gt, Gs = H // H_kt, H // H_ks
    kt_rep, ks_rep = np.repeat(kt, Gt, axis=1), np.repeat(ks, Gs, axis=1)
    a = oracle.fwd(qt, kt, qs, ks, 0.3, 0.6, causal)
    b = oracle.fwd(qt, kt_rep, qs, ks_rep, 0.3, 0.6, causal)
    for x, y in zip(a, b):
        close(x, y)
    ga = oracle.bwd(qt, kt, qs, ks, 0.3, 0.6, causal, g=g)
    gb = oracle.bwd(qt, kt_rep, qs, ks_rep, 0.3, 0.6, causal, g=g)
    close(ga[0], gb[0])
    close(ga[2], gb[2])
    # a key head's gradient is the sum over the query heads of its group
    close(ga[1], gb[1].reshape(B, H_ks, Gs, N_K, d_s).sum(axis=2), rtol=1e-11, atol=1e-14)
    close(ga[3], gb[3].reshape(B, H_kt, Gt, N_K, d_t).sum(axis=2), rtol=1e-11, atol=1e-14)


def test_grouped_heads_reject_counts_that_do_not_divide():
    qt, qs = rand((1, 4, 5, 4), 51), rand((1, 4, 5, 4), 52)
    kt, ks = rand((1, 3, 5, 4), 53), rand((1, 4, 5, 4), 54)
    with pytest.raises(ValueError):
        oracle.fwd(qt, kt, qs, ks, 0.5, 0.5, False)


# ---------------------------------------------------------------- library routine

@pytest.mark.parametrize("causal", [False, True])
def test_variants_match_torch_autograd(causal):
    # both variants at once, against torch in fp64: keys expanded to the query
    # heads with repeat_interleave (autograd sums the group's gradients) and an
    # explicit boolean mask of the visible keys
    B, H, H_kt, H_ks, N_Q, N_K, d_t, d_s = 2, 4, 2, 1, 21, 26, 8, 12
    lens = [N_K - 3, 9]
    sc_t, sc_s = 1 / math.sqrt(d_t), 1 / math.sqrt(d_s)
    arrs = (rand((B, H, N_Q, d_t), 61), rand((B, H_kt, N_K, d_t), 62),
            rand((B, H, N_Q, d_s), 63), rand((B, H_ks, N_K, d_s), 64))
    g = rand((B, H, N_Q), 65)
    T = [torch.tensor(a, dtype=torch.float64, requires_grad=True) for a in arrs]
    i = torch.arange(N_Q)[:, None]
    j = torch.arange(N_K)[None, :]
    vis = (j <= i + (N_K - N_Q)) if causal else torch.ones(N_Q, N_K, dtype=torch.bool)
    mask = vis[None, None] & (j[None, None] < torch.tensor(lens)[:, None, None, None])
    kt_e = T[1].repeat_interleave(H // H_kt, dim=1)
    ks_e = T[3].repeat_interleave(H // H_ks, dim=1)
    S_t = sc_t * T[0] @ kt_e.transpose(-1, -2)
    S_s = sc_s * T[2] @ ks_e.transpose(-1, -2)
    neg = torch.finfo(torch.float64).min
    lp = F.log_softmax(S_t.masked_fill(~mask, neg), -1)
    lq = F.log_softmax(S_s.masked_fill(~mask, neg), -1)
    kl_t = F.kl_div(lq, lp, log_target=True, reduction="none").masked_fill(~mask, 0).sum(-1)
    (kl_t * torch.tensor(g)).sum().backward()

    kl, lt, ls = oracle.fwd(*arrs, sc_t, sc_s, causal, kv_len=lens)
    np.testing.assert_allclose(kl, kl_t.detach().numpy(), rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(lt, torch.logsumexp(S_t.masked_fill(~mask, -math.inf), -1).detach().numpy(),
                               rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(ls, torch.logsumexp(S_s.masked_fill(~mask, -math.inf), -1).detach().numpy(),
                               rtol=1e-12, atol=1e-12)
    dqs, dks, dqt, dkt = oracle.bwd(*arrs, sc_t, sc_s, causal, g=g, kv_len=lens)
    for mine, leaf in ((dqt, T[0]), (dkt, T[1]), (dqs, T[2]), (dks, T[3])):
        ref = leaf.grad.numpy()
        assert mine.shape == ref.shape
        assert np.linalg.norm(mine - ref) <= 1e-10 * np.linalg.norm(ref) + 1e-14
