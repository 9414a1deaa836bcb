"""GPU padding masks and grouped key heads against the fp64 oracle.

Padding: per-batch key lengths (device int32 [B]); keys at and past a batch
element's length are hidden from every row of it.  Grouped key heads: K_t and
K_s have H_kt, H_ks heads dividing H; a key head's gradient sums over the
query heads that read it.  Lengths cover the edges of the 64-key tiles of the
forward and query-owner kernels and the 128-key items of the key-owner kernels
(0, 1, 63, 64, 65, 127, 128, 129, N_K), both masks, every kernel form (one-item
and persistent key-owner, key splits), per-row and uniform upstream gradients.
"""
import numpy as np
import pytest
import torch

import oracle
from attention_kl_divergence_attn_b200 import inputs, streamkl_fwd, streamkl_bwd, streamkl_check, StreamKLError
from attention_kl_divergence_attn_b200.autograd import streamkl_loss
from gpu_util import assert_kl, assert_lse, assert_grad, to_np, cuda

pytestmark = pytest.mark.gpu


def compare_fwd(w, x, lens_dev, lens):
    kl, lt, ls, loss = streamkl_fwd(*x, w.scale_t, w.scale_s, w.causal, kv_len=lens_dev)
    assert streamkl_check() == 0
    host = inputs.make_inputs(w)
    rkl, rlt, rls = oracle.fwd(*host, w.scale_t, w.scale_s, w.causal, kv_len=lens)
    k, t, s = to_np(kl), to_np(lt), to_np(ls)
    empty = np.isneginf(rlt)                       # rows without a visible key
    assert np.array_equal(np.isneginf(t), empty) and np.array_equal(np.isneginf(s), empty)
    assert np.all(k[empty] == 0)
    assert_kl(k[~empty], rkl[~empty], w.name)
    assert_lse(t[~empty], rlt[~empty], w.name + " lse_t")
    assert_lse(s[~empty], rls[~empty], w.name + " lse_s")
    assert abs(float(loss) - rkl.mean()) <= 1e-4 + 1e-3 * abs(rkl.mean())
    return kl, lt, ls, host


def compare_bwd(w, x, lens_dev, lens, fwd_out, host, teacher, per_row_g):
    kl, lt, ls = fwd_out
    if per_row_g:
        g = torch.randn(w.B, w.H, w.N_Q, generator=torch.Generator().manual_seed(w.seed)) / w.rows
        dkl, dloss, g_ref = g.cuda(), 0.0, g.double().numpy()
    else:
        dkl, dloss, g_ref = None, 1.5, 1.5 / w.rows
    dqs, dks, dqt, dkt = streamkl_bwd(*x, kl, lt, ls, w.scale_t, w.scale_s, w.causal, dkl=dkl, dloss=dloss,
                                      teacher_grads=teacher, kv_len=lens_dev)
    assert streamkl_check() == 0
    assert dks.shape == (w.B, w.H_ks, w.N_K, w.d_s)
    r = oracle.bwd(*host, w.scale_t, w.scale_s, w.causal, g=g_ref, teacher=teacher, kv_len=lens)
    assert_grad(to_np(dqs), r[0], w.name + " dq_s")
    assert_grad(to_np(dks), r[1], w.name + " dk_s")
    if teacher:
        assert dkt.shape == (w.B, w.H_kt, w.N_K, w.d_t)
        assert_grad(to_np(dqt), r[2], w.name + " dq_t")
        assert_grad(to_np(dkt), r[3], w.name + " dk_t")
    if lens is not None:
        # padding keys get exactly zero rows, rows of empty batch elements zero dQ
        for b, L in enumerate(lens):
            assert not dks[b, :, L:].any()
            if teacher:
                assert not dkt[b, :, L:].any()
            if L == 0:
                assert not dqs[b].any()
    return dqs, dks, dqt, dkt


CASES = [
    # (B, H, H_kt, H_ks, N_Q, N_K, d_t, d_s, causal, teacher, kv_lens)
    (4, 2, 2, 2, 300, 300, 128, 128, True, True, (300, 1, 129, 0)),       # one-item key-owner, padding
    (4, 2, 2, 2, 200, 333, 64, 64, False, True, (63, 64, 65, 333)),        # persistent key-owner (d = 64)
    (3, 2, 2, 2, 257, 520, 128, 64, False, False, (127, 128, 5)),          # persistent, staged K rows
    (2, 8, 2, 4, 256, 256, 128, 64, True, True, ()),                       # grouped heads, teacher grads
    (2, 8, 8, 2, 300, 300, 128, 128, True, False, ()),                     # grouped student heads, persistent
    (2, 6, 3, 1, 190, 410, 64, 128, False, True, (410, 77)),               # both variants together
    (1, 4, 1, 1, 128, 128, 64, 64, True, True, (100,)),                    # one key head for all
]


@pytest.mark.parametrize("per_row_g", [False, True])
@pytest.mark.parametrize("case", CASES, ids=lambda c: "x".join(map(str, c[:10])) + "_" + "-".join(map(str, c[10])))
def test_variants_match_oracle(case, per_row_g):
    B, H, H_kt, H_ks, N_Q, N_K, d_t, d_s, causal, teacher, lens = case
    w = inputs.custom(B=B, H=H, N_Q=N_Q, N_K=N_K, d_t=d_t, d_s=d_s, causal=causal, student="independent",
                      teacher_std=1.5, student_std=1.5, seed=N_Q * 3 + N_K + H_kt * 7 + H_ks,
                      h_kt=H_kt, h_ks=H_ks, kv_lens=lens)
    x = cuda(*inputs.make_inputs(w))
    lens_t = inputs.key_lengths(w)
    lens_dev = None if lens_t is None else lens_t.cuda()
    kl, lt, ls, host = compare_fwd(w, x, lens_dev, list(lens) if lens else None)
    compare_bwd(w, x, lens_dev, list(lens) if lens else None, (kl, lt, ls), host, teacher, per_row_g)


def test_grouped_heads_many_items_per_cta():
    # 2 x 8 query heads x 32 key tiles of 128 = 512 key-owner items on 148 SMs
    # (persistent kernel, several items per CTA), student keys shared by groups
    # of 4 query heads, padded batches; every element compared
    w = inputs.custom(B=2, H=8, N_Q=4096, N_K=4096, d_t=128, d_s=128, causal=True, student="independent",
                      seed=717, h_kt=8, h_ks=2, kv_lens=(4096, 2500))
    x = cuda(*inputs.make_inputs(w))
    lens = list(w.kv_lens)
    lens_dev = inputs.key_lengths(w).cuda()
    kl, lt, ls, host = compare_fwd(w, x, lens_dev, lens)
    compare_bwd(w, x, lens_dev, lens, (kl, lt, ls), host, False, False)


def test_grouped_heads_at_headline_size_sampled():
    # the 8k causal d = 128 teacher-and-student shape with 8 key heads per side:
    # one whole key head group (4 query heads) against the oracle
    w = inputs.custom(name="gqa_8k", B=1, H=32, N_Q=8192, N_K=8192, d_t=128, d_s=128, causal=True,
                      student="independent", teacher_grads=True, seed=818, h_kt=8, h_ks=8)
    x = cuda(*inputs.make_inputs(w))
    kl, lt, ls, _ = streamkl_fwd(*x, w.scale_t, w.scale_s, True)
    dqs, dks, dqt, dkt = streamkl_bwd(*x, kl, lt, ls, w.scale_t, w.scale_s, True, teacher_grads=True)
    assert streamkl_check() == 0
    g = 1.0 / w.rows
    hk = 5                                            # key head 5: query heads 20..23
    heads = [(0, h) for h in range(4 * hk, 4 * hk + 4)]
    sub = inputs.make_inputs(w, heads=heads)
    q_t, k_t, q_s, k_s = (t[:, 4 * hk:4 * hk + 4] if t.shape[1] == 32 else t[:, hk:hk + 1] for t in sub)
    rkl, _, _ = oracle.fwd(q_t, k_t, q_s, k_s, w.scale_t, w.scale_s, True)
    assert_kl(to_np(kl[:, 4 * hk:4 * hk + 4]), rkl, "gqa_8k kl")
    r = oracle.bwd(q_t, k_t, q_s, k_s, w.scale_t, w.scale_s, True, g=g, teacher=True)
    assert_grad(to_np(dks[:, hk:hk + 1]), r[1], "gqa_8k dk_s")
    assert_grad(to_np(dkt[:, hk:hk + 1]), r[3], "gqa_8k dk_t")
    assert_grad(to_np(dqs[:, 4 * hk:4 * hk + 4]), r[0], "gqa_8k dq_s")
    assert_grad(to_np(dqt[:, 4 * hk:4 * hk + 4]), r[2], "gqa_8k dq_t")


def test_cross_attention_padding_with_key_splits():
    # few query tiles and long, padded key ranges: the forward and the
    # query-owner kernel split each tile's keys; some splits then see only
    # padding and must contribute nothing
    w = inputs.custom(B=2, H=2, N_Q=256, N_K=20000, d_t=128, d_s=64, causal=False, student="independent",
                      teacher_std=2.0, student_std=2.0, seed=919, kv_lens=(20000, 500))
    x = cuda(*inputs.make_inputs(w))
    lens = list(w.kv_lens)
    lens_dev = inputs.key_lengths(w).cuda()
    kl, lt, ls, host = compare_fwd(w, x, lens_dev, lens)
    compare_bwd(w, x, lens_dev, lens, (kl, lt, ls), host, False, True)


def test_lengths_outside_the_range_are_clamped_and_reported():
    w = inputs.custom(B=2, H=2, N_Q=130, N_K=200, d_t=64, d_s=64, causal=False, student="independent", seed=1001)
    x = cuda(*inputs.make_inputs(w))
    bad = torch.tensor([-4, 999], dtype=torch.int32, device="cuda")
    good = torch.tensor([0, 200], dtype=torch.int32, device="cuda")
    a = streamkl_fwd(*x, w.scale_t, w.scale_s, False, kv_len=bad)
    with pytest.raises(StreamKLError) as e:
        streamkl_check()
    assert e.value.code == 1                           # STREAMKL_ERR_INVALID_ARG, then the word is clear
    assert streamkl_check() == 0
    b = streamkl_fwd(*x, w.scale_t, w.scale_s, False, kv_len=good)
    assert streamkl_check() == 0
    for u, v in zip(a[:3], b[:3]):
        assert torch.equal(u, v)


def test_no_padding_lengths_equal_the_plain_path():
    # lengths all equal to N_K take the padding-aware kernels but must give the
    # plain path's bits
    w = inputs.custom(B=2, H=3, N_Q=300, N_K=300, d_t=128, d_s=128, causal=True, student="independent", seed=1101)
    x = cuda(*inputs.make_inputs(w))
    full = torch.full((2,), 300, dtype=torch.int32, device="cuda")
    a = streamkl_fwd(*x, w.scale_t, w.scale_s, True)
    b = streamkl_fwd(*x, w.scale_t, w.scale_s, True, kv_len=full)
    ga = streamkl_bwd(*x, *a[:3], w.scale_t, w.scale_s, True, teacher_grads=True)
    gb = streamkl_bwd(*x, *b[:3], w.scale_t, w.scale_s, True, teacher_grads=True, kv_len=full)
    assert streamkl_check() == 0
    for u, v in zip(a[:3] + ga, b[:3] + gb):
        assert torch.equal(u, v)


def test_autograd_with_grouped_heads_and_padding():
    w = inputs.custom(B=2, H=4, N_Q=160, N_K=160, d_t=64, d_s=64, causal=True, student="independent",
                      seed=1201, h_kt=2, h_ks=1, kv_lens=(160, 90))
    host = inputs.make_inputs(w)
    x = [t.cuda().requires_grad_(True) for t in host]
    lens_dev = inputs.key_lengths(w).cuda()
    loss = streamkl_loss(*x, causal=True, temperature=2.0, kv_len=lens_dev)
    loss.backward()
    st, ss = w.scale_t / 2.0, w.scale_s / 2.0
    rkl, _, _ = oracle.fwd(*host, st, ss, True, kv_len=list(w.kv_lens))
    assert abs(float(loss) - 4.0 * rkl.mean()) <= 1e-4 + 1e-3 * abs(4.0 * rkl.mean())
    r = oracle.bwd(*host, st, ss, True, g=4.0 / w.rows, teacher=True, kv_len=list(w.kv_lens))
    for mine, ref, name in zip((x[2].grad, x[3].grad, x[0].grad, x[1].grad), r, ("dq_s", "dk_s", "dq_t", "dk_t")):
        assert_grad(to_np(mine.float()), ref, "autograd " + name)
