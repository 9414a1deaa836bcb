"""torch.autograd wrapper of the fused attention-distillation KL divergence.

The loss of knowledge distillation at temperature T ("Lecture 05 - Where It All
Lands: Quantization, Distillation, RLHF & Speculative Decoding", sections 3.1
and 3.3): both attention distributions are softened by T, P_T =
softmax(Q_t K_t^T / (T sqrt(d_t))) and Q_T = softmax(Q_s K_s^T / (T sqrt(d_s))),
and the divergence is multiplied by T^2 so that its gradients keep their size
as T changes:

    loss = T^2 * reduce_i KL(P_T,i || Q_T,i)

The forward and backward are the library's kernels ("StreamKL: Fast and
Memory-Efficient KL Divergence for Boosting Attention Distillation",
abstract: one-pass forward, recomputing backward, no N_Q x N_K buffer); this
module only chooses the scales, saves the per-row statistics between the two
passes and hands the upstream gradient to the backward without copying it to
the host.  Gradients flow to Q_s, K_s and, when they require grad, to Q_t,
K_t.  They are computed in fp32 and returned to autograd as fp32 (autograd
casts them to the bf16 of the inputs).
"""
from __future__ import annotations

import math

import torch

from . import streamkl_bwd, streamkl_fwd, streamkl_loss_reduce

_REDUCTIONS = ("mean", "sum", "none")


def _scales(d_t, d_s, temperature, scale_t, scale_s):
    T = float(temperature)
    if not (T > 0.0) or math.isinf(T):
        raise ValueError("temperature must be a positive finite number")
    st = (1.0 / math.sqrt(d_t) if scale_t is None else float(scale_t)) / T
    ss = (1.0 / math.sqrt(d_s) if scale_s is None else float(scale_s)) / T
    return st, ss, T * T


class StreamKLFunction(torch.autograd.Function):
    """loss = t2 * reduce(KL rows); see ``streamkl_loss`` for the arguments."""

    @staticmethod
    def forward(ctx, q_t, k_t, q_s, k_s, scale_t, scale_s, causal, t2, reduction, kv_len):
        kl, lse_t, lse_s, _ = streamkl_fwd(q_t, k_t, q_s, k_s, scale_t, scale_s, causal, loss_mean=False,
                                           kv_len=kv_len)
        ctx.save_for_backward(q_t, k_t, q_s, k_s, kl, lse_t, lse_s)
        ctx.cfg = (scale_t, scale_s, causal, t2, reduction, kv_len)
        ctx.mark_non_differentiable(lse_t, lse_s)
        n = kl.numel()
        if reduction == "mean":
            out = streamkl_loss_reduce(kl, t2 / n if n else 0.0)
        elif reduction == "sum":
            out = streamkl_loss_reduce(kl, t2)
        else:
            out = kl
        return out, lse_t, lse_s

    @staticmethod
    def backward(ctx, grad_out, _g_lse_t, _g_lse_s):
        q_t, k_t, q_s, k_s, kl, lse_t, lse_s = ctx.saved_tensors
        scale_t, scale_s, causal, t2, reduction, kv_len = ctx.cfg
        teacher = ctx.needs_input_grad[0] or ctx.needs_input_grad[1]
        if grad_out is None:
            return (None,) * 10
        if reduction == "none":
            dkl = grad_out.float().contiguous()
            dq_s, dk_s, dq_t, dk_t = streamkl_bwd(q_t, k_t, q_s, k_s, kl, lse_t, lse_s, scale_t, scale_s, causal,
                                                  dkl=dkl, teacher_grads=teacher, kv_len=kv_len)
        else:
            g = grad_out.float().reshape(1)
            n = kl.numel()
            scale = t2 / n if reduction == "mean" else t2
            dq_s, dk_s, dq_t, dk_t = streamkl_bwd(q_t, k_t, q_s, k_s, kl, lse_t, lse_s, scale_t, scale_s, causal,
                                                  dloss=g, dloss_scale=scale, teacher_grads=teacher, kv_len=kv_len)
        return dq_t, dk_t, dq_s, dk_s, None, None, None, None, None, None


def streamkl_loss(q_t, k_t, q_s, k_s, *, causal=False, temperature=1.0, scale_t=None, scale_s=None,
                  reduction="mean", return_lse=False, kv_len=None):
    """Distillation loss between the teacher's and the student's attention.

    q_t, k_t: teacher queries/keys [B, H, N_Q|N_K, d_t]; q_s, k_s: the
    student's [.., d_s]; contiguous CUDA bf16 (d_t, d_s in {64, 128}).
    scale_t, scale_s: logit scales before the temperature (default
    1/sqrt(d)); the kernels use scale / temperature.  reduction: "mean"
    (T^2 * mean over all B*H*N_Q rows, a 0-d tensor), "sum" (T^2 * sum), or
    "none" (the per-row KL of the softened distributions, [B, H, N_Q],
    without the T^2 factor: multiply by T^2 before reducing it yourself).
    With return_lse the per-row log-sum-exps of both softened distributions
    are returned too (no gradient).  Keys may have fewer heads than the
    queries (grouped key heads), and kv_len (int32 [B] on the device) marks
    the keys at and past each batch element's length as padding; "mean" and
    "sum" still run over every query row (reduce "none" with your own row
    weights to leave padded query rows out).
    """
    if reduction not in _REDUCTIONS:
        raise ValueError(f"reduction must be one of {_REDUCTIONS}")
    st, ss, t2 = _scales(q_t.shape[-1], q_s.shape[-1], temperature, scale_t, scale_s)
    out, lse_t, lse_s = StreamKLFunction.apply(q_t, k_t, q_s, k_s, st, ss, bool(causal), t2, reduction, kv_len)
    return (out, lse_t, lse_s) if return_lse else out
