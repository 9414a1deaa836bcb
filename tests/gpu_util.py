"""Helpers shared by the GPU parity tests (tolerances and comparisons)."""
import numpy as np
import torch

# Per-row KL: |err| <= KL_ATOL + KL_RTOL * |KL|   (fp32 logits from exact bf16
# products; fp32 online state; see the design notes for the derivation)
KL_ATOL, KL_RTOL = 1e-4, 1e-3
# Per-row LSE (natural log): fp32 accumulation of d products, fp32 log-sum-exp
LSE_ATOL, LSE_RTOL = 1e-4, 1e-5
# Gradients: relative L2 error of a whole tensor (or of a sampled slice);
# dS is rounded to bf16 before the gradient contraction
GRAD_REL_L2 = 1e-2


def to_np(t):
    return t.detach().float().cpu().double().numpy()


def assert_kl(gpu_kl, ref_kl, what=""):
    g = np.asarray(gpu_kl, dtype=np.float64).ravel()
    r = np.asarray(ref_kl, dtype=np.float64).ravel()
    assert np.all(np.isfinite(g)), f"{what}: non-finite KL"
    err = np.abs(g - r)
    bound = KL_ATOL + KL_RTOL * np.abs(r)
    worst = int(np.argmax(err / bound))
    assert np.all(err <= bound), f"{what}: KL row {worst}: gpu {g[worst]!r} oracle {r[worst]!r}"


def assert_lse(gpu, ref, what=""):
    g = np.asarray(gpu, dtype=np.float64).ravel()
    r = np.asarray(ref, dtype=np.float64).ravel()
    err = np.abs(g - r)
    bound = LSE_ATOL + LSE_RTOL * np.abs(r)
    worst = int(np.argmax(err / bound))
    assert np.all(err <= bound), f"{what}: LSE row {worst}: gpu {g[worst]!r} oracle {r[worst]!r}"


def rel_l2(a, b):
    a = np.asarray(a, dtype=np.float64).ravel()
    b = np.asarray(b, dtype=np.float64).ravel()
    nb = np.linalg.norm(b)
    return np.linalg.norm(a - b) / (nb if nb > 0 else 1.0)


def assert_grad(gpu, ref, what=""):
    g = np.asarray(gpu, dtype=np.float64)
    assert np.all(np.isfinite(g)), f"{what}: non-finite gradient"
    e = rel_l2(g, ref)
    assert e <= GRAD_REL_L2, f"{what}: rel L2 {e:.3e}"


def cuda(*ts):
    return [t.cuda() for t in ts]
