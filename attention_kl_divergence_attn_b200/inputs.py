"""Seeded synthetic inputs for the attention-KL workloads.

This module only draws random numbers and names workload shapes.  It holds
none of the method's arithmetic, so the CUDA path, the fp64 oracle, the tests
and the bench can all read the very same bf16 bytes from it.

Recipe (the same for every workload):
  * every (tensor, batch, head) slice has its own ``torch.Generator`` seeded
    with ``seed * 1_000_003 + tensor_id * 65_537 + b * 257 + h``, so a sampled
    head can be regenerated on its own without drawing the whole tensor;
  * values are fp32 ``randn`` scaled by the workload's standard deviation and
    rounded to bf16 (round-to-nearest-even, torch's ``.to(torch.bfloat16)``);
  * a "noise" student is ``teacher_fp32 + sigma * randn`` rounded once to bf16;
    an "independent" student draws its own ``randn`` with its own tensor ids.

Tensor ids: 0 = Q_t, 1 = K_t, 2 = Q_s (noise or independent), 3 = K_s.

Grouped key heads: K_t and K_s may have fewer heads than the queries
(``h_kt``, ``h_ks``, each dividing H); key head k of a tensor is drawn from
the generator of (tensor, b, k).  Padding: ``kv_lens`` gives one key length
per batch element (empty = no padding); the keys past it are drawn all the
same, so they are real data that the mask must hide.
"""
from __future__ import annotations

from dataclasses import dataclass, field, asdict
import math

import torch


@dataclass(frozen=True)
class Workload:
    """Shape and value distribution of one attention-KL problem."""

    name: str
    B: int
    H: int
    N_Q: int
    N_K: int
    d_t: int
    d_s: int
    causal: bool
    teacher_std: float = 1.0
    student: str = "noise"          # "noise" | "independent"
    student_std: float = 1.0        # std of an independent student
    noise_std: float = 0.1          # sigma of the student's additive noise
    teacher_grads: bool = False     # backward also returns dQ_t, dK_t
    seed: int = 20260
    h_kt: int = 0                   # heads of K_t (0 = H)
    h_ks: int = 0                   # heads of K_s (0 = H)
    kv_lens: tuple = ()             # per-batch key lengths (empty = no padding)

    @property
    def H_kt(self) -> int:
        return self.h_kt or self.H

    @property
    def H_ks(self) -> int:
        return self.h_ks or self.H

    @property
    def scale_t(self) -> float:
        return 1.0 / math.sqrt(self.d_t)

    @property
    def scale_s(self) -> float:
        return 1.0 / math.sqrt(self.d_s)

    @property
    def rows(self) -> int:
        return self.B * self.H * self.N_Q

    def as_dict(self) -> dict:
        d = asdict(self)
        d["scale_t"] = self.scale_t
        d["scale_s"] = self.scale_s
        return d


# The five workloads the method is exercised on.  Sizes, masks, value
# distributions and which gradients are wanted follow the problem statement of
# the fused attention-distillation KL primitive (one small self-attention
# case, three causal self-attention cases up to 32k context, and one
# long-key cross-attention case with peaked logits and d_t != d_s).
WORKLOADS = {
    "tiny_128": Workload("tiny_128", 1, 1, 128, 128, 64, 64, False,
                         student="noise", noise_std=0.1, seed=20260),
    "causal_2k_d64": Workload("causal_2k_d64", 2, 8, 2048, 2048, 64, 64, True,
                              student="noise", noise_std=0.3, seed=20261),
    "causal_8k_d128": Workload("causal_8k_d128", 1, 32, 8192, 8192, 128, 128, True,
                               student="independent", student_std=1.0,
                               teacher_grads=True, seed=20262),
    "causal_32k_d128": Workload("causal_32k_d128", 1, 16, 32768, 32768, 128, 128, True,
                                student="noise", noise_std=0.2, seed=20263),
    "cross_1k_64k": Workload("cross_1k_64k", 4, 8, 1024, 65536, 128, 64, False,
                             teacher_std=4.0, student="independent", student_std=4.0,
                             seed=20264),
}


def _gen(seed: int, tensor_id: int, b: int, h: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(seed * 1_000_003 + tensor_id * 65_537 + b * 257 + h)
    return g


def _randn(seed, tensor_id, b, h, n, d) -> torch.Tensor:
    return torch.randn(n, d, generator=_gen(seed, tensor_id, b, h), dtype=torch.float32)


def _teacher_q(w, b, h):
    return _randn(w.seed, 0, b, h, w.N_Q, w.d_t) * w.teacher_std


def _teacher_k(w, b, hk):
    return _randn(w.seed, 1, b, hk, w.N_K, w.d_t) * w.teacher_std


def _student(w, tensor_id, b, h, n, teacher):
    """Student rows of tensor 2 (queries) or 3 (keys) for head h, given the
    teacher's rows of the same head (used by a noise student)."""
    if w.student == "noise":
        if w.d_s != w.d_t:
            raise ValueError("a noise student needs d_s == d_t")
        if w.H_ks != w.H_kt:
            raise ValueError("a noise student needs as many key heads as the teacher")
        return teacher + w.noise_std * _randn(w.seed, tensor_id, b, h, n, w.d_s)
    if w.student == "independent":
        return _randn(w.seed, tensor_id, b, h, n, w.d_s) * w.student_std
    raise ValueError(w.student)


def key_head(w: Workload, h: int, teacher: bool) -> int:
    """The key head that query head h reads (grouped key heads)."""
    return h // (w.H // (w.H_kt if teacher else w.H_ks))


def head_inputs(w: Workload, b: int, h: int):
    """bf16 (Q_t, K_t, Q_s, K_s) that query head h of batch b reads, on the CPU."""
    qt = _teacher_q(w, b, h)
    qs = _student(w, 2, b, h, w.N_Q, qt)
    hkt, hks = key_head(w, h, True), key_head(w, h, False)
    kt = _teacher_k(w, b, hkt)
    ks = _student(w, 3, b, hks, w.N_K, _teacher_k(w, b, hks) if w.student == "noise" else None)
    bf = torch.bfloat16
    return qt.to(bf), kt.to(bf), qs.to(bf), ks.to(bf)


def make_inputs(w: Workload, heads=None):
    """bf16 CPU tensors Q_t [B,H,N_Q,d_t], K_t [B,H_kt,N_K,d_t], Q_s, K_s.

    ``heads`` (optional list of (b, h) query heads) fills only those slices
    (and the key heads they read) and leaves the others zero, which is how the
    CPU side regenerates a sample cheaply.
    """
    bf = torch.bfloat16
    qt = torch.zeros(w.B, w.H, w.N_Q, w.d_t, dtype=bf)
    kt = torch.zeros(w.B, w.H_kt, w.N_K, w.d_t, dtype=bf)
    qs = torch.zeros(w.B, w.H, w.N_Q, w.d_s, dtype=bf)
    ks = torch.zeros(w.B, w.H_ks, w.N_K, w.d_s, dtype=bf)
    todo = heads if heads is not None else [(b, h) for b in range(w.B) for h in range(w.H)]
    for b, h in todo:
        a, c, e, f = head_inputs(w, b, h)
        qt[b, h], qs[b, h] = a, e
        kt[b, key_head(w, h, True)], ks[b, key_head(w, h, False)] = c, f
    return qt, kt, qs, ks


def key_lengths(w: Workload):
    """Per-batch key lengths as an int32 CPU tensor, or None without padding."""
    if not w.kv_lens:
        return None
    if len(w.kv_lens) != w.B:
        raise ValueError("one key length per batch element")
    return torch.tensor(w.kv_lens, dtype=torch.int32)


def custom(name="custom", *, B=1, H=1, N_Q=128, N_K=128, d_t=64, d_s=64, causal=False,
           teacher_std=1.0, student="noise", student_std=1.0, noise_std=0.1,
           teacher_grads=False, seed=1, h_kt=0, h_ks=0, kv_lens=()) -> Workload:
    """A workload of any shape, drawn with the same recipe."""
    return Workload(name, B, H, N_Q, N_K, d_t, d_s, causal, teacher_std, student,
                    student_std, noise_std, teacher_grads, seed, h_kt, h_ks, tuple(kv_lens))


def sample_rows(w: Workload, n: int, seed: int = 7):
    """``n`` distinct flattened row ids (b*H*N_Q + h*N_Q + i), seeded."""
    g = torch.Generator().manual_seed(w.seed * 31 + seed)
    n = min(n, w.rows)
    return torch.randperm(w.rows, generator=g)[:n].sort().values


def sample_heads(w: Workload, n: int, seed: int = 11):
    """``n`` distinct (b, h) pairs, seeded."""
    g = torch.Generator().manual_seed(w.seed * 37 + seed)
    n = min(n, w.B * w.H)
    idx = torch.randperm(w.B * w.H, generator=g)[:n].sort().values.tolist()
    return [(i // w.H, i % w.H) for i in idx]
