"""streamkl_fwd_noalloc, the forward for callers that cannot allocate device memory.

Such callers (plug-in hosts that only hand out pre-planned buffers, runtimes
that forbid allocation while serving, programs whose pool owns the device)
cannot provide even the small workspace of streamkl_fwd; this entry point keeps
its scratch in a fixed array inside the library instead.  The test calls it
through the C ABI twice in a row and compares each result with streamkl_fwd on
the same inputs and with the fp64 oracle.  It lives in a file that pytest collects last, and it passes
both alone in a fresh process and after the other tests.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import attention_kl_divergence_attn_b200 as skl
from attention_kl_divergence_attn_b200 import inputs
from gpu_util import assert_kl, assert_lse, to_np

pytestmark = pytest.mark.gpu


def _p(t):
    return ctypes.c_void_p(t.data_ptr())


def test_fwd_noalloc_matches_fwd_on_two_calls_in_a_row():
    L = skl.lib()
    w = inputs.custom(B=2, H=3, N_Q=300, N_K=300, d_t=128, d_s=64, causal=True, student="independent",
                      seed=77)
    host = inputs.make_inputs(w)
    x = [t.cuda() for t in host]
    ref_kl, ref_lt, ref_ls, ref_loss = skl.streamkl_fwd(*x, w.scale_t, w.scale_s, w.causal)
    okl, olt, ols = oracle.fwd(*host, w.scale_t, w.scale_s, w.causal)
    stream = torch.cuda.current_stream()
    for call in range(2):
        kl = torch.full((w.B, w.H, w.N_Q), float("nan"), device="cuda")
        lt, ls = torch.full_like(kl, float("nan")), torch.full_like(kl, float("nan"))
        loss = torch.full((), float("nan"), device="cuda")
        status = ctypes.c_uint(12345)
        rc = L.streamkl_fwd_noalloc(*[_p(t) for t in x], w.B, w.H, w.N_Q, w.N_K, w.d_t, w.d_s,
                                    w.scale_t, w.scale_s, int(w.causal), _p(kl), _p(lt), _p(ls), _p(loss),
                                    ctypes.c_void_p(stream.cuda_stream), ctypes.byref(status))
        assert rc == 0, f"call {call}: status {rc}"
        assert status.value == 0
        torch.cuda.synchronize()
        assert_kl(to_np(kl), to_np(ref_kl), f"noalloc call {call}")
        assert_lse(to_np(lt), to_np(ref_lt), f"noalloc call {call} lse_t")
        assert_lse(to_np(ls), to_np(ref_ls), f"noalloc call {call} lse_s")
        assert abs(float(loss) - float(ref_loss)) <= 1e-4 + 1e-3 * abs(float(ref_loss))
        assert_kl(to_np(kl), okl, f"noalloc call {call} vs oracle")
        assert_lse(to_np(lt), olt, f"noalloc call {call} lse_t vs oracle")
        assert_lse(to_np(ls), ols, f"noalloc call {call} lse_s vs oracle")
        assert abs(float(loss) - okl.mean()) <= 1e-4 + 1e-3 * abs(okl.mean())
    # without a status pointer the call only enqueues
    rc = L.streamkl_fwd_noalloc(*[_p(t) for t in x], w.B, w.H, w.N_Q, w.N_K, w.d_t, w.d_s, w.scale_t,
                                w.scale_s, int(w.causal), _p(kl), _p(lt), _p(ls), None,
                                ctypes.c_void_p(stream.cuda_stream), None)
    assert rc == 0
    torch.cuda.synchronize()
    assert np.array_equal(to_np(kl), to_np(ref_kl))


def test_fwd_noalloc_rejects_bad_arguments():
    L = skl.lib()
    p = ctypes.c_void_p(16)
    rc = L.streamkl_fwd_noalloc(p, p, p, p, 1, 1, 128, 128, 96, 64, 0.1, 0.1, 0, p, p, p, None, None, None)
    assert rc == 2                                  # unsupported head dimension, nothing launched
