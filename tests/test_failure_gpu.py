"""Device failure reporting without a fault: a bounded wait that runs out.

streamkl_selftest_timeout makes one warp wait on a barrier that nothing
signals; the library's bounded wait gives up after a short budget, records a
timeout in the workspace status word and the kernel returns.  The test checks
that streamkl_check reports it (and clears it), and that the same context then
runs a forward correctly.
"""
import ctypes

import pytest
import torch

import attention_kl_divergence_attn_b200 as skl
import oracle
from attention_kl_divergence_attn_b200 import inputs
from gpu_util import assert_kl, cuda, to_np

pytestmark = pytest.mark.gpu


def test_wait_timeout_is_reported_and_context_survives():
    L = skl.lib()
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    assert L.streamkl_selftest_timeout(ctypes.c_void_p(ws.data_ptr()), 256, 20_000_000, stream) == 0
    code = ctypes.c_uint(0)
    rc = L.streamkl_check(ctypes.c_void_p(ws.data_ptr()), stream, ctypes.byref(code))
    assert rc == 4                                  # STREAMKL_ERR_TIMEOUT
    assert code.value & 1 and (code.value >> 8) & 0xFF == 63
    assert int(ws[:4].view(torch.int32).item()) == 0          # cleared by the check
    rc = L.streamkl_check(ctypes.c_void_p(ws.data_ptr()), stream, ctypes.byref(code))
    assert rc == 0 and code.value == 0
    # the context still works
    w = inputs.WORKLOADS["tiny_128"]
    t = inputs.make_inputs(w)
    kl, _, _, _ = skl.streamkl_fwd(*cuda(*t), w.scale_t, w.scale_s, w.causal)
    assert skl.streamkl_check() == 0
    r_kl, _, _ = oracle.fwd(*t, w.scale_t, w.scale_s, w.causal)
    assert_kl(to_np(kl), r_kl, "after timeout")
