"""What the GPU shape sweep (tests/test_sweep_gpu.py) reaches, checked on the CPU.

The sweep's 36 problems come from a fixed seed; this test pins that they keep
covering every kind of problem the entry points accept (both masks, both
gradient sets, mixed and equal head dimensions, padding, grouped key heads,
N_Q < N_K and N_Q > N_K, one-tile and many-tile key ranges), so that a change
to the draw cannot quietly narrow it.
"""
from test_sweep_gpu import draw


def test_the_draws_cover_the_kernel_forms():
    ws = [draw(i)[0] for i in range(36)]
    assert any(w.causal for w in ws) and any(not w.causal for w in ws)
    assert any(w.teacher_grads for w in ws) and any(not w.teacher_grads for w in ws)
    assert any(w.d_t != w.d_s for w in ws) and any(w.d_t == w.d_s == 128 for w in ws)
    assert any(w.kv_lens for w in ws)
    assert any(w.H_kt < w.H or w.H_ks < w.H for w in ws)
    assert any(w.N_Q < w.N_K for w in ws) and any(w.N_Q > w.N_K for w in ws)
    assert not any(w.causal and w.N_Q > w.N_K for w in ws)
    assert any(w.student == "noise" for w in ws) and any(w.student == "independent" for w in ws)
    assert any(w.N_K <= 64 for w in ws) and any(w.N_K > 512 for w in ws)
