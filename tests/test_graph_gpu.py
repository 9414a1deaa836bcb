"""The forward and backward can be captured into a CUDA graph and replayed.

The library launches only on the caller's stream and allocates nothing, so a
step recorded with torch.cuda.graph replays to the same bits as the eager
calls (the kernels are deterministic), including on new inputs copied into
the captured buffers.
"""
import pytest
import torch

from attention_kl_divergence_attn_b200 import inputs, streamkl_bwd, streamkl_check, streamkl_fwd

pytestmark = pytest.mark.gpu


def test_capture_and_replay():
    w = inputs.custom(B=1, H=4, N_Q=700, N_K=700, d_t=128, d_s=128, causal=True, student="independent", seed=11)
    x = [t.cuda() for t in inputs.make_inputs(w)]

    def step():
        kl, lt, ls, loss = streamkl_fwd(*x, w.scale_t, w.scale_s, True)
        g = streamkl_bwd(*x, kl, lt, ls, w.scale_t, w.scale_s, True, teacher_grads=True)
        return (kl, lt, ls, loss) + tuple(g)

    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        for _ in range(2):
            step()
    torch.cuda.current_stream().wait_stream(s)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        out = step()
    eager = [t.clone() for t in step()]
    graph.replay()
    torch.cuda.synchronize()
    assert streamkl_check() == 0
    for a, b in zip(out, eager):
        assert torch.equal(a, b)
    # new inputs through the captured buffers
    w2 = inputs.custom(B=1, H=4, N_Q=700, N_K=700, d_t=128, d_s=128, causal=True, student="noise", seed=12)
    for dst, src in zip(x, inputs.make_inputs(w2)):
        dst.copy_(src.cuda())
    graph.replay()
    eager2 = step()
    torch.cuda.synchronize()
    for a, b in zip(out, eager2):
        assert torch.equal(a, b)
