"""Argument checks of the autograd wrapper that need no GPU."""
import pytest
import torch

from attention_kl_divergence_attn_b200.autograd import streamkl_loss


def _t():
    return torch.zeros(1, 1, 4, 64, dtype=torch.bfloat16)


def test_bad_reduction_rejected():
    with pytest.raises(ValueError):
        streamkl_loss(_t(), _t(), _t(), _t(), reduction="max")


@pytest.mark.parametrize("T", [0.0, -1.0, float("inf"), float("nan")])
def test_bad_temperature_rejected(T):
    with pytest.raises(ValueError):
        streamkl_loss(_t(), _t(), _t(), _t(), temperature=T)


def test_cpu_tensors_rejected():
    with pytest.raises(TypeError):
        streamkl_loss(_t(), _t(), _t(), _t())
