"""Construction of the autograd module, on CPU: a learnable bias needs an
initial value and is a parameter from the start (no GPU call involved)."""
import math

import pytest
import torch

import padding_aware_sigmoid_b200 as sa


def test_learnable_bias_needs_an_initial_value():
    with pytest.raises(ValueError):
        sa.SigmoidAttention(learnable_bias=True)
    with pytest.raises(ValueError):
        sa.SigmoidAttention(learnable_bias=True, per_sample_bias=True, bias=-1.0)


def test_learnable_bias_is_a_parameter_before_the_first_call():
    m = sa.SigmoidAttention(learnable_bias=True, max_len=4096)
    params = list(m.parameters())
    assert len(params) == 1 and params[0] is m.b
    assert abs(m.b.item() + math.log(4096)) < 1e-6
    m2 = sa.SigmoidAttention(learnable_bias=True, bias=-2.5)
    assert m2.b.item() == -2.5
    opt = torch.optim.SGD(m2.parameters(), lr=0.1)
    assert opt.param_groups[0]["params"][0] is m2.b
    assert list(sa.SigmoidAttention().parameters()) == []
