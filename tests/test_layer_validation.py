"""MoeShuffle checks every caller tensor on the host before launching (the kernels trust shapes)."""
import pytest
import torch

from combine_moe_route_10_b200.layer import expect


def test_expect_accepts_the_right_tensor():
    expect(torch.zeros(4, 8, dtype=torch.bfloat16), (4, 8), torch.bfloat16, "x")
    expect(torch.zeros(0, 8, dtype=torch.float32), (0, 8), torch.float32, "logits")


@pytest.mark.parametrize("t,shape,dtype,err", [
    (torch.zeros(4, 8, dtype=torch.float32), (4, 8), torch.bfloat16, TypeError),   # dtype
    (torch.zeros(3, 8, dtype=torch.bfloat16), (4, 8), torch.bfloat16, ValueError),  # short: T rows
    (torch.zeros(8, 4, dtype=torch.bfloat16).t(), (4, 8), torch.bfloat16, ValueError),  # strided
    ([[0.0] * 8] * 4, (4, 8), torch.bfloat16, TypeError),                          # not a tensor
])
def test_expect_rejects(t, shape, dtype, err):
    with pytest.raises(err):
        expect(t, shape, dtype, "x")


def test_expect_checks_the_device():
    with pytest.raises(ValueError):
        expect(torch.zeros(2, 2), (2, 2), torch.float32, "x", device=torch.device("meta"))
