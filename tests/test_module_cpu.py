"""Argument checks of the PyTorch front end (no GPU needed)."""
import pytest
import torch

from linear_diffusion_cross_b200.module import (FusedLinearDiffusionCrossEntropyLoss,
                                                fused_linear_cross_entropy_loss)


def test_rejects_unknown_reduction():
    with pytest.raises(ValueError):
        FusedLinearDiffusionCrossEntropyLoss(reduction="none")


def test_rejects_mismatched_shapes():
    x = torch.zeros(4, 8, dtype=torch.bfloat16)
    w = torch.zeros(10, 16, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        fused_linear_cross_entropy_loss(x, torch.zeros(4, dtype=torch.int64), w)
    with pytest.raises(ValueError):
        fused_linear_cross_entropy_loss(x, torch.zeros(3, dtype=torch.int64),
                                        torch.zeros(10, 8, dtype=torch.bfloat16))


def test_rejects_mismatched_bias():
    x = torch.zeros(4, 8, dtype=torch.bfloat16)
    w = torch.zeros(10, 8, dtype=torch.bfloat16)
    y = torch.zeros(4, dtype=torch.int64)
    with pytest.raises((ValueError, RuntimeError)):
        fused_linear_cross_entropy_loss(x, y, w, bias=torch.zeros(9, dtype=torch.bfloat16))


def test_rejects_cpu_tensors_and_other_dtypes():
    x = torch.zeros(4, 8, dtype=torch.bfloat16)
    w = torch.zeros(10, 8, dtype=torch.bfloat16)
    y = torch.zeros(4, dtype=torch.int64)
    with pytest.raises(RuntimeError):
        fused_linear_cross_entropy_loss(x, y, w)
    with pytest.raises(TypeError):
        fused_linear_cross_entropy_loss(x, y, w.float())
