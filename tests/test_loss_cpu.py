"""The autograd entry refuses what the library cannot run, before touching it:
CPU tensors (there is no CPU path), other dtypes, mismatched shapes."""
import pytest
import torch

from lm_head_fp32_b200.loss import lm_head_cross_entropy


def test_cpu_tensors_are_refused():
    X = torch.zeros((4, 8), dtype=torch.bfloat16)
    W = torch.zeros((16, 8), dtype=torch.bfloat16)
    t = torch.zeros(4, dtype=torch.int64)
    with pytest.raises(ValueError, match="CUDA"):
        lm_head_cross_entropy(X, W, t)


@pytest.mark.gpu
def test_dtypes_and_shapes_are_checked():
    X = torch.zeros((4, 8), dtype=torch.float32, device="cuda")
    W = torch.zeros((16, 8), dtype=torch.bfloat16, device="cuda")
    t = torch.zeros(4, dtype=torch.int64, device="cuda")
    with pytest.raises(TypeError):
        lm_head_cross_entropy(X, W, t)
    with pytest.raises(ValueError):
        lm_head_cross_entropy(X.bfloat16(), W[:, :4].contiguous(), t)
    with pytest.raises(TypeError):
        lm_head_cross_entropy(X.bfloat16(), W, t.int())
