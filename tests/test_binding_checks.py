"""The Python binding's own argument checks, which run before any C call (CPU only):
tensors must be CUDA tensors of the documented dtype and rank."""
import pytest
import torch

import invariant_deterministic_04_b200 as bi


def test_cpu_tensors_are_refused_before_the_library_is_called():
    x = torch.zeros((4, 512), dtype=torch.bfloat16)
    w = torch.zeros(512, dtype=torch.bfloat16)
    with pytest.raises(TypeError, match="CUDA"):
        bi.rmsnorm(x, w)
    with pytest.raises(TypeError, match="CUDA"):
        bi.matmul(x, torch.zeros((64, 512), dtype=torch.bfloat16))
    with pytest.raises(TypeError, match="CUDA"):
        bi.log_softmax(x)
    with pytest.raises(TypeError, match="CUDA"):
        bi.sample(x, torch.zeros(4, dtype=torch.int64), torch.zeros(4, dtype=torch.int64), 0.8)


def test_wrong_dtype_is_refused():
    class FakeCuda(torch.Tensor):  # a CPU tensor that claims to be on CUDA, to reach the dtype check
        @property
        def is_cuda(self):
            return True

    x = torch.zeros((4, 512), dtype=torch.float32).as_subclass(FakeCuda)
    with pytest.raises(TypeError, match="bfloat16"):
        bi.log_softmax(x)
    y = torch.zeros((4, 512, 3), dtype=torch.bfloat16).as_subclass(FakeCuda)
    with pytest.raises(ValueError, match="2 dims"):
        bi.row_mean(y)
