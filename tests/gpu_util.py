"""Small helpers for the GPU tests (comparison of bits, tolerances)."""
import numpy as np
import torch

import oracle
import synth

# Tolerances: normwise relative error per output row against the fp64 oracle.
TOL_BF16 = 1e-2   # bf16 outputs
TOL_FP32 = 1e-5   # fp32 outputs (LM-head recompute logits)


def dev():
    return torch.device("cuda:0")


def bits(t: torch.Tensor) -> torch.Tensor:
    """Integer view of a tensor's bits (bit-exact comparison that treats NaN/-0 exactly)."""
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16)
    if t.dtype == torch.float32:
        return t.view(torch.int32)
    return t


def same_bits(a: torch.Tensor, b: torch.Tensor) -> bool:
    return a.shape == b.shape and torch.equal(bits(a.contiguous()), bits(b.contiguous()))


def max_rel(got: torch.Tensor, ref: np.ndarray) -> float:
    return float(oracle.normwise_rel_err(synth.to_f64(got.cpu()), ref).max())
