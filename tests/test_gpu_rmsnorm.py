"""RMSNorm on the GPU: parity with the fp64 oracle, bit-invariance across batch
size and row position, run-to-run bit-exactness, in-place use."""
import pytest
import torch

import invariant_deterministic_04_b200 as bi
import oracle
import synth
from gpu_util import TOL_BF16, dev, max_rel, same_bits

pytestmark = pytest.mark.gpu
EPS = 1e-6


# every register variant of the kernel (16-byte vectors per thread NV = 1, 2, 4, 8, 16),
# each also with a ragged last round (K = 136, 1032, 3080, 5128, 8200)
@pytest.mark.parametrize("M,K", [(1, 512), (7, 512), (32, 512), (129, 4096), (5, 2048), (3, 8), (4, 136),
                                 (2, 16384), (300, 1024), (3, 1032), (3, 3080), (3, 5128), (2, 8192), (2, 8200)])
def test_rmsnorm_matches_oracle(M, K):
    x, w = synth.rmsnorm_inputs(M, K, seed=M + K)
    y = bi.rmsnorm(x.to(dev()), w.to(dev()), EPS)
    ref = oracle.rmsnorm(synth.to_f64(x), synth.to_f64(w), EPS)
    assert max_rel(y, ref) <= TOL_BF16


def test_rmsnorm_constant_row_is_weight_at_eps0():
    K = 4096
    w = synth.normal_bf16((K,), 3, std=0.1, mean=1.0).to(dev())
    x = torch.full((3, K), 0.75, dtype=torch.bfloat16, device=dev())
    x[1] = -2.5
    y = bi.rmsnorm(x, w, 0.0)
    assert same_bits(y[0], w) and same_bits(y[2], w) and same_bits(y[1], -w)


@pytest.mark.parametrize("K", [512, 4096])
def test_rmsnorm_batch_invariant(K):
    M = 2048 if K == 4096 else 32
    x, w = synth.rmsnorm_inputs(M, K, seed=11)
    x, w = x.to(dev()), w.to(dev())
    full = bi.rmsnorm(x, w, EPS)
    for m in (1, 2, 7, 16, 33, 257, M - 1):
        if m <= M:
            assert same_bits(bi.rmsnorm(x[:m].contiguous(), w, EPS), full[:m])
    for r in (0, 5, M // 2, M - 1):
        assert same_bits(bi.rmsnorm(x[r:r + 1].contiguous(), w, EPS)[0], full[r])
    perm = synth.permutation(M, 12).to(dev())
    assert same_bits(bi.rmsnorm(x[perm].contiguous(), w, EPS), full[perm])


def test_rmsnorm_run_to_run_and_in_place():
    x, w = synth.rmsnorm_inputs(513, 4096, seed=13)
    x, w = x.to(dev()), w.to(dev())
    first = bi.rmsnorm(x, w, EPS)
    for _ in range(5):
        assert same_bits(bi.rmsnorm(x, w, EPS), first)
    xi = x.clone()
    bi.rmsnorm(xi, w, EPS, out=xi)
    assert same_bits(xi, first)


def test_rmsnorm_strided_rows():
    base, w = synth.rmsnorm_inputs(40, 1024, seed=14)
    base, w = base.to(dev()), w.to(dev())
    x = base[:, :512]  # ld = 1024
    y = bi.rmsnorm(x, w[:512].contiguous(), EPS)
    assert same_bits(y, bi.rmsnorm(x.contiguous(), w[:512].contiguous(), EPS))
    ref = oracle.rmsnorm(synth.to_f64(x.cpu()), synth.to_f64(w[:512].cpu()), EPS)
    assert max_rel(y, ref) <= TOL_BF16


def test_rmsnorm_full_size_65536x4096_sampled():
    # the benchmark's RMSNorm workload (512 MiB in, 512 MiB out): parity on sampled
    # rows, and each sampled row alone gives the same bits
    M, K = 65536, 4096
    x = synth.normal_bf16_device((M, K), 15, dev())
    w = synth.normal_bf16((K,), 16, std=0.1, mean=1.0).to(dev())
    y = bi.rmsnorm(x, w, EPS)
    rows = [0, 1, 4095, 32768, 65535]
    ref = oracle.rmsnorm(synth.to_f64(x[rows]), synth.to_f64(w), EPS)
    assert max_rel(y[rows], ref) <= TOL_BF16
    for r in rows:
        assert same_bits(bi.rmsnorm(x[r:r + 1].contiguous(), w, EPS)[0], y[r]), r


# Batches larger than the persistent grid (8, 4 or 2 CTAs per SM by register
# variant), so every CTA takes several rows and prefetches the next one while it
# writes the current one: every row equals the same row computed alone (grid of one
# CTA) and in a reversed batch, and sampled rows match the oracle.
@pytest.mark.parametrize("M,K", [(2500, 512), (2500, 2048), (2600, 4096), (1300, 8192), (700, 16384), (2501, 1032)])
def test_rmsnorm_rows_beyond_the_persistent_grid(M, K):
    x, w = synth.rmsnorm_inputs(M, K, seed=17 + K)
    x, w = x.to(dev()), w.to(dev())
    full = bi.rmsnorm(x, w, EPS)
    rev = torch.arange(M - 1, -1, -1, device=dev())
    assert same_bits(bi.rmsnorm(x[rev].contiguous(), w, EPS), full[rev])
    for r in (0, 1, M // 3, M - 2, M - 1):
        assert same_bits(bi.rmsnorm(x[r:r + 1].contiguous(), w, EPS)[0], full[r]), r
    rows = [0, 7, M // 2, M - 1]
    ref = oracle.rmsnorm(synth.to_f64(x[rows].cpu()), synth.to_f64(w.cpu()), EPS)
    assert max_rel(full[rows], ref) <= TOL_BF16
