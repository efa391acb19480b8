"""GPU parity and invariance of the row reductions (log_softmax, token log-probability,
mean) and of temperature sampling, through the C ABI, against the fp64 oracle.

Tolerances: fp32 outputs within 1e-5 normwise per row (log_softmax, token
log-probability) and |mean error| <= 1e-5 * mean|x| (a mean can be near zero, so
its error is bounded by the row's scale). The uniforms are compared bit for bit.
A sampled token must be the oracle's Gumbel-max winner, except that when the
oracle's top-2 scores are closer than the fp32 error bound either one counts.
"""
import numpy as np
import pytest
import torch

import invariant_deterministic_04_b200 as bi
import oracle
import synth
from gpu_util import TOL_FP32, dev, max_rel, same_bits

pytestmark = pytest.mark.gpu

# N: one 8-vector, ragged tails across the 256-thread stride, the 32000 vocabulary,
# the register-resident maximum and the re-read path above it; together every
# register variant (vectors per thread 1, 2, 4, 8, 16) and the re-read one
SIZES = [8, 1000, 2056, 6000, 12000, 32000, 32768, 40000]


def _u64(t):
    return [int(v) & (2**64 - 1) for v in t.tolist()]


@pytest.mark.parametrize("N", SIZES)
def test_log_softmax_and_token_logprob_match_oracle(N):
    M = 6
    x = synth.logits(M, N, seed=80 + N % 97)
    x[1] = 0.25                     # constant row: every entry is -log(N)
    x[2, ::3] = float("-inf")       # masked vocabulary entries
    xd = x.to(dev())
    y = bi.log_softmax(xd)
    ref = oracle.log_softmax(synth.to_f64(x))
    fin = np.isfinite(ref)
    assert np.array_equal(np.isfinite(y.cpu().numpy()), fin)
    got = y.cpu().double().numpy()
    g0, r0 = np.where(fin, got, 0), np.where(fin, ref, 0)
    err = np.abs(g0 - r0).max(axis=1) / np.abs(r0).max(axis=1)
    assert err.max() <= TOL_FP32, err
    tok = torch.tensor([(7 * m + 1) % N for m in range(M)], dtype=torch.int32)
    tok[2] = 1  # finite entry of the masked row
    lp = bi.token_logprob(xd, tok.to(dev()))
    # the same lse and the same subtraction: bit-identical to the gathered log_softmax
    assert same_bits(lp, y[torch.arange(M), tok.long().to(dev())])
    np.testing.assert_allclose(lp.cpu().double().numpy(), oracle.token_logprob(synth.to_f64(x), tok.numpy()),
                               rtol=TOL_FP32, atol=0)
    assert bi.get_device_error() == 0


@pytest.mark.parametrize("K", [8, 2048, 4096, 6000, 12000, 40000])
def test_row_mean_matches_oracle(K):
    M = 7
    x = synth.normal_bf16((M, K), 90 + K % 89, mean=0.5)
    x[3] = -1.5
    y = bi.row_mean(x.to(dev()))
    xf = synth.to_f64(x)
    err = np.abs(y.cpu().double().numpy() - oracle.row_mean(xf))
    assert np.all(err <= 1e-5 * np.abs(xf).mean(axis=1)), err
    assert y[3].item() == -1.5


def _row_mean_model(x):
    """bi_row_mean's documented order in fp32 (include/bi.h): thread t of 256 adds the
    elements of its 8-element vectors t, t+256, ... in order; inside each warp an xor
    butterfly (offsets 16, 8, 4, 2, 1) whose lane-0 value is kept; the 8 warp values
    added left to right; one division by K. Every step is an IEEE fp32 operation, so
    numpy float32 reproduces it exactly."""
    xf = synth.to_f64(x).astype(np.float32)  # bf16 -> fp32 is exact
    M, K = xf.shape
    nvec = K // 8
    s = np.zeros((M, 256), dtype=np.float32)
    for t in range(256):
        for idx in range(t, nvec, 256):
            for k in range(8):
                s[:, t] = s[:, t] + xf[:, idx * 8 + k]
    w = s.reshape(M, 8, 32)
    lanes = np.arange(32)
    for off in (16, 8, 4, 2, 1):
        w = w + w[:, :, lanes ^ off]
    tot = w[:, 0, 0]
    for i in range(1, 8):
        tot = tot + w[:, i, 0]
    return tot / np.float32(K)


@pytest.mark.parametrize("K", [8, 2056, 4096, 40000])
def test_row_mean_is_the_documented_fp32_order_bit_for_bit(K):
    x = synth.normal_bf16((5, K), 150 + K % 97, mean=0.5)
    y = bi.row_mean(x.to(dev())).cpu().numpy()
    np.testing.assert_array_equal(y, _row_mean_model(x))


@pytest.mark.parametrize("op", ["log_softmax", "mean", "sample"])
def test_rows_are_batch_invariant_and_run_to_run(op):
    M, N = 301, 32000
    x = synth.logits(M, N, seed=95).to(dev())
    seeds = synth.request_seeds(M, 96).to(dev())
    steps = torch.arange(M, dtype=torch.int64, device=dev()) % 7
    run = {
        "log_softmax": lambda a, s, t: bi.log_softmax(a),
        "mean": lambda a, s, t: bi.row_mean(a),
        "sample": lambda a, s, t: bi.sample(a, s, t, 0.8),
    }[op]
    full = run(x, seeds, steps)
    assert same_bits(run(x, seeds, steps), full)
    perm = synth.permutation(M, 97).to(dev())
    assert same_bits(run(x[perm].contiguous(), seeds[perm].contiguous(), steps[perm].contiguous()), full[perm])
    for m in (0, 150, 300):
        for lo, hi in ((m, m + 1), (max(0, m - 3), m + 1)):
            part = run(x[lo:hi].contiguous(), seeds[lo:hi].contiguous(), steps[lo:hi].contiguous())
            assert same_bits(part, full[lo:hi]), (op, lo, hi)


def test_sampling_uniforms_are_the_oracle_bits():
    M, V = 5, 1032
    seeds = synth.request_seeds(M, 100)
    seeds[0] = 0
    seeds[1] = -1  # 2^64 - 1
    steps = torch.tensor([0, 1, 2**40 + 3, 7, 123456], dtype=torch.int64)
    u = bi.sampling_uniforms(seeds.to(dev()), steps.to(dev()), V).cpu().double().numpy()
    for m, (s, t) in enumerate(zip(_u64(seeds), _u64(steps))):
        assert np.array_equal(u[m], oracle.sampling_uniforms(s, t, V)), m


@pytest.mark.parametrize("T", [0.3, 1.0, 1.7])
def test_sample_matches_oracle_gumbel_max(T):
    M, V = 12, 32000
    x = synth.logits(M, V, seed=101)
    seeds = synth.request_seeds(M, 102)
    steps = torch.arange(M, dtype=torch.int64) * 5
    tok = bi.sample(x.to(dev()), seeds.to(dev()), steps.to(dev()), T).cpu().numpy()
    xf = synth.to_f64(x)
    for m, (s, t) in enumerate(zip(_u64(seeds), _u64(steps))):
        sc = oracle.gumbel_scores(xf[m], T, oracle.sampling_uniforms(s, t, V))
        top = oracle.argmax_lowest(sc)
        srt = np.sort(sc)
        bound = 2e-5 * (1.0 + abs(srt[-1]))  # fp32 error of 1/T, two logs and one FMA
        assert sc[tok[m]] >= srt[-1] - bound, m
        if srt[-1] - srt[-2] > bound:
            assert tok[m] == top, m


def test_sample_low_temperature_is_greedy():
    # at T = 1e-3 logits 1 apart are 1000 apart after the division, far more than the
    # Gumbel noise (within [-2.9, 16.7] for 23-bit uniforms): the draw is the argmax
    M, V = 16, 64
    g = synth.generator(104)
    x = torch.stack([torch.randperm(V, generator=g) for _ in range(M)]).to(torch.bfloat16)
    seeds = synth.request_seeds(M, 105)
    steps = torch.arange(M, dtype=torch.int64)
    tok = bi.sample(x.to(dev()), seeds.to(dev()), steps.to(dev()), 1e-3).cpu()
    assert torch.equal(tok.long(), torch.argmax(x.float(), dim=1))


def test_sample_nan_row_reports_and_leaves_other_rows_alone():
    # a row of NaN logits has no maximum: token 0 and BI_ERR_DEVICE_INDEX; the
    # other rows draw what they draw alone
    M, V = 4, 1000
    x = synth.logits(M, V, seed=106)
    x[2] = float("nan")
    seeds = synth.request_seeds(M, 107).to(dev())
    steps = torch.arange(M, dtype=torch.int64, device=dev())
    xd = x.to(dev())
    tok = bi.sample(xd, seeds, steps, 0.9)
    assert bi.get_device_error() == 8
    assert int(tok[2]) == 0
    for m in (0, 1, 3):
        one = bi.sample(xd[m:m + 1].contiguous(), seeds[m:m + 1].contiguous(), steps[m:m + 1].contiguous(), 0.9)
        assert int(one[0]) == int(tok[m]), m
    assert bi.get_device_error() == 0


def test_sample_frequencies_follow_softmax():
    # 4000 requests (seeds) sampling the same 8-entry row: the token frequencies
    # follow softmax(x / T)
    n, T = 4000, 1.3
    row = torch.tensor([0.0, 1.0, 2.0, -1.0, 0.5, -3.0, 1.5, 0.25], dtype=torch.bfloat16)
    x = row[None].repeat(n, 1).to(dev())
    seeds = torch.arange(n, dtype=torch.int64, device=dev())
    steps = torch.full((n,), 11, dtype=torch.int64, device=dev())
    tok = bi.sample(x, seeds, steps, T).cpu().numpy()
    counts = np.bincount(tok, minlength=8)
    p = np.exp(row.double().numpy() / T)
    p /= p.sum()
    sigma = np.sqrt(n * p * (1 - p))
    assert np.all(np.abs(counts - n * p) < 4.5 * sigma), (counts, n * p)


def test_reductions_full_size_4096x32000_sampled():
    # the benchmark's reductions workload: log_softmax, token log-probability and
    # sampling of 4096 rows of 32000 logits, checked on sampled rows
    M, V, T = 4096, 32000, 0.8
    x = synth.normal_bf16_device((M, V), 120, dev(), std=3.0)
    tok = torch.randint(0, V, (M,), generator=synth.generator(121), dtype=torch.int32)
    seeds = synth.request_seeds(M, 122)
    steps = torch.arange(M, dtype=torch.int64) % 13
    y = bi.log_softmax(x)
    lp = bi.token_logprob(x, tok.to(dev()))
    st = bi.sample(x, seeds.to(dev()), steps.to(dev()), T).cpu().numpy()
    rows = [0, 1, 2047, 4095]
    xf = synth.to_f64(x[rows])
    ref = oracle.log_softmax(xf)
    err = np.abs(y[rows].cpu().double().numpy() - ref).max(axis=1) / np.abs(ref).max(axis=1)
    assert err.max() <= TOL_FP32, err
    np.testing.assert_allclose(lp[rows].cpu().double().numpy(), oracle.token_logprob(xf, tok.numpy()[rows]),
                               rtol=TOL_FP32, atol=0)
    sd, sp = _u64(seeds), _u64(steps)
    for i, m in enumerate(rows):
        sc = oracle.gumbel_scores(xf[i], T, oracle.sampling_uniforms(sd[m], sp[m], V))
        srt = np.sort(sc)
        bound = 2e-5 * (1.0 + abs(srt[-1]))
        assert sc[st[m]] >= srt[-1] - bound, m
        if srt[-1] - srt[-2] > bound:
            assert st[m] == oracle.argmax_lowest(sc), m
    assert bi.get_device_error() == 0


def test_bad_token_gives_nan_and_device_index_error():
    x = synth.logits(2, 64, seed=103).to(dev())
    out = bi.token_logprob(x, torch.tensor([3, 64], dtype=torch.int32, device=dev()))
    assert bi.get_device_error() == 8
    assert torch.isfinite(out[0]) and torch.isnan(out[1])
    assert bi.get_device_error() == 0
