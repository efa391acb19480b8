"""Pins for the oracle's row reductions (log_softmax, token log-probability, mean),
its Philox4x64-10 generator and its temperature sampler (CPU only).

Each pin comes from outside the oracle: closed forms, pure-Python brute force,
library routines (scipy's log_softmax, numpy's mean, numpy's own Philox bit
generator) and distributional facts (Gumbel-max draws follow softmax(x / T)).
A plausible slip — a missing max shift, a sign error in the Gumbel variate, x * T
instead of x / T, a wrong Philox constant, round or output word — fails one of them.
"""
import math
import warnings

import numpy as np
import pytest
import scipy.special

import oracle


# ---------------------------------------------------------------------------
# log_softmax / token log-probability


@pytest.mark.parametrize("N", [1, 2, 7, 32000])
@pytest.mark.parametrize("c", [0.0, -3.25, 41.0])
def test_log_softmax_constant_row_is_minus_log_n(N, c):
    y = oracle.log_softmax(np.full((1, N), c))
    np.testing.assert_allclose(y, -math.log(N), rtol=0, atol=1e-12)


@pytest.mark.parametrize("a,b", [(0.0, 1.0), (2.5, -4.0), (1000.0, 1000.0), (-750.0, -745.0)])
def test_log_softmax_two_values_closed_form(a, b):
    y = oracle.log_softmax(np.array([[a, b]]))
    # log(e^a / (e^a + e^b)) = -log(1 + e^(b - a)), written without overflow
    assert y[0, 0] == pytest.approx(-math.log1p(math.exp(b - a)) if b <= a else (a - b) - math.log1p(math.exp(a - b)),
                                    abs=1e-12)
    assert y[0, 1] == pytest.approx(-math.log1p(math.exp(a - b)) if a <= b else (b - a) - math.log1p(math.exp(b - a)),
                                    abs=1e-12)


def test_log_softmax_rows_far_apart():
    # each row is shifted by its own maximum: rows 1800 apart still give -log N,
    # and the token log-probability of any entry is the same
    x = np.array([[900.0, 900.0, 900.0], [-900.0, -900.0, -900.0]])
    np.testing.assert_allclose(oracle.log_softmax(x), -math.log(3), rtol=0, atol=1e-12)
    np.testing.assert_allclose(oracle.token_logprob(x, np.array([2, 0])), -math.log(3), rtol=0, atol=1e-12)


def test_log_softmax_matches_library_and_normalises():
    rng = np.random.default_rng(0)
    x = rng.normal(0, 3, size=(5, 1000))
    y = oracle.log_softmax(x)
    np.testing.assert_allclose(y, scipy.special.log_softmax(x, axis=-1), rtol=0, atol=1e-12)
    np.testing.assert_allclose(np.exp(y).sum(axis=-1), 1.0, rtol=0, atol=1e-12)
    np.testing.assert_allclose(oracle.log_softmax(x + 123.0), y, rtol=0, atol=1e-11)


def test_token_logprob_bruteforce():
    x = [[0.5, -1.0, 2.0, 0.0], [3.0, 3.0, -2.0, 1.0]]
    tok = [2, 1]
    got = oracle.token_logprob(np.array(x), np.array(tok))
    for m in range(2):
        den = sum(math.exp(v) for v in x[m])
        assert got[m] == pytest.approx(math.log(math.exp(x[m][tok[m]]) / den), abs=1e-13)


# ---------------------------------------------------------------------------
# mean


@pytest.mark.parametrize("K", [1, 8, 4096])
def test_row_mean_closed_forms(K):
    assert oracle.row_mean(np.full((1, K), -1.75))[0] == -1.75
    assert oracle.row_mean(np.arange(K, dtype=np.float64)[None])[0] == pytest.approx((K - 1) / 2, abs=1e-12)


def test_row_mean_library_and_bruteforce():
    rng = np.random.default_rng(1)
    x = rng.normal(0, 1, size=(4, 777))
    np.testing.assert_allclose(oracle.row_mean(x), np.mean(x, axis=-1), rtol=0, atol=1e-15)
    small = [[1.0, 2.0, 4.0], [-1.0, 0.5, 0.25]]
    assert list(oracle.row_mean(np.array(small))) == [sum(r) / 3 for r in small]


# ---------------------------------------------------------------------------
# Philox4x64-10 against numpy's independent implementation


def _words(v, n):
    return [np.uint64((v >> (64 * i)) & (2**64 - 1)) for i in range(n)]


@pytest.mark.parametrize("counter,key", [(0, 0), (5, 7), (2**64 - 1, 1), (2**128 - 2, 2**64 + 3),
                                         (2**64 - 3, 123456789 + (987654321 << 64))])
def test_philox_matches_numpy_bit_generator(counter, key):
    # numpy's Philox bit generator is Philox4x64-10; it increments its 256-bit counter
    # before each block, so its first block is the one at counter + 1
    with warnings.catch_warnings():
        warnings.simplefilter("ignore")
        raw = np.random.Philox(counter=counter, key=key).random_raw(12)
    for b in range(3):
        got = oracle.philox4x64_10(_words(counter + 1 + b, 4), _words(key, 2))
        assert [int(v) for v in got] == [int(v) for v in raw[4 * b:4 * b + 4]]


def test_sampling_uniforms_layout_and_range():
    seed, step, V = 0x1234_5678_9ABC_DEF0, 17, 1003
    u = oracle.sampling_uniforms(seed, step, V)
    # u_i = (top 23 bits of 32-bit half i mod 2 (low, high) of word (i mod 8) div 2 of
    # block (i div 8, step) + 1/2) * 2^-23, by Python integers
    for i in (0, 1, 2, 3, 7, 8, 9, 998, 1002):
        words = oracle.philox4x64_10(_words(i // 8, 1) + [np.uint64(step), np.uint64(0), np.uint64(0)],
                                     [np.uint64(seed), np.uint64(0)])
        half = (int(words[(i % 8) // 2]) >> (32 * (i % 2))) & 0xFFFFFFFF
        assert u[i] == ((half >> 9) + 0.5) / 2**23
    assert np.all((u > 0) & (u < 1))
    assert np.all((u * 2**23 - 0.5) == np.floor(u * 2**23))
    assert np.all(u.astype(np.float32).astype(np.float64) == u)  # exact in fp32
    # a row's draws do not depend on the vocabulary size asked for (nor on anything but seed, step, i)
    np.testing.assert_array_equal(oracle.sampling_uniforms(seed, step, 10), u[:10])
    assert not np.array_equal(oracle.sampling_uniforms(seed, step + 1, 10), u[:10])
    assert not np.array_equal(oracle.sampling_uniforms(seed + 1, step, 10), u[:10])


# ---------------------------------------------------------------------------
# Temperature sampling (Gumbel-max)


def test_sample_low_temperature_is_greedy():
    # the Gumbel variate lies in [-2.9, 16.7] for u in [2^-24, 1 - 2^-24]; at T = 1e-3
    # the logits are 1000 apart after division by T, far more than the noise: greedy
    rng = np.random.default_rng(2)
    x = rng.permutation(64).astype(np.float64)[None].repeat(8, axis=0)
    tok = oracle.sample(x, 1e-3, seeds=np.arange(8), steps=np.zeros(8, dtype=np.int64))
    assert list(tok) == [int(np.argmax(x[0]))] * 8


@pytest.mark.parametrize("T", [1.0, 2.0])
def test_sample_frequencies_follow_softmax(T):
    x = np.array([0.0, 1.0, 2.0, -1.0])
    n = 4000
    counts = np.zeros(4)
    for seed in range(n):
        counts[oracle.sample(x[None], T, seeds=[seed], steps=[3])[0]] += 1
    p = np.exp(x / T) / np.exp(x / T).sum()
    sigma = np.sqrt(n * p * (1 - p))
    assert np.all(np.abs(counts - n * p) < 4.5 * sigma), (counts, n * p)
    # and not the distribution of the other temperature (x * T or a flipped variate would match neither)
    other = np.exp(x * T) / np.exp(x * T).sum() if T != 1.0 else np.exp(-x) / np.exp(-x).sum()
    assert np.any(np.abs(counts - n * other) > 6 * np.sqrt(n * other * (1 - other)))


def test_sample_rows_do_not_depend_on_the_batch():
    # each row's token is a function of its own logits, seed and step: sampling a
    # batch gives, row by row, what sampling each row alone gives
    rng = np.random.default_rng(4)
    x = rng.normal(0, 0.5, size=(8, 64))
    seeds = np.array([11, 12, 13, 14, 15, 16, 17, 18])
    steps = np.array([0, 5, 5, 9, 2, 7, 1, 3])
    batch = oracle.sample(x, 1.0, seeds, steps)
    alone = [oracle.sample(x[m:m + 1], 1.0, seeds[m:m + 1], steps[m:m + 1])[0] for m in range(8)]
    assert list(batch) == alone
    # and the draw moves with the seed and with the step (64 near-uniform choices)
    assert len({int(oracle.sample(x[:1], 1.0, [s], [0])[0]) for s in range(16)}) > 4
    assert len({int(oracle.sample(x[:1], 1.0, [11], [t])[0]) for t in range(16)}) > 4


def test_gumbel_scores_closed_form():
    u = np.array([math.exp(-1.0), math.exp(-math.exp(-2.0))])  # -log(-log u) = 0 and 2
    np.testing.assert_allclose(oracle.gumbel_scores(np.array([3.0, -1.0]), 2.0, u), [1.5, 1.5], rtol=0, atol=1e-12)
