"""bi_matmul on the GPU (tcgen05 + TMA): parity with the fp64 oracle, exact
small-integer products (pins the shared-memory layout and descriptors),
row-position independence inside a 128-row tile, ragged products on CTA-pair
(256-row) tiles, bit-invariance across the M
sweep at K=4096, N in {4096, 6144, 14336}, run-to-run bit-exactness, and the
RMSNorm -> matmul chain of the 32 x 512 -> 1024 configuration."""
import numpy as np
import pytest
import torch

import invariant_deterministic_04_b200 as bi
import oracle
import synth
from gpu_util import TOL_BF16, dev, max_rel, same_bits

pytestmark = pytest.mark.gpu

M_SWEEP = [1, 2, 3, 4, 7, 8, 13, 16, 32, 33, 64, 127, 128, 255, 256, 257, 512, 1023, 1024, 2047, 2048]


@pytest.mark.parametrize("M,N,K", [(300, 520, 512), (1, 256, 64), (128, 256, 128), (129, 264, 192),
                                   (32, 1024, 512), (5, 8, 64), (257, 4096, 1024),
                                   (130, 520, 16384)])  # a long K: 256 blocks accumulated in TMEM
def test_matmul_matches_oracle(M, N, K):
    a, w = synth.matmul_inputs(M, N, K, seed=M * 7 + N + K)
    c = bi.matmul(a.to(dev()), w.to(dev()))
    assert max_rel(c, oracle.matmul(synth.to_f64(a), synth.to_f64(w))) <= TOL_BF16


# Ragged products on CTA pairs (256-row tiles; on a 148-SM B200 (1100, 4000), (1000,
# 5992) and (513, 6152) take 192-wide tiles, the others 256-wide): a last pair tile whose
# second CTA holds no valid row (M = 1100, 1000) or part of one (M = 200), a last tile
# whose W half lies past N, a 32-column chunk cut by N (N = 5992, 4104, 6152), odd M, and
# last rounds with a few tiles (M = 1024, 2047 at N = 14336) or a partial W slice
# (M = 513, N = 6152).
@pytest.mark.parametrize("M,N,K", [(1100, 4000, 512), (1000, 5992, 320), (2047, 4104, 256), (600, 6000, 1024),
                                   (1024, 14336, 128), (2047, 14336, 64), (513, 6152, 256), (200, 14336, 64)])
def test_matmul_pair_tiles_match_oracle(M, N, K):
    assert bi.matmul_tile_m(M, N) == 256
    a, w = synth.matmul_inputs(M, N, K, seed=M + N + K)
    c = bi.matmul(a.to(dev()), w.to(dev()))
    assert max_rel(c, oracle.matmul(synth.to_f64(a), synth.to_f64(w))) <= TOL_BF16
    # the same rows on single-CTA tiles (fewer than 256 rows) give the same bits
    for r0 in (0, M - 7):
        assert same_bits(bi.matmul(a[r0:r0 + 7].to(dev()), w.to(dev())), c[r0:r0 + 7]), r0


def test_matmul_small_integers_exact():
    # entries in {-1, 0, 1}: every product and partial sum is an integer below 2^24
    # and |C| <= K = 192 fits bf16 exactly, so any layout slip shows as a wrong integer.
    g = synth.generator(21)
    M, N, K = 200, 520, 192
    a = torch.randint(-1, 2, (M, K), generator=g).to(torch.bfloat16)
    w = torch.randint(-1, 2, (N, K), generator=g).to(torch.bfloat16)
    c = bi.matmul(a.to(dev()), w.to(dev())).cpu()
    ref = oracle.matmul(synth.to_f64(a), synth.to_f64(w))
    np.testing.assert_array_equal(synth.to_f64(c), ref)


def test_matmul_one_hot_rows_select_weight_columns():
    N, K = 512, 256
    _, w = synth.matmul_inputs(1, N, K, seed=22)
    ks = [0, 1, 63, 64, 100, 255]
    a = torch.zeros((len(ks), K), dtype=torch.bfloat16)
    for m, k in enumerate(ks):
        a[m, k] = 1.0
    c = bi.matmul(a.to(dev()), w.to(dev())).cpu()
    for m, k in enumerate(ks):
        assert same_bits(c[m], w[:, k].contiguous())


def test_matmul_row_position_independent():
    # Each row computed alone (M = 1, tile row 0) equals the same row computed at
    # tile row r % 128 of a 300-row batch, bit for bit.
    M, N, K = 300, 512, 1024
    a, w = synth.matmul_inputs(M, N, K, seed=23)
    a, w = a.to(dev()), w.to(dev())
    full = bi.matmul(a, w)
    for r in range(M):
        assert same_bits(bi.matmul(a[r:r + 1].contiguous(), w)[0], full[r]), r


@pytest.mark.parametrize("N", [4096, 6144, 14336])
def test_matmul_batch_invariant_over_m_sweep(N):
    K = 4096
    a, w = synth.matmul_inputs(2048, N, K, seed=24)
    a, w = a.to(dev()), w.to(dev())
    full = bi.matmul(a, w)
    for m in M_SWEEP:
        assert same_bits(bi.matmul(a[:m].contiguous(), w), full[:m]), m
    # the sweep crosses tile widths (on a 148-SM B200: 32/64/128/256, and 192 at N = 6144)
    # and both tile heights: 128-row tiles on one CTA, 256-row tiles on a CTA pair
    assert len({bi.matmul_tile_n(m, N) for m in M_SWEEP + [2048]}) >= 2
    assert {bi.matmul_tile_m(m, N) for m in M_SWEEP + [2048]} == {128, 256}
    # rows in a permuted batch and a batch taken from the middle
    perm = synth.permutation(2048, 25).to(dev())
    assert same_bits(bi.matmul(a[perm].contiguous(), w), full[perm])
    assert same_bits(bi.matmul(a[1000:1037].contiguous(), w), full[1000:1037])
    # full-size parity on sampled rows
    rows = [0, 1, 127, 128, 1023, 2047]
    ref = oracle.matmul(synth.to_f64(a[rows].cpu()), synth.to_f64(w.cpu()))
    assert max_rel(full[rows], ref) <= TOL_BF16


def test_matmul_run_to_run():
    a, w = synth.matmul_inputs(2048, 6144, 4096, seed=26)
    a, w = a.to(dev()), w.to(dev())
    first = bi.matmul(a, w)
    for _ in range(3):
        assert same_bits(bi.matmul(a, w), first)


def test_matmul_strided_operands_and_output():
    a, w = synth.matmul_inputs(100, 512, 1024, seed=27)
    a, w = a.to(dev()), w.to(dev())
    out = torch.zeros((100, 1024), dtype=torch.bfloat16, device=dev())
    bi.matmul(a[:, :512], w[:, :512], out=out[:, 256:768])
    ref = bi.matmul(a[:, :512].contiguous(), w[:, :512].contiguous())
    assert same_bits(out[:, 256:768], ref)
    assert int(out[:, :256].abs().sum()) == 0 and int(out[:, 768:].abs().sum()) == 0


def test_rmsnorm_matmul_chain_32x512x1024():
    x, wn = synth.rmsnorm_inputs(32, 512, seed=0)
    _, W = synth.matmul_inputs(32, 1024, 512, seed=2)
    xd, wnd, Wd = x.to(dev()), wn.to(dev()), W.to(dev())
    c = bi.matmul(bi.rmsnorm(xd, wnd, 1e-6), Wd)
    for m in (1, 2, 7, 16):
        for start in (0, 32 - m):
            sub = bi.matmul(bi.rmsnorm(xd[start:start + m].contiguous(), wnd, 1e-6), Wd)
            assert same_bits(sub, c[start:start + m])
    # the chain in double, no bf16 intermediate
    ref = oracle.matmul(oracle.rmsnorm(synth.to_f64(x), synth.to_f64(wn), 1e-6), synth.to_f64(W))
    assert max_rel(c, ref) <= TOL_BF16


def _multi_inputs(M, Ns, K, seed):
    a = synth.normal_bf16((M, K), seed)
    ws = [synth.normal_bf16((n, K), seed + 1 + j, std=0.02) for j, n in enumerate(Ns)]
    return a.to(dev()), [w.to(dev()) for w in ws]


# Several products with one A in one call: each output equals bi_matmul's, bit for bit,
# whether the call runs them as one joint launch on CTA pairs (every product on pair
# tiles: M >= 129 here, and at N = 4096 from M = 600 on) or as separate launches.
@pytest.mark.parametrize("M", [1, 64, 128, 129, 255, 256, 300, 512, 1023, 2048])
def test_matmul_multi_equals_separate_calls(M):
    a, ws = _multi_inputs(M, [4096, 6144, 14336], 4096, seed=60 + M)
    cs = bi.matmul_multi(a, ws)
    for w, c in zip(ws, cs):
        assert same_bits(c, bi.matmul(a, w)), (M, w.shape[0])


def test_matmul_multi_ragged_two_and_one_products_and_strided_outputs():
    # ragged N and M; on a 148-SM B200 the first call runs as one joint launch on
    # 256-wide pair tiles (485 tiles; alone, N = 4000 would take 192-wide ones)
    a, ws = _multi_inputs(1100, [4000, 6152, 14336], 512, seed=70)
    cs = bi.matmul_multi(a, ws)
    for w, c in zip(ws, cs):
        assert same_bits(c, bi.matmul(a, w))
    ref = oracle.matmul(synth.to_f64(a[::97].cpu()), synth.to_f64(ws[1].cpu()))
    assert max_rel(cs[1][::97], ref) <= TOL_BF16
    # two products, written into column ranges of one wider output
    big = torch.full((1100, 4000 + 6152 + 8), float("nan"), dtype=torch.bfloat16, device=dev())
    outs = [big[:, :4000], big[:, 4000:4000 + 6152]]
    bi.matmul_multi(a, ws[:2], outs=outs)
    assert same_bits(outs[0], cs[0]) and same_bits(outs[1], cs[1])
    assert torch.isnan(big[:, -8:].float()).all()  # columns past the outputs untouched
    # one product: the same as bi_matmul
    assert same_bits(bi.matmul_multi(a, ws[2:])[0], cs[2])
    # a mix where one product alone would not use pair tiles (narrow N): separate launches
    a2, ws2 = _multi_inputs(300, [264, 14336], 256, seed=71)
    for w, c in zip(ws2, bi.matmul_multi(a2, ws2)):
        assert same_bits(c, bi.matmul(a2, w))
