"""bi_lmhead_argmax on the GPU: greedy tokens, recompute flags and fp32 logits
against the fp64 oracle; planted margins; bit-invariance across batch size;
thresholds that force or forbid the recompute; full size M=64, V=32000, K=2048."""
import numpy as np
import pytest
import torch

import invariant_deterministic_04_b200 as bi
import oracle
import synth
from gpu_util import TOL_FP32, dev, same_bits

pytestmark = pytest.mark.gpu
TAU = 0.5


def _check_against_oracle(h, w, tau, tokens, rec, logits):
    r = oracle.lmhead(synth.to_f64(h), synth.to_f64(w), tau)
    rec = rec.cpu().numpy().astype(bool)
    tokens = tokens.cpu().numpy()
    # the recompute decision: compared where the oracle's bf16 margin is clearly on one side
    # (a 1-ulp difference in a bf16 logit can move the margin by up to 2 bf16 ulps)
    top = np.abs(r["logits"]).max(axis=1)
    band = 2 * 2.0 ** (np.floor(np.log2(np.maximum(top, 1e-30))) - 7)
    clear = np.abs(r["margin_bf16"] - tau) > band
    assert (rec[clear] == r["recompute"][clear]).all()
    # recomputed rows: fp32 logits within 1e-5 normwise, token = exact argmax whenever
    # the exact top-2 margin exceeds the fp32 error bound
    if rec.any():
        lg = logits.cpu().numpy()[rec]
        err = oracle.normwise_rel_err(lg, r["logits"][rec])
        assert err.max() <= TOL_FP32, err.max()
        bound = 4 * TOL_FP32 * top[rec]
        ok = r["margin"][rec] > bound
        assert (tokens[rec][ok] == r["tokens"][rec][ok]).all()
    # first-pass rows: token = argmax of the bf16-rounded logits where those have a clear top-1
    keep = ~rec & clear
    assert (tokens[keep] == r["tokens_bf16"][keep]).all()
    return r, rec


@pytest.mark.parametrize("M,V,K", [(9, 1000, 256), (1, 32000, 2048), (64, 32000, 2048), (40, 4096, 512),
                                   (4, 32000, 2048), (3, 16384, 512),
                                   (2, 1000, 4096),   # the streaming recompute's largest K
                                   (4, 1000, 4160),   # K > 4096: the tiled recompute
                                   (5, 1000, 4096),   # the largest K of the W-streaming recompute
                                   (6, 2000, 4160)])  # K > 4096: the 64-row tiled recompute
def test_lmhead_matches_oracle(M, V, K):
    h, w = synth.lmhead_inputs(M, V, K, seed=M + V)
    tok, rec, lg = bi.lmhead_argmax(h.to(dev()), w.to(dev()), TAU, want_logits=True)
    _check_against_oracle(h, w, TAU, tok, rec, lg)
    # rows that were not recomputed are left untouched in logits_fp32
    norec = ~rec.cpu().bool()
    assert torch.isnan(lg.cpu()[norec]).all()


def test_lmhead_planted_margins():
    K, V = 128, 512
    _, w = synth.lmhead_inputs(1, V, K, seed=70)
    h = torch.zeros((5, K), dtype=torch.bfloat16)
    h[0, 0] = h[1, 1] = h[2, 2] = h[3, 3] = 1.0
    h[4, 4] = h[4, 5] = 1.0
    w[:, :6] = w[:, :6].clamp(-1, 1)
    w[7, 0], w[30, 0] = 3.0, 2.875      # margin 0.125 -> recompute, token 7
    w[12, 1], w[40, 1] = 8.0, 3.0       # margin 5 -> first pass, token 12
    w[5, 2], w[6, 2] = 2.0, 2.0         # exact tie -> margin 0, lowest index wins
    w[9, 3], w[20, 3] = 4.0, 3.5        # margin exactly 0.5 is not below 0.5 -> first pass
    # row 4: logits 256 (token 0) and 256 + 0.625 (token 1). Between 256 and 512 bf16
    # values are 2 apart, so the first pass sees a tie (margin 0, token 0); the fp32
    # recompute sees 256.625 and must return token 1.
    w[0, 4], w[0, 5] = 256.0, 0.0
    w[1, 4], w[1, 5] = 256.0, 0.625
    tok, rec, lg = bi.lmhead_argmax(h.to(dev()), w.to(dev()), TAU, want_logits=True)
    assert tok.cpu().tolist() == [7, 12, 5, 9, 1]
    assert rec.cpu().tolist() == [1, 0, 1, 0, 1]
    assert float(lg[0, 7]) == 3.0 and float(lg[0, 30]) == 2.875
    assert float(lg[4, 1]) == 256.625 and float(lg[4, 0]) == 256.0
    # the first pass alone (bf16 logits) could not tell rows 4's two tokens apart
    first = bi.matmul(h.to(dev()), w.to(dev()))
    assert float(first[4, 0]) == float(first[4, 1]) == 256.0


def test_lmhead_thresholds_force_or_forbid_recompute():
    h, w = synth.lmhead_inputs(16, 4096, 512, seed=71)
    hd, wd = h.to(dev()), w.to(dev())
    _, rec0, _ = bi.lmhead_argmax(hd, wd, 0.0)
    assert int(rec0.sum()) == 0
    tok, rec1, lg = bi.lmhead_argmax(hd, wd, float("inf"), want_logits=True)
    assert int(rec1.sum()) == 16
    assert (tok.cpu() == torch.argmax(lg.cpu(), dim=1).to(torch.int32)).all()


def _fp32_fma_chain(h, w):
    """fp32 logits computed as the header specifies: one FMA chain per logit in ascending
    k, acc = fma(h[k], w[k], acc) from 0. A product of two bf16 values is exact in fp64,
    so float64(acc) + h*w is the exact sum here and one rounding to fp32 is the fused
    result."""
    hf, wf = synth.to_f64(h), synth.to_f64(w)
    acc = np.zeros((hf.shape[0], wf.shape[0]), dtype=np.float32)
    for k in range(hf.shape[1]):
        acc = (acc.astype(np.float64) + np.outer(hf[:, k], wf[:, k])).astype(np.float32)
    return acc


@pytest.mark.parametrize("M,V,K", [(1, 1000, 256),     # W-streaming recompute of a single row
                                   (2, 520, 128),      # the 8-row streaming kernel, two rows used
                                   (3, 1000, 256),
                                   (4, 4096, 1024),
                                   (10, 1000, 256),    # a group of eight rows, then a group of two
                                   (30, 520, 128)])    # the 64-row tiled recompute
def test_lmhead_recompute_is_the_documented_fp32_chain_bit_for_bit(M, V, K):
    # threshold inf flags every row; each path that produces fp32 logits must give
    # exactly the ascending-k fp32 FMA chain
    h, w = synth.lmhead_inputs(M, V, K, seed=400 + M)
    tok, rec, lg = bi.lmhead_argmax(h.to(dev()), w.to(dev()), float("inf"), want_logits=True)
    assert int(rec.sum()) == M
    np.testing.assert_array_equal(lg.cpu().numpy(), _fp32_fma_chain(h, w))


def test_lmhead_batch_invariant():
    M, V, K = 64, 32000, 2048
    h, w = synth.lmhead_inputs(M, V, K, seed=72)
    hd, wd = h.to(dev()), w.to(dev())
    tok, rec, lg = bi.lmhead_argmax(hd, wd, TAU, want_logits=True)
    for r in (0, 13, 63):
        t1, r1, l1 = bi.lmhead_argmax(hd[r:r + 1].contiguous(), wd, TAU, want_logits=True)
        assert int(t1[0]) == int(tok[r]) and int(r1[0]) == int(rec[r])
        if int(r1[0]):
            assert same_bits(l1[0], lg[r])
    # small batches put their flagged rows through the streaming recompute (one row, or
    # groups of 8), the 64-row batch through the tiled one: the same bits
    for m in (1, 2, 4, 5, 7, 33):
        t2, r2, l2 = bi.lmhead_argmax(hd[:m].contiguous(), wd, TAU, want_logits=True)
        assert torch.equal(t2, tok[:m]) and torch.equal(r2, rec[:m])
        mask = r2.bool()
        assert same_bits(l2[mask], lg[:m][mask])
    t3, r3, _ = bi.lmhead_argmax(hd, wd, TAU)
    assert torch.equal(t3, tok) and torch.equal(r3, rec)
