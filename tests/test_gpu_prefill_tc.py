"""Tensor-core causal prefill (bi_attention_prefill_tc): parity with the fp64 oracle,
whole vs chunked bit-identity (uneven chunks, appends between them), agreement with
the CUDA-core prefill within the bf16 tolerance, and the 4096-token configuration
(whole vs 8 x 512 chunks)."""
import numpy as np
import pytest
import torch

import invariant_deterministic_04_b200 as bi
import oracle
import synth
from gpu_util import TOL_BF16, dev, max_rel, same_bits

pytestmark = pytest.mark.gpu


def _dev(kv):
    return synth.PagedKV(kv.k_cache.to(dev()), kv.v_cache.to(dev()), kv.page_table.to(dev()),
                         kv.seq_lens.to(dev()), kv.max_pages)


@pytest.mark.parametrize("D,Hq,Hkv", [(128, 32, 8), (64, 32, 8), (128, 16, 8), (128, 32, 4)])  # groups 4, 4, 2, 8
def test_prefill_tc_matches_oracle(D, Hq, Hkv):
    S = 300
    q, qs, qp, kv = synth.prefill_inputs([S], Hq, Hkv, D, seed=70 + D + Hq)
    kvd = _dev(kv)
    out = bi.attention_prefill_tc(q.to(dev()), 0, 0, kvd.k_cache, kvd.v_cache, kvd.page_table)
    assert torch.isfinite(out.float()).all()
    rows = [0, 1, 2, 15, 16, 127, 128, 129, 200, 255, 256, 299]
    ref = oracle.attention_prefill(synth.to_f64(q)[rows], qs.numpy()[rows], qp.numpy()[rows],
                                   synth.to_f64(kv.k_cache), synth.to_f64(kv.v_cache), kv.page_table.numpy())
    assert max_rel(out.cpu()[rows], ref) <= TOL_BF16
    assert bi.get_device_error() == 0


@pytest.mark.parametrize("D,Hq,Hkv", [(128, 32, 8), (64, 32, 8)])
def test_prefill_tc_whole_equals_chunked_and_agrees_with_cuda_cores(D, Hq, Hkv):
    S = 1100
    q, qs, qp, kv = synth.prefill_inputs([S], Hq, Hkv, D, seed=73 + D)
    kvd = _dev(kv)
    qd = q.to(dev())
    whole = bi.attention_prefill_tc(qd, 0, 0, kvd.k_cache, kvd.v_cache, kvd.page_table)
    for _ in range(2):
        assert same_bits(bi.attention_prefill_tc(qd, 0, 0, kvd.k_cache, kvd.v_cache, kvd.page_table), whole)
    # uneven chunks, each appended to an empty (NaN) store before its own attention
    t = torch.arange(S)
    pages = kv.page_table[0, t // 16].long()
    k_tok = kv.k_cache[pages, :, t % 16, :].contiguous().to(dev())
    v_tok = kv.v_cache[pages, :, t % 16, :].contiguous().to(dev())
    ek = torch.full_like(kvd.k_cache, float("nan"))
    ev = torch.full_like(kvd.v_cache, float("nan"))
    chunked = torch.empty_like(whole)
    bounds = [0, 77, 128, 333, 512, 513, 1000, 1099, 1100]  # includes 1-row chunks
    for c0, c1 in zip(bounds[:-1], bounds[1:]):
        sl = slice(c0, c1)
        bi.kv_append(k_tok[sl], v_tok[sl], qs[sl].to(dev()), qp[sl].to(dev()), ek, ev, kvd.page_table)
        chunked[sl] = bi.attention_prefill_tc(qd[sl].contiguous(), 0, c0, ek, ev, kvd.page_table)
    assert same_bits(chunked, whole)
    cuda_cores = bi.attention_prefill(qd, qs.to(dev()), qp.to(dev()), kvd.k_cache, kvd.v_cache, kvd.page_table)
    assert max_rel(whole, synth.to_f64(cuda_cores.cpu())) <= TOL_BF16
    assert bi.get_device_error() == 0


def test_prefill_tc_large_score_jumps_take_the_rescale_path():
    # With q, k ~ N(0, 1) no later block's maximum exceeds the running reference
    # point by the lazy threshold (8 in log2 units), so O is never rescaled after
    # the first block. Keys at positions >= 130 scaled by 8 raise the block maxima
    # by about 20 (natural units) and force the rescale in the blocks after the jump
    # (thousands of times over the 300 rows x 32 heads). Parity with the oracle and
    # whole vs chunked bits must still hold.
    S, Hq, Hkv, D = 300, 32, 8, 128
    q, qs, qp, kv = synth.prefill_inputs([S], Hq, Hkv, D, seed=77)
    t = torch.arange(S)
    pages = kv.page_table[0, t // 16].long()
    big = t >= 130
    k = kv.k_cache.clone()
    k[pages[big], :, (t % 16)[big], :] = (k[pages[big], :, (t % 16)[big], :].float() * 8).to(torch.bfloat16)
    kv = synth.PagedKV(k, kv.v_cache, kv.page_table, kv.seq_lens, kv.max_pages)
    kvd = _dev(kv)
    qd = q.to(dev())
    out = bi.attention_prefill_tc(qd, 0, 0, kvd.k_cache, kvd.v_cache, kvd.page_table)
    assert torch.isfinite(out.float()).all()
    ref = oracle.attention_prefill(synth.to_f64(q), qs.numpy(), qp.numpy(), synth.to_f64(kv.k_cache),
                                   synth.to_f64(kv.v_cache), kv.page_table.numpy())
    assert max_rel(out.cpu(), ref) <= TOL_BF16
    for c0, c1 in ((0, 130), (130, 200), (200, 300)):  # the jump at a chunk start and inside one
        part = bi.attention_prefill_tc(qd[c0:c1].contiguous(), 0, c0, kvd.k_cache, kvd.v_cache, kvd.page_table)
        assert same_bits(part, out[c0:c1]), c0
    assert bi.get_device_error() == 0


def test_prefill_tc_full_size_4096_whole_vs_8_chunks():
    S, Hq, Hkv, D = 4096, 32, 8, 128
    kv = synth.paged_kv_device([S], Hkv, D, seed=60, max_pages=S // 16, device=dev())
    q = synth.normal_bf16((S, Hq, D), 61).to(dev())
    whole = bi.attention_prefill_tc(q, 0, 0, kv.k_cache, kv.v_cache, kv.page_table)
    for c0 in range(0, S, 512):
        part = bi.attention_prefill_tc(q[c0:c0 + 512].contiguous(), 0, c0, kv.k_cache, kv.v_cache, kv.page_table)
        assert same_bits(part, whole[c0:c0 + 512]), c0
    rows = [0, 511, 512, 2048, 4095]
    k, v, pt = synth.sequence_pages(kv, 0, S)
    ref = oracle.attention_prefill(synth.to_f64(q[rows].cpu()), np.zeros(len(rows), dtype=np.int64), np.array(rows),
                                   synth.to_f64(k), synth.to_f64(v), pt.numpy())
    assert max_rel(whole[rows], ref) <= TOL_BF16


def test_prefill_tc_validation_and_device_errors():
    # odd query-head group: refused on the host; bad page id: recorded on the device, no fault
    S, D = 200, 128
    q, qs, qp, kv = synth.prefill_inputs([S], 24, 8, D, seed=75)
    kvd = _dev(kv)
    with pytest.raises(bi.BIError, match="UNSUPPORTED"):
        bi.attention_prefill_tc(q.to(dev()), 0, 0, kvd.k_cache, kvd.v_cache, kvd.page_table)
    q, qs, qp, kv = synth.prefill_inputs([S], 32, 8, D, seed=76)
    kvd = _dev(kv)
    pt = kvd.page_table.clone()
    pt[0, 3] = kv.k_cache.shape[0] + 5  # outside the store
    bi.attention_prefill_tc(q.to(dev()), 0, 0, kvd.k_cache, kvd.v_cache, pt)
    torch.cuda.synchronize()
    assert bi.get_device_error() == 8
    # the context stays usable and the next call is correct
    out = bi.attention_prefill_tc(q.to(dev()), 0, 0, kvd.k_cache, kvd.v_cache, kvd.page_table)
    rows = [0, 199]
    ref = oracle.attention_prefill(synth.to_f64(q)[rows], qs.numpy()[rows], qp.numpy()[rows],
                                   synth.to_f64(kv.k_cache), synth.to_f64(kv.v_cache), kv.page_table.numpy())
    assert max_rel(out.cpu()[rows], ref) <= TOL_BF16
    assert bi.get_device_error() == 0
