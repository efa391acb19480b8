"""Attention over the paged store on the GPU: decode and causal prefill parity
with the fp64 oracle, closed forms, NaN-poisoned stale slots, bit-invariance
across batch size / order / page placement, whole vs chunked prefill, prefill
row == decode row, device-side index errors, and full-size sampled parity
(32 q-heads / 8 kv-heads, D=128, lengths ~ U[1, 32768], B=256; S=4096 prefill
whole vs 8 x 512 chunks)."""
import math

import numpy as np
import pytest
import torch

import invariant_deterministic_04_b200 as bi
import oracle
import synth
from gpu_util import TOL_BF16, dev, max_rel, same_bits

pytestmark = pytest.mark.gpu


def _to_dev(kv):
    return synth.PagedKV(kv.k_cache.to(dev()), kv.v_cache.to(dev()), kv.page_table.to(dev()),
                         kv.seq_lens.to(dev()), kv.max_pages)


def _decode(q, kv, **kw):
    return bi.attention_decode(q, kv.k_cache, kv.v_cache, kv.page_table, kv.seq_lens, **kw)


def _oracle_decode(q, kv):
    return oracle.attention_decode(synth.to_f64(q), synth.to_f64(kv.k_cache), synth.to_f64(kv.v_cache),
                                   kv.page_table.cpu().numpy(), kv.seq_lens.cpu().numpy())


# every instantiation of the split kernel: D in {64, 128} x group size Hq/Hkv in {1, 2, 4, 8}
@pytest.mark.parametrize("Hq,Hkv,D", [(32, 8, 128), (32, 8, 64), (8, 8, 128), (32, 4, 128), (16, 8, 64), (8, 1, 64),
                                      (16, 8, 128), (8, 8, 64)])
def test_decode_matches_oracle(Hq, Hkv, D):
    lens = [1, 16, 17, 255, 256, 257, 700, 513]
    q, kv = synth.decode_inputs(len(lens), Hq, Hkv, D, max_len=800, seed=Hq + Hkv + D, lens=lens)
    out = _decode(q.to(dev()), _to_dev(kv))
    assert torch.isfinite(out.float()).all()  # NaN in stale slots never reaches a result
    assert max_rel(out, _oracle_decode(q, kv)) <= TOL_BF16
    assert bi.get_device_error() == 0


def test_decode_closed_forms():
    # L = 1 returns v0 exactly; identical keys return the mean of the visible values
    q, kv = synth.decode_inputs(2, 32, 8, 128, max_len=300, seed=31, lens=[1, 300], poison_tail=True)
    k = kv.k_cache.clone()
    p1 = kv.page_table[1, :19]
    k[p1] = k[int(p1[0]), :, 0:1, :]  # every slot of sequence 1 holds the same key (per kv-head)
    kv = synth.PagedKV(k, kv.v_cache, kv.page_table, kv.seq_lens, kv.max_pages)
    out = _decode(q.to(dev()), _to_dev(kv)).cpu()
    v0 = kv.v_cache[int(kv.page_table[0, 0]), :, 0, :]  # [Hkv, D]
    assert same_bits(out[0], v0.repeat_interleave(4, dim=0))
    vals = np.stack([synth.to_f64(kv.v_cache[int(kv.page_table[1, t // 16]), :, t % 16, :]) for t in range(300)])
    mean = vals.mean(axis=0).repeat(4, axis=0)
    assert max_rel(out[1], mean) <= TOL_BF16


def test_decode_zero_length_sequences_give_zero_rows():
    # a sequence of length 0 sees no key: its rows are +0 in every bit, and the
    # other rows keep the bits they have alone. The pages stay allocated (lengths
    # 1, 40, 1) so only seq_lens says the outer two are empty.
    q, kv = synth.decode_inputs(3, 32, 8, 128, max_len=64, seed=35, lens=[1, 40, 1])
    kv = synth.PagedKV(kv.k_cache, kv.v_cache, kv.page_table, torch.tensor([0, 40, 0], dtype=torch.int32),
                       kv.max_pages)
    qd, kvd = q.to(dev()), _to_dev(kv)
    out = _decode(qd, kvd)
    assert bi.get_device_error() == 0
    assert bool((out[0].view(torch.int16) == 0).all()) and bool((out[2].view(torch.int16) == 0).all())
    one = bi.attention_decode(qd[1:2].contiguous(), kvd.k_cache, kvd.v_cache, kvd.page_table[1:2].contiguous(),
                              kvd.seq_lens[1:2].contiguous())
    assert same_bits(one[0], out[1])
    # every sequence empty: no split at all, all rows zero
    empty = bi.attention_decode(qd, kvd.k_cache, kvd.v_cache, kvd.page_table,
                                torch.zeros(3, dtype=torch.int32, device=dev()))
    assert bi.get_device_error() == 0
    assert bool((empty.view(torch.int16) == 0).all())


def test_decode_batch_invariant_and_run_to_run():
    lens = [3000, 1, 257, 4096, 77, 1500, 256, 999]
    q, kv = synth.decode_inputs(len(lens), 32, 8, 128, max_len=4096, seed=32, lens=lens)
    qd, kvd = q.to(dev()), _to_dev(kv)
    full = _decode(qd, kvd)
    for _ in range(3):
        assert same_bits(_decode(qd, kvd), full)
    # each sequence alone
    for b in range(len(lens)):
        one = bi.attention_decode(qd[b:b + 1].contiguous(), kvd.k_cache, kvd.v_cache,
                                  kvd.page_table[b:b + 1].contiguous(), kvd.seq_lens[b:b + 1].contiguous())
        assert same_bits(one[0], full[b]), b
    # batch order permuted
    perm = synth.permutation(len(lens), 33).to(dev())
    outp = bi.attention_decode(qd[perm].contiguous(), kvd.k_cache, kvd.v_cache, kvd.page_table[perm].contiguous(),
                               kvd.seq_lens[perm].contiguous())
    assert same_bits(outp, full[perm])


def test_decode_heads_per_warp_do_not_change_bits():
    """Decode reduces a (row, kv-head, split) with all 4 query heads of the kv-head on
    one warp when the batch's items fill the GPU, with 2 or 1 per warp when they fill
    at most a half or a quarter of it (on a 148-SM B200: 8 rows of 4096 tokens take
    4 per warp, 5 of them 2, 3 of them 1). Every head's bits are the same."""
    lens = [4096] * 8
    q, kv = synth.decode_inputs(8, 32, 8, 128, max_len=4096, seed=90, lens=lens)
    qd, kvd = q.to(dev()), _to_dev(kv)
    full = _decode(qd, kvd)
    for sub in ([0, 2, 4, 6, 7], [1, 3, 5], [6]):
        s = torch.tensor(sub, device=dev())
        part = bi.attention_decode(qd[s].contiguous(), kvd.k_cache, kvd.v_cache, kvd.page_table[s].contiguous(),
                                   kvd.seq_lens[s].contiguous())
        assert same_bits(part, full[s]), sub
    kv_sub = synth.PagedKV(kv.k_cache, kv.v_cache, kv.page_table[[6]], kv.seq_lens[[6]], kv.max_pages)
    assert max_rel(full[6:7], _oracle_decode(q[6:7], kv_sub)) <= TOL_BF16
    assert bi.get_device_error() == 0


@pytest.mark.parametrize("D", [128, 64])
def test_decode_combine_width_does_not_change_bits(D):
    """96 sequences x 32 heads fold their splits with D / 32 (or D / 64) dims per
    lane; 3 sequences with one dim per lane over D / 32 warps. Same bits, and the
    oracle agrees with both."""
    q, kv = synth.decode_inputs(96, 32, 8, D, max_len=1300, seed=70 + D)
    qd, kvd = q.to(dev()), _to_dev(kv)
    full = _decode(qd, kvd)
    sub = [0, 41, 95]
    s = torch.tensor(sub, device=dev())
    few = bi.attention_decode(qd[s].contiguous(), kvd.k_cache, kvd.v_cache, kvd.page_table[s].contiguous(),
                              kvd.seq_lens[s].contiguous())
    assert same_bits(few, full[s])
    kv_sub = synth.PagedKV(kv.k_cache, kv.v_cache, kv.page_table[sub], kv.seq_lens[sub], kv.max_pages)
    assert max_rel(few, _oracle_decode(q[sub], kv_sub)) <= TOL_BF16


def test_decode_invariant_to_physical_page_placement():
    lens = [1000, 333]
    q, kv = synth.decode_inputs(2, 32, 8, 64, max_len=1024, seed=34, lens=lens)
    ref = _decode(q.to(dev()), _to_dev(kv))
    n = kv.num_pages
    perm = synth.permutation(n, 35)
    k2, v2 = torch.empty_like(kv.k_cache), torch.empty_like(kv.v_cache)
    k2[perm], v2[perm] = kv.k_cache, kv.v_cache
    pt2 = torch.where(kv.page_table >= 0, perm.to(torch.int32)[kv.page_table.clamp(min=0).long()], kv.page_table)
    kv2 = synth.PagedKV(k2, v2, pt2.to(torch.int32), kv.seq_lens, kv.max_pages)
    assert same_bits(_decode(q.to(dev()), _to_dev(kv2)), ref)


def _prefill(q, q_seq, q_pos, kv):
    return bi.attention_prefill(q, q_seq, q_pos, kv.k_cache, kv.v_cache, kv.page_table)


@pytest.mark.parametrize("D", [128, 64])
def test_prefill_matches_oracle(D):
    lens = [300, 45]
    q, qs, qp, kv = synth.prefill_inputs(lens, 32, 8, D, seed=40 + D)
    out = _prefill(q.to(dev()), qs.to(dev()), qp.to(dev()), _to_dev(kv)).cpu()
    rows = [0, 1, 15, 16, 100, 255, 256, 257, 299, 300, 320, 344]
    ref = oracle.attention_prefill(synth.to_f64(q)[rows], qs.numpy()[rows], qp.numpy()[rows],
                                   synth.to_f64(kv.k_cache), synth.to_f64(kv.v_cache), kv.page_table.numpy())
    assert max_rel(out[rows], ref) <= TOL_BF16


def test_prefill_row_equals_decode_row():
    S = 700
    q, qs, qp, kv = synth.prefill_inputs([S], 32, 8, 128, seed=42)
    kvd = _to_dev(kv)
    pre = _prefill(q.to(dev()), qs.to(dev()), qp.to(dev()), kvd)
    for p in (0, 15, 255, 256, 511, 699):
        lens = torch.tensor([p + 1], dtype=torch.int32, device=dev())
        dec = bi.attention_decode(q[p:p + 1].to(dev()), kvd.k_cache, kvd.v_cache, kvd.page_table, lens)
        assert same_bits(dec[0], pre[p]), p


@pytest.mark.parametrize("Hq,Hkv,D", [(32, 8, 128), (32, 4, 64), (8, 1, 128)])
def test_prefill_rows_in_any_order_and_mix(Hq, Hkv, D):
    """Rows of three sequences in sequence order, then in a seeded shuffle (the
    prefill kernel's windows of consecutive rows then mix sequences, so rows that
    share a page-table row are scattered): every row keeps its bits, and equals the
    decode of that row."""
    lens = [300, 37, 530]
    q, qs, qp, kv = synth.prefill_inputs(lens, Hq, Hkv, D, seed=80 + D)
    kvd = _to_dev(kv)
    qd, qsd, qpd = q.to(dev()), qs.to(dev()), qp.to(dev())
    ordered = _prefill(qd, qsd, qpd, kvd)
    perm = synth.permutation(q.shape[0], 81).to(dev())
    shuffled = _prefill(qd[perm].contiguous(), qsd[perm].contiguous(), qpd[perm].contiguous(), kvd)
    assert same_bits(shuffled, ordered[perm])
    for row in (0, 299, 300, 336, 337, 600, 866):
        b, p = int(qs[row]), int(qp[row])
        n = torch.tensor([p + 1], dtype=torch.int32, device=dev())
        dec = bi.attention_decode(qd[row:row + 1].contiguous(), kvd.k_cache, kvd.v_cache,
                                  kvd.page_table[b:b + 1].contiguous(), n)
        assert same_bits(dec[0], ordered[row]), row
    assert bi.get_device_error() == 0


def test_prefill_whole_equals_chunked_with_appends():
    # Whole: every token's K/V written, then one prefill call over all rows.
    # Chunked: the store starts empty (NaN); for each chunk its K/V are appended,
    # then only its rows are prefilled against the cached prefix.
    S, Hq, Hkv, D = 1100, 32, 8, 128
    q, qs, qp, kv = synth.prefill_inputs([S], Hq, Hkv, D, seed=43)
    kvd = _to_dev(kv)
    whole = _prefill(q.to(dev()), qs.to(dev()), qp.to(dev()), kvd)
    # token-major K/V of the sequence, gathered from the store
    t = torch.arange(S)
    pages = kv.page_table[0, t // 16].long()
    k_tok = kv.k_cache[pages, :, t % 16, :].contiguous()  # [S, Hkv, D]
    v_tok = kv.v_cache[pages, :, t % 16, :].contiguous()
    empty_k = torch.full_like(kvd.k_cache, float("nan"))
    empty_v = torch.full_like(kvd.v_cache, float("nan"))
    chunked = torch.empty_like(whole)
    for c0 in range(0, S, 512):
        c1 = min(S, c0 + 512)
        sl = slice(c0, c1)
        bi.kv_append(k_tok[sl].to(dev()), v_tok[sl].to(dev()), qs[sl].to(dev()), qp[sl].to(dev()), empty_k, empty_v,
                     kvd.page_table)
        chunked[sl] = bi.attention_prefill(q[sl].to(dev()), qs[sl].to(dev()), qp[sl].to(dev()), empty_k, empty_v,
                                           kvd.page_table)
    assert same_bits(chunked, whole)
    assert bi.get_device_error() == 0


def test_device_index_errors_are_reported_not_faulted():
    q, kv = synth.decode_inputs(2, 32, 8, 128, max_len=64, seed=44, lens=[40, 20])
    kvd = _to_dev(kv)
    pt = kvd.page_table.clone()
    pt[0, 1] = kv.num_pages + 5  # page id outside the store
    bi.attention_decode(q.to(dev()), kvd.k_cache, kvd.v_cache, pt, kvd.seq_lens)
    assert bi.get_device_error() == 8
    lens = torch.tensor([40, 4 * 16 + 1], dtype=torch.int32, device=dev())  # beyond the page table
    out = bi.attention_decode(q.to(dev()), kvd.k_cache, kvd.v_cache, kvd.page_table, lens)
    assert bi.get_device_error() == 8
    assert int(out[1].float().abs().sum()) == 0
    assert bi.get_device_error() == 0


def test_bounded_wait_expires_with_status_and_context_stays_usable():
    # a wait on an mbarrier that nothing completes gives up after 50 ms
    assert bi.get_device_error() == 0
    bi.selftest_wait_timeout(50)
    assert bi.get_device_error() == 7  # BI_ERR_DEVICE_TIMEOUT
    q, kv = synth.decode_inputs(2, 32, 8, 128, max_len=300, seed=45, lens=[300, 17])
    out = _decode(q.to(dev()), _to_dev(kv))
    assert max_rel(out, _oracle_decode(q, kv)) <= TOL_BF16
    assert bi.get_device_error() == 0


# ---------------------------------------------------------------------------
# Full-size configurations (sampled oracle rows)


def _sample_decode_rows(q, kv, bs):
    refs = []
    for b in bs:
        L = int(kv.seq_lens[b])
        k, v, pt = synth.sequence_pages(kv, b, L)
        refs.append(oracle.attention_decode(synth.to_f64(q[b:b + 1].cpu()), synth.to_f64(k), synth.to_f64(v),
                                            pt.numpy(), np.array([L]))[0])
    return np.stack(refs)


def test_decode_full_size_b256_sampled():
    B, Hq, Hkv, D, Lmax = 256, 32, 8, 128, 32768
    lens = synth.decode_lengths(B, Lmax, seed=50)
    kv = synth.paged_kv_device(lens, Hkv, D, seed=51, max_pages=Lmax // 16, device=dev())
    q = synth.normal_bf16((B, Hq, D), 52).to(dev())
    out = _decode(q, kv)
    bs = [0, 1, int(torch.argmax(lens)), int(torch.argmin(lens)), 100, 255]
    assert max_rel(out[bs], _sample_decode_rows(q, kv, bs)) <= TOL_BF16
    # invariance at full size: a small batch drawn from the big one
    sub = torch.tensor([255, 3, 100], device=dev())
    outs = bi.attention_decode(q[sub].contiguous(), kv.k_cache, kv.v_cache, kv.page_table[sub].contiguous(),
                               kv.seq_lens[sub].contiguous())
    assert same_bits(outs, out[sub])
    assert bi.get_device_error() == 0


def test_prefill_full_size_4096_whole_vs_8_chunks():
    S, Hq, Hkv, D = 4096, 32, 8, 128
    kv = synth.paged_kv_device([S], Hkv, D, seed=60, max_pages=S // 16, device=dev())
    q = synth.normal_bf16((S, Hq, D), 61).to(dev())
    qs = torch.zeros(S, dtype=torch.int32, device=dev())
    qp = torch.arange(S, dtype=torch.int32, device=dev())
    whole = _prefill(q, qs, qp, kv)
    for c0 in range(0, S, 512):
        part = _prefill(q[c0:c0 + 512].contiguous(), qs[c0:c0 + 512].contiguous(), qp[c0:c0 + 512].contiguous(), kv)
        assert same_bits(part, whole[c0:c0 + 512]), c0
    rows = [0, 511, 512, 2048, 4095]
    k, v, pt = synth.sequence_pages(kv, 0, S)
    ref = oracle.attention_prefill(synth.to_f64(q[rows].cpu()), np.zeros(len(rows), dtype=np.int64), np.array(rows),
                                   synth.to_f64(k), synth.to_f64(v), pt.numpy())
    assert max_rel(whole[rows], ref) <= TOL_BF16
