"""bi_attention_decode_static: decode attention that allocates nothing.

Some callers cannot allocate device memory at the point where they run decode
attention (a plugin inside a framework that owns all device memory, or a
latency-critical path that may not pay cudaMalloc's device-wide synchronisation),
so they cannot supply the workspace bi_attention_decode needs. This entry point
keeps its scratch in a fixed 32 MiB array inside the library instead.

The GPU test calls it through the C ABI twice in a row, on different inputs (the
second call finds the first call's leftovers in the shared array), and compares
each result with bi_attention_decode on the same inputs. This file is collected
last so that a run stopping at the first failure has already run every other test.
"""
import ctypes

import pytest
import torch

import invariant_deterministic_04_b200 as bi
import synth
from gpu_util import TOL_BF16, dev, max_rel, same_bits

P = 0x10000  # aligned stand-in address for host-side validation (never dereferenced)


def test_static_decode_host_validation():
    L = bi.lib()
    f = L.bi_attention_decode_static
    assert f(None, P, P, 100, P, 64, P, P, 4, 32, 8, 128, 0.088, None) == 1          # BI_ERR_NULL
    assert f(P, P, P, 100, P, 64, P, P, -1, 32, 8, 128, 0.088, None) == 2            # BI_ERR_SHAPE
    assert f(P, P, P, 100, P, 64, P, P, 0, 32, 8, 128, 0.088, None) == 0             # empty batch: no-op
    # a request needing more scratch than the fixed array is refused before any launch
    need = L.bi_attention_workspace_size(256, 32, 128, 2048)
    assert need > bi.STATIC_SCRATCH_BYTES
    assert f(P, P, P, 100, P, 2048, P, P, 256, 32, 8, 128, 0.088, None) == 4        # BI_ERR_WORKSPACE
    # shape errors are reported as such even when the size query would pass
    assert f(P, P, P, 100, P, 64, P, P, 4, 0, 8, 128, 0.088, None) == 2              # Hq = 0: BI_ERR_SHAPE
    assert f(P, P, P, 100, P, 64, P, P, 4, 32, 8, 96, 0.088, None) == 5              # D = 96: BI_ERR_UNSUPPORTED
    # the smallest batch whose scratch no longer fits is refused; the one below it fits exactly
    B = max_batch_in_scratch(L, 16)
    assert L.bi_attention_workspace_size(B, 32, 128, 16) <= bi.STATIC_SCRATCH_BYTES
    assert L.bi_attention_workspace_size(B + 1, 32, 128, 16) > bi.STATIC_SCRATCH_BYTES
    assert f(P, P, P, 100, P, 16, P, P, B + 1, 32, 8, 128, 0.088, None) == 4


def max_batch_in_scratch(L, max_pages):
    """Largest batch whose decode scratch (Hq 32, D 128) fits the fixed array."""
    B = 1
    while L.bi_attention_workspace_size(B + 1, 32, 128, max_pages) <= bi.STATIC_SCRATCH_BYTES:
        B += 1
    return B


@pytest.mark.gpu
def test_static_decode_matches_workspace_decode_on_two_calls_in_a_row():
    cases = [
        ([4096, 1, 257, 3000, 77, 1500], 90),   # first call: 6 sequences, many splits
        ([513, 16, 2048], 91),                  # second call: fewer rows, stale scratch left behind
    ]
    results = []
    for lens, seed in cases:
        q, kv = synth.decode_inputs(len(lens), 32, 8, 128, max_len=4096, seed=seed, lens=lens)
        qd = q.to(dev())
        kc, vc, pt, sl = kv.k_cache.to(dev()), kv.v_cache.to(dev()), kv.page_table.to(dev()), kv.seq_lens.to(dev())
        assert bi.attention_workspace_size(len(lens), 32, 128, kv.max_pages) <= bi.STATIC_SCRATCH_BYTES
        got = bi.attention_decode_static(qd, kc, vc, pt, sl)
        ref = bi.attention_decode(qd, kc, vc, pt, sl)
        torch.cuda.synchronize()
        results.append((got.clone(), ref))
    for got, ref in results:
        assert max_rel(got, synth.to_f64(ref.cpu())) <= TOL_BF16
        assert same_bits(got, ref)
    assert bi.get_device_error() == 0


@pytest.mark.gpu
@pytest.mark.parametrize("max_pages,long_lens", [(16, []), (2048, [32768, 20000])])
def test_static_decode_with_scratch_filled_to_its_end(max_pages, long_lens):
    # The largest batch that fits: the split partials of the last rows lie at the
    # end of the fixed array (with one page per sequence the scratch is filled to
    # its last byte). Two call shapes: thousands of one-split rows, and a few rows
    # with up to 128 splits next to short ones.
    L = bi.lib()
    B = max_batch_in_scratch(L, max_pages)
    assert L.bi_attention_workspace_size(B, 32, 128, max_pages) > bi.STATIC_SCRATCH_BYTES - (2 << 20)
    g = synth.generator(92 + max_pages)
    short = torch.randint(1, 257, (B - len(long_lens),), generator=g).tolist()
    lens = long_lens + short
    q, kv = synth.decode_inputs(B, 32, 8, 128, max_len=max_pages * 16, seed=93, lens=lens)
    assert kv.max_pages == max_pages
    qd = q.to(dev())
    kc, vc, ptd, sl = kv.k_cache.to(dev()), kv.v_cache.to(dev()), kv.page_table.to(dev()), kv.seq_lens.to(dev())
    got = bi.attention_decode_static(qd, kc, vc, ptd, sl)
    ref = bi.attention_decode(qd, kc, vc, ptd, sl)
    torch.cuda.synchronize()
    assert same_bits(got, ref)
    assert bi.get_device_error() == 0
