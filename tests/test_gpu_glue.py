"""Decoder glue on the GPU (row gather, RoPE, SwiGLU, residual add): parity with the
fp64 oracle and bit-invariance across batch size."""
import numpy as np
import pytest
import torch

import invariant_deterministic_04_b200 as bi
import oracle
import synth
from gpu_util import TOL_BF16, dev, max_rel, same_bits
from invariant_deterministic_04_b200.llama import rope_cos_sin

pytestmark = pytest.mark.gpu


def test_gather_rows_copies_and_flags_bad_ids():
    src = synth.normal_bf16((100, 2048), 1).to(dev())
    idx = torch.tensor([5, 0, 99, 5, 42], dtype=torch.int32, device=dev())
    out = bi.gather_rows(src, idx)
    assert same_bits(out, src[idx.long()])
    bad = torch.tensor([3, 100], dtype=torch.int32, device=dev())
    out2 = bi.gather_rows(src, bad)
    assert bi.get_device_error() == 8
    assert same_bits(out2[0], src[3]) and int(out2[1].float().abs().sum()) == 0


@pytest.mark.parametrize("H,D", [(32, 64), (8, 64), (32, 128)])
def test_rope_matches_oracle_and_is_row_invariant(H, D):
    T = 37
    x = synth.normal_bf16((T, H, D), 2)
    pos = torch.randint(0, 384, (T,), generator=synth.generator(3), dtype=torch.int32)
    table = rope_cos_sin(384, D, 10000.0, dev())
    xd = x.to(dev()).clone()
    bi.rope(xd, pos.to(dev()), table)
    ref = oracle.rope(synth.to_f64(x), pos.numpy())
    assert max_rel(xd, ref) <= TOL_BF16
    one = x[7:8].to(dev()).clone()
    bi.rope(one, pos[7:8].to(dev()), table)
    assert same_bits(one[0], xd[7])
    # strided rows: the q block of a fused QKV row
    fused = synth.normal_bf16((T, H * D + 256), 4).to(dev())
    view = fused[:, : H * D].view(T, H, D)
    expect = view.clone()
    bi.rope(expect, pos.to(dev()), table)
    bi.rope(view, pos.to(dev()), table)
    assert same_bits(view, expect)


def _rope_model(x, pos, table):
    """bi_rope's documented fp32 arithmetic (include/bi.h): with (c, s) from the fp32
    table, y1 = fma(a, c, -(b s)) and y2 = fma(b, c, a s), each rounded to bf16 (nearest
    even). b s is one fp32 product; a c is exact in fp64 (8 x 24 significant bits), so
    one rounding of a c - (b s) to fp32 is the fused result."""
    xf = synth.to_f64(x)
    half = x.shape[2] // 2
    cs = table.cpu().double().numpy()[np.asarray(pos, dtype=np.int64)]  # [T, D/2, 2]
    c, s = cs[..., 0][:, None, :], cs[..., 1][:, None, :]
    a, b = xf[..., :half], xf[..., half:]
    bs = (b * s).astype(np.float32).astype(np.float64)
    as_ = (a * s).astype(np.float32).astype(np.float64)
    y = np.concatenate([(a * c - bs).astype(np.float32), (b * c + as_).astype(np.float32)], axis=-1)
    return torch.from_numpy(y).to(torch.bfloat16)


@pytest.mark.parametrize("H,D", [(32, 64), (32, 128)])
def test_rope_is_the_documented_fp32_arithmetic_bit_for_bit(H, D):
    T = 37
    x = synth.normal_bf16((T, H, D), 9)
    pos = torch.randint(0, 384, (T,), generator=synth.generator(10), dtype=torch.int32)
    table = rope_cos_sin(384, D, 10000.0, dev())
    xd = x.to(dev()).clone()
    bi.rope(xd, pos.to(dev()), table)
    assert same_bits(xd.cpu(), _rope_model(x, pos.numpy(), table))


def test_swiglu_and_add_match_oracle():
    gu = synth.normal_bf16((33, 2 * 8192), 5)
    out = bi.swiglu(gu.to(dev()))
    assert max_rel(out, oracle.swiglu(synth.to_f64(gu))) <= TOL_BF16
    assert same_bits(bi.swiglu(gu[10:11].to(dev()))[0], out[10])
    a, b = synth.normal_bf16((9, 2048), 6), synth.normal_bf16((9, 2048), 7)
    s = bi.add(a.to(dev()), b.to(dev()))
    assert max_rel(s, synth.to_f64(a) + synth.to_f64(b)) <= TOL_BF16
    # the documented arithmetic exactly: one fp32 add, rounded to bf16 (nearest even)
    assert same_bits(s.cpu(), (a.float() + b.float()).to(torch.bfloat16))
    ad = a.to(dev())
    bi.add(ad, b.to(dev()), out=ad)
    assert same_bits(ad, s)
