"""Pins for the fp64 oracle (CPU only).

The oracle is checked against things other than itself: hand-derived values
(tests/golden), closed forms, pure-Python brute force on tiny inputs, a library
bf16 cast, and invariants. Each test is chosen so that a plausible slip in the
oracle (dropped eps or weight, mean vs sum, transposed operand, wrong GQA
mapping, off-by-one causal mask, wrong page lookup, wrong tie-break) fails it.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "closed_forms.json")


def _cases(op):
    with open(GOLDEN) as f:
        return [c for c in json.load(f)["cases"] if c["op"] == op]


# ---------------------------------------------------------------------------
# RMSNorm


@pytest.mark.parametrize("case", _cases("rmsnorm"))
def test_rmsnorm_golden(case):
    y = oracle.rmsnorm(np.array(case["x"]), np.array(case["w"]), case["eps"])
    np.testing.assert_allclose(y, np.array(case["expected"]), rtol=0, atol=1e-14)


@pytest.mark.parametrize("c", [0.75, -2.5, 1e-3, 37.0])
@pytest.mark.parametrize("K", [1, 8, 512])
def test_rmsnorm_constant_row(c, K):
    w = synth.to_f64(synth.normal_bf16((K,), 5, std=0.1, mean=1.0))
    eps = 1e-6
    y = oracle.rmsnorm(np.full((1, K), c), w, eps)
    np.testing.assert_allclose(y[0], w * c / math.sqrt(c * c + eps), rtol=1e-14, atol=0)
    # eps = 0: a constant row normalises to w (sign of c) exactly
    y0 = oracle.rmsnorm(np.full((1, K), c), w, 0.0)
    np.testing.assert_allclose(y0[0], w * math.copysign(1.0, c), rtol=1e-15, atol=0)


def test_rmsnorm_scale_invariance_at_eps0():
    x = synth.to_f64(synth.normal_bf16((4, 96), 1))
    w = synth.to_f64(synth.normal_bf16((96,), 2, std=0.1, mean=1.0))
    y = oracle.rmsnorm(x, w, 0.0)
    for a in (0.125, 3.0, -7.5):
        np.testing.assert_allclose(oracle.rmsnorm(a * x, w, 0.0), math.copysign(1, a) * y, rtol=1e-13, atol=1e-15)


def test_rmsnorm_bruteforce():
    x = synth.to_f64(synth.normal_bf16((3, 13), 3))
    w = synth.to_f64(synth.normal_bf16((13,), 4, std=0.1, mean=1.0))
    eps = 0.25
    y = oracle.rmsnorm(x, w, eps)
    for m in range(3):
        ms = math.fsum(v * v for v in x[m]) / 13
        r = 1.0 / math.sqrt(ms + eps)
        for k in range(13):
            assert abs(y[m, k] - x[m, k] * r * w[k]) <= 1e-14 * (1 + abs(y[m, k]))


def test_rmsnorm_rows_independent():
    x = synth.to_f64(synth.normal_bf16((9, 40), 6))
    w = synth.to_f64(synth.normal_bf16((40,), 7, std=0.1, mean=1.0))
    full = oracle.rmsnorm(x, w, 1e-6)
    for m in range(9):
        np.testing.assert_array_equal(oracle.rmsnorm(x[m:m + 1], w, 1e-6)[0], full[m])


# ---------------------------------------------------------------------------
# MatMul


@pytest.mark.parametrize("case", _cases("matmul"))
def test_matmul_golden(case):
    c = oracle.matmul(np.array(case["a"]), np.array(case["w"]))
    np.testing.assert_array_equal(c, np.array(case["expected"]))


def test_matmul_one_hot_rows_pick_weight_columns():
    N, K = 7, 11
    w = synth.to_f64(synth.normal_bf16((N, K), 8, std=0.02))
    ks = [0, 3, 10, 5]
    a = np.zeros((len(ks), K))
    for m, k in enumerate(ks):
        a[m, k] = 1.0
    c = oracle.matmul(a, w)
    for m, k in enumerate(ks):
        np.testing.assert_array_equal(c[m], w[:, k])


def test_matmul_small_integers_exact_bruteforce():
    rng = np.random.default_rng(0)
    M, N, K = 5, 6, 9
    a = rng.integers(-8, 9, (M, K))
    w = rng.integers(-8, 9, (N, K))
    c = oracle.matmul(a.astype(float), w.astype(float))
    for m in range(M):
        for n in range(N):
            assert c[m, n] == sum(int(a[m, k]) * int(w[n, k]) for k in range(K))


# ---------------------------------------------------------------------------
# Attention


@pytest.mark.parametrize("case", _cases("attention"))
def test_attention_golden(case):
    out = oracle.softmax_attend(np.array(case["q"]), np.array(case["keys"]), np.array(case["vals"]),
                                1.0 / math.sqrt(len(case["q"])))
    np.testing.assert_allclose(out, np.array(case["expected"]), rtol=0, atol=1e-15)


def test_attention_split_merge_algebra_equals_full_softmax():
    # Partials (m, l, o) of consecutive key splits, folded left with
    # m = max(m1, m2), l = l1 e^(m1-m) + l2 e^(m2-m), o = o1 e^(m1-m) + o2 e^(m2-m),
    # give o / l = the softmax over all keys (an identity, exact up to rounding in fp64).
    rng = np.random.default_rng(21)
    D, L, split = 16, 700, 256
    q = rng.normal(size=D)
    keys, vals = rng.normal(size=(L, D)), rng.normal(size=(L, D))
    scale = 1.0 / math.sqrt(D)
    m, l, o = -math.inf, 0.0, np.zeros(D)
    for s0 in range(0, L, split):
        sc = keys[s0:s0 + split] @ q * scale
        m2 = sc.max()
        e = np.exp(sc - m2)
        l2, o2 = e.sum(), e @ vals[s0:s0 + split]
        mn = max(m, m2)
        a, b = math.exp(m - mn) if m > -math.inf else 0.0, math.exp(m2 - mn)
        m, l, o = mn, l * a + l2 * b, o * a + o2 * b
    np.testing.assert_allclose(oracle.softmax_attend(q, keys, vals, scale), o / l, rtol=0, atol=1e-14)


def test_attention_key_order_does_not_matter():
    rng = np.random.default_rng(22)
    q, keys, vals = rng.normal(size=8), rng.normal(size=(50, 8)), rng.normal(size=(50, 8))
    perm = rng.permutation(50)
    np.testing.assert_allclose(oracle.softmax_attend(q, keys[perm], vals[perm], 0.3),
                               oracle.softmax_attend(q, keys, vals, 0.3), rtol=0, atol=1e-15)


def _tiny_paged(lens, Hkv=2, D=8, seed=0):
    return synth.paged_kv(lens, Hkv, D, seed=seed, poison_tail=False)


def test_attention_single_key_returns_its_value():
    kv = _tiny_paged([1, 1], Hkv=2, D=8)
    q = synth.to_f64(synth.normal_bf16((2, 4, 8), 1))
    out = oracle.attention_decode(q, synth.to_f64(kv.k_cache), synth.to_f64(kv.v_cache),
                                  kv.page_table.numpy(), kv.seq_lens.numpy())
    v = synth.to_f64(kv.v_cache)
    for b in range(2):
        p = int(kv.page_table[b, 0])
        for h in range(4):
            np.testing.assert_array_equal(out[b, h], v[p, h // 2, 0])


def test_attention_identical_keys_give_mean_of_values():
    L, D = 37, 8
    kv = _tiny_paged([L], Hkv=1, D=D)
    k = synth.to_f64(kv.k_cache)
    v = synth.to_f64(kv.v_cache)
    k[:] = k[int(kv.page_table[0, 0]), 0, 0]  # every slot holds the same key
    q = synth.to_f64(synth.normal_bf16((1, 2, D), 3))
    out = oracle.attention_decode(q, k, v, kv.page_table.numpy(), kv.seq_lens.numpy())
    vals = np.array([v[int(kv.page_table[0, t // 16]), 0, t % 16] for t in range(L)])
    for h in range(2):
        np.testing.assert_allclose(out[0, h], vals.mean(axis=0), rtol=0, atol=1e-14)


def test_attention_gqa_head_mapping():
    # kv-head g holds the constant value g+1; q-head h must read kv-head h // (Hq/Hkv)
    Hq, Hkv, D, L = 8, 2, 4, 20
    kv = _tiny_paged([L], Hkv=Hkv, D=D)
    v = synth.to_f64(kv.v_cache)
    for g in range(Hkv):
        v[:, g] = g + 1.0
    q = synth.to_f64(synth.normal_bf16((1, Hq, D), 4))
    out = oracle.attention_decode(q, synth.to_f64(kv.k_cache), v, kv.page_table.numpy(), kv.seq_lens.numpy())
    for h in range(Hq):
        np.testing.assert_allclose(out[0, h], np.full(D, h // (Hq // Hkv) + 1.0), rtol=0, atol=1e-14)


def test_attention_two_keys_closed_form_scale():
    D = 16
    k = np.zeros((1, 1, 16, D))
    v = np.zeros((1, 1, 16, D))
    k[0, 0, 0, 0] = 1.0
    k[0, 0, 1, 1] = 1.0
    v[0, 0, 0, 2] = 1.0
    v[0, 0, 1, 3] = 1.0
    q = np.zeros((1, 1, D))
    q[0, 0, 0], q[0, 0, 1] = 3.0, -1.0
    out = oracle.attention_decode(q, k, v, np.array([[0]]), np.array([2]))
    a, b = 3.0 / math.sqrt(D), -1.0 / math.sqrt(D)
    np.testing.assert_allclose(out[0, 0, 2], math.exp(a) / (math.exp(a) + math.exp(b)), rtol=1e-15)
    np.testing.assert_allclose(out[0, 0, 3], math.exp(b) / (math.exp(a) + math.exp(b)), rtol=1e-15)


def _bruteforce_head(qv, k, v, page_row, L, g):
    """Pure-Python attention of one query vector over tokens 0..L-1 of kv-head g,
    each token looked up as (page_row[t // 16], slot t % 16); plain softmax
    without max subtraction (the scores are small in these cases)."""
    D = len(qv)
    rows = [(page_row[t // 16], t % 16) for t in range(L)]
    w = [math.exp(sum(qv[d] * k[p, g, s, d] for d in range(D)) / math.sqrt(D)) for p, s in rows]
    z = math.fsum(w)
    return [math.fsum(w[i] * v[p, g, s, d] for i, (p, s) in enumerate(rows)) / z for d in range(D)]


def test_attention_bruteforce_through_page_table():
    lens = [5, 33, 18]
    Hq, Hkv, D = 4, 2, 8
    kv = _tiny_paged(lens, Hkv=Hkv, D=D, seed=9)
    q = synth.to_f64(synth.normal_bf16((3, Hq, D), 10))
    k = synth.to_f64(kv.k_cache)
    v = synth.to_f64(kv.v_cache)
    pt = kv.page_table.tolist()
    out = oracle.attention_decode(q, k, v, np.array(pt), np.array(lens))
    for b, L in enumerate(lens):
        for h in range(Hq):
            ref = _bruteforce_head(q[b, h], k, v, pt[b], L, h // (Hq // Hkv))
            np.testing.assert_allclose(out[b, h], ref, rtol=0, atol=1e-13)


def test_attention_empty_sequence_gives_zeros():
    # a sequence of length 0 sees no key: its rows are zero, the others are unaffected
    lens = [0, 5, 0]
    kv = _tiny_paged([1, 5, 1], Hkv=1, D=8, seed=18)
    q = synth.to_f64(synth.normal_bf16((3, 2, 8), 19))
    k, v, pt = synth.to_f64(kv.k_cache), synth.to_f64(kv.v_cache), kv.page_table.numpy()
    out = oracle.attention_decode(q, k, v, pt, np.array(lens))
    assert np.all(out[0] == 0) and np.all(out[2] == 0)
    for h in range(2):
        np.testing.assert_allclose(out[1, h], _bruteforce_head(q[1, h], k, v, pt[1].tolist(), 5, 0), rtol=0, atol=1e-13)


def test_prefill_rows_of_two_sequences_bruteforce():
    # rows of two sequences, shuffled together: each row reads its own sequence's
    # pages, keys 0..p inclusive of its position p
    lens = [21, 35]
    Hq, Hkv, D = 4, 2, 8
    q, q_seq, q_pos, kv = synth.prefill_inputs(lens, Hq, Hkv, D, seed=17)
    perm = np.random.default_rng(5).permutation(sum(lens))
    q = synth.to_f64(q)[perm]
    seq, pos = q_seq.numpy()[perm], q_pos.numpy()[perm]
    k, v, pt = synth.to_f64(kv.k_cache), synth.to_f64(kv.v_cache), kv.page_table.tolist()
    out = oracle.attention_prefill(q, seq, pos, k, v, np.array(pt))
    for r in range(len(perm)):
        for h in range(Hq):
            ref = _bruteforce_head(q[r, h], k, v, pt[seq[r]], int(pos[r]) + 1, h // (Hq // Hkv))
            np.testing.assert_allclose(out[r, h], ref, rtol=0, atol=1e-13)


def test_attention_invariant_to_physical_page_placement():
    lens = [70]
    kv = _tiny_paged(lens, Hkv=1, D=8, seed=11)
    q = synth.to_f64(synth.normal_bf16((1, 2, 8), 12))
    k, v, pt = synth.to_f64(kv.k_cache), synth.to_f64(kv.v_cache), kv.page_table.numpy().copy()
    ref = oracle.attention_decode(q, k, v, pt, np.array(lens))
    perm = np.random.default_rng(1).permutation(k.shape[0])
    k2, v2 = np.empty_like(k), np.empty_like(v)
    k2[perm], v2[perm] = k, v
    pt2 = np.where(pt >= 0, perm[np.maximum(pt, 0)], -1)
    out = oracle.attention_decode(q, k2, v2, pt2, np.array(lens))
    np.testing.assert_array_equal(out, ref)


def test_prefill_mask_is_causal_and_inclusive():
    # key at position p is made dominant for the query at p: it must be seen;
    # the key at p+1 is made even more dominant: it must not be seen.
    L, D, p = 40, 8, 21
    kv = _tiny_paged([L], Hkv=1, D=D, seed=13)
    k, v = synth.to_f64(kv.k_cache), synth.to_f64(kv.v_cache)
    pt = kv.page_table.numpy()
    q = np.zeros((1, 1, D))
    q[0, 0, 0] = 1.0
    k[:, :, :, 0] = 0.0
    k[pt[0, p // 16], 0, p % 16, 0] = 200.0
    k[pt[0, (p + 1) // 16], 0, (p + 1) % 16, 0] = 400.0
    out = oracle.attention_prefill(q, np.array([0]), np.array([p]), k, v, pt)
    np.testing.assert_allclose(out[0, 0], v[pt[0, p // 16], 0, p % 16], rtol=0, atol=1e-12)


def test_prefill_row_equals_decode_of_prefix():
    lens = [50]
    q, q_seq, q_pos, kv = synth.prefill_inputs(lens, 4, 2, 8, seed=14)
    k, v, pt = synth.to_f64(kv.k_cache), synth.to_f64(kv.v_cache), kv.page_table.numpy()
    pre = oracle.attention_prefill(synth.to_f64(q), q_seq.numpy(), q_pos.numpy(), k, v, pt)
    for p in (0, 15, 16, 49):
        dec = oracle.attention_decode(synth.to_f64(q)[p:p + 1], k, v, pt, np.array([p + 1]))
        np.testing.assert_array_equal(pre[p], dec[0])


# ---------------------------------------------------------------------------
# LM head


@pytest.mark.parametrize("case", _cases("lmhead"))
def test_lmhead_golden(case):
    r = oracle.lmhead(np.array(case["h"]), np.array(case["w"]), case["threshold"])
    assert r["tokens"][0] == case["expected"]["token"]
    assert r["margin"][0] == case["expected"]["margin"]
    assert bool(r["recompute"][0]) == case["expected"]["recompute"]


def test_lmhead_planted_margins():
    K, V = 16, 50
    w = synth.to_f64(synth.normal_bf16((V, K), 15, std=0.02))
    h = np.zeros((2, K))
    h[0, 0] = h[1, 1] = 1.0
    w[:, 0] = np.clip(w[:, 0], -1, 1)
    w[:, 1] = np.clip(w[:, 1], -1, 1)
    w[7, 0], w[30, 0] = 3.0, 2.875      # margin 0.125 -> recompute
    w[12, 1], w[40, 1] = 8.0, 3.0       # margin 5 -> no recompute
    r = oracle.lmhead(h, w, 0.5)
    assert list(r["tokens"]) == [7, 12]
    assert list(r["recompute"]) == [True, False]
    assert r["margin"][0] == 0.125 and r["margin"][1] == 5.0
    # a margin exactly at the threshold is not below it: no recompute
    h3 = np.zeros((1, K))
    h3[0, 2] = 1.0
    w[:, 2] = np.clip(w[:, 2], -1, 1)
    w[3, 2], w[20, 2] = 4.0, 3.5
    r3 = oracle.lmhead(h3, w, 0.5)
    assert r3["tokens"][0] == 3 and r3["margin"][0] == 0.5 and not r3["recompute"][0]


def test_lmhead_margin_is_taken_on_bf16_rounded_logits():
    # bf16 values between 256 and 512 are 2 apart, so 256.625 rounds to 256: the
    # exact margin 0.625 would not ask for a recompute, but the bf16 logits tie
    # (margin 0 < 0.5), and their argmax is the lower index while the exact
    # argmax is the higher one
    vals = [256.0, 256.625, 1.0, -3.0]
    r = oracle.lmhead(np.array([[1.0]]), np.array(vals).reshape(4, 1), 0.5)
    assert r["tokens"][0] == 1 and r["margin"][0] == 0.625
    assert r["tokens_bf16"][0] == 0 and r["margin_bf16"][0] == 0.0 and r["recompute"][0]


def test_lmhead_bruteforce_argmax_and_ties():
    vals = [0.25, -1.0, 0.75, 0.75, 0.5, -0.125, 0.75, 0.0]
    h = np.array([[1.0]])
    w = np.array(vals).reshape(8, 1)
    r = oracle.lmhead(h, w, 0.5)
    best = max(range(8), key=lambda i: (vals[i], -i))
    assert best == 2 and r["tokens"][0] == 2  # lowest index among the tied maxima
    assert r["margin"][0] == 0.0 and r["recompute"][0]


def test_round_to_bf16_matches_library_cast():
    x = np.concatenate([
        synth.to_f64(synth.normal_bf16((4096,), 16)) * (1 + 2.0 ** -9),
        np.random.default_rng(2).normal(size=4096) * 10,
        np.array([1 + 2.0 ** -8, 1 + 3 * 2.0 ** -8, -(1 + 2.0 ** -8), 0.0, 2.0 ** -130]),
    ])
    ref = torch.from_numpy(x.astype(np.float32)).to(torch.bfloat16).to(torch.float64).numpy()
    np.testing.assert_array_equal(oracle.round_to_bf16(x), ref)
    assert oracle.round_to_bf16(np.array([1 + 2.0 ** -8]))[0] == 1.0
    assert oracle.round_to_bf16(np.array([1 + 3 * 2.0 ** -8]))[0] == 1 + 2.0 ** -6


def test_normwise_rel_err():
    ref = np.array([[2.0, -4.0, 1.0], [0.0, 0.0, 0.0]])
    got = np.array([[2.0, -4.02, 1.01], [0.0, 1e-3, 0.0]])
    e = oracle.normwise_rel_err(got, ref)
    np.testing.assert_allclose(e, [0.02 / 4.0, 1e-3])


# ---------------------------------------------------------------------------
# Decoder glue: RoPE, SwiGLU, one decoder layer


@pytest.mark.parametrize("case", _cases("rope"))
def test_rope_golden(case):
    out = oracle.rope(np.array(case["x"]), np.array(case["pos"]), case["theta"])
    np.testing.assert_allclose(out, np.array(case["expected"]), rtol=0, atol=1e-13)


def test_rope_identity_norms_and_composition():
    x = synth.to_f64(synth.normal_bf16((5, 3, 64), 80))
    np.testing.assert_array_equal(oracle.rope(x, np.zeros(5)), x)  # position 0: no rotation
    pos = np.array([1, 7, 100, 383, 5000])
    y = oracle.rope(x, pos)
    pair = lambda z: np.hypot(z[..., :32], z[..., 32:])
    np.testing.assert_allclose(pair(y), pair(x), rtol=1e-13)  # rotations keep each pair's length
    np.testing.assert_allclose(oracle.rope(oracle.rope(x, pos), pos + 3), oracle.rope(x, 2 * pos + 3), atol=1e-10)
    # the lowest frequency pair (i = D/2 - 1) turns by pos * theta^(-(D-2)/D)
    ang = 100 * 10000.0 ** (-62 / 64)
    z = np.zeros((1, 1, 64))
    z[0, 0, 31] = 1.0
    r = oracle.rope(z, np.array([100]))
    assert abs(r[0, 0, 31] - math.cos(ang)) < 1e-15 and abs(r[0, 0, 63] - math.sin(ang)) < 1e-15


@pytest.mark.parametrize("case", _cases("swiglu"))
def test_swiglu_golden(case):
    np.testing.assert_allclose(oracle.swiglu(np.array(case["gate_up"])), np.array(case["expected"]), rtol=1e-15)


def test_silu_limits():
    assert oracle.silu(np.array([0.0]))[0] == 0.0
    assert abs(oracle.silu(np.array([40.0]))[0] - 40.0) < 1e-15
    assert abs(oracle.silu(np.array([-40.0]))[0]) < 1e-15


def test_decoder_layer_structure():
    # With wo = wdown = 0 the layer is the identity on h; with one kv head and
    # identical keys the attention output is the mean of the values.
    rng = np.random.default_rng(3)
    Hd, nh, nkv, F = 16, 4, 2, 24
    D = Hd // nh
    w = dict(wqkv=rng.normal(0, 0.2, ((nh + 2 * nkv) * D, Hd)), wo=np.zeros((Hd, Hd)),
             wgu=rng.normal(0, 0.2, (2 * F, Hd)), wdown=np.zeros((Hd, F)), attn_norm=np.ones(Hd),
             mlp_norm=np.ones(Hd))
    h = rng.normal(size=(3, Hd))
    out = oracle.decoder_layer(h, [0, 0, 1], [0, 1, 0], {}, {}, w, nh, nkv)
    np.testing.assert_array_equal(out, h)
    # a row that sees only itself: attention returns its own value vector, so with
    # wo = I the update is exactly v (rotation does not touch v)
    w2 = dict(w, wo=np.eye(Hd))
    out2 = oracle.decoder_layer(h[:1], [0], [0], {}, {}, w2, nh, nkv)
    x = oracle.rmsnorm(h[:1], w["attn_norm"], 1e-6)
    v = oracle.matmul(x, w["wqkv"])[:, (nh + nkv) * D:].reshape(1, nkv, D)
    expect = h[:1] + np.repeat(v, nh // nkv, axis=1).reshape(1, Hd)
    np.testing.assert_allclose(out2, expect, rtol=1e-13, atol=1e-13)


def test_decoder_layer_attention_closed_form():
    # One head, D = 2, eps = 0, Wq = Wk = Wv = wo = I, wdown = 0. Rows h0 = e0 at
    # position 0 and h1 = e1 at position 1 of one sequence; RMSNorm makes x_t =
    # sqrt(2) h_t. At D = 2 RoPE turns the one pair by pos radians, so
    # q1 = k1 = sqrt(2) (-sin 1, cos 1) and k0 = sqrt(2) e0. With scale 1/sqrt(2) row 1
    # scores key 0 at -sqrt(2) sin 1 and key 1 at sqrt(2); row 0 sees only itself.
    I2 = np.eye(2)
    w = dict(wqkv=np.vstack([I2, I2, I2]), wo=I2, wgu=np.zeros((2, 2)), wdown=np.zeros((2, 1)),
             attn_norm=np.ones(2), mlp_norm=np.ones(2))
    r2 = math.sqrt(2)
    s0, s1 = -r2 * math.sin(1.0), r2
    p0 = math.exp(s0) / (math.exp(s0) + math.exp(s1))
    expect = np.array([[1 + r2, 0.0], [r2 * p0, 1 + r2 * (1 - p0)]])
    out = oracle.decoder_layer(np.eye(2), [0, 0], [0, 1], {}, {}, w, 1, 1, eps=0.0)
    np.testing.assert_allclose(out, expect, rtol=0, atol=1e-14)
    # row 1 alone, position 0 supplied by the cache (key as rotated at position 0,
    # a value of our choosing): the same weights p0, 1 - p0 mix that value and v1
    v0 = np.array([0.25, -0.75])
    out1 = oracle.decoder_layer(np.eye(2)[1:], [0], [1], {0: (r2 * I2[0])[None, None]}, {0: v0[None, None]},
                                w, 1, 1, eps=0.0)
    np.testing.assert_allclose(out1[0], I2[1] + p0 * v0 + (1 - p0) * r2 * I2[1], rtol=0, atol=1e-14)


def test_decoder_layer_mlp_closed_form():
    # wo = 0 removes attention. The MLP sees x = rmsnorm(h) * mlp_norm: for h = e0,
    # eps = 0 and mlp_norm = (1/2, 3), x = (sqrt(2)/2, 0). wgu rows (1, 0), (1, 0)
    # make gate = up = a = sqrt(2)/2, and wdown = (1, 0)^T puts silu(a) * a on column 0.
    a = math.sqrt(2) / 2
    w = dict(wqkv=np.ones((6, 2)), wo=np.zeros((2, 2)), wgu=np.array([[1.0, 0.0], [1.0, 0.0]]),
             wdown=np.array([[1.0], [0.0]]), attn_norm=np.full(2, 5.0), mlp_norm=np.array([0.5, 3.0]))
    out = oracle.decoder_layer(np.array([[1.0, 0.0]]), [0], [0], {}, {}, w, 1, 1, eps=0.0)
    np.testing.assert_allclose(out, [[1 + a * a / (1 + math.exp(-a)), 0.0]], rtol=0, atol=1e-15)
