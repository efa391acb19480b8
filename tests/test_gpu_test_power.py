"""Power of the GPU parity tests (CPU only): would they see a wrong kernel?

A GPU parity test runs a kernel on fixed seeded inputs and requires its output to
lie within a tolerance of the oracle's (normwise 1e-2 per row for bf16 outputs). A
kernel bug slips through when its output stays inside that tolerance on those
inputs. Here each plausible kernel bug is emulated in fp64 on the CPU: a dropped
last page, split or 16-byte vector, a split combine without its rescaling, a wrong
GQA head mapping or scale, an off-by-one causal mask, a wrong page lookup, an
unwritten ragged tail. The emulation runs on exactly the inputs of the GPU parity
test it targets, and must fail that test's own assertion on at least one of its
cases, so the GPU test would fail on such a kernel.

Out of reach by design: changes smaller than the tolerance, e.g. eps placed outside
the square root of RMSNorm (about 1e-6 here) or fp32 instead of fp64 accumulation.
"""
from __future__ import annotations

import math

import numpy as np
import pytest

import oracle
import synth
from gpu_util import TOL_BF16
from test_oracle_mutants import _mutated

PAGE = 16


def _fails_parity(buggy: np.ndarray, ref: np.ndarray) -> bool:
    """True when `max_rel(got, ref) <= TOL_BF16`, the GPU tests' assertion, is false
    for got = buggy (NaN counts as a failure, as it does there)."""
    err = oracle.normwise_rel_err(oracle.round_to_bf16(np.nan_to_num(buggy, nan=np.inf)), ref).max()
    return not (err <= TOL_BF16)


# ---------------------------------------------------------------------------
# Decode attention: the cases of test_decode_matches_oracle

DECODE_CASES = [(32, 8, 128), (32, 8, 64), (8, 8, 128), (32, 4, 128), (16, 8, 64), (8, 1, 64)]
DECODE_LENS = [1, 16, 17, 255, 256, 257, 700, 513]


def _decode_case(Hq, Hkv, D):
    q, kv = synth.decode_inputs(len(DECODE_LENS), Hq, Hkv, D, max_len=800, seed=Hq + Hkv + D, lens=DECODE_LENS)
    return (synth.to_f64(q), synth.to_f64(kv.k_cache), synth.to_f64(kv.v_cache), kv.page_table.numpy(),
            kv.seq_lens.numpy())


def _split_combine(q, k, v, pt, lens, rescale=True):
    """Decode by fixed 256-token splits folded left; without `rescale` the split
    partials are added as if they shared one maximum (a missing exp(m_s - M))."""
    B, Hq, D = q.shape
    group = Hq // k.shape[1]
    out = np.zeros_like(q)
    for b in range(B):
        L = int(lens[b])
        keys_all = [oracle.gather_kv(k, pt[b], g, L) for g in range(k.shape[1])]
        vals_all = [oracle.gather_kv(v, pt[b], g, L) for g in range(k.shape[1])]
        for h in range(Hq):
            g = h // group
            M, Lsum, O = -math.inf, 0.0, np.zeros(D)
            parts = []
            for s0 in range(0, L, 256):
                sc = keys_all[g][s0:s0 + 256] @ q[b, h] / math.sqrt(D)
                m = sc.max()
                e = np.exp(sc - m)
                parts.append((m, e.sum(), e @ vals_all[g][s0:s0 + 256]))
            if not parts:
                continue
            M = max(p[0] for p in parts)
            for m, l, o in parts:
                w = math.exp(m - M) if rescale else 1.0
                Lsum, O = Lsum + w * l, O + w * o
            out[b, h] = O / Lsum
    return out


def _decode_bugs():
    def scale_over_d(q, k, v, pt, lens):
        return oracle.attention_decode(q, k, v, pt, lens, scale=1.0 / q.shape[2])

    def drop_last_token(q, k, v, pt, lens):
        return oracle.attention_decode(q, k, v, pt, lens - 1)

    def drop_partial_page(q, k, v, pt, lens):
        return oracle.attention_decode(q, k, v, pt, (lens // PAGE) * PAGE)

    def drop_last_split(q, k, v, pt, lens):
        return oracle.attention_decode(q, k, v, pt, ((lens - 1) // 256) * 256)

    def combine_without_rescale(q, k, v, pt, lens):
        return _split_combine(q, k, v, pt, lens, rescale=False)

    def mutant(name, old, new):
        def run(monkeypatch):
            monkeypatch.setattr(oracle, name, _mutated(name, old, new))
        return run

    return {
        "scale 1/D instead of 1/sqrt(D)": (scale_over_d, None),
        "last token of each sequence dropped": (drop_last_token, None),
        "last partial page dropped": (drop_partial_page, None),
        "last 256-token split dropped": (drop_last_split, None),
        "split partials combined without exp(m_s - M)": (combine_without_rescale, None),
        "GQA heads interleaved (h -> kv-head h mod Hkv)":
            (None, mutant("attention_rows", "h = g * group + j", "h = j * Hkv + g")),
        "logical page index used as the physical page":
            (None, mutant("gather_kv", "pages = np.asarray(page_row, dtype=np.int64)[t // PAGE]",
                          "pages = t // PAGE")),
        "kv-head 0 read for every query head":
            (None, mutant("gather_kv", "cache[pages, g, t % PAGE]", "cache[pages, 0, t % PAGE]")),
    }


DECODE_BUGS = _decode_bugs()


def test_controls_pass_parity():
    # the correct results, rounded to bf16, pass every case of each GPU test: a
    # "caught" above is the bug's doing, not the rounding's
    for case in DECODE_CASES:
        q, k, v, pt, lens = _decode_case(*case)
        ref = oracle.attention_decode(q, k, v, pt, lens)
        assert not _fails_parity(ref, ref)
    for M, K in RMS_CASES:
        x, w = (synth.to_f64(t) for t in synth.rmsnorm_inputs(M, K, seed=M + K))
        assert not _fails_parity(oracle.rmsnorm(x, w, EPS), oracle.rmsnorm(x, w, EPS))
    for M, N, K in MM_CASES:
        a, w = (synth.to_f64(t) for t in synth.matmul_inputs(M, N, K, seed=M * 7 + N + K))
        assert not _fails_parity(oracle.matmul(a, w), oracle.matmul(a, w))


def test_split_combine_emulation_is_exact_when_rescaled():
    q, k, v, pt, lens = _decode_case(32, 8, 64)
    ref = oracle.attention_decode(q, k, v, pt, lens)
    np.testing.assert_allclose(_split_combine(q, k, v, pt, lens), ref, rtol=0, atol=1e-12)


@pytest.mark.parametrize("bug", list(DECODE_BUGS))
def test_decode_parity_sees(bug, monkeypatch):
    fn, patch = DECODE_BUGS[bug]
    caught = []
    for case in DECODE_CASES:
        q, k, v, pt, lens = _decode_case(*case)
        ref = oracle.attention_decode(q, k, v, pt, lens)
        if patch is None:
            buggy = fn(q, k, v, pt, lens)
        else:
            with monkeypatch.context() as mp:
                patch(mp)
                with np.errstate(all="ignore"):
                    buggy = oracle.attention_decode(q, k, v, pt, lens)
        caught.append(_fails_parity(buggy, ref))
    assert any(caught), f"{bug}: inside the tolerance in every case"


# ---------------------------------------------------------------------------
# Prefill attention: the cases of test_prefill_matches_oracle

PREFILL_ROWS = [0, 1, 15, 16, 100, 255, 256, 257, 299, 300, 320, 344]


def _prefill_case(D):
    q, qs, qp, kv = synth.prefill_inputs([300, 45], 32, 8, D, seed=40 + D)
    r = PREFILL_ROWS
    return (synth.to_f64(q)[r], qs.numpy()[r], qp.numpy()[r], synth.to_f64(kv.k_cache), synth.to_f64(kv.v_cache),
            kv.page_table.numpy())


PREFILL_BUGS = {
    "causal mask excludes the row's own position": ("np.asarray(q_pos) + 1", "np.asarray(q_pos)"),
    "causal mask lets in the next position": ("np.asarray(q_pos) + 1", "np.asarray(q_pos) + 2"),
    "every row reads sequence 0": ("np.asarray(q_seq),", "np.zeros(len(q_seq), dtype=np.int64),"),
}


@pytest.mark.parametrize("bug", list(PREFILL_BUGS))
def test_prefill_parity_sees(bug, monkeypatch):
    old, new = PREFILL_BUGS[bug]
    caught = []
    for D in (128, 64):
        q, qs, qp, k, v, pt = _prefill_case(D)
        ref = oracle.attention_prefill(q, qs, qp, k, v, pt)
        # a row that would read past its sequence reads the store's next slot, which
        # the inputs fill with NaN (stale data); index the page table safely
        with monkeypatch.context() as mp:
            mp.setattr(oracle, "attention_prefill", _mutated("attention_prefill", old, new))
            with np.errstate(all="ignore"):
                buggy = oracle.attention_prefill(q, qs, qp, k, v, np.where(pt < 0, pt.max(), pt))
        caught.append(_fails_parity(buggy, ref))
    assert any(caught), f"{bug}: inside the tolerance in every case"


# ---------------------------------------------------------------------------
# RMSNorm: the cases of test_rmsnorm_matches_oracle

RMS_CASES = [(1, 512), (7, 512), (32, 512), (129, 4096), (5, 2048), (3, 8), (4, 136), (2, 16384), (300, 1024)]
EPS = 1e-6

RMS_BUGS = {
    "sum of squares misses the row's last 16-byte vector":
        lambda x, w: x / np.sqrt((x[:, :-8] ** 2).sum(axis=1, keepdims=True) / x.shape[1] + EPS) * w,
    "sum instead of mean": lambda x, w: x / np.sqrt((x ** 2).sum(axis=1, keepdims=True) + EPS) * w,
    "weight not applied": lambda x, w: oracle.rmsnorm(x, np.ones_like(w), EPS),
    "weight read one 16-byte vector late": lambda x, w: oracle.rmsnorm(x, np.roll(w, -8), EPS),
    "row scaled by the next row's rms": lambda x, w: x / np.sqrt(
        np.roll((x ** 2).mean(axis=1, keepdims=True), -1, axis=0) + EPS) * w,
}


@pytest.mark.parametrize("bug", list(RMS_BUGS))
def test_rmsnorm_parity_sees(bug):
    caught = []
    for M, K in RMS_CASES:
        x, w = synth.rmsnorm_inputs(M, K, seed=M + K)
        x, w = synth.to_f64(x), synth.to_f64(w)
        caught.append(_fails_parity(RMS_BUGS[bug](x, w), oracle.rmsnorm(x, w, EPS)))
    assert any(caught), f"{bug}: inside the tolerance in every case"


def test_a_dropped_vector_is_seen_only_at_small_k():
    # the ragged small-K cases carry the check: at K >= 512 one 8-element vector
    # moves the rms by less than the tolerance
    bug = RMS_BUGS["sum of squares misses the row's last 16-byte vector"]
    seen = {}
    for M, K in RMS_CASES:
        x, w = synth.rmsnorm_inputs(M, K, seed=M + K)
        x, w = synth.to_f64(x), synth.to_f64(w)
        seen[K] = _fails_parity(bug(x, w), oracle.rmsnorm(x, w, EPS))
    assert seen[8] and seen[136] and not seen[4096]


# ---------------------------------------------------------------------------
# MatMul: the cases of test_matmul_matches_oracle

MM_CASES = [(300, 520, 512), (1, 256, 64), (128, 256, 128), (129, 264, 192), (32, 1024, 512), (5, 8, 64),
            (257, 4096, 1024)]

MM_BUGS = {
    "last 64-wide K block dropped": lambda a, w: oracle.matmul(a[:, :-64], w[:, :-64]),
    "first K block accumulated twice": lambda a, w: oracle.matmul(a, w) + oracle.matmul(a[:, :64], w[:, :64]),
    "columns past the last full 256-wide tile left at zero":
        lambda a, w: np.where(np.arange(w.shape[0]) < (w.shape[0] // 256) * 256, oracle.matmul(a, w), 0.0),
    "rows of a ragged last tile read from the tile's first row":
        lambda a, w: oracle.matmul(a[np.minimum(np.arange(a.shape[0]), (a.shape[0] - 1) // 128 * 128)], w),
    "K blocks taken in the wrong 64-column order for W":
        lambda a, w: oracle.matmul(a, np.roll(w, 64, axis=1)),
}


@pytest.mark.parametrize("bug", list(MM_BUGS))
def test_matmul_parity_sees(bug):
    caught = []
    for M, N, K in MM_CASES:
        a, w = synth.matmul_inputs(M, N, K, seed=M * 7 + N + K)
        a, w = synth.to_f64(a), synth.to_f64(w)
        caught.append(_fails_parity(MM_BUGS[bug](a, w), oracle.matmul(a, w)))
    assert any(caught), f"{bug}: inside the tolerance in every case"


# ---------------------------------------------------------------------------
# LM head: the cases of test_gpu_lmhead.py (oracle comparison, planted margins,
# thresholds that force or forbid the recompute)

LM_CASES = [(9, 1000, 256), (1, 32000, 2048), (64, 32000, 2048), (40, 4096, 512), (6, 2000, 4160)]
TAU = 0.5


def _first_argmax(v, highest):
    idx = np.flatnonzero(v == v.max())
    return int(idx[-1] if highest else idx[0])


def _lm_emulate(h, w, tau, bug):
    """What bi_lmhead_argmax returns (tokens, recomputed, fp32 logits or NaN) for a
    correct kernel (bug None) or for one with the named bug."""
    r = oracle.lmhead(h, w, tau)
    lb = oracle.round_to_bf16(r["logits"])
    b1 = np.array([oracle.top2(row)[0] for row in lb])
    b2 = np.array([oracle.top2(row)[2] for row in lb])
    margin = (b1.astype(np.float32) - b2.astype(np.float32)).astype(np.float64)
    if bug == "top-2 margin taken from the fp32 accumulators, not the bf16 logits":
        margin = r["margin"]
    rec = margin <= tau if bug == "threshold test is <= instead of <" else margin < tau
    lg32 = r["logits"].astype(np.float32).astype(np.float64)
    if bug == "recompute done in bf16":
        lg32 = lb
    if bug == "recompute drops the last 64-wide K block":
        lg32 = oracle.matmul(h[:, :-64], w[:, :-64]).astype(np.float32).astype(np.float64)
    highest = bug == "ties go to the highest index"
    first = np.array([_first_argmax(row, highest) for row in lb])
    second = np.array([_first_argmax(row, highest) for row in lg32])
    if bug == "recomputed rows keep the first-pass token":
        second = first
    tokens = np.where(rec, second, first)
    logits = np.where(rec[:, None], lg32, np.nan)
    return tokens, rec, logits


LM_BUGS = ["threshold test is <= instead of <", "top-2 margin taken from the fp32 accumulators, not the bf16 logits",
           "recompute done in bf16", "recompute drops the last 64-wide K block", "ties go to the highest index",
           "recomputed rows keep the first-pass token"]


def _planted_inputs():
    K, V = 128, 512
    _, w = synth.lmhead_inputs(1, V, K, seed=70)
    h = np.zeros((5, K))
    h[0, 0] = h[1, 1] = h[2, 2] = h[3, 3] = 1.0
    h[4, 4] = h[4, 5] = 1.0
    w = synth.to_f64(w)
    w[:, :6] = np.clip(w[:, :6], -1, 1)
    w[7, 0], w[30, 0] = 3.0, 2.875
    w[12, 1], w[40, 1] = 8.0, 3.0
    w[5, 2], w[6, 2] = 2.0, 2.0
    w[9, 3], w[20, 3] = 4.0, 3.5
    w[0, 4], w[0, 5] = 256.0, 0.0
    w[1, 4], w[1, 5] = 256.0, 0.625
    return h, w


def _lm_tests_fail(bug, cases):
    """True when some assertion of the LM-head GPU tests fails on the emulated output."""
    import torch
    from test_gpu_lmhead import _check_against_oracle

    try:
        for h, w in cases:
            tok, rec, lg = _lm_emulate(h, w, TAU, bug)
            ht = torch.from_numpy(h).to(torch.bfloat16)
            wt = torch.from_numpy(w).to(torch.bfloat16)
            _check_against_oracle(ht, wt, TAU, torch.from_numpy(tok), torch.from_numpy(rec.astype(np.int32)),
                                  torch.from_numpy(lg.astype(np.float32)))
            assert np.isnan(lg[~rec]).all()
        h, w = _planted_inputs()
        tok, rec, lg = _lm_emulate(h, w, TAU, bug)
        assert tok.tolist() == [7, 12, 5, 9, 1] and rec.astype(int).tolist() == [1, 0, 1, 0, 1]
        assert lg[0, 7] == 3.0 and lg[0, 30] == 2.875 and lg[4, 1] == 256.625 and lg[4, 0] == 256.0
        h, w = (synth.to_f64(t) for t in synth.lmhead_inputs(16, 4096, 512, seed=71))
        assert _lm_emulate(h, w, 0.0, bug)[1].sum() == 0
        tok, rec, lg = _lm_emulate(h, w, math.inf, bug)
        assert rec.sum() == 16 and (tok == np.argmax(lg, axis=1)).all()
    except AssertionError:
        return True
    return False


@pytest.fixture(scope="module")
def lm_cases():
    return [tuple(synth.to_f64(t) for t in synth.lmhead_inputs(M, V, K, seed=M + V)) for M, V, K in LM_CASES]


def test_lmhead_control_passes(lm_cases):
    assert not _lm_tests_fail(None, lm_cases)


@pytest.mark.parametrize("bug", LM_BUGS)
def test_lmhead_tests_see(bug, lm_cases):
    assert _lm_tests_fail(bug, lm_cases), f"{bug}: every LM-head GPU test would pass"


# ---------------------------------------------------------------------------
# Tensor-core prefill: the cases of test_prefill_tc_matches_oracle (one sequence
# of 300 rows, sampled rows, three head configurations)

TC_CASES = [(128, 32, 8), (64, 32, 8), (128, 16, 8)]
TC_ROWS = [0, 1, 2, 15, 16, 127, 128, 129, 200, 255, 256, 299]


def _tc_case(D, Hq, Hkv):
    q, qs, qp, kv = synth.prefill_inputs([300], Hq, Hkv, D, seed=70 + D + Hq)
    r = TC_ROWS
    return (synth.to_f64(q)[r], qs.numpy()[r], qp.numpy()[r], synth.to_f64(kv.k_cache), synth.to_f64(kv.v_cache),
            kv.page_table.numpy())


def _tc_bug_keys_of_block_skipped(q, qs, qp, k, v, pt, block):
    """A schedule that drops one whole 64-key block (e.g. an off-by-one block count):
    keys of that block are removed from every row that would see them. A row whose
    keys all lie in that block keeps them (the emulation understates the bug there)."""
    out = np.zeros_like(q)
    D = q.shape[2]
    group = q.shape[1] // k.shape[1]
    for i in range(q.shape[0]):
        L = int(qp[i]) + 1
        keep = [t for t in range(L) if t // 64 != block] or list(range(L))
        for h in range(q.shape[1]):
            keys = oracle.gather_kv(k, pt[int(qs[i])], h // group, L)[keep]
            vals = oracle.gather_kv(v, pt[int(qs[i])], h // group, L)[keep]
            out[i, h] = oracle.softmax_attend(q[i, h], keys, vals, 1.0 / math.sqrt(D))
    return out


TC_BUGS = {
    "diagonal block's mask excludes the row's own key":
        lambda q, qs, qp, k, v, pt: oracle.attention_rows(q, k, v, pt, qs, qp, None),
    "diagonal block's mask lets in the next key":
        lambda q, qs, qp, k, v, pt: oracle.attention_rows(q, k, v, pt, qs, qp + 2, None),
    "first 64-key block skipped": lambda *a: _tc_bug_keys_of_block_skipped(*a, block=0),
    "second 64-key block skipped": lambda *a: _tc_bug_keys_of_block_skipped(*a, block=1),
    "tile B computed with tile A's query head":
        lambda q, qs, qp, k, v, pt: oracle.attention_prefill(np.repeat(q[:, 0::2], 2, axis=1), qs, qp, k, v, pt),
}


@pytest.mark.parametrize("bug", list(TC_BUGS))
def test_prefill_tc_parity_sees(bug):
    caught = []
    for case in TC_CASES:
        q, qs, qp, k, v, pt = _tc_case(*case)
        ref = oracle.attention_prefill(q, qs, qp, k, v, pt)
        with np.errstate(all="ignore"):
            buggy = TC_BUGS[bug](q, qs, qp, k, v, np.where(pt < 0, pt.max(), pt))
        caught.append(_fails_parity(buggy, ref))
    assert any(caught), f"{bug}: inside the tolerance in every case"


# ---------------------------------------------------------------------------
# Decoder glue: the cases of test_gpu_glue.py (RoPE at three head shapes; SwiGLU)

ROPE_CASES = [(32, 64), (8, 64), (32, 128)]


def _rope_case(H, D):
    import torch
    x = synth.to_f64(synth.normal_bf16((37, H, D), 2))
    pos = torch.randint(0, 384, (37,), generator=synth.generator(3), dtype=torch.int32).numpy()
    return x, pos


def _rope_interleaved(x, pos):
    T, H, D = x.shape
    inv = 10000.0 ** (-2.0 * np.arange(D // 2) / D)
    ang = pos[:, None].astype(np.float64) * inv[None, :]
    c, s = np.cos(ang)[:, None, :], np.sin(ang)[:, None, :]
    a, b = x[..., 0::2], x[..., 1::2]
    out = np.empty_like(x)
    out[..., 0::2], out[..., 1::2] = a * c - b * s, b * c + a * s
    return out


ROPE_BUGS = {
    "position off by one": lambda x, pos: oracle.rope(x, pos + 1),
    "rotation the other way": lambda x, pos: oracle.rope(x, -pos),
    "interleaved pairs instead of halves": _rope_interleaved,
    "frequency exponent i/D instead of 2i/D": lambda x, pos: oracle.rope(x, pos, theta=100.0),
}


@pytest.mark.parametrize("bug", list(ROPE_BUGS))
def test_rope_parity_sees(bug):
    caught = []
    for H, D in ROPE_CASES:
        x, pos = _rope_case(H, D)
        caught.append(_fails_parity(ROPE_BUGS[bug](x, pos), oracle.rope(x, pos)))
    assert any(caught), f"{bug}: inside the tolerance in every case"


SWIGLU_BUGS = {
    "gate and up halves swapped": lambda gu: oracle.swiglu(np.concatenate([gu[:, gu.shape[1] // 2:],
                                                                            gu[:, : gu.shape[1] // 2]], axis=1)),
    "sigmoid instead of silu": lambda gu: (1 / (1 + np.exp(-gu[:, : gu.shape[1] // 2]))) * gu[:, gu.shape[1] // 2:],
    "gate times up without the activation": lambda gu: gu[:, : gu.shape[1] // 2] * gu[:, gu.shape[1] // 2:],
}


@pytest.mark.parametrize("bug", list(SWIGLU_BUGS))
def test_swiglu_parity_sees(bug):
    gu = synth.to_f64(synth.normal_bf16((33, 2 * 8192), 5))
    assert _fails_parity(SWIGLU_BUGS[bug](gu), oracle.swiglu(gu)), f"{bug}: inside the tolerance"
