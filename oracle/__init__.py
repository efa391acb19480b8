"""fp64 CPU oracle for the batch-invariant forward-pass kernels.

TEST INFRASTRUCTURE ONLY. Nothing on the product path imports this package:
only the tests, the smoke check and the benchmark's CPU-baseline leg may call it.
It shares no code with the CUDA library; inputs come from ``synth`` as exact
float64 widenings of the bf16 bits the GPU saw.

Every function evaluates the plain mathematical definition in float64, with no
blocking, splitting or reordering of its own: the batch-invariant GPU kernels
reach the same mathematical result in one fixed fp32 order, so the definition is
the reference. Sources (web pages on batch invariance):

* "Defeating Nondeterminism in LLM Inference" technical summary (mobiles-han
  blog), section 対応策：バッチ不変なカーネル設計, kernel table rows RMSNorm,
  MatMul and Attention — the three operations and what each must keep fixed.
* same blog, usage article, section 注意点・補足実装 (FixedAttention sketch) —
  the cache and the current chunk are joined into one layout before attention.
* "Greedy Decoding Is Not Precision-Invariant" (arXiv 2609.26621), abstract —
  the top-2 logit margin at the LM head decides greedy flips; the LM head is
  recomputed in FP32 only when that margin is below a threshold.
* same summary, section 他の演算子 (RMSNorm, MatMul, mean/reduction etc.) —
  log_softmax and mean are replaced by batch-invariant kernels too; Techzine,
  "Thinking Machines wil AI voorspelbaarder maken" — sampling and training must
  be bit-identical for on-policy RL; French "température zéro" blog, section "Le
  mensonge de la température zéro" — sampling made deterministic only in theory.

Readings where the pages are silent (each is pinned by a test):
* RMSNorm: y = x / sqrt(mean(x^2) + eps) * w, eps inside the root.
* MatMul: C = A @ W^T with W stored [N, K].
* Attention: softmax(q . k * scale) v with scale = 1/sqrt(D); q-head h reads
  kv-head h // (Hq/Hkv); a query at absolute position p sees keys 0..p
  (inclusive); decode queries see keys 0..L-1.
* LM head: greedy token = argmax of the logits, lowest index on ties; the
  recompute decision compares the top-2 margin of the bf16-rounded logits,
  taken in fp32, against the threshold.
* Sampling at temperature T > 0 (no page gives a method): the Gumbel-max rule
  over Philox4x64-10 uniforms keyed by the request's seed and step, so a row's
  draws never depend on the batch. The sampler and the generator are algorithms,
  not definitions: the oracle follows their published steps.

Parity pins: every function here is pinned (tests/test_oracle.py).
"""
from __future__ import annotations

import math

import numpy as np

PAGE = 16  # tokens per KV page of the unified store


# ---------------------------------------------------------------------------
# RMSNorm — "Defeating Nondeterminism" summary, kernel table, row RMSNorm


def rmsnorm(x: np.ndarray, w: np.ndarray, eps: float) -> np.ndarray:
    """y[m, :] = x[m, :] / sqrt(mean_k x[m, k]^2 + eps) * w, in float64."""
    x = np.asarray(x, dtype=np.float64)
    w = np.asarray(w, dtype=np.float64)
    ms = np.mean(x * x, axis=-1, keepdims=True)
    return x / np.sqrt(ms + eps) * w


# ---------------------------------------------------------------------------
# MatMul — same table, row MatMul


def matmul(a: np.ndarray, w: np.ndarray) -> np.ndarray:
    """C[m, n] = sum_k A[m, k] * W[n, k] (W stored [N, K]), in float64."""
    return np.asarray(a, dtype=np.float64) @ np.asarray(w, dtype=np.float64).T


# ---------------------------------------------------------------------------
# Attention over the unified paged store — same table, row Attention, and the
# FixedAttention sketch (cache and current tokens in one layout)


def gather_kv(cache: np.ndarray, page_row: np.ndarray, g: int, n_tokens: int) -> np.ndarray:
    """Tokens 0..n_tokens-1 of kv-head g, read through one page-table row.

    cache is [num_pages, Hkv, PAGE, D]; token t sits in slot t % PAGE of
    physical page page_row[t // PAGE].
    """
    t = np.arange(n_tokens)
    pages = np.asarray(page_row, dtype=np.int64)[t // PAGE]
    return np.asarray(cache[pages, g, t % PAGE], dtype=np.float64)


def softmax_attend(q: np.ndarray, keys: np.ndarray, vals: np.ndarray, scale: float) -> np.ndarray:
    """softmax(keys @ q * scale) @ vals for one query vector, max-subtracted, float64."""
    s = keys @ np.asarray(q, dtype=np.float64) * scale
    e = np.exp(s - s.max())
    return (e @ vals) / e.sum()


def attention_rows(q, k_cache, v_cache, page_table, row_page, row_len, scale=None):
    """Attention for a list of query rows.

    q: [R, Hq, D]; row r reads page-table row row_page[r] and sees keys
    0..row_len[r]-1. Returns [R, Hq, D] float64. A row with no visible key
    returns zeros.
    """
    q = np.asarray(q, dtype=np.float64)
    k_cache = np.asarray(k_cache, dtype=np.float64)
    v_cache = np.asarray(v_cache, dtype=np.float64)
    R, Hq, D = q.shape
    Hkv = k_cache.shape[1]
    group = Hq // Hkv
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    out = np.zeros((R, Hq, D), dtype=np.float64)
    for r in range(R):
        L = int(row_len[r])
        if L <= 0:
            continue
        prow = np.asarray(page_table[int(row_page[r])])
        for g in range(Hkv):
            keys = gather_kv(k_cache, prow, g, L)
            vals = gather_kv(v_cache, prow, g, L)
            for j in range(group):
                h = g * group + j
                out[r, h] = softmax_attend(q[r, h], keys, vals, scale)
    return out


def attention_decode(q, k_cache, v_cache, page_table, seq_lens, scale=None):
    """Decode: query b (one new token per sequence) sees keys 0..seq_lens[b]-1."""
    B = np.asarray(q).shape[0]
    return attention_rows(q, k_cache, v_cache, page_table, np.arange(B), np.asarray(seq_lens), scale)


def attention_prefill(q, q_seq, q_pos, k_cache, v_cache, page_table, scale=None):
    """Causal prefill: the query at absolute position p of sequence s sees keys 0..p of s."""
    return attention_rows(q, k_cache, v_cache, page_table, np.asarray(q_seq),
                          np.asarray(q_pos) + 1, scale)


# ---------------------------------------------------------------------------
# LM head with the margin test — "Greedy Decoding Is Not Precision-Invariant",
# abstract (selective FP32 LM-head recompute below a margin threshold)


def round_to_bf16(x: np.ndarray) -> np.ndarray:
    """Round float64 values to bf16 as the GPU epilogue does (fp64 -> fp32 RNE, fp32 -> bf16 RNE).

    Works on the fp32 bit pattern: add 0x7FFF plus the lowest kept bit, then
    truncate the low 16 bits. NaN/inf are not expected here.
    """
    f = np.asarray(x, dtype=np.float64).astype(np.float32)
    bits = f.view(np.uint32).astype(np.uint64)
    lsb = (bits >> 16) & 1
    rounded = ((bits + 0x7FFF + lsb) >> 16) << 16
    return rounded.astype(np.uint32).view(np.float32).astype(np.float64)


def argmax_lowest(v: np.ndarray) -> int:
    """Index of the largest value, lowest index among equals."""
    v = np.asarray(v)
    return int(np.flatnonzero(v == v.max())[0])


def top2(v: np.ndarray):
    """(top1 value, top1 index, top2 value, top2 index) with lowest-index tie-break."""
    v = np.asarray(v, dtype=np.float64)
    i1 = argmax_lowest(v)
    rest = v.copy()
    rest[i1] = -np.inf
    i2 = argmax_lowest(rest)
    return v[i1], i1, v[i2], i2


def lmhead(h: np.ndarray, w: np.ndarray, threshold: float):
    """Greedy LM head.

    Returns a dict with
      logits  [M, V] float64 (exact),
      tokens  [M] int: argmax of the exact logits,
      margin  [M] float64: exact top1 - top2,
      margin_bf16 [M] float64: top1 - top2 of the bf16-rounded logits
                  (the quantity the first pass thresholds),
      recompute [M] bool: margin_bf16 < threshold,
      tokens_bf16 [M] int: argmax of the bf16-rounded logits.
    """
    logits = matmul(h, w)
    M = logits.shape[0]
    tokens = np.empty(M, dtype=np.int64)
    tokens_bf16 = np.empty(M, dtype=np.int64)
    margin = np.empty(M)
    margin_bf16 = np.empty(M)
    lb = round_to_bf16(logits)
    for m in range(M):
        v1, i1, v2, _ = top2(logits[m])
        tokens[m], margin[m] = i1, v1 - v2
        b1, j1, b2, _ = top2(lb[m])
        tokens_bf16[m] = j1
        margin_bf16[m] = float(np.float32(b1) - np.float32(b2))
    return dict(logits=logits, tokens=tokens, margin=margin, margin_bf16=margin_bf16,
                recompute=margin_bf16 < threshold, tokens_bf16=tokens_bf16)


# ---------------------------------------------------------------------------
# Row reductions and sampling — "Defeating Nondeterminism" summary, section
# 他の演算子 (RMSNorm, MatMul, mean/reduction etc.): log_softmax and mean are among
# the operations replaced by batch-invariant kernels, and a mean must be reduced in
# one fixed order (no split, or a split of fixed size only). Why logprobs and
# sampled tokens must match bit for bit: Techzine, "Thinking Machines wil AI
# voorspelbaarder maken" (training and sampling bit-identical, hence truly
# on-policy RL) and the hakusoku page's discussion of trainer/sampler numerics;
# the French "température zéro" blog, section "Le mensonge de la température
# zéro", on sampling made deterministic in theory but not in practice.


def log_softmax(x: np.ndarray) -> np.ndarray:
    """y[m, i] = x[m, i] - log(sum_j exp(x[m, j])), in float64 (max-shifted)."""
    x = np.asarray(x, dtype=np.float64)
    mx = x.max(axis=-1, keepdims=True)
    return x - (mx + np.log(np.exp(x - mx).sum(axis=-1, keepdims=True)))


def token_logprob(x: np.ndarray, tokens: np.ndarray) -> np.ndarray:
    """log_softmax(x)[m, tokens[m]]: the log-probability of each row's token."""
    ls = log_softmax(x)
    return ls[np.arange(ls.shape[0]), np.asarray(tokens, dtype=np.int64)]


def row_mean(x: np.ndarray) -> np.ndarray:
    """y[m] = sum_k x[m, k] / K, in float64."""
    x = np.asarray(x, dtype=np.float64)
    return x.sum(axis=-1) / x.shape[-1]


# Philox4x64-10, the counter-based generator of Salmon, Moraes, Dror and Shaw,
# "Parallel random numbers: as easy as 1, 2, 3" (SC 2011): ten rounds of two 64x64
# -> 128-bit multiplications on a 256-bit counter under a 128-bit key, with a Weyl
# increment of the key between rounds. Written from that definition; its outputs
# are pinned against numpy's independent implementation.
_PHILOX_M = (np.uint64(0xD2E7470EE14C6C93), np.uint64(0xCA5A826395121157))
_PHILOX_W = (np.uint64(0x9E3779B97F4A7C15), np.uint64(0xBB67AE8584CAA73B))
_LO32 = np.uint64(0xFFFFFFFF)


def _mulhilo64(a, b):
    """(high, low) 64-bit halves of the 128-bit product a * b (uint64 arrays)."""
    a = np.asarray(a, dtype=np.uint64)
    b = np.asarray(b, dtype=np.uint64)
    s32 = np.uint64(32)
    a0, a1 = a & _LO32, a >> s32
    b0, b1 = b & _LO32, b >> s32
    p00, p01, p10, p11 = a0 * b0, a0 * b1, a1 * b0, a1 * b1
    mid = (p00 >> s32) + (p01 & _LO32) + (p10 & _LO32)
    hi = p11 + (p01 >> s32) + (p10 >> s32) + (mid >> s32)
    with np.errstate(over="ignore"):
        lo = a * b
    return hi, lo


def philox4x64_10(ctr, key):
    """Philox4x64-10 block: ctr = 4 uint64 words (arrays broadcast), key = 2 words.

    Returns the 4 output words. Round: (x0, x1, x2, x3) -> (hi(M1 x2) ^ x1 ^ k0,
    lo(M1 x2), hi(M0 x0) ^ x3 ^ k1, lo(M0 x0)); then k += (W0, W1).
    """
    x = [np.asarray(c, dtype=np.uint64) for c in ctr]
    k0, k1 = (np.asarray(k, dtype=np.uint64) for k in key)
    with np.errstate(over="ignore"):
        for _ in range(10):
            hi0, lo0 = _mulhilo64(_PHILOX_M[0], x[0])
            hi1, lo1 = _mulhilo64(_PHILOX_M[1], x[2])
            x = [hi1 ^ x[1] ^ k0, lo1, hi0 ^ x[3] ^ k1, lo0]
            k0 = k0 + _PHILOX_W[0]
            k1 = k1 + _PHILOX_W[1]
    return x


def sampling_uniforms(seed: int, step: int, V: int) -> np.ndarray:
    """The uniform u_i in (0, 1) drawn for vocabulary entry i of one row.

    Reading (the pages give no generator): the row's request seed is the key
    (seed, 0); the counter is (i div 8, step, 0, 0); one block's four 64-bit words
    give eight 32-bit halves, entry i taking word (i mod 8) div 2, its low half for
    even i and its high half for odd i; u_i = (top 23 bits of that half + 1/2) *
    2^-23 — exactly representable in fp32, never 0 or 1. It depends only on
    (seed, step, i), never on the batch.
    """
    i = np.arange(V, dtype=np.uint64)
    z = np.zeros(V, dtype=np.uint64)
    words = philox4x64_10((i >> np.uint64(3), np.full(V, step, dtype=np.uint64), z, z),
                          (np.uint64(seed), np.uint64(0)))
    w = np.choose(((i >> np.uint64(1)) & np.uint64(3)).astype(np.int64), words)
    half = np.where((i & np.uint64(1)) == 0, w & _LO32, w >> np.uint64(32))
    return ((half >> np.uint64(9)).astype(np.float64) + 0.5) * 2.0 ** -23


def gumbel_scores(x: np.ndarray, temperature: float, u: np.ndarray) -> np.ndarray:
    """x_i / T + g_i with the Gumbel variate g_i = -log(-log(u_i)), in float64."""
    x = np.asarray(x, dtype=np.float64)
    return x / temperature - np.log(-np.log(np.asarray(u, dtype=np.float64)))


def sample(x: np.ndarray, temperature: float, seeds, steps) -> np.ndarray:
    """Temperature sampling by the Gumbel-max rule: token = argmax_i (x_i / T + g_i).

    argmax of logits plus independent Gumbel noise is a draw from softmax(x / T)
    (Gumbel 1954; the "Gumbel-max trick"). One row per request; lowest index wins
    ties. x: [M, V].
    """
    x = np.asarray(x, dtype=np.float64)
    M, V = x.shape
    out = np.empty(M, dtype=np.int64)
    for m in range(M):
        out[m] = argmax_lowest(gumbel_scores(x[m], temperature, sampling_uniforms(int(seeds[m]), int(steps[m]), V)))
    return out


# ---------------------------------------------------------------------------
# Normwise error used by every parity test


def normwise_rel_err(got: np.ndarray, ref: np.ndarray) -> np.ndarray:
    """Per row: max |got - ref| / max |ref| (rows are the leading axes flattened)."""
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    g = got.reshape(-1, got.shape[-1])
    r = ref.reshape(-1, ref.shape[-1])
    den = np.abs(r).max(axis=1)
    den[den == 0] = 1.0
    return np.abs(g - r).max(axis=1) / den


# ---------------------------------------------------------------------------
# Decoder-step glue (plain Llama operations, no page describes them): rotary
# embedding (rotate-half), SwiGLU, and one decoder layer chained in float64.


def rope(x: np.ndarray, pos: np.ndarray, theta: float = 10000.0) -> np.ndarray:
    """Rotary embedding, rotate-half form, in float64.

    x: [T, H, D]; for i < D/2 the pair (x[i], x[i + D/2]) of token t is rotated by
    the angle pos[t] * theta^(-2i/D).
    """
    x = np.asarray(x, dtype=np.float64)
    T, H, D = x.shape
    half = D // 2
    inv = theta ** (-2.0 * np.arange(half) / D)
    ang = np.asarray(pos, dtype=np.float64)[:, None] * inv[None, :]  # [T, half]
    c, s = np.cos(ang)[:, None, :], np.sin(ang)[:, None, :]
    a, b = x[..., :half], x[..., half:]
    return np.concatenate([a * c - b * s, b * c + a * s], axis=-1)


def silu(g: np.ndarray) -> np.ndarray:
    g = np.asarray(g, dtype=np.float64)
    return g / (1.0 + np.exp(-g))


def swiglu(gate_up: np.ndarray) -> np.ndarray:
    """silu(gate) * up with gate = first half of the columns, up = second half."""
    gu = np.asarray(gate_up, dtype=np.float64)
    F = gu.shape[-1] // 2
    return silu(gu[..., :F]) * gu[..., F:]


def decoder_layer(h, rows_seq, rows_pos, past_k, past_v, w, n_heads, n_kv, eps=1e-6, theta=10000.0):
    """One pre-norm Llama decoder layer over query rows, in float64.

    h: [T, Hd] hidden rows; row t is token rows_pos[t] of sequence rows_seq[t].
    past_k/past_v: dict seq -> [L, n_kv, D] keys/values already in the cache for
    positions 0..L-1 (already rotated). w: dict with wqkv [(n_heads+2 n_kv) D, Hd],
    wo [Hd, Hd], wgu [2F, Hd], wdown [Hd, F], attn_norm, mlp_norm [Hd].
    The rows' own keys/values are appended (positions must continue the cache) and
    each row attends causally over its sequence. Returns the new h [T, Hd].
    """
    h = np.asarray(h, dtype=np.float64)
    T, Hd = h.shape
    D = Hd // n_heads
    x = rmsnorm(h, w["attn_norm"], eps)
    qkv = matmul(x, w["wqkv"])
    q = qkv[:, : n_heads * D].reshape(T, n_heads, D)
    k = qkv[:, n_heads * D: (n_heads + n_kv) * D].reshape(T, n_kv, D)
    v = qkv[:, (n_heads + n_kv) * D:].reshape(T, n_kv, D)
    q = rope(q, rows_pos, theta)
    k = rope(k, rows_pos, theta)
    keys = {s: np.asarray(past_k[s], dtype=np.float64) for s in past_k}
    vals = {s: np.asarray(past_v[s], dtype=np.float64) for s in past_v}
    for t in range(T):
        s, p = int(rows_seq[t]), int(rows_pos[t])
        kk = keys.setdefault(s, np.zeros((0, n_kv, D)))
        assert kk.shape[0] == p, "rows must extend their sequence's cache in order"
        keys[s] = np.concatenate([kk, k[t:t + 1]])
        vals[s] = np.concatenate([vals.setdefault(s, np.zeros((0, n_kv, D))), v[t:t + 1]])
    att = np.empty((T, n_heads, D))
    group = n_heads // n_kv
    for t in range(T):
        s, p = int(rows_seq[t]), int(rows_pos[t])
        for hh in range(n_heads):
            g = hh // group
            att[t, hh] = softmax_attend(q[t, hh], keys[s][: p + 1, g], vals[s][: p + 1, g], 1.0 / math.sqrt(D))
    h = h + matmul(att.reshape(T, Hd), w["wo"])
    x = rmsnorm(h, w["mlp_norm"], eps)
    h = h + matmul(swiglu(matmul(x, w["wgu"])), w["wdown"])
    return h
