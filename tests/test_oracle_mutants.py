"""Strength of the oracle's pins: planted mistakes must be caught (CPU only).

Each mutant is one plausible slip written into a copy of an oracle function's
source: a dropped term, a wrong sign, axis, index or constant, a transposed or
swapped operand, an off-by-one mask, a wrong tie-break or rounding. The mutated
function replaces the oracle's for the duration of one test, and the pins of
test_oracle.py and test_oracle_reductions.py run against it. The mutant is caught
when at least one pin fails. A control run checks that every pin passes on the
unmutated oracle, so a harness error cannot pass for a catch.

The mistakes are planted in the oracle only, on the CPU; nothing here touches the
GPU path.
"""
from __future__ import annotations

import __future__
import functools
import inspect
import textwrap

import numpy as np
import pytest

import oracle
import test_oracle
import test_oracle_reductions

# pins that take seconds run last, so most mutants stop at a fast one
_SLOW = ("test_sample_frequencies_follow_softmax",)


def _expand(fn):
    """The pytest parametrisations of a pin, as argument-free callables."""
    combos = [{}]
    for mark in getattr(fn, "pytestmark", []):
        if mark.name != "parametrize":
            continue
        names, values = mark.args[0], mark.args[1]
        names = [n.strip() for n in names.split(",")] if isinstance(names, str) else list(names)
        combos = [{**c, **dict(zip(names, v if len(names) > 1 else (v,)))} for c in combos for v in values]
    return [(fn.__name__, functools.partial(fn, **c)) for c in combos]


def _pins():
    out = []
    for mod in (test_oracle, test_oracle_reductions):
        for name, fn in inspect.getmembers(mod, inspect.isfunction):
            if name.startswith("test_") and fn.__module__ == mod.__name__:
                out += _expand(fn)
    return out


PINS = _pins()


def _first_failure(prefer=()):
    """Name and error of the first pin that fails, or None. Pins whose names
    contain one of `prefer` run first."""
    order = sorted(PINS, key=lambda p: (not any(s in p[0] for s in prefer), p[0] in _SLOW))
    for name, pin in order:
        try:
            pin()
        except Exception as e:  # noqa: BLE001 - any failure of a pin catches the mutant
            return name, f"{type(e).__name__}: {str(e)[:120]}"
    return None


def _mutated(name, old, new):
    """oracle.<name> rebuilt from its source with `old` replaced by `new` (once)."""
    src = textwrap.dedent(inspect.getsource(getattr(oracle, name)))
    assert src.count(old) == 1, f"{name}: {old!r} occurs {src.count(old)} times"
    code = compile(src.replace(old, new), f"<mutant of oracle.{name}>", "exec",
                   flags=__future__.annotations.compiler_flag, dont_inherit=True)
    ns = {}
    exec(code, vars(oracle), ns)  # globals are the oracle's, so its other functions resolve as usual
    return ns[name]


# (oracle function, text replaced, replacement, pins to try first)
SOURCE_MUTANTS = [
    # RMSNorm
    ("rmsnorm", "np.mean(x * x", "np.sum(x * x", "rmsnorm"),
    ("rmsnorm", "np.sqrt(ms + eps)", "(np.sqrt(ms) + eps)", "rmsnorm"),
    ("rmsnorm", "ms + eps", "ms", "rmsnorm"),
    ("rmsnorm", "np.sqrt(ms + eps) * w", "np.sqrt(ms + eps)", "rmsnorm"),
    ("rmsnorm", "axis=-1, keepdims=True", "axis=0, keepdims=True", "rmsnorm"),
    ("rmsnorm", "x / np.sqrt", "x * np.sqrt", "rmsnorm"),
    ("rmsnorm", "x * x", "np.abs(x)", "rmsnorm"),
    # MatMul
    ("matmul", "dtype=np.float64) @", "dtype=np.float32) @", "matmul"),
    ("matmul", "dtype=np.float64).T", "dtype=np.float64)", "matmul"),
    # paged gather
    ("gather_kv", "pages = np.asarray(page_row, dtype=np.int64)[t // PAGE]",
     "pages = np.asarray(page_row, dtype=np.int64)[t % PAGE]", "attention"),
    ("gather_kv", "pages = np.asarray(page_row, dtype=np.int64)[t // PAGE]", "pages = t // PAGE", "attention"),
    ("gather_kv", "cache[pages, g, t % PAGE]", "cache[pages, 0, t % PAGE]", "attention"),
    ("gather_kv", "cache[pages, g, t % PAGE]", "cache[pages, g, t // PAGE]", "attention"),
    # softmax · V
    ("softmax_attend", "np.float64) * scale", "np.float64)", "attention"),
    ("softmax_attend", "(e @ vals) / e.sum()", "(e @ vals)", "attention"),
    ("softmax_attend", "(e @ vals)", "(e @ keys)", "attention"),
    ("softmax_attend", "np.exp(s - s.max())", "np.exp(s.max() - s)", "attention"),
    # attention rows, decode, prefill
    ("attention_rows", "h = g * group + j", "h = j * Hkv + g", "attention"),
    ("attention_rows", "group = Hq // Hkv", "group = Hkv", "attention"),
    ("attention_rows", "scale = 1.0 / math.sqrt(D)", "scale = 1.0 / D", "attention"),
    ("attention_rows", "L = int(row_len[r])", "L = int(row_len[r]) - 1", "attention"),
    ("attention_rows", "page_table[int(row_page[r])]", "page_table[r]", "prefill"),
    ("attention_rows", "if L <= 0:", "if L < 0:", "attention"),
    ("attention_decode", "np.asarray(seq_lens), scale", "np.asarray(seq_lens) - 1, scale", "attention"),
    ("attention_prefill", "np.asarray(q_pos) + 1", "np.asarray(q_pos)", "prefill"),
    ("attention_prefill", "np.asarray(q_pos) + 1", "np.asarray(q_pos) + 2", "prefill"),
    ("attention_prefill", "np.asarray(q_seq),", "np.zeros(len(q_seq), dtype=np.int64),", "prefill"),
    # bf16 rounding, argmax, top-2, LM head
    ("round_to_bf16", "0x7FFF + lsb", "0x7FFF", "bf16"),
    ("round_to_bf16", "0x7FFF + lsb", "0x8000", "bf16"),
    ("round_to_bf16", "bits + 0x7FFF + lsb", "bits", "bf16"),
    ("argmax_lowest", "[0]", "[-1]", "lmhead"),
    ("top2", "rest[i1] = -np.inf", "rest[i1] = rest[i1]", "lmhead"),
    ("top2", "return v[i1], i1, v[i2], i2", "return v[i1], i1, v[i1], i2", "lmhead"),
    ("lmhead", "recompute=margin_bf16 < threshold", "recompute=margin_bf16 <= threshold", "lmhead"),
    ("lmhead", "top2(lb[m])", "top2(logits[m])", "lmhead"),
    ("lmhead", "lb = round_to_bf16(logits)", "lb = logits", "lmhead"),
    ("lmhead", "i1, v1 - v2", "i1, v2 - v1", "lmhead"),
    ("lmhead", "tokens_bf16[m] = j1", "tokens_bf16[m] = i1", "lmhead"),
    # row reductions
    ("log_softmax", ".sum(axis=-1, keepdims=True)", ".mean(axis=-1, keepdims=True)", "log_softmax"),
    ("log_softmax", "x - (mx + np.log", "x - (np.log", "log_softmax"),
    ("log_softmax", "mx = x.max(axis=-1, keepdims=True)", "mx = x.max()", "log_softmax"),
    ("token_logprob", "np.asarray(tokens, dtype=np.int64)]", "np.asarray(tokens, dtype=np.int64) - 1]", "token"),
    ("token_logprob", "ls[np.arange(ls.shape[0]), ", "ls[0, ", "token"),
    ("row_mean", "/ x.shape[-1]", "/ (x.shape[-1] - 1)", "row_mean"),
    ("row_mean", "x.sum(axis=-1)", "x.sum(axis=0)", "row_mean"),
    # Philox4x64-10 and the uniforms
    ("_mulhilo64", " + (mid >> s32)", "", "philox"),
    ("_mulhilo64", "mid = (p00 >> s32) + ", "mid = ", "philox"),
    ("philox4x64_10", "range(10)", "range(9)", "philox"),
    ("philox4x64_10", "hi1 ^ x[1] ^ k0", "hi1 ^ x[1] ^ k1", "philox"),
    ("philox4x64_10", "x = [hi1 ^ x[1] ^ k0, lo1, hi0 ^ x[3] ^ k1, lo0]",
     "x = [hi0 ^ x[1] ^ k0, lo0, hi1 ^ x[3] ^ k1, lo1]", "philox"),
    ("philox4x64_10", "k0 = k0 + _PHILOX_W[0]", "k0 = k0 + _PHILOX_W[1]", "philox"),
    ("philox4x64_10", "_mulhilo64(_PHILOX_M[1], x[2])", "_mulhilo64(_PHILOX_M[1], x[1])", "philox"),
    ("sampling_uniforms", "i >> np.uint64(3), np.full", "i >> np.uint64(2), np.full", "uniforms"),
    ("sampling_uniforms", "w & _LO32, w >> np.uint64(32)", "w >> np.uint64(32), w & _LO32", "uniforms"),
    ("sampling_uniforms", "(half >> np.uint64(9))", "(half >> np.uint64(8))", "uniforms"),
    ("sampling_uniforms", ".astype(np.float64) + 0.5)", ".astype(np.float64) + 0.0)", "uniforms"),
    ("sampling_uniforms", "(i >> np.uint64(3), np.full(V, step, dtype=np.uint64), z, z)",
     "(np.full(V, step, dtype=np.uint64), i >> np.uint64(3), z, z)", "uniforms"),
    ("sampling_uniforms", "(np.uint64(seed), np.uint64(0))", "(np.uint64(0), np.uint64(seed))", "uniforms"),
    ("sampling_uniforms", "((i >> np.uint64(1)) & np.uint64(3))", "(i & np.uint64(3))", "uniforms"),
    # Gumbel-max sampling
    ("gumbel_scores", "x / temperature - np.log", "x * temperature - np.log", "sample"),
    ("gumbel_scores", "x / temperature - np.log", "x / temperature + np.log", "sample"),
    ("gumbel_scores", "np.log(-np.log(", "(-np.log(", "gumbel"),
    ("sample", "int(seeds[m])", "int(seeds[0])", "sample"),
    ("sample", "int(steps[m])", "int(steps[0])", "sample"),
    ("sample", "gumbel_scores(x[m], temperature,", "gumbel_scores(x[m], 1.0,", "sample"),
    # error measure
    ("normwise_rel_err", "den = np.abs(r).max(axis=1)", "den = np.abs(g).max(axis=1)", "normwise"),
    # decoder glue
    ("rope", "-2.0 * np.arange(half) / D", "-1.0 * np.arange(half) / D", "rope"),
    ("rope", "a * c - b * s, b * c + a * s", "a * c + b * s, b * c - a * s", "rope"),
    ("rope", "a, b = x[..., :half], x[..., half:]", "a, b = x[..., 0::2], x[..., 1::2]", "rope"),
    ("rope", "np.asarray(pos, dtype=np.float64)[:, None]", "(np.asarray(pos, dtype=np.float64)[:, None] + 1)",
     "rope"),
    ("silu", "g / (1.0 + np.exp(-g))", "1.0 / (1.0 + np.exp(-g))", "silu"),
    ("silu", "np.exp(-g)", "np.exp(g)", "silu"),
    ("swiglu", "silu(gu[..., :F]) * gu[..., F:]", "gu[..., :F] * silu(gu[..., F:])", "swiglu"),
    # one decoder layer
    ("decoder_layer", 'x = rmsnorm(h, w["attn_norm"], eps)', "x = h", "decoder"),
    ("decoder_layer", 'x = rmsnorm(h, w["mlp_norm"], eps)', 'x = rmsnorm(h, w["attn_norm"], eps)', "decoder"),
    ("decoder_layer", "q = rope(q, rows_pos, theta)", "q = q", "decoder"),
    ("decoder_layer", "k = rope(k, rows_pos, theta)", "k = k", "decoder"),
    ("decoder_layer", "keys[s][: p + 1, g], vals[s][: p + 1, g]", "keys[s][:, g], vals[s][:, g]", "decoder"),
    ("decoder_layer", "g = hh // group", "g = hh % n_kv", "decoder"),
    ("decoder_layer", "1.0 / math.sqrt(D))", "1.0 / D)", "decoder"),
    ("decoder_layer", "v = qkv[:, (n_heads + n_kv) * D:]", "v = qkv[:, n_heads * D: (n_heads + n_kv) * D]",
     "decoder"),
    ("decoder_layer", 'h = h + matmul(att.reshape(T, Hd), w["wo"])', 'h = matmul(att.reshape(T, Hd), w["wo"])',
     "decoder"),
    ("decoder_layer", "h = h + matmul(swiglu(", "h = matmul(swiglu(", "decoder"),
    ("decoder_layer", "vals = {s: np.asarray(past_v[s]", "vals = {s: np.asarray(past_k[s]", "decoder"),
    ("decoder_layer", "keys = {s: np.asarray(past_k[s], dtype=np.float64)",
     "keys = {s: 0 * np.asarray(past_k[s], dtype=np.float64)", "decoder"),
]

# (oracle attribute, wrong value, pins to try first)
VALUE_MUTANTS = [
    ("_PHILOX_M", tuple(reversed(oracle._PHILOX_M)), "philox"),
    ("_PHILOX_W", tuple(reversed(oracle._PHILOX_W)), "philox"),
    ("PAGE", 8, "attention"),
]


def test_every_pin_passes_on_the_oracle():
    assert len(PINS) > 60
    assert _first_failure() is None


@pytest.mark.parametrize("name,old,new,prefer", SOURCE_MUTANTS,
                         ids=[f"{m[0]}:{i}" for i, m in enumerate(SOURCE_MUTANTS)])
def test_source_mutant_is_caught(monkeypatch, name, old, new, prefer):
    monkeypatch.setattr(oracle, name, _mutated(name, old, new))
    with np.errstate(all="ignore"):
        caught = _first_failure((prefer,))
    assert caught is not None, f"no pin fails when oracle.{name} has {old!r} -> {new!r}"


@pytest.mark.parametrize("name,value,prefer", VALUE_MUTANTS, ids=[m[0] for m in VALUE_MUTANTS])
def test_value_mutant_is_caught(monkeypatch, name, value, prefer):
    monkeypatch.setattr(oracle, name, value)
    with np.errstate(all="ignore"):
        caught = _first_failure((prefer,))
    assert caught is not None, f"no pin fails when oracle.{name} = {value!r}"
