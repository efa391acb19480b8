"""Verify-and-rollback selective determinism (LLM-42 as the French "température zéro"
blog describes it, section "Vous n'avez pas à le payer partout") on the random Llama.

* certified requests end with exactly the streams of pure batch-invariant greedy
  decoding, whatever the nondeterministic fast path proposed and however it was
  batched; requests that are not certified keep the fast path's tokens;
* BI_LLM42_REPORT=<path> also times, at 64 prompts x 128 tokens, 256 generated:
  pure invariant decoding, verify-and-rollback with all / a quarter / no requests
  certified, and writes the acceptance rate and tokens/s as JSON.
"""
import json
import os

import numpy as np
import pytest

import synth
from gpu_util import dev
from invariant_deterministic_04_b200.llama import FastBiLlama, run_schedule
from invariant_deterministic_04_b200.verify import FastPathLlama, generate, timed_generate

pytestmark = pytest.mark.gpu


def _models(cfg, w, S, max_pos, window):
    fast = FastPathLlama(cfg, w, S, max_pos, dev())
    inv = FastBiLlama(cfg, w, S, max_pos, dev(), max_want=S * window)
    return fast, inv


def test_certified_streams_equal_invariant_decoding():
    cfg = synth.LLAMA_CFG
    S, P, G, window = 12, 48, 40, 6
    w = synth.llama_weights(cfg, seed=0, device=dev())
    prompts = synth.prompts(S, P, cfg["vocab"], seed=3)
    ref, _, _ = run_schedule(FastBiLlama(cfg, w, S, P + G, dev()), prompts, G, seed=4)
    certified = np.arange(S) % 2 == 0
    for seed in (5, 6):  # two different load patterns on the fast path
        fast, inv = _models(cfg, w, S, P + G, window)
        out, st = generate(fast, inv, prompts, G, certified, window, seed)
        assert out.shape == (S, G)
        np.testing.assert_array_equal(out[certified], ref[certified])
        assert st["accepted"] <= st["proposed"]
        assert st["verify_rows"] == st["proposed"]
    report = os.environ.get("BI_LLM42_REPORT")
    if report:
        _report(report)


def _report(path):
    cfg = synth.LLAMA_CFG
    S, P, G, window = 64, 128, 256, 8
    w = synth.llama_weights(cfg, seed=0, device=dev())
    prompts = synth.prompts(S, P, cfg["vocab"], seed=0)
    res = {"prompts": S, "prompt_len": P, "generated": G, "window": window}
    inv_model = FastBiLlama(cfg, w, S, P + G, dev())
    run_schedule(inv_model, prompts, 8, seed=0)  # warm-up
    import time

    import torch

    torch.cuda.synchronize()
    t0 = time.perf_counter()
    ref, steps, _ = run_schedule(FastBiLlama(cfg, w, S, P + G, dev()), prompts, G, seed=1)
    torch.cuda.synchronize()
    res["invariant_tokens_per_s"] = S * G / (time.perf_counter() - t0)
    for name, frac in (("all", 1.0), ("quarter", 0.25), ("none", 0.0)):
        certified = np.arange(S) < int(S * frac)
        fast, inv = _models(cfg, w, S, P + G, window)
        generate(fast, inv, prompts[:4], 8, certified[:4], window, seed=0)  # warm-up (flashinfer plans, kernels)
        fast, inv = _models(cfg, w, S, P + G, window)
        (out, st), sec = timed_generate(fast, inv, prompts, G, certified, window, seed=2)
        assert np.array_equal(out[certified], ref[certified])
        res[f"certified_{name}"] = {"tokens_per_s": S * G / sec, "acceptance": st["accepted"] / max(1, st["proposed"]),
                                    "rollbacks": st["rolled_back"], "rounds": st["rounds"],
                                    "verify_rows": st["verify_rows"], "fast_rows": st["fast_rows"]}
    with open(path, "w") as f:
        json.dump(res, f, indent=1)
    print(json.dumps(res))
