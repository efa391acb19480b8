#!/usr/bin/env python
"""Benchmark of the batch-invariant kernels (one JSON line on rank 0).

Step (the default workload "k4096_m2048"): one batch of M=2048 rows at hidden
size K=4096 goes through bi_rmsnorm and then, in one bi_matmul_multi call, the
matmuls against three weights with N = 4096, 6144 and 14336 (each product bit-identical
to bi_matmul alone; one launch over the three products' tiles): the RMSNorm-then-matmul configuration
swept by the invariance tests, at its largest batch. `value` is the matmul
throughput of the whole step (2*M*K*sum(N) FLOPs / step time, the RMSNorm
included in the time), summed over all GPUs; every GPU runs its own replica
(rows are independent, nothing is exchanged), so scaling is weak.

Also reported on rank 0 at N=1: the per-kernel roofline of the dominant kernel
(the tcgen05 matmul), the slowdown against the non-invariant path (cuBLAS via
torch.matmul + F.rms_norm) on the same box, an end-to-end figure through the
public API with host buffers, the clocks seen during the timed region, the fp64
CPU oracle timed on a bounded sample, and (``--rows``, default on) one
measurement of every other hot-path kernel: RMSNorm bandwidth, decode attention
bandwidth, causal prefill throughput, the LM head, the row reductions, and the
random-Llama decoder under mixed batching (streams per prompt, tokens/s,
recompute rate, against stock torch ops); and (``--sweeps``, default
on) the configuration sweeps: bi_matmul over M = 1..2048 at K = 4096 for N = 4096,
6144 and 14336 (W warm and W cold), RMSNorm over the same M at hidden 4096, and
decode attention over B = 1..256 with lengths ~ U[1, 32768], each entry with its
fraction of the applicable peak.

``--impl reference`` times the fp64 CPU oracle on the same workload and metric
(bounded samples per step) and prints the reference line.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402
import torch.distributed as dist  # noqa: E402

import synth  # noqa: E402

METRIC = "bi-matmul TFLOP/s, RMSNorm/attn HBM GB/s, % roofline, slowdown vs non-invariant"
K_HIDDEN = 4096
NS = (4096, 6144, 14336)
EPS = 1e-6
WORKLOAD = "k4096_m2048"


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return {"hbm_gbs": float(p["hbm_gbs"]), "bf16_tflops": float(p["bf16_tflops"]),
                "bf16_tflops_sustained": float(p["bf16_tflops_sustained"]), "sm_max_mhz": float(p.get("sm_max_mhz", 1965)),
                "source": "measured"}
    except Exception:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "sm_max_mhz": 1965.0,
                "source": "fallback"}


# ---------------------------------------------------------------------------
# distributed plumbing (timing only; no data-path collective)


def init_dist():
    """Process group from the torchrun environment. A rank that fails or never joins ends the
    others' next collective with an error after BI_PG_TIMEOUT_S seconds (default 300)
    instead of a hang."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1 and not dist.is_initialized():
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        timeout = datetime.timedelta(seconds=float(os.environ.get("BI_PG_TIMEOUT_S", "300")))
        dist.init_process_group(backend=backend, timeout=timeout)
    return rank, world, local


def barrier(world):
    if world > 1:
        dist.barrier()


def aggregate(units: float, ms: float, world: int, device=None):
    """Whole-job (sum of units, max of elapsed ms) over ranks."""
    if world <= 1:
        return units, ms
    t = torch.tensor([units], dtype=torch.float64, device=device)
    m = torch.tensor([ms], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    dist.all_reduce(m, op=dist.ReduceOp.MAX)
    return float(t.item()), float(m.item())


# ---------------------------------------------------------------------------
# clocks during the timed region


class ClockSampler:
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.QUERY}",
                                          "--format=csv,noheader,nounits", "-lms", "50"],
                                         stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return None
        mhz = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        maxmhz = max(float(r[2]) for r in rows if r[2].replace(".", "").isdigit())
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower().startswith("active")})
        busy = [m for m in mhz if m > 0.5 * maxmhz] or mhz
        return {"sm_mhz": statistics.median(busy), "sm_max_mhz": maxmhz, "reasons": reasons,
                "samples": len(rows)}


# ---------------------------------------------------------------------------
# the step


class Workload:
    """Resident inputs of the default step (weights + two rotating activation sets)."""

    def __init__(self, M: int, device):
        self.M = M
        self.device = device
        xs = [synth.normal_bf16((M, K_HIDDEN), 100 + i) for i in range(2)]
        self.x = [x.to(device) for x in xs]
        self.wn = synth.normal_bf16((K_HIDDEN,), 110, std=0.1, mean=1.0).to(device)
        self.W = [synth.normal_bf16((n, K_HIDDEN), 120 + j, std=0.02).to(device) for j, n in enumerate(NS)]
        self.y = torch.empty((M, K_HIDDEN), dtype=torch.bfloat16, device=device)
        self.C = [torch.empty((M, n), dtype=torch.bfloat16, device=device) for n in NS]
        self.flops = 2.0 * M * K_HIDDEN * sum(NS)
        self.rms_bytes = 4.0 * M * K_HIDDEN + 2.0 * K_HIDDEN
        self.launches_per_step = 2  # the RMSNorm, then the three products in one bi_matmul_multi call


def step_ours(bi, wl: Workload, i: int, ev=None):
    """RMSNorm then the three matmuls of the normalised rows (one bi_matmul_multi call: one
    launch on CTA-pair tiles at M = 2048). ev: optional (start, end) event pairs per call."""
    if ev is None:
        bi.rmsnorm(wl.x[i % 2], wl.wn, EPS, out=wl.y)
        bi.matmul_multi(wl.y, wl.W, outs=wl.C)
        return
    ev[0][0].record()
    bi.rmsnorm(wl.x[i % 2], wl.wn, EPS, out=wl.y)
    ev[0][1].record()
    ev[1][0].record()
    bi.matmul_multi(wl.y, wl.W, outs=wl.C)
    ev[1][1].record()


def step_cublas(wl: Workload, i: int):
    y = torch.nn.functional.rms_norm(wl.x[i % 2], (K_HIDDEN,), wl.wn, EPS)
    for W, C in zip(wl.W, wl.C):
        torch.matmul(y, W.t(), out=C)


def time_loop(fn, steps: int, warmup: int, world: int):
    for i in range(warmup):
        fn(i)
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s.record()
    for i in range(steps):
        fn(i)
    e.record()
    torch.cuda.synchronize()
    barrier(world)
    return s.elapsed_time(e)


def e2e_pipelined(bi, wl, xh, steps: int, warmup: int, world: int):
    """Device time of `steps` end-to-end steps through the public calls. Every step copies
    its input from pinned host memory to the device (its own stream), runs the RMSNorm and
    the three matmuls (the current stream) and copies all three outputs back to pinned host
    memory (a third stream). Two device buffers of the input and of the outputs let step
    i's copies run under the neighbouring steps' kernels; events keep each buffer's
    writer, reader and copy in order. The timed region ends when the last output copy has
    landed."""
    comp = torch.cuda.current_stream()
    h2d, d2h = torch.cuda.Stream(), torch.cuda.Stream()
    xd = [torch.empty_like(wl.x[0]) for _ in range(2)]
    cd = [[torch.empty_like(c) for c in wl.C] for _ in range(2)]
    ch = [[torch.empty(c.shape, dtype=c.dtype).pin_memory() for c in wl.C] for _ in range(2)]
    ev_in = [torch.cuda.Event() for _ in range(2)]    # input of the buffer's step is on the device
    ev_comp = [torch.cuda.Event() for _ in range(2)]  # its kernels are done (input read, outputs written)
    ev_out = [torch.cuda.Event() for _ in range(2)]   # its outputs are on the host

    def run(i):
        b = i % 2
        with torch.cuda.stream(h2d):
            if i >= 2:
                h2d.wait_event(ev_comp[b])  # step i-2 has read xd[b]
            xd[b].copy_(xh[b], non_blocking=True)
            ev_in[b].record(h2d)
        comp.wait_event(ev_in[b])
        if i >= 2:
            comp.wait_event(ev_out[b])  # step i-2's outputs have left cd[b]
        bi.rmsnorm(xd[b], wl.wn, EPS, out=wl.y)
        bi.matmul_multi(wl.y, wl.W, outs=cd[b])
        ev_comp[b].record(comp)
        with torch.cuda.stream(d2h):
            d2h.wait_event(ev_comp[b])
            for C, H in zip(cd[b], ch[b]):
                H.copy_(C, non_blocking=True)
            ev_out[b].record(d2h)

    for i in range(warmup):
        run(i)
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s.record(comp)
    for i in range(steps):
        run(i)
    comp.wait_stream(d2h)
    e.record(comp)
    torch.cuda.synchronize()
    barrier(world)
    return s.elapsed_time(e)


def traffic_from_profile():
    """Per-launch DRAM bytes of the step's matmul launch (the three products) from the
    committed ncu summary, or None if gemm.cuh changed since it was captured."""
    path = os.path.join(ROOT, "profiles", "gemm_bf16_pair_kernel_traffic.txt")
    src = os.path.join(ROOT, "invariant_deterministic_04_b200", "csrc", "gemm.cuh")
    try:
        rec = {}
        with open(path) as f:
            for line in f:
                if ":" in line and not line.startswith("#"):
                    k, v = line.split(":", 1)
                    rec[k.strip()] = v.strip()
        with open(src, "rb") as f:
            h = hashlib.sha256(f.read()).hexdigest()
        if rec.get("gemm_cuh_sha256") != h:
            return None
        return int(rec["dram_bytes_per_launch"])
    except Exception:
        return None


# ---------------------------------------------------------------------------
# CPU oracle timing (bounded sample)


def oracle_step_sample(rows: int, seed: int = 0):
    """fp64 oracle on `rows` rows of the step: RMSNorm then the three matmuls. Returns (flops, seconds)."""
    import oracle

    x = synth.to_f64(synth.normal_bf16((rows, K_HIDDEN), 100 + seed))
    wn = synth.to_f64(synth.normal_bf16((K_HIDDEN,), 110, std=0.1, mean=1.0))
    Ws = [synth.to_f64(synth.normal_bf16((n, K_HIDDEN), 120 + j, std=0.02)) for j, n in enumerate(NS)]
    t0 = time.perf_counter()
    y = oracle.rmsnorm(x, wn, EPS)
    for W in Ws:
        oracle.matmul(y, W)
    return 2.0 * rows * K_HIDDEN * sum(NS), time.perf_counter() - t0


def cpu_threads():
    try:
        from threadpoolctl import threadpool_info

        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return os.cpu_count() or 1


def cpu_baseline(budget_s: float = 10.0):
    """The oracle on about budget_s seconds of the step: a row sample if a whole step takes
    longer, else whole 2048-row steps repeated."""
    rows = 32
    flops, t = oracle_step_sample(rows)
    rows = int(max(32, min(2048, rows * budget_s / max(t, 1e-3))))
    flops, t = oracle_step_sample(rows, seed=1)
    reps = 1
    if rows == 2048 and t < budget_s:
        reps = max(1, int(budget_s / max(t, 1e-3)))
        for i in range(reps - 1):
            f, dt = oracle_step_sample(rows, seed=2 + i % 2)
            flops += f
            t += dt
    what = f"{reps} whole steps of 2048 rows" if rows == 2048 else f"{rows} of the 2048 rows of one step"
    out = {"value": flops / t / 1e12, "unit": "TFLOP/s", "cores": cpu_threads(), "kind": "oracle",
           "sample": f"fp64 numpy oracle: RMSNorm + matmuls (N=4096,6144,14336; K=4096), {what}, {t:.1f} s"}
    # the same oracle on one core: a 32-row sample of the step (about two seconds)
    try:
        from threadpoolctl import threadpool_limits

        with threadpool_limits(limits=1):
            f1, t1 = oracle_step_sample(32, seed=3)
        out["one_core"] = {"value": f1 / t1 / 1e12, "unit": "TFLOP/s", "sample": f"32 of the 2048 rows, {t1:.1f} s"}
    except Exception as e:  # threadpoolctl missing or the BLAS not controllable
        out["one_core"] = f"unavailable: {type(e).__name__}"
    return out


# ---------------------------------------------------------------------------
# other hot-path kernels (one measurement each, rank 0)


def _events_ms(fn, iters=10, warmup=3):
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s.record()
    for _ in range(iters):
        fn()
    e.record()
    torch.cuda.synchronize()
    return s.elapsed_time(e) / iters


def _graph_us(fn, n=20, reps=10):
    """Device microseconds per call of fn, from a CUDA graph of n calls replayed reps times."""
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        for _ in range(3):
            fn()
    torch.cuda.current_stream().wait_stream(side)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for _ in range(n):
            fn()
    g.replay()
    torch.cuda.synchronize()
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s.record()
    for _ in range(reps):
        g.replay()
    e.record()
    torch.cuda.synchronize()
    del g
    return s.elapsed_time(e) * 1e3 / (n * reps)


def other_rows(bi, device, pk, only=None):
    out = {}
    want = (lambda name: only is None or only == name)
    if want("chain"):
        out.update(_row_chain(bi, device))
    # RMSNorm bandwidth at a size far above L2 (M = 65536, K = 4096: 1 GiB in + out)
    if want("rmsnorm"):
        out.update(_row_rmsnorm(bi, device, pk))
    if want("decode"):
        out.update(_row_decode(bi, device, pk))
    if want("prefill"):
        out.update(_row_prefill(bi, device, pk))
    if want("lmhead"):
        out.update(_row_lmhead(bi, device, pk))
    if want("reduce"):
        out.update(_row_reduce(bi, device, pk))
    if want("config5"):
        out.update(_row_config5(bi, device, pk))
    return out


def _row_chain(bi, device):
    """Config 1: RMSNorm (K = 512) then the matmul 512 -> 1024 on 32 rows, x ~ N(0, 1),
    w = 1 + N(0, 0.1), W ~ N(0, 0.02). Reported: microseconds per chain (two launches,
    CUDA-graph replays, inputs warm: the whole chain is 1.3 MB), the same for F.rms_norm +
    torch.matmul, and whether rows 0..m-1 and the last m rows recomputed as batches of
    m = 1, 2, 7, 16 equal the 32-row batch bit for bit. Launch- and latency-bound: the
    chain is 33.6 MFLOP and 1.1 MB."""
    x, wn = synth.rmsnorm_inputs(32, 512, seed=0)
    _, W = synth.matmul_inputs(32, 1024, 512, seed=2)
    x, wn, W = x.to(device), wn.to(device), W.to(device)
    y = torch.empty_like(x)
    c = torch.empty((32, 1024), dtype=torch.bfloat16, device=device)

    def chain():
        bi.rmsnorm(x, wn, 1e-6, out=y)
        bi.matmul(y, W, out=c)

    us = _graph_per_call_us([chain] * 16)  # per closure: one RMSNorm and one matmul launch
    full = bi.matmul(bi.rmsnorm(x, wn, 1e-6), W)
    same = True
    for m in (1, 2, 7, 16):
        for start in (0, 32 - m):
            part = bi.matmul(bi.rmsnorm(x[start:start + m].contiguous(), wn, 1e-6), W)
            same = same and bool(torch.equal(part.view(torch.int16), full[start:start + m].view(torch.int16)))
    def ref():
        torch.matmul(torch.nn.functional.rms_norm(x, (512,), wn, 1e-6), W.t(), out=c)

    ref_us = _graph_per_call_us([ref] * 16)
    return {"chain_m32_k512_n1024": {"us": round(us, 2), "rows_bit_identical_m1_2_7_16": same,
                                     "noninvariant_us": round(ref_us, 2), "slowdown": round(us / ref_us, 3)}}


def _row_config5(bi, device, pk, repeats=3, base_repeats=2):
    """The random-init Llama decoder (16 layers, hidden 2048, 32/8 heads, SwiGLU 8192,
    vocab 32000, weights ~ N(0, 0.02), seed 0): 64 prompts of 128 tokens, 256 greedy
    tokens each, under random mixed batching (batch ~ U[1, 64] per step, random
    subsets and order, prefill chunks mixed with decode tokens; schedule seed r for
    repeat r). Reported: the most distinct 256-token streams any prompt produced over
    the repeats (1 = bit-identical), wall-clock tokens/s, the share of LM-head rows
    that took the FP32 recompute, and the same for stock torch ops (cuBLAS,
    F.rms_norm, padded attention, matmul + argmax) on the same weights."""
    from invariant_deterministic_04_b200.llama import BaselineLlama, FastBiLlama, run_repeats, run_schedule

    cfg = synth.LLAMA_CFG
    w = synth.llama_weights(cfg, seed=0, device=device)
    prompts = synth.prompts(64, 128, cfg["vocab"], seed=0)
    run_schedule(FastBiLlama(cfg, w, 64, 128 + 8, device), prompts, 8, seed=10_000)  # warm-up
    inv = run_repeats(FastBiLlama, cfg, w, prompts, 256, repeats, device)
    base = run_repeats(BaselineLlama, cfg, w, prompts, 256, base_repeats, device)
    diverging = int((base["first"] != inv["first"]).any(axis=1).sum())
    row = {"repeats": repeats, "max_unique_streams_per_prompt": inv["max_unique"],
           "tokens_per_s": round(inv["tokens_per_s"], 1), "recompute_rate": round(inv["recompute_rate"], 4),
           "baseline_repeats": base_repeats, "baseline_max_unique_streams_per_prompt": base["max_unique"],
           "baseline_mean_unique_streams_per_prompt": round(float(base["unique_per_seq"].mean()), 2),
           "baseline_prompts_diverging_from_invariant": diverging,
           "baseline_tokens_per_s": round(base["tokens_per_s"], 1),
           "speed_vs_baseline": round(inv["tokens_per_s"] / base["tokens_per_s"], 3)}
    del w
    torch.cuda.empty_cache()
    return {"config5_llama_64x128_gen256": row}


def _row_rmsnorm(bi, device, pk):
    out = {}
    M = 65536
    x = torch.randn((M, K_HIDDEN), device=device, dtype=torch.float32).to(torch.bfloat16)
    w = synth.normal_bf16((K_HIDDEN,), 110, std=0.1, mean=1.0).to(device)
    y = torch.empty_like(x)
    ms = _events_ms(lambda: bi.rmsnorm(x, w, EPS, out=y))
    ms_ref = _events_ms(lambda: torch.nn.functional.rms_norm(x, (K_HIDDEN,), w, EPS))
    gbs = (4.0 * M * K_HIDDEN + 2 * K_HIDDEN) / ms / 1e6
    out["rmsnorm_m65536_k4096"] = {"GB/s": round(gbs, 1), "frac_hbm": round(gbs / pk["hbm_gbs"], 3), "ms": round(ms, 4),
                                   "slowdown_vs_F.rms_norm": round(ms / ms_ref, 3)}
    return out


def _row_decode(bi, device, pk):
    out = {}
    # decode attention: B=64 sequences, lengths ~ U[1, 32768], GQA 32/8, D=128
    B, Lmax = 64, 32768
    lens = synth.decode_lengths(B, Lmax, seed=50)
    kv = synth.paged_kv_device(lens, 8, 128, seed=51, max_pages=Lmax // 16, device=device)
    q = synth.normal_bf16((B, 32, 128), 52).to(device)
    ws = torch.empty(bi.attention_workspace_size(B, 32, 128, kv.max_pages), dtype=torch.uint8, device=device)
    o = torch.empty_like(q)
    ms = _events_ms(lambda: bi.attention_decode(q, kv.k_cache, kv.v_cache, kv.page_table, kv.seq_lens, out=o,
                                                workspace=ws))
    kv_bytes = 4096.0 * int(lens.sum())  # K and V: L * Hkv * D * 2 bytes * 2
    gbs = kv_bytes / ms / 1e6
    out["decode_b64_l32k"] = {"GB/s": round(gbs, 1), "frac_hbm": round(gbs / pk["hbm_gbs"], 3), "ms": round(ms, 4),
                              "kv_bytes": kv_bytes}
    # non-invariant comparison: flashinfer's paged decode with its own split-KV heuristic, same store
    try:
        import flashinfer

        npages = [(int(L) + 15) // 16 for L in lens.tolist()]
        indptr = torch.tensor([0] + list(np.cumsum(npages)), dtype=torch.int32, device=device)
        indices = torch.cat([kv.page_table[b, :n] for b, n in enumerate(npages)]).contiguous()
        last = torch.tensor([(int(L) - 1) % 16 + 1 for L in lens.tolist()], dtype=torch.int32, device=device)
        fws = torch.empty(256 << 20, dtype=torch.uint8, device=device)
        wrapper = flashinfer.BatchDecodeWithPagedKVCacheWrapper(fws, kv_layout="HND")
        wrapper.plan(indptr, indices, last, 32, 8, 128, 16, q_data_type=torch.bfloat16, kv_data_type=torch.bfloat16)
        fo = wrapper.run(q, (kv.k_cache, kv.v_cache))
        ms_ref = _events_ms(lambda: wrapper.run(q, (kv.k_cache, kv.v_cache)))
        err = float(((fo.float() - o.float()).abs().max() / o.float().abs().max()).item())
        out["decode_b64_l32k"].update({"flashinfer_ms": round(ms_ref, 4), "slowdown_vs_flashinfer": round(ms / ms_ref, 3),
                                       "flashinfer_GB/s": round(kv_bytes / ms_ref / 1e6, 1),
                                       "max_rel_diff_vs_flashinfer": round(err, 5)})
    except Exception as e:  # the comparison path is optional
        out["decode_b64_l32k"]["flashinfer"] = f"unavailable: {type(e).__name__}: {str(e)[:120]}"
    return out


def _row_prefill(bi, device, pk):
    out = {}
    # causal prefill, one sequence of 4096 tokens
    S = 4096
    kvp = synth.paged_kv_device([S], 8, 128, seed=60, max_pages=S // 16, device=device)
    qp = synth.normal_bf16((S, 32, 128), 61).to(device)
    qs = torch.zeros(S, dtype=torch.int32, device=device)
    qpos = torch.arange(S, dtype=torch.int32, device=device)
    wsp = torch.empty(bi.attention_workspace_size(S, 32, 128, kvp.max_pages), dtype=torch.uint8, device=device)
    op = torch.empty_like(qp)
    ms = _events_ms(lambda: bi.attention_prefill(qp, qs, qpos, kvp.k_cache, kvp.v_cache, kvp.page_table, out=op,
                                                 workspace=wsp), iters=3, warmup=1)
    flops = 2.0 * 32 * 128 * S * (S + 1)  # q.k and p.v over the visible keys
    alu_peak = 148 * 128 * 2 * pk["sm_max_mhz"] * 1e6 / 1e12
    out["prefill_s4096"] = {"TFLOP/s": round(flops / ms / 1e9, 2), "frac_fp32_alu": round(flops / ms / 1e9 / alu_peak, 3),
                            "ms": round(ms, 3)}
    # the tensor-core prefill (same whole/chunked invariance, different fixed arithmetic)
    try:
        otc = torch.empty_like(qp)
        ms_tc = _events_ms(lambda: bi.attention_prefill_tc(qp, 0, 0, kvp.k_cache, kvp.v_cache, kvp.page_table, out=otc),
                           iters=10, warmup=2)
        out["prefill_s4096"].update({"tc_ms": round(ms_tc, 4), "tc_TFLOP/s": round(flops / ms_tc / 1e9, 1),
                                     "tc_frac_bf16_tensor": round(flops / ms_tc / 1e9 / pk["bf16_tflops"], 3)})
    except Exception as e:
        out["prefill_s4096"]["tc"] = f"unavailable: {type(e).__name__}: {str(e)[:120]}"
    # non-invariant comparison: torch SDPA (flash, tensor cores) on the same K/V laid out contiguously
    try:
        t = torch.arange(S, device=device)
        pages = kvp.page_table[0, t // 16].long()
        kc = kvp.k_cache[pages, :, t % 16, :].permute(1, 0, 2).unsqueeze(0)  # [1, 8, S, D]
        vc = kvp.v_cache[pages, :, t % 16, :].permute(1, 0, 2).unsqueeze(0)
        qs4 = qp.permute(1, 0, 2).unsqueeze(0)  # [1, 32, S, D]
        sdpa = torch.nn.functional.scaled_dot_product_attention
        ms_ref = _events_ms(lambda: sdpa(qs4, kc, vc, is_causal=True, enable_gqa=True), iters=10, warmup=2)
        out["prefill_s4096"].update({"sdpa_ms": round(ms_ref, 4), "slowdown_vs_sdpa": round(ms / ms_ref, 2)})
        if "tc_ms" in out["prefill_s4096"]:
            out["prefill_s4096"]["tc_slowdown_vs_sdpa"] = round(out["prefill_s4096"]["tc_ms"] / ms_ref, 2)
    except Exception as e:
        out["prefill_s4096"]["sdpa"] = f"unavailable: {type(e).__name__}: {str(e)[:120]}"
    return out


def _row_lmhead(bi, device, pk):
    out = {}
    # LM head: 64 rows, vocabulary 32000, hidden 2048
    h = synth.normal_bf16((64, 2048), 70).to(device)
    Wl = synth.normal_bf16((32000, 2048), 71, std=0.02).to(device)
    tok = torch.empty(64, dtype=torch.int32, device=device)
    rec = torch.empty(64, dtype=torch.int32, device=device)
    wsl = torch.empty(bi.lmhead_workspace_size(64, 32000), dtype=torch.uint8, device=device)
    ms = _events_ms(lambda: bi.lmhead_argmax(h, Wl, 0.5, tokens=tok, recomputed=rec, workspace=wsl))
    ms_ref = _events_ms(lambda: torch.argmax(torch.matmul(h, Wl.t()), dim=1))
    out["lmhead_m64_v32000"] = {"ms": round(ms, 4), "recomputed_rows": int(rec.sum()),
                                "slowdown_vs_cublas_argmax": round(ms / ms_ref, 3)}
    # batch 4 with trained-model-like margins (the greedy-decoding abstract's setting):
    # no row near a tie, then one row near a tie; device time from CUDA-graph replays
    for ties in (0, 1):
        h4, W4 = synth.lmhead_planted(4, 32000, 2048, seed=72, ties=ties)
        h4, W4 = h4.to(device), W4.to(device)
        t4 = torch.empty(4, dtype=torch.int32, device=device)
        r4 = torch.empty(4, dtype=torch.int32, device=device)
        ws4 = torch.empty(bi.lmhead_workspace_size(4, 32000), dtype=torch.uint8, device=device)
        us = _graph_us(lambda: bi.lmhead_argmax(h4, W4, 0.5, tokens=t4, recomputed=r4, workspace=ws4))
        us_ref = _graph_us(lambda: torch.argmax(torch.matmul(h4, W4.t()), dim=1))
        out[f"lmhead_m4_v32000_{ties}tie"] = {"us": round(us, 2), "recomputed_rows": int(r4.sum()),
                                             "cublas_argmax_us": round(us_ref, 2),
                                             "overhead_vs_cublas_argmax": round(us / us_ref - 1, 3)}
    return out


def _row_reduce(bi, device, pk):
    out = {}
    hbm = pk["hbm_gbs"]
    # log-probabilities of a 4096-token sequence over a 32000 vocabulary (bf16 in,
    # fp32 out: 786 MB, far above L2), its token log-probabilities, and sampling
    M, V = 4096, 32000
    x = synth.logits(M, V, seed=110).to(device)
    y = torch.empty((M, V), dtype=torch.float32, device=device)
    tok = torch.randint(0, V, (M,), generator=synth.generator(111), dtype=torch.int32).to(device)
    lp = torch.empty(M, dtype=torch.float32, device=device)
    seeds = synth.request_seeds(M, 112).to(device)
    steps = torch.zeros(M, dtype=torch.int64, device=device)
    st = torch.empty(M, dtype=torch.int32, device=device)
    ms = _events_ms(lambda: bi.log_softmax(x, out=y))
    ms_ref = _events_ms(lambda: torch.log_softmax(x, dim=-1, dtype=torch.float32))
    gbs = M * V * 6 / ms / 1e6
    out["log_softmax_m4096_v32000"] = {"ms": round(ms, 4), "GB/s": round(gbs, 1), "frac_hbm": round(gbs / hbm, 3),
                                       "slowdown_vs_torch": round(ms / ms_ref, 3)}
    ms = _events_ms(lambda: bi.token_logprob(x, tok, out=lp))
    gbs = M * V * 2 / ms / 1e6
    out["token_logprob_m4096_v32000"] = {"ms": round(ms, 4), "GB/s": round(gbs, 1), "frac_hbm": round(gbs / hbm, 3)}
    ms = _events_ms(lambda: bi.sample(x, seeds, steps, 0.8, out=st))
    # non-invariant comparison: torch's Gumbel-max with its own generator (batch-dependent draws)
    ms_ref = _events_ms(lambda: torch.argmax(x.float() / 0.8 - torch.log(-torch.log(torch.rand_like(x, dtype=torch.float32))),
                                             dim=-1))
    gbs = M * V * 2 / ms / 1e6
    out["sample_m4096_v32000"] = {"ms": round(ms, 4), "GB/s": round(gbs, 1), "frac_hbm": round(gbs / hbm, 3),
                                  "slowdown_vs_torch_gumbel": round(ms / ms_ref, 3)}
    # a decode-sized batch: 20 launches captured in a CUDA graph, so the host's
    # per-call cost does not hide the device time
    xs, s64, t64, o64 = x[:64].contiguous(), seeds[:64].contiguous(), steps[:64].contiguous(), st[:64]
    out["sample_m64_v32000"] = {"us": round(_graph_us(lambda: bi.sample(xs, s64, t64, 0.8, out=o64)), 2)}
    out["log_softmax_m64_v32000"] = {"us": round(_graph_us(lambda: bi.log_softmax(xs, out=y[:64])), 2)}
    # row means of 65536 x 4096 bf16 (512 MiB)
    xm = synth.normal_bf16((65536, 4096), 113, mean=0.5).to(device)
    ym = torch.empty(65536, dtype=torch.float32, device=device)
    ms = _events_ms(lambda: bi.row_mean(xm, out=ym))
    ms_ref = _events_ms(lambda: torch.mean(xm, dim=-1, dtype=torch.float32))
    gbs = xm.numel() * 2 / ms / 1e6
    out["row_mean_m65536_k4096"] = {"ms": round(ms, 4), "GB/s": round(gbs, 1), "frac_hbm": round(gbs / hbm, 3),
                                    "slowdown_vs_torch": round(ms / ms_ref, 3)}
    return out


# ---------------------------------------------------------------------------
# the configuration sweeps: bi_matmul over M (K=4096, three N, W warm and W cold),
# RMSNorm over M at hidden 4096, decode attention over the batch size


M_SWEEP = [1, 2, 3, 4, 7, 8, 13, 16, 32, 33, 64, 127, 128, 255, 256, 257, 512, 1023, 1024, 2047, 2048]
B_SWEEP = [1, 2, 4, 8, 16, 32, 64, 128, 256]


def _graph_per_call_us(calls, reps=5):
    """Device microseconds per call: the calls (closures issuing one launch each) are
    captured back to back in one CUDA graph, replayed `reps` times between two CUDA
    events, and the time is divided by the number of calls. Graph replay keeps the
    device busy from one launch to the next, so neither the host's issue cost nor the
    overhead of an event pair is counted. Callers rotate through inputs whose total
    size exceeds L2 (126 MB) to time them cold, or repeat one input to time it warm."""
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        for fn in calls[:2]:
            fn()
    torch.cuda.current_stream().wait_stream(side)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for fn in calls:
            fn()
    g.replay()
    torch.cuda.synchronize()
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s.record()
    for _ in range(reps):
        g.replay()
    e.record()
    torch.cuda.synchronize()
    del g
    return s.elapsed_time(e) * 1e3 / (len(calls) * reps)


def _copies(nbytes_one, floor=384 << 20, cap=64):
    """Number of rotating copies whose total exceeds `floor` bytes (three times L2)."""
    return int(max(2, min(cap, -(-floor // max(1, nbytes_one)))))


# tcgen05 dependent-accumulation step: one 128 x N x 16 MMA into the accumulator the
# previous one wrote costs about 83 SM cycles for N <= 128, 98 for N = 192 and 130
# for N = 256 (measured on this B200 with probes/mma_chain.cu). Every output tile is
# one such chain of K/16 MMAs, so no tile finishes in less than K/16 steps.
MMA_CHAIN_CYCLES = {32: 83.0, 64: 83.0, 128: 83.0, 192: 97.6, 256: 130.0}


def sweep_matmul(bi, device, pk, clocks_mhz, ms_list=M_SWEEP, calls=12):
    """One entry per (M, N): bi_matmul and cuBLAS (torch.matmul), each as CUDA-graph
    replays of back-to-back launches. W warm: one W repeated (it stays in L2). W cold:
    launches rotate through copies of W larger than L2 together (A, the activations,
    stays resident, as between the layers of a model). Fractions: of the bf16 burst
    peak; of the roofline max(FLOPs / peak, bytes / HBM); of the chain bound
    max(roofline time, K/16 chain steps at the sampled SM clock)."""
    A = synth.normal_bf16((2048, K_HIDDEN), 100).to(device)
    out = []
    for j, n in enumerate(NS):
        W = synth.normal_bf16((n, K_HIDDEN), 120 + j, std=0.02).to(device)
        R = _copies(W.numel() * 2)
        Ws = [W] + [W.clone() for _ in range(R - 1)]
        C = torch.empty((2048, n), dtype=torch.bfloat16, device=device)
        for m in ms_list:
            a, c = A[:m], C[:m]
            flops = 2.0 * m * n * K_HIDDEN
            byts = 2.0 * (m * K_HIDDEN + n * K_HIDDEN + m * n)
            roof_ms = max(flops / pk["bf16_tflops"] / 1e9, byts / pk["hbm_gbs"] / 1e6)
            tile_n = bi.matmul_tile_n(m, n)
            chain_ms = (K_HIDDEN / 16) * MMA_CHAIN_CYCLES[tile_n] / (clocks_mhz * 1e3)
            warm = _graph_per_call_us([lambda: bi.matmul(a, W, out=c)] * calls) / 1e3
            cold = _graph_per_call_us([lambda w=Ws[i % R]: bi.matmul(a, w, out=c) for i in range(max(calls, R))]) / 1e3
            ref = _graph_per_call_us([lambda w=Ws[i % R]: torch.matmul(a, w.t(), out=c)
                                      for i in range(max(calls, R))]) / 1e3
            out.append({"M": m, "N": n, "tile_m": bi.matmul_tile_m(m, n), "tile_n": tile_n,
                        "warm_us": round(warm * 1e3, 2), "warm_tflops": round(flops / warm / 1e9, 1),
                        "warm_frac_peak": round(flops / warm / 1e9 / pk["bf16_tflops"], 3),
                        "cold_us": round(cold * 1e3, 2), "cold_tflops": round(flops / cold / 1e9, 1),
                        "cold_frac_peak": round(flops / cold / 1e9 / pk["bf16_tflops"], 3),
                        "cold_frac_roofline": round(roof_ms / cold, 3),
                        "cold_frac_hbm": round(byts / cold / 1e6 / pk["hbm_gbs"], 3),
                        "cold_frac_chain_bound": round(max(roof_ms, chain_ms) / cold, 3),
                        "cublas_cold_us": round(ref * 1e3, 2), "slowdown_vs_cublas": round(cold / ref, 3)})
        del W, Ws, C
    return out


def sweep_rmsnorm(bi, device, pk, ms_list=M_SWEEP):
    """RMSNorm at hidden 4096 over M, CUDA-graph replays of back-to-back launches
    rotating through (x, y) pairs larger than L2 together (up to 64 pairs; below
    M = 64 the rows stay in L2 whatever the rotation): GB/s of x in + y out + w,
    fraction of the HBM copy peak, and F.rms_norm on the same rows."""
    wn = synth.normal_bf16((K_HIDDEN,), 110, std=0.1, mean=1.0).to(device)
    out = []
    for m in ms_list:
        R = _copies(2 * 2 * m * K_HIDDEN)
        xs = [synth.normal_bf16_device((m, K_HIDDEN), 130 + i, device) for i in range(R)]
        ys = [torch.empty_like(x) for x in xs]
        t = _graph_per_call_us([lambda i=i: bi.rmsnorm(xs[i], wn, EPS, out=ys[i]) for i in range(R)] * max(1, 16 // R))
        ref = _graph_per_call_us([lambda i=i: torch.nn.functional.rms_norm(xs[i], (K_HIDDEN,), wn, EPS)
                                  for i in range(R)] * max(1, 16 // R))
        gbs = (4.0 * m * K_HIDDEN + 2 * K_HIDDEN) / t / 1e3
        out.append({"M": m, "us": round(t, 2), "GB/s": round(gbs, 1), "frac_hbm": round(gbs / pk["hbm_gbs"], 3),
                    "slowdown_vs_F.rms_norm": round(t / ref, 3), "rotating_buffers": R})
        del xs, ys
    return out


def sweep_decode(bi, device, pk, bs=B_SWEEP):
    """Decode attention (32 q-heads / 8 kv-heads, D 128, 16-token pages) over the batch
    size, from one store of 256 sequences with lengths ~ U[1, 32768] (17 GB of K/V).
    Each B is timed as CUDA-graph replays of back-to-back launches over disjoint
    batches of B sequences (sequences rB .. rB + B - 1 for r = 0 .. 256/B - 1, at most
    16 batches), so consecutive launches read different K/V: KV bytes of all
    launches / their time, against the HBM copy peak."""
    Bmax, Lmax = max(bs), 32768
    lens = synth.decode_lengths(Bmax, Lmax, seed=50)
    kv = synth.paged_kv_device(lens, 8, 128, seed=51, max_pages=Lmax // 16, device=device)
    q = synth.normal_bf16((Bmax, 32, 128), 52).to(device)
    o = torch.empty_like(q)
    out = []
    for B in bs:
        R = max(1, min(16, Bmax // B))
        ws = torch.empty(bi.attention_workspace_size(B, 32, 128, kv.max_pages), dtype=torch.uint8, device=device)
        calls = []
        for r in range(R):
            sl = slice(r * B, (r + 1) * B)
            calls.append(lambda sl=sl: bi.attention_decode(q[sl], kv.k_cache, kv.v_cache, kv.page_table[sl],
                                                           kv.seq_lens[sl], out=o[sl], workspace=ws))
        reps = max(1, 16 // R)
        t = _graph_per_call_us(calls * reps if R < 16 else calls)
        tokens = int(lens[: R * B].sum())
        kv_bytes = 4096.0 * tokens / R
        gbs = kv_bytes / t / 1e3
        out.append({"B": B, "batches": R, "kv_tokens_per_launch": round(tokens / R), "us": round(t, 2),
                    "GB/s": round(gbs, 1), "frac_hbm": round(gbs / pk["hbm_gbs"], 3)})
        del ws
    del kv
    return out


def run_sweeps(bi, device, pk, clocks_mhz=None):
    res = {"matmul_k4096": sweep_matmul(bi, device, pk, clocks_mhz or pk["sm_max_mhz"]),
           "rmsnorm_k4096": sweep_rmsnorm(bi, device, pk),
           "decode_h32_8_d128_l32k": sweep_decode(bi, device, pk)}
    torch.cuda.empty_cache()
    return res


def run_sweep(bi, device, pk):
    """--sweep: the sweeps alone, one JSON line per entry."""
    for name, entries in run_sweeps(bi, device, pk).items():
        for e in entries:
            print(json.dumps({"sweep": name, **e}), flush=True)


# ---------------------------------------------------------------------------


PROFILE_CASES = ("decode_b16", "decode_b4", "decode_b1", "prefill_s4096", "rmsnorm", "lmhead_m4", "lmhead_m64", "matmul_small")


def profile_case(bi, device, name):
    """A few plain launches of one kernel case, for an ncu capture (nothing timed):
    decode_b16 / decode_b4 = decode attention over the first 16 / 4 sequences of the
    decode sweep's lengths (~ U[1, 32768]; 1.1 GB of K/V for 16); decode_b1 = decode attention over
    one sequence of 16384 tokens (64 splits, 67 MB of K/V); prefill_s4096 = causal
    prefill of one 4096-token sequence on the CUDA cores; rmsnorm = RMSNorm at 65536 x 4096
    then 2048 x 4096; lmhead_m4 = the LM head at 4 rows, V = 32000, K = 2048, with no
    near-tie and with one (then the cuBLAS matmul + argmax of the same shapes);
    lmhead_m64 = the LM head at 64 rows, V = 32000, K = 2048, random N(0, 0.02) weights
    (53 rows flagged);
    matmul_small = bi_matmul at M = 1 and 128, K = N = 4096."""
    if name in ("decode_b16", "decode_b4"):
        nb = 16 if name == "decode_b16" else 4
        lens = synth.decode_lengths(16, 32768, seed=50)[:nb]
        kv = synth.paged_kv_device(lens, 8, 128, seed=51, max_pages=2048, device=device)
        q = synth.normal_bf16((nb, 32, 128), 52).to(device)
        o = torch.empty_like(q)
        ws = torch.empty(bi.attention_workspace_size(nb, 32, 128, kv.max_pages), dtype=torch.uint8, device=device)
        for _ in range(3):
            bi.attention_decode(q, kv.k_cache, kv.v_cache, kv.page_table, kv.seq_lens, out=o, workspace=ws)
    elif name == "decode_b1":
        kv = synth.paged_kv_device([16384], 8, 128, seed=51, max_pages=2048, device=device)
        q = synth.normal_bf16((1, 32, 128), 52).to(device)
        o = torch.empty_like(q)
        ws = torch.empty(bi.attention_workspace_size(1, 32, 128, kv.max_pages), dtype=torch.uint8, device=device)
        for _ in range(3):
            bi.attention_decode(q, kv.k_cache, kv.v_cache, kv.page_table, kv.seq_lens, out=o, workspace=ws)
    elif name == "prefill_s4096":
        S = 4096
        kv = synth.paged_kv_device([S], 8, 128, seed=60, max_pages=S // 16, device=device)
        q = synth.normal_bf16((S, 32, 128), 61).to(device)
        qs = torch.zeros(S, dtype=torch.int32, device=device)
        qpos = torch.arange(S, dtype=torch.int32, device=device)
        o = torch.empty_like(q)
        ws = torch.empty(bi.attention_workspace_size(S, 32, 128, kv.max_pages), dtype=torch.uint8, device=device)
        for _ in range(2):
            bi.attention_prefill(q, qs, qpos, kv.k_cache, kv.v_cache, kv.page_table, out=o, workspace=ws)
    elif name == "lmhead_m64":
        h = synth.normal_bf16((64, 2048), 70).to(device)
        Wl = synth.normal_bf16((32000, 2048), 71, std=0.02).to(device)
        tok = torch.empty(64, dtype=torch.int32, device=device)
        rec = torch.empty(64, dtype=torch.int32, device=device)
        wsl = torch.empty(bi.lmhead_workspace_size(64, 32000), dtype=torch.uint8, device=device)
        for _ in range(3):
            bi.lmhead_argmax(h, Wl, 0.5, tokens=tok, recomputed=rec, workspace=wsl)
    elif name == "rmsnorm":
        for M in (65536, 2048):
            x = synth.normal_bf16_device((M, K_HIDDEN), 15, device)
            w = synth.normal_bf16((K_HIDDEN,), 16, std=0.1, mean=1.0).to(device)
            y = torch.empty_like(x)
            for _ in range(3):
                bi.rmsnorm(x, w, EPS, out=y)
    elif name == "lmhead_m4":
        for ties in (0, 1):
            h, W = synth.lmhead_planted(4, 32000, 2048, seed=72, ties=ties)
            h, W = h.to(device), W.to(device)
            for _ in range(2):
                bi.lmhead_argmax(h, W, 0.5)
            torch.argmax(torch.matmul(h, W.t()), dim=1)
    elif name == "matmul_small":
        A = synth.normal_bf16((128, K_HIDDEN), 100).to(device)
        W = synth.normal_bf16((4096, K_HIDDEN), 120, std=0.02).to(device)
        for m in (1, 128):
            for _ in range(2):
                bi.matmul(A[:m], W)
    torch.cuda.synchronize()
    print(json.dumps({"profile_case": name, "done": True}))


def ours_config(M, world):
    """The workload description both arms print (the same dict, so the two lines compare)."""
    return {"workload": WORKLOAD, "M": M, "K": K_HIDDEN, "N": list(NS), "step": "bi_rmsnorm + bi_matmul_multi (the three products, one launch)",
            "parallelism": f"replicas x{world}",
            "l2": "working set > L2 (201 MB of weights per step; two activation buffers rotate)"}


def run_reference(args, rank, world):
    """The fp64 CPU oracle on the same workload and metric (bounded samples per step)."""
    if rank != 0:
        return
    total = args.steps + args.warmup
    flops, t = oracle_step_sample(8)
    per = max(1, min(2048, int(8 * (90.0 / total) / max(t, 1e-3))))
    for i in range(args.warmup):
        oracle_step_sample(per, seed=i % 2)
    fl, tt = 0.0, 0.0
    for i in range(args.steps):
        f, s = oracle_step_sample(per, seed=i % 2)
        fl += f
        tt += s
    v = fl / tt / 1e12
    sample = f"fp64 numpy oracle, {per} of the 2048 rows per step (RMSNorm + matmuls N=4096,6144,14336; K=4096)"
    line = {"impl": "reference", "metric": METRIC, "value": v, "unit": "TFLOP/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": tt / args.steps * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": ours_config(2048, world),
            "cpu_baseline": {"value": v, "unit": "TFLOP/s", "cores": cpu_threads(), "kind": "oracle", "sample": sample},
            "e2e": {"value": v, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def run_ours(args, rank, world, local):
    import invariant_deterministic_04_b200 as bi

    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    bi.lib()
    pk = peaks()
    wl = Workload(args.M, device)

    # device-timed steps, with per-kernel events inside the timed region
    nk = wl.launches_per_step
    evs = [[[torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)] for _ in range(nk)]
           for _ in range(args.steps)]
    for i in range(args.warmup):
        step_ours(bi, wl, i)
    torch.cuda.synchronize()
    sampler = ClockSampler(local) if rank == 0 else None
    if sampler:
        sampler.start()
    barrier(world)
    torch.cuda.synchronize()
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s.record()
    for i in range(args.steps):
        step_ours(bi, wl, i, evs[i])
    e.record()
    torch.cuda.synchronize()
    barrier(world)
    clocks = sampler.stop() if sampler else None
    ms_total = s.elapsed_time(e)
    kernel_ms = [sum(evs[i][j][0].elapsed_time(evs[i][j][1]) for i in range(args.steps)) for j in range(nk)]
    units, ms_max = aggregate(wl.flops * args.steps, ms_total, world, device)
    value = units / (ms_max / 1e3) / 1e12
    gpu_launches = nk * args.steps

    # end to end through the public API: pinned host input in, all outputs back to pinned host memory
    xh = [wl.x[j].cpu().pin_memory() for j in range(2)]
    e2e_steps = max(10, min(args.steps, 100))
    e2e_ms = e2e_pipelined(bi, wl, xh, e2e_steps, 3, world)
    e2e_units, e2e_max = aggregate(wl.flops * e2e_steps, e2e_ms, world, device)
    h2d = wl.M * K_HIDDEN * 2
    d2h = sum(wl.M * n * 2 for n in NS)

    # non-invariant path on the same box
    ref_ms = time_loop(lambda i: step_cublas(wl, i), args.steps, args.warmup, world)

    if rank != 0:
        return
    # roofline of the dominant kernel: the tcgen05 matmul, one joint launch of the three
    # products per step (the launch the committed ncu capture covers)
    big_flops = 2.0 * wl.M * K_HIDDEN * sum(NS)
    big_ms = kernel_ms[1] / args.steps
    achieved = big_flops / (big_ms / 1e3) / 1e12
    gemm_ms = sum(kernel_ms[1:])
    step_gemm_tflops = 2.0 * wl.M * K_HIDDEN * sum(NS) * args.steps / (gemm_ms / 1e3) / 1e12
    # The denominator follows the regime the run was in: the burst peak (cuBLAS timed
    # alone, clocks at their maximum) while the SM clock stayed near its maximum, the
    # sustained one (seconds of back-to-back GEMMs under the power cap) when the
    # sampled median clock fell below 95 % of the maximum, or the timed region lasted
    # longer than two seconds.
    sm_mhz = (clocks or {}).get("sm_mhz")
    sm_max = (clocks or {}).get("sm_max_mhz") or pk["sm_max_mhz"]
    sustained = ms_total > 2000.0 or (sm_mhz is not None and sm_mhz < 0.95 * sm_max)
    peak = pk["bf16_tflops_sustained"] if sustained else pk["bf16_tflops"]
    roof = {"bound": "tensor",
            "kernel": ("gemm_bf16_pair_kernel<256> (tcgen05.mma.cta_group::2, 256 x 256 tiles on SM pairs), "
                       "one launch of the three products M=2048 K=4096 N=4096+6144+14336"),
            "achieved": round(achieved, 1), "peak": peak, "unit": "TFLOP/s",
            "frac": round(achieved / peak, 3),
            "peak_kind": (f"bf16 {'sustained' if sustained else 'burst'} ({pk['source']}); timed region "
                          f"{ms_total / 1e3:.3f} s, median SM clock {sm_mhz} of {sm_max} MHz"),
            "frac_of_burst": round(achieved / pk["bf16_tflops"], 3),
            "frac_of_sustained": round(achieved / pk["bf16_tflops_sustained"], 3), "traffic": traffic_from_profile(),
            "algorithmic_bytes_per_launch": 2 * (wl.M * K_HIDDEN + sum(NS) * K_HIDDEN + wl.M * sum(NS)),
            "launch_ms": round(big_ms, 4), "all_matmul_launches_tflops": round(step_gemm_tflops, 1),
            "kernel_share": round(gemm_ms / sum(kernel_ms), 3)}
    if roof["traffic"] is None:
        roof["traffic_note"] = ("gemm.cuh differs from the file the committed ncu counters "
                                "(profiles/gemm_bf16_pair_kernel_traffic.txt) were taken with")
    rms_ms = kernel_ms[0] / args.steps
    line = {
        "metric": METRIC, "value": round(value, 2), "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms_max / args.steps, 4), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": ours_config(wl.M, world),
        "roofline": roof,
        "rmsnorm_in_step": {"GB/s": round(wl.rms_bytes / rms_ms / 1e6, 1), "ms": round(rms_ms, 4),
                            "note": ("16 MiB in + 16 MiB out per launch, one event pair per launch inside the "
                                     "step: it includes the event gaps and the write-back of the previous step's "
                                     "matmul outputs (up to 96 MiB of dirty lines) that its reads evict from L2; "
                                     "the launch on its own is sweeps.rmsnorm_k4096 at M = 2048")},
        "slowdown_vs_noninvariant": round((ms_total / args.steps) / (ref_ms / args.steps), 3),
        "noninvariant_ms_per_step": round(ref_ms / args.steps, 4),
        "e2e": {"value": round(e2e_units / (e2e_max / 1e3) / 1e12, 2), "unit": "TFLOP/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "steps": e2e_steps,
                "overlap": "input copy, kernels and output copy on three streams, two device buffers of each"},
        "gpu_launches": gpu_launches,
        "clocks": clocks,
    }
    if world == 1 and not args.no_cpu:
        line["cpu_baseline"] = cpu_baseline(args.cpu_budget)
    if world == 1 and (args.rows or args.sweeps):
        del wl
        torch.cuda.empty_cache()
    if world == 1 and args.rows:
        line["rows"] = other_rows(bi, device, pk)
    if world == 1 and args.sweeps:
        line["sweeps"] = run_sweeps(bi, device, pk, (clocks or {}).get("sm_mhz"))
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1500)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--M", type=int, default=2048)
    ap.add_argument("--rows", dest="rows", action="store_true", default=True)
    ap.add_argument("--no-rows", dest="rows", action="store_false")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--sweeps", dest="sweeps", action="store_true", default=True,
                    help="add the matmul / RMSNorm / decode sweeps to the line (default on)")
    ap.add_argument("--no-sweeps", dest="sweeps", action="store_false")
    ap.add_argument("--sweep", action="store_true", help="only the sweeps, one JSON line per entry")
    ap.add_argument("--row", choices=["chain", "rmsnorm", "decode", "prefill", "lmhead", "reduce", "config5"], default=None,
                    help="measure only this hot-path kernel (for profiling) and print its line")
    ap.add_argument("--cpu-budget", type=float, default=10.0)
    ap.add_argument("--profile", choices=PROFILE_CASES, default=None,
                    help="run a few plain launches of one kernel case (for an ncu capture) and exit")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    rank, world, local = init_dist()
    try:
        if args.profile is not None:
            import invariant_deterministic_04_b200 as bi

            torch.cuda.set_device(local)
            profile_case(bi, torch.device("cuda", local), args.profile)
        elif args.sweep:
            import invariant_deterministic_04_b200 as bi

            torch.cuda.set_device(local)
            run_sweep(bi, torch.device("cuda", local), peaks())
        elif args.row is not None:
            import invariant_deterministic_04_b200 as bi

            torch.cuda.set_device(local)
            print(json.dumps({"row": args.row, **other_rows(bi, torch.device("cuda", local), peaks(), only=args.row)}))
        elif args.impl == "reference":
            run_reference(args, rank, world)
        else:
            run_ours(args, rank, world, local)
    finally:
        if world > 1 and dist.is_initialized():
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
