"""Random-init Llama-style decoder on the batch-invariant kernels, with a mixed-batch
greedy scheduler (test harness for the 1000-repeat determinism check).

Every operation of a step runs in libbi through the binding: row gather (embedding),
RMSNorm, the tcgen05 matmul, RoPE, KV append into the paged store, causal attention
over the store (prefill chunks and decode tokens in one call), SwiGLU, residual add
and the LM head with its selective FP32 recompute. Torch only provides memory.

``BaselineLlama`` runs the same weights through stock torch ops (cuBLAS matmuls,
F.rms_norm, padded batched attention, matmul + argmax LM head): the non-invariant
comparison path.
"""
from __future__ import annotations

import math
import time

import numpy as np
import torch

import invariant_deterministic_04_b200 as bi

PAGE = 16


def rope_cos_sin(max_pos: int, D: int, theta: float, device) -> torch.Tensor:
    """fp32 [max_pos, D/2, 2] table of (cos, sin) of pos * theta^(-2i/D), built in double."""
    half = D // 2
    inv = np.power(theta, -2.0 * np.arange(half) / D)
    ang = np.arange(max_pos, dtype=np.float64)[:, None] * inv[None, :]
    return torch.from_numpy(np.stack([np.cos(ang), np.sin(ang)], axis=-1).astype(np.float32)).to(device)


class PagedStore:
    """Per-layer K/V stores [num_pages, Hkv, 16, D] and one page-table row per sequence
    (pages of a sequence are a fixed, shuffled set of physical pages)."""

    def __init__(self, layers, n_seqs, max_pos, kv_heads, head_dim, device, seed=0):
        self.max_pages = math.ceil(max_pos / PAGE)
        n = n_seqs * self.max_pages
        perm = torch.randperm(n, generator=torch.Generator().manual_seed(seed)).to(torch.int32)
        self.page_table = perm.view(n_seqs, self.max_pages).contiguous().to(device)
        shape = (n, kv_heads, PAGE, head_dim)
        self.k = [torch.zeros(shape, dtype=torch.bfloat16, device=device) for _ in range(layers)]
        self.v = [torch.zeros(shape, dtype=torch.bfloat16, device=device) for _ in range(layers)]


class BiLlama:
    def __init__(self, cfg, weights, n_seqs, max_pos, device, threshold=0.5):
        self.cfg, self.w, self.device, self.threshold = cfg, weights, device, threshold
        self.store = PagedStore(cfg["layers"], n_seqs, max_pos, cfg["kv_heads"], cfg["head_dim"], device)
        self.table = rope_cos_sin(max_pos, cfg["head_dim"], cfg["theta"], device)
        self.recomputed = 0
        self.lm_rows = 0

    def hidden(self, seqs, poss, toks, n_layers=None):
        """Hidden rows after the first n_layers decoder layers (all by default)."""
        c, w, st, dev = self.cfg, self.w, self.store, self.device
        nh, nkv, D, H = c["heads"], c["kv_heads"], c["head_dim"], c["hidden"]
        T = len(toks)
        meta = torch.tensor(np.stack([seqs, poss, toks]).astype(np.int32)).pin_memory().to(dev, non_blocking=True)
        q_seq, q_pos, ids = meta[0], meta[1], meta[2]
        h = bi.gather_rows(w["embed"], ids)
        x = torch.empty_like(h)
        for l, lw in enumerate(w["layers"][:n_layers]):
            bi.rmsnorm(h, lw["attn_norm"], c["eps"], out=x)
            qkv = bi.matmul(x, lw["wqkv"])
            q = qkv[:, : nh * D].view(T, nh, D)
            k = qkv[:, nh * D: (nh + nkv) * D].view(T, nkv, D)
            v = qkv[:, (nh + nkv) * D:].view(T, nkv, D)
            bi.rope(q, q_pos, self.table)
            bi.rope(k, q_pos, self.table)
            bi.kv_append(k, v, q_seq, q_pos, st.k[l], st.v[l], st.page_table)
            att = bi.attention_prefill(q, q_seq, q_pos, st.k[l], st.v[l], st.page_table)
            o = bi.matmul(att.view(T, nh * D), lw["wo"])
            bi.add(h, o, out=h)
            bi.rmsnorm(h, lw["mlp_norm"], c["eps"], out=x)
            a = bi.swiglu(bi.matmul(x, lw["wgu"]))
            bi.add(h, bi.matmul(a, lw["wdown"]), out=h)
        return h

    def forward(self, seqs, poss, toks, want):
        """Rows (seqs[t], poss[t], toks[t]); returns greedy tokens for the row indices in `want`."""
        c, w, dev = self.cfg, self.w, self.device
        h = self.hidden(seqs, poss, toks)
        if not want:
            return np.zeros(0, dtype=np.int64)
        sel = torch.tensor(np.asarray(want, dtype=np.int32)).to(dev)
        hs = bi.rmsnorm(bi.gather_rows(h, sel), w["final_norm"], c["eps"])
        tok, rec, _ = bi.lmhead_argmax(hs, w["lm_head"], self.threshold)
        out = tok.cpu().numpy()
        self.recomputed += int(rec.sum())
        self.lm_rows += len(want)
        return out


class BaselineLlama(BiLlama):
    """Same weights and store, stock torch ops (the non-invariant path)."""

    def forward(self, seqs, poss, toks, want):
        c, w, st, dev = self.cfg, self.w, self.store, self.device
        nh, nkv, D, H = c["heads"], c["kv_heads"], c["head_dim"], c["hidden"]
        T = len(toks)
        q_seq = torch.tensor(np.asarray(seqs, dtype=np.int64), device=dev)
        q_pos = torch.tensor(np.asarray(poss, dtype=np.int64), device=dev)
        ids = torch.tensor(np.asarray(toks, dtype=np.int64), device=dev)
        cs = self.table[q_pos]  # [T, D/2, 2]
        cos, sin = cs[..., 0][:, None, :], cs[..., 1][:, None, :]

        def rot(t):
            a, b = t[..., : D // 2].float(), t[..., D // 2:].float()
            return torch.cat([a * cos - b * sin, b * cos + a * sin], -1).to(torch.bfloat16)

        maxlen = int(q_pos.max()) + 1
        span = torch.arange(maxlen, device=dev)
        pages = st.page_table[q_seq][:, span // PAGE].long()  # [T, maxlen]
        slot = (span % PAGE)[None, :].expand(T, maxlen)
        mask = (span[None, :] <= q_pos[:, None])
        h = torch.nn.functional.embedding(ids, w["embed"])
        for l, lw in enumerate(w["layers"]):
            x = torch.nn.functional.rms_norm(h, (H,), lw["attn_norm"], c["eps"])
            qkv = x @ lw["wqkv"].t()
            q = rot(qkv[:, : nh * D].view(T, nh, D))
            k = rot(qkv[:, nh * D: (nh + nkv) * D].view(T, nkv, D))
            v = qkv[:, (nh + nkv) * D:].view(T, nkv, D)
            pg = st.page_table[q_seq, q_pos // PAGE].long()
            st.k[l][pg, :, q_pos % PAGE] = k
            st.v[l][pg, :, q_pos % PAGE] = v
            K = st.k[l][pages, :, slot].repeat_interleave(nh // nkv, dim=2)  # [T, maxlen, nh, D]
            V = st.v[l][pages, :, slot].repeat_interleave(nh // nkv, dim=2)
            s = torch.einsum("thd,tjhd->thj", q, K) / math.sqrt(D)
            s = s.float().masked_fill(~mask[:, None, :], float("-inf"))
            p = torch.softmax(s, dim=-1).to(torch.bfloat16)
            att = torch.einsum("thj,tjhd->thd", p, V).reshape(T, nh * D)
            h = h + att @ lw["wo"].t()
            x = torch.nn.functional.rms_norm(h, (H,), lw["mlp_norm"], c["eps"])
            gu = x @ lw["wgu"].t()
            F = gu.shape[1] // 2
            h = h + (torch.nn.functional.silu(gu[:, :F]) * gu[:, F:]) @ lw["wdown"].t()
        if not want:
            return np.zeros(0, dtype=np.int64)
        hs = torch.nn.functional.rms_norm(h[torch.tensor(want, device=dev)], (H,), w["final_norm"], c["eps"])
        return torch.argmax(hs @ w["lm_head"].t(), dim=-1).cpu().numpy()


def run_schedule(model, prompts: np.ndarray, gen_len: int, seed: int, max_batch: int = 64, max_chunk: int = 128):
    """Greedy generation of gen_len tokens for every prompt under a random mixed batching.

    Each step draws a batch size ~ U[1, max_batch] and a random subset, in random order,
    of the unfinished sequences; a sequence still in its prompt contributes a random
    chunk of its remaining prompt (U[1, min(remaining, max_chunk)] tokens), one that is
    generating contributes its newest token. Returns (tokens [S, gen_len], steps, rows).
    """
    rng = np.random.default_rng(seed)
    S, P = prompts.shape
    done = np.zeros(S, dtype=np.int64)
    gen = [[] for _ in range(S)]
    steps = rows_total = 0
    while True:
        cand = [s for s in range(S) if len(gen[s]) < gen_len]
        if not cand:
            break
        b = int(rng.integers(1, max_batch + 1))
        pick = rng.permutation(cand)[:b]
        seqs, poss, toks, want, owner = [], [], [], [], []
        for s in pick:
            if done[s] < P:
                n = int(rng.integers(1, min(P - done[s], max_chunk) + 1))
                for i in range(n):
                    seqs.append(s)
                    poss.append(done[s] + i)
                    toks.append(prompts[s, done[s] + i])
                done[s] += n
                if done[s] == P:
                    want.append(len(toks) - 1)
                    owner.append(s)
            else:
                seqs.append(s)
                poss.append(P + len(gen[s]) - 1)
                toks.append(gen[s][-1])
                want.append(len(toks) - 1)
                owner.append(s)
        out = model.forward(seqs, poss, toks, want)
        for s, t in zip(owner, out):
            gen[s].append(int(t))
        steps += 1
        rows_total += len(toks)
    return np.array(gen, dtype=np.int64), steps, rows_total


def run_repeats(model_cls, cfg, weights, prompts, gen_len, repeats, device, seed0=0, **kw):
    """Run `repeats` schedules (seed seed0 + r); returns per-sequence unique-stream counts and stats."""
    S, P = prompts.shape
    seen = [dict() for _ in range(S)]
    first = None
    t_total = 0.0
    tokens = 0
    model = model_cls(cfg, weights, S, P + gen_len, device, **kw)
    for r in range(repeats):
        torch.cuda.synchronize()
        t0 = time.perf_counter()
        gen, steps, rows = run_schedule(model, prompts, gen_len, seed0 + r)
        torch.cuda.synchronize()
        t_total += time.perf_counter() - t0
        tokens += gen.size
        if first is None:
            first = gen
        for s in range(S):
            key = gen[s].tobytes()
            seen[s][key] = seen[s].get(key, 0) + 1
    uniq = np.array([len(d) for d in seen])
    return dict(unique_per_seq=uniq, max_unique=int(uniq.max()), first=first, tokens_per_s=tokens / t_total,
                seconds=t_total, recompute_rate=(model.recomputed / model.lm_rows) if model.lm_rows else None)
