"""Random-init Llama-style decoder on the batch-invariant kernels, with a mixed-batch
greedy scheduler: the model of the 1000-repeat determinism check and of the
config-5 benchmark row.

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


class FastBiLlama(BiLlama):
    """BiLlama with preallocated buffers and direct C-ABI calls (raw pointers, no
    per-call tensor checks): the same kernels and arguments, less host overhead."""

    def __init__(self, cfg, weights, n_seqs, max_pos, device, threshold=0.5, max_rows=8192, max_want=64):
        super().__init__(cfg, weights, n_seqs, max_pos, device, threshold)
        c = cfg
        H, nh, nkv, D, F, V = (c[k] for k in ("hidden", "heads", "kv_heads", "head_dim", "ffn", "vocab"))
        self.L = bi.lib()
        e = lambda *shape: torch.empty(shape, dtype=torch.bfloat16, device=device)
        self.h, self.x, self.o = e(max_rows, H), e(max_rows, H), e(max_rows, H)
        self.qkv, self.att = e(max_rows, (nh + 2 * nkv) * D), e(max_rows, nh * D)
        self.gu, self.a = e(max_rows, 2 * F), e(max_rows, F)
        self.meta = torch.empty((3, max_rows), dtype=torch.int32, device=device)
        # ring of pinned staging buffers; a buffer is refilled only after its last copy completed
        self.meta_host = [torch.empty((3, max_rows), dtype=torch.int32).pin_memory() for _ in range(4)]
        self.meta_ev = [torch.cuda.Event() for _ in range(4)]
        self.meta_i = 0
        self.sel = torch.empty(max_want, dtype=torch.int32, device=device)
        self.hs, self.hn = e(max_want, H), e(max_want, H)
        self.tok = torch.empty(max_want, dtype=torch.int32, device=device)
        self.rec = torch.empty(max_want, dtype=torch.int32, device=device)
        self.ws_att = torch.empty(bi.attention_workspace_size(max_rows, nh, D, self.store.max_pages),
                                  dtype=torch.uint8, device=device)
        self.ws_lm = torch.empty(bi.lmhead_workspace_size(max_want, V), dtype=torch.uint8, device=device)
        self.max_rows, self.max_want = max_rows, max_want

    def _ok(self, name, status):
        if status != 0:
            raise bi.BIError(name, status)

    def hidden(self, seqs, poss, toks, n_layers=None):
        c, w, st, L = self.cfg, self.w, self.store, self.L
        H, nh, nkv, D, F = (c[k] for k in ("hidden", "heads", "kv_heads", "head_dim", "ffn"))
        T = len(toks)
        assert T <= self.max_rows
        s = torch.cuda.current_stream().cuda_stream
        i = self.meta_i = (self.meta_i + 1) % len(self.meta_host)
        mh = self.meta_host[i]
        self.meta_ev[i].synchronize()
        mh[0, :T] = torch.from_numpy(np.asarray(seqs, dtype=np.int32))
        mh[1, :T] = torch.from_numpy(np.asarray(poss, dtype=np.int32))
        mh[2, :T] = torch.from_numpy(np.asarray(toks, dtype=np.int32))
        self.meta[:, :T].copy_(mh[:, :T], non_blocking=True)
        self.meta_ev[i].record()
        mp = self.meta.data_ptr()
        q_seq, q_pos, ids = mp, mp + 4 * self.max_rows, mp + 8 * self.max_rows
        QKV = (nh + 2 * nkv) * D
        h, x, o, qkv, att, gu, a = (t.data_ptr() for t in (self.h, self.x, self.o, self.qkv, self.att, self.gu, self.a))
        E = w["embed"]
        self._ok("gather", L.bi_gather_rows(E.data_ptr(), H, E.shape[0], ids, T, H, h, H, s))
        npages, maxp, pt = st.k[0].shape[0], st.max_pages, st.page_table.data_ptr()
        tab = self.table.data_ptr()
        scale = 1.0 / math.sqrt(D)
        ws, wsb = self.ws_att.data_ptr(), self.ws_att.numel()
        n_seqs = st.page_table.shape[0]
        for l, lw in enumerate(w["layers"][:n_layers]):
            kc, vc = st.k[l].data_ptr(), st.v[l].data_ptr()
            self._ok("rmsnorm", L.bi_rmsnorm(h, H, lw["attn_norm"].data_ptr(), x, H, T, H, c["eps"], s))
            self._ok("qkv", L.bi_matmul(x, H, lw["wqkv"].data_ptr(), H, qkv, QKV, T, QKV, H, s))
            self._ok("rope q", L.bi_rope(qkv, QKV, T, nh, D, q_pos, tab, self.table.shape[0], s))
            self._ok("rope k", L.bi_rope(qkv + 2 * nh * D, QKV, T, nkv, D, q_pos, tab, self.table.shape[0], s))
            self._ok("append", L.bi_kv_append(qkv + 2 * nh * D, qkv + 2 * (nh + nkv) * D, QKV, q_seq, q_pos, kc, vc,
                                              npages, pt, n_seqs, maxp, T, nkv, D, s))
            self._ok("attn", L.bi_attention_prefill(qkv, QKV, q_seq, q_pos, kc, vc, npages, pt, n_seqs, maxp, att, T,
                                                    nh, nkv, D, scale, ws, wsb, s))
            self._ok("o", L.bi_matmul(att, nh * D, lw["wo"].data_ptr(), nh * D, o, H, T, H, nh * D, s))
            self._ok("add", L.bi_add(h, o, h, T * H, s))
            self._ok("rmsnorm", L.bi_rmsnorm(h, H, lw["mlp_norm"].data_ptr(), x, H, T, H, c["eps"], s))
            self._ok("gu", L.bi_matmul(x, H, lw["wgu"].data_ptr(), H, gu, 2 * F, T, 2 * F, H, s))
            self._ok("swiglu", L.bi_swiglu(gu, 2 * F, a, F, T, F, s))
            self._ok("down", L.bi_matmul(a, F, lw["wdown"].data_ptr(), F, o, H, T, H, F, s))
            self._ok("add", L.bi_add(h, o, h, T * H, s))
        return self.h[:T]

    def forward(self, seqs, poss, toks, want):
        c, w, L = self.cfg, self.w, self.L
        H, V = c["hidden"], c["vocab"]
        self.hidden(seqs, poss, toks)
        n = len(want)
        if n == 0:
            return np.zeros(0, dtype=np.int64)
        s = torch.cuda.current_stream().cuda_stream
        self.sel[:n].copy_(torch.from_numpy(np.asarray(want, dtype=np.int32)), non_blocking=True)
        self._ok("select", L.bi_gather_rows(self.h.data_ptr(), H, len(toks), self.sel.data_ptr(), n, H,
                                            self.hs.data_ptr(), H, s))
        self._ok("final norm", L.bi_rmsnorm(self.hs.data_ptr(), H, w["final_norm"].data_ptr(), self.hn.data_ptr(), H,
                                            n, H, c["eps"], s))
        self._ok("lm head", L.bi_lmhead_argmax(self.hn.data_ptr(), H, w["lm_head"].data_ptr(), n, V, H, self.threshold,
                                               self.tok.data_ptr(), self.rec.data_ptr(), None,
                                               self.ws_lm.data_ptr(), self.ws_lm.numel(), s))
        out = self.tok[:n].cpu().numpy()
        self.recomputed += int(self.rec[:n].sum())
        self.lm_rows += n
        return out
