"""Selective determinism by verify and rollback, on the config-5 random Llama.

Source: French "température zéro" blog, section "Vous n'avez pas à le payer partout":
LLM-42 keeps a fast nondeterministic path and enforces determinism with a light
verify-and-rollback loop that re-uses existing kernels, so only the traffic that
needs determinism pays; the verifier recomputes what must be certified and rolls
back where it disagrees.

Here:
* the fast path (``FastPathLlama``) is stock-library decoding — cuBLAS matmuls,
  F.rms_norm and flashinfer's paged decode attention with its own split heuristic —
  run under a load-dependent batch composition, so its numerics drift with the load;
* every request proposes ``window`` tokens per round on the fast path;
* for a certified request the batch-invariant path re-runs the window as one
  prefill chunk (the last committed token and the first window-1 proposals, at
  their positions) and yields the invariant next token at every position; the
  longest agreeing prefix is accepted, and at the first disagreement the invariant
  token is committed and the rest of the window is dropped (rollback). K/V written
  for dropped positions are overwritten later and never read before that, since a
  row only reads keys at or before its own position;
* requests that are not certified keep the fast path's tokens.

Because the invariant prefill of a row equals the invariant decode of that row bit
for bit (batch invariance plus decode == prefill), a certified stream is exactly the
stream of pure invariant greedy decoding, whatever the fast path proposed.
"""
from __future__ import annotations

import time

import numpy as np
import torch

from .llama import PAGE, BaselineLlama, FastBiLlama


class FastPathLlama(BaselineLlama):
    """The nondeterministic fast path: stock torch / cuBLAS / flashinfer kernels."""

    def __init__(self, cfg, weights, n_seqs, max_pos, device, **kw):
        super().__init__(cfg, weights, n_seqs, max_pos, device)
        import flashinfer

        self.fws = torch.empty(256 << 20, dtype=torch.uint8, device=device)
        self.dec = flashinfer.BatchDecodeWithPagedKVCacheWrapper(self.fws, kv_layout="HND")
        self.pt_host = self.store.page_table.cpu()

    def decode(self, seqs, poss, toks):
        """One token per row (rows are distinct sequences); returns the greedy next tokens."""
        c, w, st, dev = self.cfg, self.w, self.store, self.device
        nh, nkv, D, H = c["heads"], c["kv_heads"], c["head_dim"], c["hidden"]
        T = len(toks)
        q_seq = torch.tensor(np.asarray(seqs, dtype=np.int64), device=dev)
        q_pos = torch.tensor(np.asarray(poss, dtype=np.int64), device=dev)
        ids = torch.tensor(np.asarray(toks, dtype=np.int64), device=dev)
        cs = self.table[q_pos]
        cos, sin = cs[..., 0][:, None, :], cs[..., 1][:, None, :]

        def rot(t):
            a, b = t[..., : D // 2].float(), t[..., D // 2:].float()
            return torch.cat([a * cos - b * sin, b * cos + a * sin], -1).to(torch.bfloat16)

        npages = [p // PAGE + 1 for p in poss]
        pt = self.pt_host
        indptr = torch.tensor([0] + list(np.cumsum(npages)), dtype=torch.int32, device=dev)
        indices = torch.cat([pt[s, :n] for s, n in zip(seqs, npages)]).to(dev)
        last = torch.tensor([p % PAGE + 1 for p in poss], dtype=torch.int32, device=dev)
        self.dec.plan(indptr, indices, last, nh, nkv, D, PAGE, q_data_type=torch.bfloat16,
                      kv_data_type=torch.bfloat16)
        pg = st.page_table[q_seq, q_pos // PAGE].long()
        h = torch.nn.functional.embedding(ids, w["embed"])
        for l, lw in enumerate(w["layers"]):
            x = torch.nn.functional.rms_norm(h, (H,), lw["attn_norm"], c["eps"])
            qkv = x @ lw["wqkv"].t()
            q = rot(qkv[:, : nh * D].view(T, nh, D))
            st.k[l][pg, :, q_pos % PAGE] = rot(qkv[:, nh * D: (nh + nkv) * D].view(T, nkv, D))
            st.v[l][pg, :, q_pos % PAGE] = qkv[:, (nh + nkv) * D:].view(T, nkv, D)
            att = self.dec.run(q.contiguous(), (st.k[l], st.v[l])).reshape(T, nh * D)
            h = h + att @ lw["wo"].t()
            x = torch.nn.functional.rms_norm(h, (H,), lw["mlp_norm"], c["eps"])
            gu = x @ lw["wgu"].t()
            F = gu.shape[1] // 2
            h = h + (torch.nn.functional.silu(gu[:, :F]) * gu[:, F:]) @ lw["wdown"].t()
        hs = torch.nn.functional.rms_norm(h, (H,), w["final_norm"], c["eps"])
        return torch.argmax(hs @ w["lm_head"].t(), dim=-1).cpu().numpy()


def generate(fast: FastPathLlama, inv: FastBiLlama | None, prompts: np.ndarray, gen_len: int,
             certified: np.ndarray, window: int, seed: int):
    """Verify-and-rollback generation. Returns (streams [S, gen_len], stats).

    The fast path decodes with a load-dependent batch composition (each round the
    active requests are shuffled and cut into random sub-batches).
    """
    rng = np.random.default_rng(seed)
    S, P = prompts.shape
    cert = np.flatnonzero(certified)
    # prompts: the fast path prefills every request; the invariant path the certified ones
    rows = [(s, p, prompts[s, p]) for s in range(S) for p in range(P)]
    want = [s * P + P - 1 for s in range(S)]
    first_fast = fast.forward([r[0] for r in rows], [r[1] for r in rows], [r[2] for r in rows], want)
    gen = [[int(first_fast[s])] for s in range(S)]
    if len(cert):
        crow = [(s, p, prompts[s, p]) for s in cert for p in range(P)]
        first_inv = inv.forward([r[0] for r in crow], [r[1] for r in crow], [r[2] for r in crow],
                                [i * P + P - 1 for i in range(len(cert))])
        for s, t in zip(cert, first_inv):
            gen[s][0] = int(t)
    stats = dict(proposed=0, accepted=0, rolled_back=0, verify_rows=0, fast_rows=0, rounds=0)
    while True:
        active = [s for s in range(S) if len(gen[s]) < gen_len]
        if not active:
            break
        stats["rounds"] += 1
        base = {s: len(gen[s]) for s in active}
        k = {s: min(window, gen_len - base[s]) for s in active}
        prop = {s: [] for s in active}
        for j in range(max(k.values())):
            todo = [s for s in active if j < k[s]]
            order = rng.permutation(todo)
            cuts = np.sort(rng.choice(np.arange(1, len(order)), size=min(len(order) - 1, int(rng.integers(0, 4))),
                                      replace=False)) if len(order) > 1 else []
            for part in np.split(order, cuts):
                if len(part) == 0:
                    continue
                seqs = [int(s) for s in part]
                poss = [P + base[s] + j - 1 for s in seqs]
                toks = [prop[s][-1] if j else gen[s][-1] for s in seqs]
                out = fast.decode(seqs, poss, toks)
                stats["fast_rows"] += len(seqs)
                for s, t in zip(seqs, out):
                    prop[s].append(int(t))
        vs = [s for s in active if certified[s]]
        if vs:
            seqs, poss, toks, want = [], [], [], []
            for s in vs:
                inputs = [gen[s][-1]] + prop[s][: k[s] - 1]
                for j, t in enumerate(inputs):
                    seqs.append(s)
                    poss.append(P + base[s] - 1 + j)
                    toks.append(t)
                    want.append(len(toks) - 1)
            ref = inv.forward(seqs, poss, toks, want)
            stats["verify_rows"] += len(toks)
            i = 0
            for s in vs:
                a = [int(t) for t in ref[i: i + k[s]]]
                i += k[s]
                n = 0
                while n < k[s] and prop[s][n] == a[n]:
                    n += 1
                stats["proposed"] += k[s]
                stats["accepted"] += n
                if n < k[s]:
                    stats["rolled_back"] += 1
                    gen[s].extend(a[: n + 1])   # agreeing prefix, then the invariant token
                else:
                    gen[s].extend(a)
        for s in active:
            if not certified[s]:
                gen[s].extend(prop[s])
    return np.array(gen, dtype=np.int64), stats


def timed_generate(*args, **kw):
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    out = generate(*args, **kw)
    torch.cuda.synchronize()
    return out, time.perf_counter() - t0
