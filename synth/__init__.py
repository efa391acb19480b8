"""Seeded synthetic inputs for the batch-invariant kernels.

This module only draws random numbers and lays them out; it holds none of the
arithmetic of the operations under test. Both the CUDA-path tests/benchmark and
the fp64 oracle tests take their inputs from here, so the two sides see the same
bf16 bits.

Recipe (all on the CPU, ``torch.Generator`` seeded per call):
  * normals are drawn in fp32 and cast to bf16 with round-to-nearest-even;
  * RMSNorm: x ~ N(0, 1), weight = 1 + N(0, 0.1);
  * matmul: A ~ N(0, 1), W ~ N(0, 0.02), W stored [N, K] (nn.Linear layout);
  * attention: q, k, v ~ N(0, 1); K/V live in a paged store of 16-token pages
    ``[num_pages, Hkv, 16, D]``; each sequence's logical pages map to a seeded
    random permutation of the physical pages; page-table entries past a
    sequence's last page are -1; decode lengths ~ U[1, max_len];
  * LM head: h ~ N(0, 1), W ~ N(0, 0.02) stored [V, K];
  * logits for log_softmax / sampling: N(0, 3^2) bf16 rows (the spread of a
    trained LM head's logits); row means: x ~ N(0.5, 1);
  * request seeds: uniform 64-bit words; decode steps: small integers.
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import numpy as np
import torch

PAGE = 16  # tokens per KV page


def generator(seed: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    return g


def normal_bf16(shape, seed: int, std: float = 1.0, mean: float = 0.0) -> torch.Tensor:
    """fp32 N(mean, std^2) draws cast to bf16 (round to nearest even)."""
    x = torch.randn(tuple(shape), generator=generator(seed), dtype=torch.float32)
    if std != 1.0:
        x = x * std
    if mean != 0.0:
        x = x + mean
    return x.to(torch.bfloat16)


def to_f64(t: torch.Tensor) -> np.ndarray:
    """Exact widening of a bf16 (or fp32) tensor to a float64 numpy array."""
    return t.detach().to("cpu").to(torch.float64).numpy()


# ---------------------------------------------------------------------------
# RMSNorm / matmul


def rmsnorm_inputs(M: int, K: int, seed: int = 0):
    x = normal_bf16((M, K), seed)
    w = normal_bf16((K,), seed + 1, std=0.1, mean=1.0)
    return x, w


def matmul_inputs(M: int, N: int, K: int, seed: int = 0):
    a = normal_bf16((M, K), seed)
    w = normal_bf16((N, K), seed + 1, std=0.02)
    return a, w


# ---------------------------------------------------------------------------
# Paged KV store


@dataclass
class PagedKV:
    k_cache: torch.Tensor  # bf16 [num_pages, Hkv, PAGE, D]
    v_cache: torch.Tensor  # bf16 [num_pages, Hkv, PAGE, D]
    page_table: torch.Tensor  # int32 [num_seqs, max_pages]; -1 past the last page
    seq_lens: torch.Tensor  # int32 [num_seqs]
    max_pages: int

    @property
    def num_pages(self) -> int:
        return int(self.k_cache.shape[0])


def decode_lengths(B: int, max_len: int, seed: int) -> torch.Tensor:
    """Per-sequence KV lengths ~ U[1, max_len] (inclusive)."""
    return torch.randint(1, max_len + 1, (B,), generator=generator(seed), dtype=torch.int64).to(torch.int32)


def paged_kv(seq_lens, Hkv: int, D: int, seed: int = 0, max_pages: int | None = None,
             spare_pages: int = 3, poison_tail: bool = True) -> PagedKV:
    """Random K/V for the given lengths, scattered over a shuffled page pool.

    ``poison_tail`` writes NaN into the slots of each sequence's last page that
    lie past its length (and into the spare pages), the way a reused page of a
    real cache holds stale data; a kernel must never read them into a result.
    """
    lens = [int(v) for v in (seq_lens.tolist() if torch.is_tensor(seq_lens) else seq_lens)]
    B = len(lens)
    npages_seq = [math.ceil(L / PAGE) for L in lens]
    if max_pages is None:
        max_pages = max(npages_seq + [1])
    assert all(n <= max_pages for n in npages_seq)
    total = sum(npages_seq) + spare_pages
    k = normal_bf16((total, Hkv, PAGE, D), seed)
    v = normal_bf16((total, Hkv, PAGE, D), seed + 1)
    perm = torch.randperm(total, generator=generator(seed + 2)).to(torch.int32)
    pt = torch.full((B, max_pages), -1, dtype=torch.int32)
    pos = 0
    for b, n in enumerate(npages_seq):
        pt[b, :n] = perm[pos:pos + n]
        pos += n
    if poison_tail:
        nan = torch.tensor(float("nan"), dtype=torch.bfloat16)
        for b, L in enumerate(lens):
            if L % PAGE:
                p = int(pt[b, (L - 1) // PAGE])
                k[p, :, L % PAGE:, :] = nan
                v[p, :, L % PAGE:, :] = nan
        for p in perm[pos:].tolist():
            k[p] = nan
            v[p] = nan
    return PagedKV(k, v, pt, torch.tensor(lens, dtype=torch.int32), max_pages)


def decode_inputs(B: int, Hq: int, Hkv: int, D: int, max_len: int, seed: int = 0,
                  lens=None, poison_tail: bool = True):
    if lens is None:
        lens = decode_lengths(B, max_len, seed + 10)
    kv = paged_kv(lens, Hkv, D, seed=seed + 20, max_pages=math.ceil(max_len / PAGE),
                  poison_tail=poison_tail)
    q = normal_bf16((B, Hq, D), seed + 30)
    return q, kv


def prefill_inputs(seq_lens, Hq: int, Hkv: int, D: int, seed: int = 0, max_len: int | None = None):
    """Queries for every position of every sequence, plus its (seq, pos) tags.

    Rows are ordered sequence by sequence, position ascending.
    """
    lens = [int(v) for v in seq_lens]
    max_pages = math.ceil((max_len or max(lens)) / PAGE)
    kv = paged_kv(lens, Hkv, D, seed=seed + 20, max_pages=max_pages, poison_tail=True)
    T = sum(lens)
    q = normal_bf16((T, Hq, D), seed + 30)
    q_seq = torch.cat([torch.full((L,), b, dtype=torch.int32) for b, L in enumerate(lens)])
    q_pos = torch.cat([torch.arange(L, dtype=torch.int32) for L in lens])
    return q, q_seq, q_pos, kv


# ---------------------------------------------------------------------------
# LM head


def lmhead_inputs(M: int, V: int, K: int, seed: int = 0):
    h = normal_bf16((M, K), seed)
    w = normal_bf16((V, K), seed + 1, std=0.02)
    return h, w


def lmhead_planted(M: int, V: int, K: int, seed: int, ties: int):
    """LM-head inputs with a trained-model-like margin structure: W ~ N(0, 0.02) [V, K];
    row m of h is N(0, 1) plus 40 times the weight row of a seeded target token, so that
    token's logit stands far above the rest; each of the first `ties` rows is instead
    20 * (w_a / |w_a|^2 + w_b / |w_b|^2) for two targets a, b (no noise), so logits a and
    b are both about 20 and nearly tied at the top."""
    W = normal_bf16((V, K), seed, std=0.02)
    g = generator(seed + 1)
    tgt = torch.randint(0, V, (M, 2), generator=g)
    h = torch.randn((M, K), generator=g, dtype=torch.float32)
    Wf = W.float()
    for m in range(M):
        if m < ties:
            wa, wb = Wf[tgt[m, 0]], Wf[tgt[m, 1]]
            h[m] = 20.0 * (wa / wa.dot(wa) + wb / wb.dot(wb))
        else:
            h[m] += 40.0 * Wf[tgt[m, 0]]
    return h.to(torch.bfloat16), W


def logits(M: int, V: int, seed: int = 0, std: float = 3.0) -> torch.Tensor:
    """bf16 [M, V] logit rows ~ N(0, std^2)."""
    return normal_bf16((M, V), seed, std=std)


def request_seeds(M: int, seed: int) -> torch.Tensor:
    """[M] int64 tensor holding uniform 64-bit words (the bits of uint64 request seeds)."""
    g = generator(seed)
    hi = torch.randint(0, 2**32, (M,), generator=g, dtype=torch.int64)
    lo = torch.randint(0, 2**32, (M,), generator=g, dtype=torch.int64)
    return (hi << 32) | lo


def permutation(n: int, seed: int) -> torch.Tensor:
    return torch.randperm(n, generator=generator(seed))


# ---------------------------------------------------------------------------
# Full-size paged stores, generated on the GPU from a seed (the CPU generator
# would take minutes for tens of GB). Same recipe as paged_kv.


def _device_normal_bf16(shape, gen, device, chunk_elems=1 << 28):
    out = torch.empty(shape, dtype=torch.bfloat16, device=device)
    flat = out.view(-1)
    for s in range(0, flat.numel(), chunk_elems):
        e = min(flat.numel(), s + chunk_elems)
        flat[s:e] = torch.randn(e - s, generator=gen, device=device, dtype=torch.float32).to(torch.bfloat16)
    return out


def normal_bf16_device(shape, seed: int, device, std: float = 1.0, mean: float = 0.0) -> torch.Tensor:
    """Seeded N(mean, std^2) bf16 draws made on the device (for inputs of several GB,
    too slow to draw on the host). Same distribution as normal_bf16, other values."""
    gen = torch.Generator(device=device)
    gen.manual_seed(int(seed))
    x = _device_normal_bf16(shape, gen, device)
    if std != 1.0 or mean != 0.0:
        x = (x.float() * std + mean).to(torch.bfloat16)
    return x


def paged_kv_device(seq_lens, Hkv: int, D: int, seed: int, max_pages: int, device, spare_pages: int = 1) -> PagedKV:
    lens = [int(v) for v in (seq_lens.tolist() if torch.is_tensor(seq_lens) else seq_lens)]
    B = len(lens)
    npages_seq = [math.ceil(L / PAGE) for L in lens]
    total = sum(npages_seq) + spare_pages
    gen = torch.Generator(device=device)
    gen.manual_seed(int(seed))
    k = _device_normal_bf16((total, Hkv, PAGE, D), gen, device)
    v = _device_normal_bf16((total, Hkv, PAGE, D), gen, device)
    perm = torch.randperm(total, generator=generator(seed + 2)).to(torch.int32)
    pt = torch.full((B, max_pages), -1, dtype=torch.int32)
    pos = 0
    for b, n in enumerate(npages_seq):
        pt[b, :n] = perm[pos:pos + n]
        pos += n
    # stale data past each sequence's length and in the spare pages
    nan = float("nan")
    tails = [(int(pt[b, (L - 1) // PAGE]), L % PAGE) for b, L in enumerate(lens) if L % PAGE]
    for p, s in tails:
        k[p, :, s:, :] = nan
        v[p, :, s:, :] = nan
    for p in perm[pos:].tolist():
        k[p] = nan
        v[p] = nan
    return PagedKV(k, v, pt.to(device), torch.tensor(lens, dtype=torch.int32, device=device), max_pages)


def sequence_pages(kv: PagedKV, b: int, L: int):
    """CPU copy of one sequence's pages as a private store (pages renumbered 0..n-1)."""
    n = math.ceil(L / PAGE)
    pages = kv.page_table[b, :n].to(torch.int64)
    k = kv.k_cache[pages].cpu()
    v = kv.v_cache[pages].cpu()
    return k, v, torch.arange(n, dtype=torch.int32).view(1, n)


# ---------------------------------------------------------------------------
# Random-init Llama-style decoder weights and prompts (drawn on the GPU from a
# seed; N(0, 0.02) for every matrix, norm weights 1, no biases).


LLAMA_CFG = dict(layers=16, hidden=2048, heads=32, kv_heads=8, head_dim=64, ffn=8192, vocab=32000, eps=1e-6,
                 theta=10000.0)


def llama_weights(cfg: dict, seed: int, device):
    gen = torch.Generator(device=device)
    gen.manual_seed(int(seed))
    H, nh, nkv, D, F, V = (cfg[k] for k in ("hidden", "heads", "kv_heads", "head_dim", "ffn", "vocab"))

    def nrm(shape):
        return _device_normal_bf16(shape, gen, device).mul_(0.02)

    ones = lambda n: torch.ones(n, dtype=torch.bfloat16, device=device)
    layers = [dict(wqkv=nrm(((nh + 2 * nkv) * D, H)), wo=nrm((H, nh * D)), wgu=nrm((2 * F, H)), wdown=nrm((H, F)),
                   attn_norm=ones(H), mlp_norm=ones(H)) for _ in range(cfg["layers"])]
    return dict(embed=nrm((V, H)), layers=layers, final_norm=ones(H), lm_head=nrm((V, H)))


def prompts(n: int, length: int, vocab: int, seed: int) -> np.ndarray:
    """n prompts of `length` token ids ~ U[0, vocab)."""
    return torch.randint(0, vocab, (n, length), generator=generator(seed), dtype=torch.int64).numpy()
