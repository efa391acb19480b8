"""Python binding of libbi, the batch-invariant forward-pass kernels for B200.

Argument marshalling only: every step of every operation runs in the CUDA
kernels behind the C ABI declared in include/bi.h. PyTorch provides device
memory and the current stream. There is no CPU or library fallback: if
libbi.so is missing or fails to load, every call raises ``BIError``.

Operations (see include/bi.h for the exact contracts):
  rmsnorm, matmul, matmul_multi, matmul_tile_n, matmul_tile_m, attention_decode, attention_decode_static, attention_prefill,
  kv_append, lmhead_argmax, gather_rows, rope, swiglu, add, log_softmax,
  token_logprob, row_mean, sampling_uniforms, sample, get_device_error.
"""
from __future__ import annotations

import contextlib
import ctypes
import math
import os

import torch

from ._build import LIB_PATH, build_library  # noqa: F401

PAGE_TOKENS = 16
KV_SPLIT = 256

_STATUS = {
    0: "BI_OK", 1: "BI_ERR_NULL", 2: "BI_ERR_SHAPE", 3: "BI_ERR_ALIGN", 4: "BI_ERR_WORKSPACE",
    5: "BI_ERR_UNSUPPORTED", 6: "BI_ERR_CUDA", 7: "BI_ERR_DEVICE_TIMEOUT", 8: "BI_ERR_DEVICE_INDEX",
}


class BIError(RuntimeError):
    def __init__(self, where: str, status: int):
        self.status = status
        super().__init__(f"{where}: {_STATUS.get(status, status)}")


_P, _I64, _I32, _F, _SZ = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_float, ctypes.c_size_t

_SIGNATURES = {
    "bi_status_string": ([_I32], ctypes.c_char_p),
    "bi_version": ([], _I32),
    "bi_rmsnorm": ([_P, _I64, _P, _P, _I64, _I64, _I64, _F, _P], _I32),
    "bi_matmul": ([_P, _I64, _P, _I64, _P, _I64, _I64, _I64, _I64, _P], _I32),
    "bi_matmul_multi": ([_P, _I64, _I32, _P, _P, _P, _P, _P, _I64, _I64, _P], _I32),
    "bi_matmul_tile_n": ([_I64, _I64], _I32),
    "bi_matmul_tile_m": ([_I64, _I64], _I32),
    "bi_attention_workspace_size": ([_I64, _I32, _I32, _I32], _SZ),
    "bi_attention_decode": ([_P, _P, _P, _I64, _P, _I32, _P, _P, _I32, _I32, _I32, _I32, _F, _P, _SZ, _P], _I32),
    "bi_attention_decode_static": ([_P, _P, _P, _I64, _P, _I32, _P, _P, _I32, _I32, _I32, _I32, _F, _P], _I32),
    "bi_attention_prefill": ([_P, _I64, _P, _P, _P, _P, _I64, _P, _I32, _I32, _P, _I32, _I32, _I32, _I32, _F, _P, _SZ,
                              _P], _I32),
    "bi_attention_prefill_tc": ([_P, _I64, _I32, _I32, _I32, _P, _P, _I64, _P, _I32, _I32, _P, _I32, _I32, _I32, _F,
                                 _P], _I32),
    "bi_kv_append": ([_P, _P, _I64, _P, _P, _P, _P, _I64, _P, _I32, _I32, _I32, _I32, _I32, _P], _I32),
    "bi_gather_rows": ([_P, _I64, _I64, _P, _I64, _I64, _P, _I64, _P], _I32),
    "bi_rope": ([_P, _I64, _I64, _I32, _I32, _P, _P, _I32, _P], _I32),
    "bi_swiglu": ([_P, _I64, _P, _I64, _I64, _I64, _P], _I32),
    "bi_add": ([_P, _P, _P, _I64, _P], _I32),
    "bi_lmhead_workspace_size": ([_I64, _I64], _SZ),
    "bi_lmhead_argmax": ([_P, _I64, _P, _I64, _I64, _I64, _F, _P, _P, _P, _P, _SZ, _P], _I32),
    "bi_log_softmax": ([_P, _I64, _P, _I64, _I64, _I64, _P], _I32),
    "bi_token_logprob": ([_P, _I64, _P, _P, _I64, _I64, _P], _I32),
    "bi_row_mean": ([_P, _I64, _P, _I64, _I64, _P], _I32),
    "bi_sampling_uniforms": ([_P, _P, _P, _I64, _I64, _I64, _P], _I32),
    "bi_sample": ([_P, _I64, _P, _P, _F, _P, _I64, _I64, _P], _I32),
    "bi_get_device_error": ([ctypes.POINTER(ctypes.c_int32)], _I32),
    "bi_selftest_wait_timeout": ([_I32, _P], _I32),
}

_lib = None
_load_error = None


def lib() -> ctypes.CDLL:
    """The loaded libbi.so (raises BIError-like RuntimeError if it cannot be loaded)."""
    global _lib, _load_error
    if _lib is not None:
        return _lib
    if _load_error is None:
        if not os.path.exists(LIB_PATH):
            _load_error = f"{LIB_PATH} is missing; build it with __graft_entry__.build() (nvcc, sm_100a)"
        else:
            try:
                handle = ctypes.CDLL(LIB_PATH)
                for name, (args, ret) in _SIGNATURES.items():
                    fn = getattr(handle, name)
                    fn.argtypes, fn.restype = args, ret
                _lib = handle
                return _lib
            except OSError as e:  # pragma: no cover
                _load_error = f"cannot load {LIB_PATH}: {e}"
    raise RuntimeError(_load_error)


def _check(where: str, status: int):
    if status != 0:
        raise BIError(where, status)


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


@contextlib.contextmanager
def _on(device, stream):
    """Launch context: the tensors' device, and the caller's stream if one was given.

    Under it, temporaries (workspace, outputs) are allocated on the stream the
    kernels run on, so the caching allocator cannot hand their memory to other
    work before those kernels are done with it. A stream of another device is
    refused (its kernels would get this device's pointers)."""
    if stream is not None and getattr(stream, "device", device) != device:
        raise ValueError(f"stream is on {stream.device}, the tensors on {device}")
    with torch.cuda.device(device):
        if stream is None:
            yield
        else:
            with torch.cuda.stream(stream):
                yield


def _same_device(first: torch.Tensor, *others):
    """The device of `first`; every other tensor given (None entries skipped) must be on it."""
    d = first.device
    for t in others:
        if t is not None and t.device != d:
            raise ValueError(f"all tensors must be on {d}; got one on {t.device}")
    return d


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _req(t: torch.Tensor, dtype, name: str, dims: int | None = None):
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if dims is not None and t.dim() != dims:
        raise ValueError(f"{name} must have {dims} dims, got {tuple(t.shape)}")


def _contig(t: torch.Tensor, name: str):
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _out(t: torch.Tensor, dtype, shape, name: str, strided_rows: bool = False):
    """Check a caller-supplied output (the C calls write exactly `shape` through its
    pointer, and a row stride where they take one): dtype, shape, and contiguous
    storage, or contiguous rows (unit inner stride) when `strided_rows`."""
    _req(t, dtype, name, len(shape))
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    if strided_rows:
        if t.stride(-1) != 1:
            raise ValueError(f"{name} rows must be contiguous")
    else:
        _contig(t, name)
    return t


# ---------------------------------------------------------------------------


def rmsnorm(x: torch.Tensor, w: torch.Tensor, eps: float = 1e-6, out: torch.Tensor | None = None, stream=None):
    """y = bf16(x * rsqrt(mean(x^2) + eps) * w), one fixed reduction order per row."""
    _req(x, torch.bfloat16, "x", 2)
    _req(w, torch.bfloat16, "w", 1)
    _contig(w, "w")
    if x.stride(1) != 1:
        raise ValueError("x rows must be contiguous")
    M, K = x.shape
    device = _same_device(x, w, out)
    if out is not None:
        _out(out, torch.bfloat16, (M, K), "out", strided_rows=True)
    with _on(device, stream):
        y = torch.empty_like(x, memory_format=torch.contiguous_format) if out is None else out
        _check("bi_rmsnorm", lib().bi_rmsnorm(_ptr(x), x.stride(0), _ptr(w), _ptr(y), y.stride(0), M, K, eps,
                                             _stream()))
    return y


def matmul(a: torch.Tensor, w: torch.Tensor, out: torch.Tensor | None = None, stream=None):
    """C = A W^T with A [M, K], W [N, K] (nn.Linear layout), bf16 out; every element is one
    ascending-k chain of tcgen05 MMAs, the same for every M."""
    _req(a, torch.bfloat16, "a", 2)
    _req(w, torch.bfloat16, "w", 2)
    if a.stride(1) != 1 or w.stride(1) != 1:
        raise ValueError("a and w rows must be contiguous")
    M, K = a.shape
    N = w.shape[0]
    if w.shape[1] != K:
        raise ValueError(f"inner dimensions differ: {tuple(a.shape)} x {tuple(w.shape)}^T")
    device = _same_device(a, w, out)
    if out is not None:
        _out(out, torch.bfloat16, (M, N), "out", strided_rows=True)
    with _on(device, stream):
        c = torch.empty((M, N), dtype=torch.bfloat16, device=device) if out is None else out
        _check("bi_matmul", lib().bi_matmul(_ptr(a), a.stride(0), _ptr(w), w.stride(0), _ptr(c), c.stride(0), M, N,
                                           K, _stream()))
    return c


MATMUL_MULTI_MAX = 3


def matmul_multi(a: torch.Tensor, ws, outs=None, stream=None):
    """[A W_g^T for each W_g in ws] in one call (at most MATMUL_MULTI_MAX products), each
    bit-identical to matmul(a, W_g); one launch when every product runs on CTA-pair tiles."""
    ws = list(ws)
    if not 1 <= len(ws) <= MATMUL_MULTI_MAX:
        raise ValueError(f"between 1 and {MATMUL_MULTI_MAX} weight matrices, got {len(ws)}")
    _req(a, torch.bfloat16, "a", 2)
    if a.stride(1) != 1:
        raise ValueError("a rows must be contiguous")
    M, K = a.shape
    for g, w in enumerate(ws):
        _req(w, torch.bfloat16, f"ws[{g}]", 2)
        if w.stride(1) != 1:
            raise ValueError(f"ws[{g}] rows must be contiguous")
        if w.shape[1] != K:
            raise ValueError(f"inner dimensions differ: {tuple(a.shape)} x {tuple(w.shape)}^T")
    if outs is not None:
        outs = list(outs)
        if len(outs) != len(ws):
            raise ValueError(f"{len(ws)} weight matrices but {len(outs)} outputs")
        for g, (w, c) in enumerate(zip(ws, outs)):
            _out(c, torch.bfloat16, (M, w.shape[0]), f"outs[{g}]", strided_rows=True)
    device = _same_device(a, *ws, *(outs or []))
    n = len(ws)
    with _on(device, stream):
        cs = [torch.empty((M, w.shape[0]), dtype=torch.bfloat16, device=device) for w in ws] if outs is None else outs
        wp = (ctypes.c_void_p * n)(*[w.data_ptr() for w in ws])
        cp = (ctypes.c_void_p * n)(*[c.data_ptr() for c in cs])
        ldw = (ctypes.c_int64 * n)(*[w.stride(0) for w in ws])
        ldc = (ctypes.c_int64 * n)(*[c.stride(0) for c in cs])
        ns = (ctypes.c_int64 * n)(*[w.shape[0] for w in ws])
        _check("bi_matmul_multi", lib().bi_matmul_multi(_ptr(a), a.stride(0), n, wp, ldw, cp, ldc, ns, M, K,
                                                         _stream()))
    return cs


def matmul_tile_n(M: int, N: int) -> int:
    """Tile width bi_matmul uses for an M x N product on the current device (a
    scheduling choice; it does not enter the arithmetic of an element)."""
    w = int(lib().bi_matmul_tile_n(M, N))
    if w < 0:
        raise RuntimeError("bi_matmul_tile_n: device query failed")
    return w


def matmul_tile_m(M: int, N: int) -> int:
    """Tile rows bi_matmul uses for an M x N product on the current device: 128 (one
    CTA per tile) or 256 (a pair of CTAs per tile); a scheduling choice like the width."""
    r = int(lib().bi_matmul_tile_m(M, N))
    if r < 0:
        raise RuntimeError("bi_matmul_tile_m: device query failed")
    return r


def attention_workspace_size(rows: int, Hq: int, D: int, max_pages_per_seq: int) -> int:
    return int(lib().bi_attention_workspace_size(rows, Hq, D, max_pages_per_seq))


def _check_workspace(workspace):
    """A caller-supplied workspace: any dtype, CUDA, contiguous (its byte size is what counts)."""
    if workspace is not None:
        if not isinstance(workspace, torch.Tensor) or not workspace.is_cuda:
            raise TypeError("workspace must be a CUDA tensor")
        _contig(workspace, "workspace")


def _workspace(nbytes: int, device, workspace):
    """(tensor, bytes): the caller's workspace, else a fresh one (call under _on)."""
    if workspace is not None:
        return workspace, workspace.numel() * workspace.element_size()
    return torch.empty(max(nbytes, 1), dtype=torch.uint8, device=device), nbytes


def attention_decode(q, k_cache, v_cache, page_table, seq_lens, scale: float | None = None, out=None,
                     workspace=None, stream=None):
    """Decode attention over the paged store; q [B, Hq, D] -> out [B, Hq, D]."""
    _req(q, torch.bfloat16, "q", 3)
    _req(k_cache, torch.bfloat16, "k_cache", 4)
    _req(v_cache, torch.bfloat16, "v_cache", 4)
    _req(page_table, torch.int32, "page_table", 2)
    _req(seq_lens, torch.int32, "seq_lens", 1)
    for t, n in ((q, "q"), (k_cache, "k_cache"), (v_cache, "v_cache"), (page_table, "page_table"),
                 (seq_lens, "seq_lens")):
        _contig(t, n)
    B, Hq, D = q.shape
    num_pages, Hkv = k_cache.shape[0], k_cache.shape[1]
    if k_cache.shape != v_cache.shape or k_cache.shape[2] != PAGE_TOKENS or k_cache.shape[3] != D:
        raise ValueError("k_cache/v_cache must be [num_pages, Hkv, 16, D]")
    if page_table.shape[0] < B or seq_lens.shape[0] < B:
        raise ValueError("page_table and seq_lens need a row per sequence")
    maxp = page_table.shape[1]
    scale = 1.0 / math.sqrt(D) if scale is None else scale
    device = _same_device(q, k_cache, v_cache, page_table, seq_lens, out, workspace)
    if out is not None:
        _out(out, torch.bfloat16, (B, Hq, D), "out")
    _check_workspace(workspace)
    with _on(device, stream):
        out = torch.empty_like(q) if out is None else out
        ws, nbytes = _workspace(attention_workspace_size(B, Hq, D, maxp), device, workspace)
        _check("bi_attention_decode", lib().bi_attention_decode(
            _ptr(q), _ptr(k_cache), _ptr(v_cache), num_pages, _ptr(page_table), maxp, _ptr(seq_lens), _ptr(out),
            B, Hq, Hkv, D, scale, _ptr(ws), nbytes, _stream()))
    return out


STATIC_SCRATCH_BYTES = 32 << 20


def attention_decode_static(q, k_cache, v_cache, page_table, seq_lens, scale: float | None = None, out=None,
                            stream=None):
    """Decode attention that allocates nothing: its scratch is a fixed 32 MiB array inside
    libbi (for callers that cannot allocate device memory). Same result as attention_decode.
    Calls that overlap on the GPU share that array and must be serialised by the caller."""
    _req(q, torch.bfloat16, "q", 3)
    _req(k_cache, torch.bfloat16, "k_cache", 4)
    _req(v_cache, torch.bfloat16, "v_cache", 4)
    _req(page_table, torch.int32, "page_table", 2)
    _req(seq_lens, torch.int32, "seq_lens", 1)
    for t, n in ((q, "q"), (k_cache, "k_cache"), (v_cache, "v_cache"), (page_table, "page_table"),
                 (seq_lens, "seq_lens")):
        _contig(t, n)
    B, Hq, D = q.shape
    num_pages, Hkv = k_cache.shape[0], k_cache.shape[1]
    if k_cache.shape != v_cache.shape or k_cache.shape[2] != PAGE_TOKENS or k_cache.shape[3] != D:
        raise ValueError("k_cache/v_cache must be [num_pages, Hkv, 16, D]")
    if page_table.shape[0] < B or seq_lens.shape[0] < B:
        raise ValueError("page_table and seq_lens need a row per sequence")
    scale = 1.0 / math.sqrt(D) if scale is None else scale
    device = _same_device(q, k_cache, v_cache, page_table, seq_lens, out)
    if out is not None:
        _out(out, torch.bfloat16, (B, Hq, D), "out")
    with _on(device, stream):
        out = torch.empty_like(q) if out is None else out
        _check("bi_attention_decode_static", lib().bi_attention_decode_static(
            _ptr(q), _ptr(k_cache), _ptr(v_cache), num_pages, _ptr(page_table), page_table.shape[1], _ptr(seq_lens),
            _ptr(out), B, Hq, Hkv, D, scale, _stream()))
    return out


def _rows3(t: torch.Tensor, name: str):
    """[T, H, D] view whose rows may be strided (e.g. a slice of a fused QKV output)."""
    if t.dim() != 3 or t.stride(2) != 1 or t.stride(1) != t.shape[2]:
        raise ValueError(f"{name} must be [T, H, D] with contiguous heads (row stride free)")
    return t.stride(0)


def attention_prefill(q, q_seq, q_pos, k_cache, v_cache, page_table, scale: float | None = None, out=None,
                      workspace=None, stream=None):
    """Causal prefill; row t of q [T, Hq, D] sees keys 0..q_pos[t] of sequence q_seq[t].

    A decode token is a row at its sequence's newest position, so one call may mix
    prefill chunks and decode tokens. q's rows may be strided (a fused QKV slice).
    """
    _req(q, torch.bfloat16, "q", 3)
    _req(q_seq, torch.int32, "q_seq", 1)
    _req(q_pos, torch.int32, "q_pos", 1)
    _req(k_cache, torch.bfloat16, "k_cache", 4)
    _req(v_cache, torch.bfloat16, "v_cache", 4)
    _req(page_table, torch.int32, "page_table", 2)
    for t, n in ((q_seq, "q_seq"), (q_pos, "q_pos"), (k_cache, "k_cache"), (v_cache, "v_cache"),
                 (page_table, "page_table")):
        _contig(t, n)
    ldq = _rows3(q, "q")
    T, Hq, D = q.shape
    num_pages, Hkv = k_cache.shape[0], k_cache.shape[1]
    if k_cache.shape != v_cache.shape or k_cache.shape[2] != PAGE_TOKENS or k_cache.shape[3] != D:
        raise ValueError("k_cache/v_cache must be [num_pages, Hkv, 16, D]")
    if q_seq.shape[0] != T or q_pos.shape[0] != T:
        raise ValueError("q_seq and q_pos need one entry per query row")
    num_seqs, maxp = page_table.shape
    scale = 1.0 / math.sqrt(D) if scale is None else scale
    device = _same_device(q, q_seq, q_pos, k_cache, v_cache, page_table, out, workspace)
    if out is not None:
        _out(out, torch.bfloat16, (T, Hq, D), "out")
    _check_workspace(workspace)
    with _on(device, stream):
        out = torch.empty((T, Hq, D), dtype=torch.bfloat16, device=device) if out is None else out
        ws, nbytes = _workspace(attention_workspace_size(T, Hq, D, maxp), device, workspace)
        _check("bi_attention_prefill", lib().bi_attention_prefill(
            _ptr(q), ldq, _ptr(q_seq), _ptr(q_pos), _ptr(k_cache), _ptr(v_cache), num_pages, _ptr(page_table),
            num_seqs, maxp, _ptr(out), T, Hq, Hkv, D, scale, _ptr(ws), nbytes, _stream()))
    return out


def attention_prefill_tc(q, seq: int, pos0: int, k_cache, v_cache, page_table, scale: float | None = None, out=None,
                         stream=None):
    """Causal prefill of positions pos0 .. pos0+T-1 of one sequence on tensor cores (q [T, Hq, D])."""
    _req(q, torch.bfloat16, "q", 3)
    _req(k_cache, torch.bfloat16, "k_cache", 4)
    _req(v_cache, torch.bfloat16, "v_cache", 4)
    _req(page_table, torch.int32, "page_table", 2)
    for t, n in ((k_cache, "k_cache"), (v_cache, "v_cache"), (page_table, "page_table")):
        _contig(t, n)
    ldq = _rows3(q, "q")
    T, Hq, D = q.shape
    num_pages, Hkv = k_cache.shape[0], k_cache.shape[1]
    if k_cache.shape != v_cache.shape or k_cache.shape[2] != PAGE_TOKENS or k_cache.shape[3] != D:
        raise ValueError("k_cache/v_cache must be [num_pages, Hkv, 16, D]")
    num_seqs, maxp = page_table.shape
    scale = 1.0 / math.sqrt(D) if scale is None else scale
    device = _same_device(q, k_cache, v_cache, page_table, out)
    if out is not None:
        _out(out, torch.bfloat16, (T, Hq, D), "out")
    with _on(device, stream):
        out = torch.empty((T, Hq, D), dtype=torch.bfloat16, device=device) if out is None else out
        _check("bi_attention_prefill_tc", lib().bi_attention_prefill_tc(
            _ptr(q), ldq, seq, pos0, T, _ptr(k_cache), _ptr(v_cache), num_pages, _ptr(page_table), num_seqs, maxp,
            _ptr(out), Hq, Hkv, D, scale, _stream()))
    return out


def kv_append(k_new, v_new, q_seq, q_pos, k_cache, v_cache, page_table, stream=None):
    """Write k_new/v_new [T, Hkv, D] (rows may be strided) into the paged store at (q_seq[t], q_pos[t])."""
    for t, n in ((k_new, "k_new"), (v_new, "v_new"), (k_cache, "k_cache"), (v_cache, "v_cache")):
        _req(t, torch.bfloat16, n)
    for t, n in ((k_cache, "k_cache"), (v_cache, "v_cache")):
        _contig(t, n)
    for t, n in ((q_seq, "q_seq"), (q_pos, "q_pos"), (page_table, "page_table")):
        _req(t, torch.int32, n)
        _contig(t, n)
    ld = _rows3(k_new, "k_new")
    if _rows3(v_new, "v_new") != ld or v_new.shape != k_new.shape:
        raise ValueError("k_new and v_new must have the same shape and row stride")
    T, Hkv, D = k_new.shape
    if q_seq.shape != (T,) or q_pos.shape != (T,):
        raise ValueError("q_seq and q_pos need one entry per new row")
    if k_cache.dim() != 4 or k_cache.shape != v_cache.shape or k_cache.shape[1:] != (Hkv, PAGE_TOKENS, D):
        raise ValueError("k_cache/v_cache must be [num_pages, Hkv, 16, D] matching k_new")
    if page_table.dim() != 2:
        raise ValueError("page_table must be [num_seqs, max_pages]")
    num_seqs, maxp = page_table.shape
    device = _same_device(k_new, v_new, q_seq, q_pos, k_cache, v_cache, page_table)
    with _on(device, stream):
        _check("bi_kv_append", lib().bi_kv_append(
            _ptr(k_new), _ptr(v_new), ld, _ptr(q_seq), _ptr(q_pos), _ptr(k_cache), _ptr(v_cache), k_cache.shape[0],
            _ptr(page_table), num_seqs, maxp, T, Hkv, D, _stream()))


def gather_rows(src, idx, out=None, stream=None):
    """out[m] = src[idx[m]] (embedding lookup / row selection)."""
    _req(src, torch.bfloat16, "src", 2)
    _req(idx, torch.int32, "idx", 1)
    _contig(idx, "idx")
    if src.stride(1) != 1:
        raise ValueError("src rows must be contiguous")
    M, W = idx.shape[0], src.shape[1]
    device = _same_device(src, idx, out)
    if out is not None:
        _out(out, torch.bfloat16, (M, W), "out", strided_rows=True)
    with _on(device, stream):
        out = torch.empty((M, W), dtype=torch.bfloat16, device=device) if out is None else out
        _check("bi_gather_rows", lib().bi_gather_rows(_ptr(src), src.stride(0), src.shape[0], _ptr(idx), M, W,
                                                      _ptr(out), out.stride(0), _stream()))
    return out


def rope(x, pos, cos_sin, stream=None):
    """In-place rotary embedding on x [T, H, D] (rows may be strided); cos_sin fp32 [max_pos, D/2, 2]."""
    _req(x, torch.bfloat16, "x", 3)
    _req(pos, torch.int32, "pos", 1)
    _req(cos_sin, torch.float32, "cos_sin", 3)
    _contig(pos, "pos")
    _contig(cos_sin, "cos_sin")
    ldx = _rows3(x, "x")
    T, H, D = x.shape
    if cos_sin.shape[1:] != (D // 2, 2):
        raise ValueError("cos_sin must be [max_pos, D/2, 2]")
    if pos.shape != (T,):
        raise ValueError("pos needs one entry per row of x")
    device = _same_device(x, pos, cos_sin)
    with _on(device, stream):
        _check("bi_rope", lib().bi_rope(_ptr(x), ldx, T, H, D, _ptr(pos), _ptr(cos_sin), cos_sin.shape[0],
                                        _stream()))
    return x


def swiglu(gate_up, out=None, stream=None):
    """out = silu(gate_up[:, :F]) * gate_up[:, F:] with F = gate_up.shape[1] // 2."""
    _req(gate_up, torch.bfloat16, "gate_up", 2)
    if gate_up.stride(1) != 1:
        raise ValueError("gate_up rows must be contiguous")
    M, F2 = gate_up.shape
    F = F2 // 2
    device = _same_device(gate_up, out)
    if out is not None:
        _out(out, torch.bfloat16, (M, F), "out", strided_rows=True)
    with _on(device, stream):
        out = torch.empty((M, F), dtype=torch.bfloat16, device=device) if out is None else out
        _check("bi_swiglu", lib().bi_swiglu(_ptr(gate_up), gate_up.stride(0), _ptr(out), out.stride(0), M, F,
                                            _stream()))
    return out


def add(a, b, out=None, stream=None):
    """out = a + b elementwise (bf16 in, fp32 add, bf16 out); out may be a or b."""
    for t, n in ((a, "a"), (b, "b")):
        _req(t, torch.bfloat16, n)
        _contig(t, n)
    if a.shape != b.shape:
        raise ValueError("a and b must have the same shape")
    device = _same_device(a, b, out)
    if out is not None:
        _out(out, torch.bfloat16, tuple(a.shape), "out")
    with _on(device, stream):
        out = torch.empty_like(a) if out is None else out
        _check("bi_add", lib().bi_add(_ptr(a), _ptr(b), _ptr(out), a.numel(), _stream()))
    return out


def lmhead_workspace_size(M: int, V: int) -> int:
    return int(lib().bi_lmhead_workspace_size(M, V))


def lmhead_argmax(h, w, margin_threshold: float = 0.5, want_logits: bool = False, tokens=None, recomputed=None,
                  logits_fp32=None, workspace=None, stream=None):
    """Greedy tokens with the selective FP32 recompute.

    Returns (tokens int32 [M], recomputed int32 [M], logits_fp32 [M, V] or None).
    """
    _req(h, torch.bfloat16, "h", 2)
    _req(w, torch.bfloat16, "w", 2)
    _contig(w, "w")
    if h.stride(1) != 1:
        raise ValueError("h rows must be contiguous")
    M, K = h.shape
    V = w.shape[0]
    if w.shape[1] != K:
        raise ValueError(f"h has {K} columns but w has {w.shape[1]}")
    dev = _same_device(h, w, tokens, recomputed, logits_fp32, workspace)
    if tokens is not None:
        _out(tokens, torch.int32, (M,), "tokens")
    if recomputed is not None:
        _out(recomputed, torch.int32, (M,), "recomputed")
    if logits_fp32 is not None:
        _out(logits_fp32, torch.float32, (M, V), "logits_fp32")
    _check_workspace(workspace)
    with _on(dev, stream):
        tokens = torch.empty(M, dtype=torch.int32, device=dev) if tokens is None else tokens
        recomputed = torch.empty(M, dtype=torch.int32, device=dev) if recomputed is None else recomputed
        if want_logits and logits_fp32 is None:
            logits_fp32 = torch.full((M, V), float("nan"), dtype=torch.float32, device=dev)
        ws, nbytes = _workspace(lmhead_workspace_size(M, V), dev, workspace)
        _check("bi_lmhead_argmax", lib().bi_lmhead_argmax(
            _ptr(h), h.stride(0), _ptr(w), M, V, K, margin_threshold, _ptr(tokens), _ptr(recomputed),
            _ptr(logits_fp32), _ptr(ws), nbytes, _stream()))
    return tokens, recomputed, logits_fp32


def _rows2(x: torch.Tensor, name: str):
    _req(x, torch.bfloat16, name, 2)
    if x.stride(1) != 1:
        raise ValueError(f"{name} rows must be contiguous")
    return x.shape


def _u64(t: torch.Tensor, name: str, M: int):
    if not isinstance(t, torch.Tensor) or not t.is_cuda or t.dtype not in (torch.int64, torch.uint64):
        raise TypeError(f"{name} must be a CUDA int64/uint64 tensor (raw 64-bit words)")
    if t.shape != (M,):
        raise ValueError(f"{name} must have shape ({M},)")
    _contig(t, name)


def log_softmax(x, out=None, stream=None):
    """fp32 log_softmax of each bf16 row, one fixed reduction order per row."""
    M, N = _rows2(x, "x")
    device = _same_device(x, out)
    if out is not None:
        _out(out, torch.float32, (M, N), "out", strided_rows=True)
    with _on(device, stream):
        y = torch.empty((M, N), dtype=torch.float32, device=device) if out is None else out
        _check("bi_log_softmax", lib().bi_log_softmax(_ptr(x), x.stride(0), _ptr(y), y.stride(0), M, N, _stream()))
    return y


def token_logprob(x, tokens, out=None, stream=None):
    """fp32 log-probability of tokens[m] under log_softmax(x[m])."""
    M, N = _rows2(x, "x")
    _out(tokens, torch.int32, (M,), "tokens")
    device = _same_device(x, tokens, out)
    if out is not None:
        _out(out, torch.float32, (M,), "out")
    with _on(device, stream):
        out = torch.empty(M, dtype=torch.float32, device=device) if out is None else out
        _check("bi_token_logprob", lib().bi_token_logprob(_ptr(x), x.stride(0), _ptr(tokens), _ptr(out), M, N,
                                                         _stream()))
    return out


def row_mean(x, out=None, stream=None):
    """fp32 mean of each bf16 row, one fixed reduction order per row."""
    M, K = _rows2(x, "x")
    device = _same_device(x, out)
    if out is not None:
        _out(out, torch.float32, (M,), "out")
    with _on(device, stream):
        out = torch.empty(M, dtype=torch.float32, device=device) if out is None else out
        _check("bi_row_mean", lib().bi_row_mean(_ptr(x), x.stride(0), _ptr(out), M, K, _stream()))
    return out


def sampling_uniforms(seeds, steps, V: int, out=None, stream=None):
    """The (0, 1) uniforms the sampler draws for rows (seed, step): fp32 [M, V]."""
    M = seeds.shape[0]
    _u64(seeds, "seeds", M)
    _u64(steps, "steps", M)
    device = _same_device(seeds, steps, out)
    if out is not None:
        _out(out, torch.float32, (M, V), "out", strided_rows=True)
    with _on(device, stream):
        u = torch.empty((M, V), dtype=torch.float32, device=device) if out is None else out
        _check("bi_sampling_uniforms", lib().bi_sampling_uniforms(_ptr(seeds), _ptr(steps), _ptr(u), u.stride(0), M,
                                                                 V, _stream()))
    return u


def sample(logits, seeds, steps, temperature: float, out=None, stream=None):
    """Gumbel-max temperature sampling: int32 [M] tokens from bf16 logits [M, V]."""
    M, V = _rows2(logits, "logits")
    _u64(seeds, "seeds", M)
    _u64(steps, "steps", M)
    device = _same_device(logits, seeds, steps, out)
    if out is not None:
        _out(out, torch.int32, (M,), "out")
    with _on(device, stream):
        out = torch.empty(M, dtype=torch.int32, device=device) if out is None else out
        _check("bi_sample", lib().bi_sample(_ptr(logits), logits.stride(0), _ptr(seeds), _ptr(steps), temperature,
                                           _ptr(out), M, V, _stream()))
    return out


def selftest_wait_timeout(limit_ms: int = 50, stream=None):
    """Launch a kernel whose bounded wait is made to expire (records BI_ERR_DEVICE_TIMEOUT)."""
    _check("bi_selftest_wait_timeout", lib().bi_selftest_wait_timeout(limit_ms, _stream(stream)))


def get_device_error() -> int:
    """Read and clear the device error word (synchronises the device)."""
    code = ctypes.c_int32(0)
    _check("bi_get_device_error", lib().bi_get_device_error(ctypes.byref(code)))
    return int(code.value)
