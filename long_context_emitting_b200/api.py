"""Tensor-level entry points: PyTorch CUDA tensors in, C-ABI calls out.

Each function checks dtypes/devices/contiguity, allocates outputs and the
workspace with PyTorch when the caller passes none, and calls the entry point
of the same name in libkascade.so on the current CUDA stream.  All arithmetic
runs in the library's kernels; CPU tensors are rejected.
"""
from __future__ import annotations

import math
from typing import Optional

import torch

from . import binding
from .binding import Shape, check

HEAD_DIM = 128
TILE = 128


def _lib():
    return binding.load()


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _need_cuda(name: str, t: torch.Tensor, dtype: torch.dtype) -> None:
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor (the library has no CPU path)")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _need_size(name: str, t: torch.Tensor, dtype: torch.dtype, n: int) -> None:
    """A contiguous CUDA tensor of ``dtype`` with at least ``n`` elements: the
    kernels read or write that many from its start, and nothing checks the
    size below this layer."""
    _need_cuda(name, t, dtype)
    if t.numel() < n:
        raise ValueError(f"{name} has {t.numel()} elements; this call needs at least {n}")


def _ws_bytes(ws: torch.Tensor) -> int:
    """Byte size of a caller's workspace tensor (any dtype)."""
    if not isinstance(ws, torch.Tensor) or not ws.is_cuda or not ws.is_contiguous():
        raise ValueError("ws must be a contiguous CUDA tensor")
    return ws.numel() * ws.element_size()


_DATA_DTYPES = (torch.bfloat16, torch.float16)


def _data_suffix(*ts) -> str:
    """'' for bfloat16 q/k/v/out, '_f16' for float16 (all of one call alike)."""
    dt = ts[0].dtype
    if dt not in _DATA_DTYPES or any(t.dtype != dt for t in ts):
        raise TypeError("q, k, v must all be bfloat16 or all float16")
    return "_f16" if dt == torch.float16 else ""


def _stream() -> int:
    return torch.cuda.current_stream().cuda_stream


def k_for_len(n: int) -> int:
    """Top-k size for a context of n keys (the library's rule)."""
    return int(_lib().kascade_k_for_len(int(n)))


def device_status(stream: Optional[int] = None) -> int:
    """Wait for the stream and return/clear the sticky device status code."""
    return int(_lib().kascade_get_device_status(_stream() if stream is None else stream))


def selftest_wait_timeout(spin: bool = False, stream: Optional[int] = None) -> int:
    """Run the bounded-wait diagnostic (about 2 s on the GPU) and return the
    device status it leaves: KASCADE_ERR_TIMEOUT when the wait gave up."""
    st = _stream() if stream is None else stream
    check(_lib().kascade_selftest_wait_timeout(1 if spin else 0, st), "kascade_selftest_wait_timeout")
    return device_status(st)


def workspace(nbytes: int, device) -> torch.Tensor:
    return torch.empty(max(int(nbytes), 16), dtype=torch.uint8, device=device)


# ---------------------------------------------------------------- decode ----
def decode_anchor_workspace_bytes(B, Hq, Hkv, max_T) -> int:
    return int(_lib().kascade_decode_anchor_workspace_bytes(Shape(B, Hq, Hkv, HEAD_DIM), max_T))


def decode_anchor(q, k, v, kv_off, seq_len, max_T: int, scale: float, Hkv: int,
                  out=None, lse=None, pooled=None, ld_pooled: Optional[int] = None, ws=None):
    """Dense decode attention + GQA-pooled probabilities (kascade_decode_anchor; the
    _f16 entry point when q, k, v are float16)."""
    B, Hq, d = q.shape
    sfx = _data_suffix(q, k, v)
    for name, t in (("q", q), ("k", k), ("v", v)):
        _need_cuda(name, t, q.dtype)
    _need_size("kv_off", kv_off, torch.int64, B)
    _need_size("seq_len", seq_len, torch.int32, B)
    dev = q.device
    if ld_pooled is None:
        ld_pooled = (max_T + 3) // 4 * 4
    out = torch.empty(B, Hq, d, dtype=q.dtype, device=dev) if out is None else out
    lse = torch.empty(B, Hq, dtype=torch.float32, device=dev) if lse is None else lse
    pooled = torch.empty(B, Hkv, ld_pooled, dtype=torch.float32, device=dev) if pooled is None else pooled
    _need_size("out", out, q.dtype, B * Hq * d)
    _need_size("lse", lse, torch.float32, B * Hq)
    _need_size("pooled", pooled, torch.float32, B * Hkv * ld_pooled)
    shape = Shape(B, Hq, Hkv, d)
    need = _lib().kascade_decode_anchor_workspace_bytes(shape, max_T)
    ws = workspace(need, dev) if ws is None else ws
    rc = getattr(_lib(), "kascade_decode_anchor" + sfx)(shape, _ptr(q), _ptr(k), _ptr(v), _ptr(kv_off), _ptr(seq_len),
                                      int(max_T), float(scale), _ptr(out), _ptr(lse), _ptr(pooled),
                                      int(ld_pooled), _ptr(ws), _ws_bytes(ws), _stream())
    check(rc, "kascade_decode_anchor" + sfx)
    return out, lse, pooled


def decode_reuse_workspace_bytes(B, Hq, Hkv, k_max) -> int:
    return int(_lib().kascade_decode_reuse_workspace_bytes(Shape(B, Hq, Hkv, HEAD_DIM), k_max))


def decode_reuse(q, k, v, kv_off, seq_len, idx, idx_k, head_map, scale: float, Hkv: int,
                 out=None, lse=None, ws=None):
    """Sparse decode attention over anchor indices via a head map (kascade_decode_reuse;
    the _f16 entry point when q, k, v are float16)."""
    B, Hq, d = q.shape
    sfx = _data_suffix(q, k, v)
    for name, t in (("q", q), ("k", k), ("v", v)):
        _need_cuda(name, t, q.dtype)
    k_max = idx.shape[-1]
    _need_size("kv_off", kv_off, torch.int64, B)
    _need_size("seq_len", seq_len, torch.int32, B)
    _need_size("idx", idx, torch.int32, B * Hkv * k_max)
    _need_size("idx_k", idx_k, torch.int32, B * Hkv)
    _need_size("head_map", head_map, torch.int32, Hkv)
    dev = q.device
    out = torch.empty(B, Hq, d, dtype=q.dtype, device=dev) if out is None else out
    lse = torch.empty(B, Hq, dtype=torch.float32, device=dev) if lse is None else lse
    _need_size("out", out, q.dtype, B * Hq * d)
    _need_size("lse", lse, torch.float32, B * Hq)
    shape = Shape(B, Hq, Hkv, d)
    need = _lib().kascade_decode_reuse_workspace_bytes(shape, k_max)
    ws = workspace(need, dev) if ws is None else ws
    rc = getattr(_lib(), "kascade_decode_reuse" + sfx)(shape, _ptr(q), _ptr(k), _ptr(v), _ptr(kv_off), _ptr(seq_len),
                                     _ptr(idx), _ptr(idx_k), int(k_max), _ptr(head_map),
                                     float(scale), _ptr(out), _ptr(lse), _ptr(ws), _ws_bytes(ws),
                                     _stream())
    check(rc, "kascade_decode_reuse" + sfx)
    return out, lse


# ------------------------------------------------------------ decode, paged ----
def _need_pages(k_pages, v_pages, block_table, B: int, Hkv: int, page_size: int, d: int,
                dtype: torch.dtype = torch.bfloat16) -> None:
    """Page store [num_pages, Hkv, page_size, d] (K and V alike) and a block
    table with a row of page numbers for each of the B sequences."""
    _need_cuda("k_pages", k_pages, dtype)
    _need_cuda("v_pages", v_pages, dtype)
    _need_cuda("block_table", block_table, torch.int32)
    if k_pages.dim() != 4 or tuple(k_pages.shape[1:]) != (Hkv, page_size, d):
        raise ValueError(f"k_pages must be [num_pages, {Hkv}, {page_size}, {d}], got {tuple(k_pages.shape)}")
    if v_pages.shape != k_pages.shape:
        raise ValueError("v_pages must have the shape of k_pages")
    if block_table.dim() != 2 or block_table.shape[0] < B:
        raise ValueError(f"block_table must be [>= {B}, max_pages], got {tuple(block_table.shape)}")


def decode_anchor_paged(q, k_pages, v_pages, block_table, page_size: int, seq_len, max_T: int,
                        scale: float, Hkv: int, out=None, lse=None, pooled=None,
                        ld_pooled: Optional[int] = None, ws=None):
    """kascade_decode_anchor over a paged cache (see paging.to_paged); the _f16
    entry point when q and the pages are float16."""
    B, Hq, d = q.shape
    sfx = _data_suffix(q, k_pages, v_pages)
    _need_cuda("q", q, q.dtype)
    _need_pages(k_pages, v_pages, block_table, B, Hkv, page_size, d, q.dtype)
    _need_size("seq_len", seq_len, torch.int32, B)
    dev = q.device
    if ld_pooled is None:
        ld_pooled = (max_T + 3) // 4 * 4
    out = torch.empty(B, Hq, d, dtype=q.dtype, device=dev) if out is None else out
    lse = torch.empty(B, Hq, dtype=torch.float32, device=dev) if lse is None else lse
    pooled = torch.empty(B, Hkv, ld_pooled, dtype=torch.float32, device=dev) if pooled is None else pooled
    _need_size("out", out, q.dtype, B * Hq * d)
    _need_size("lse", lse, torch.float32, B * Hq)
    _need_size("pooled", pooled, torch.float32, B * Hkv * ld_pooled)
    shape = Shape(B, Hq, Hkv, d)
    need = _lib().kascade_decode_anchor_workspace_bytes(shape, max_T)
    ws = workspace(need, dev) if ws is None else ws
    rc = getattr(_lib(), "kascade_decode_anchor_paged" + sfx)(
        shape, _ptr(q), _ptr(k_pages), _ptr(v_pages), int(k_pages.shape[0]), _ptr(block_table),
        int(block_table.shape[1]), int(page_size), _ptr(seq_len), int(max_T), float(scale),
        _ptr(out), _ptr(lse), _ptr(pooled), int(ld_pooled), _ptr(ws), _ws_bytes(ws), _stream())
    check(rc, "kascade_decode_anchor_paged" + sfx)
    return out, lse, pooled


def decode_reuse_paged(q, k_pages, v_pages, block_table, page_size: int, seq_len, idx, idx_k,
                       head_map, scale: float, Hkv: int, out=None, lse=None, ws=None):
    """kascade_decode_reuse over a paged cache (see paging.to_paged); the _f16
    entry point when q and the pages are float16."""
    B, Hq, d = q.shape
    sfx = _data_suffix(q, k_pages, v_pages)
    _need_cuda("q", q, q.dtype)
    _need_pages(k_pages, v_pages, block_table, B, Hkv, page_size, d, q.dtype)
    k_max = idx.shape[-1]
    _need_size("seq_len", seq_len, torch.int32, B)
    _need_size("idx", idx, torch.int32, B * Hkv * k_max)
    _need_size("idx_k", idx_k, torch.int32, B * Hkv)
    _need_size("head_map", head_map, torch.int32, Hkv)
    dev = q.device
    out = torch.empty(B, Hq, d, dtype=q.dtype, device=dev) if out is None else out
    lse = torch.empty(B, Hq, dtype=torch.float32, device=dev) if lse is None else lse
    _need_size("out", out, q.dtype, B * Hq * d)
    _need_size("lse", lse, torch.float32, B * Hq)
    shape = Shape(B, Hq, Hkv, d)
    need = _lib().kascade_decode_reuse_workspace_bytes(shape, k_max)
    ws = workspace(need, dev) if ws is None else ws
    rc = getattr(_lib(), "kascade_decode_reuse_paged" + sfx)(
        shape, _ptr(q), _ptr(k_pages), _ptr(v_pages), int(k_pages.shape[0]), _ptr(block_table),
        int(block_table.shape[1]), int(page_size), _ptr(seq_len), _ptr(idx), _ptr(idx_k),
        int(k_max), _ptr(head_map), float(scale), _ptr(out), _ptr(lse), _ptr(ws), _ws_bytes(ws),
        _stream())
    check(rc, "kascade_decode_reuse_paged" + sfx)
    return out, lse


# ------------------------------------------------------------------ topk ----
def topk(scores, row_len, row_k, k_max: int, out=None):
    """Row-wise Top-k (ties to lower index, ascending output; tail = -1)."""
    _need_cuda("scores", scores, torch.float32)
    ld = scores.shape[-1]
    rows = scores.numel() // ld if ld else 0
    _need_size("row_len", row_len, torch.int32, rows)
    _need_size("row_k", row_k, torch.int32, rows)
    out = torch.empty(rows, k_max, dtype=torch.int32, device=scores.device) if out is None else out
    _need_size("out", out, torch.int32, rows * k_max)
    rc = _lib().kascade_topk(_ptr(scores), int(rows), int(ld), _ptr(row_len), _ptr(row_k),
                             int(k_max), _ptr(out), None, 0, _stream())
    check(rc, "kascade_topk")
    return out


# --------------------------------------------------------------- prefill ----
def prefill_anchor_workspace_bytes(B, Hq, Hkv, N) -> int:
    return int(_lib().kascade_prefill_anchor_workspace_bytes(Shape(B, Hq, Hkv, HEAD_DIM), N))


def _need_kv_like(k, v, B: int, N: int, d: int) -> None:
    """Prefill K and V as [B, Hkv, N, d], the same shape."""
    if k.dim() != 4 or k.shape[0] != B or k.shape[2] != N or k.shape[3] != d:
        raise ValueError(f"k must be [{B}, Hkv, {N}, {d}], got {tuple(k.shape)}")
    if v.shape != k.shape:
        raise ValueError("v must have the shape of k")


def prefill_anchor(q, k, v, scale: float, out=None, lse=None, pooled=None, ws=None):
    """Dense causal prefill attention + tile-pooled probabilities (kascade_prefill_anchor;
    the _f16 entry point when q, k, v are float16)."""
    B, Hq, N, d = q.shape
    Hkv = k.shape[1]
    sfx = _data_suffix(q, k, v)
    for name, t in (("q", q), ("k", k), ("v", v)):
        _need_cuda(name, t, q.dtype)
    _need_kv_like(k, v, B, N, d)
    dev = q.device
    out = torch.empty_like(q) if out is None else out
    lse = torch.empty(B, Hq, N, dtype=torch.float32, device=dev) if lse is None else lse
    if pooled is None:
        pooled = torch.empty(B, N // TILE, Hkv, N, dtype=torch.float32, device=dev)
    _need_size("out", out, q.dtype, q.numel())
    _need_size("lse", lse, torch.float32, B * Hq * N)
    _need_size("pooled", pooled, torch.float32, B * (N // TILE) * Hkv * N)
    shape = Shape(B, Hq, Hkv, d)
    need = _lib().kascade_prefill_anchor_workspace_bytes(shape, N)
    ws = workspace(need, dev) if ws is None else ws
    rc = getattr(_lib(), "kascade_prefill_anchor" + sfx)(shape, int(N), _ptr(q), _ptr(k), _ptr(v), float(scale),
                                       _ptr(out), _ptr(lse), _ptr(pooled), _ptr(ws), _ws_bytes(ws),
                                       _stream())
    check(rc, "kascade_prefill_anchor" + sfx)
    return out, lse, pooled


def prefill_reuse_workspace_bytes(B, Hq, Hkv, N, k_max) -> int:
    return int(_lib().kascade_prefill_reuse_workspace_bytes(Shape(B, Hq, Hkv, HEAD_DIM), N, k_max))


def prefill_reuse(q, k, v, idx, idx_k, head_map, scale: float, out=None, lse=None, ws=None):
    """Sparse causal prefill attention over tile indices + diagonal (kascade_prefill_reuse;
    the _f16 entry point when q, k, v are float16)."""
    B, Hq, N, d = q.shape
    Hkv = k.shape[1]
    sfx = _data_suffix(q, k, v)
    for name, t in (("q", q), ("k", k), ("v", v)):
        _need_cuda(name, t, q.dtype)
    _need_kv_like(k, v, B, N, d)
    k_max = idx.shape[-1]
    n_tiles = N // TILE
    _need_size("idx", idx, torch.int32, B * n_tiles * Hkv * k_max)
    _need_size("idx_k", idx_k, torch.int32, B * n_tiles * Hkv)
    _need_size("head_map", head_map, torch.int32, Hkv)
    dev = q.device
    out = torch.empty_like(q) if out is None else out
    lse = torch.empty(B, Hq, N, dtype=torch.float32, device=dev) if lse is None else lse
    _need_size("out", out, q.dtype, q.numel())
    _need_size("lse", lse, torch.float32, B * Hq * N)
    shape = Shape(B, Hq, Hkv, d)
    need = _lib().kascade_prefill_reuse_workspace_bytes(shape, N, k_max)
    ws = workspace(need, dev) if ws is None else ws
    rc = getattr(_lib(), "kascade_prefill_reuse" + sfx)(shape, int(N), _ptr(q), _ptr(k), _ptr(v), _ptr(idx),
                                      _ptr(idx_k), int(k_max), _ptr(head_map), float(scale),
                                      _ptr(out), _ptr(lse), _ptr(ws), _ws_bytes(ws), _stream())
    check(rc, "kascade_prefill_reuse" + sfx)
    return out, lse


# ----------------------------------------------------------- calibration ----
def similarity_rows(p_b, row_len, row_k, idx_a, idx_b, b_row=None, a_row=None, out=None):
    """Per-row similarity ratio (kascade_similarity_rows): fp64 [n_out].

    Row r compares the Top-k set idx_a[a_row[r]] with idx_b[b_row[r]] on the
    distribution p_b[b_row[r]] (identity maps when b_row / a_row are None).
    """
    _need_cuda("p_b", p_b, torch.float32)
    ld = p_b.shape[-1]
    rows = p_b.numel() // ld if ld else 0
    k_max = idx_a.shape[-1]
    for name, t, n in (("row_len", row_len, rows), ("row_k", row_k, rows),
                       ("idx_a", idx_a, rows * k_max), ("idx_b", idx_b, rows * k_max)):
        _need_size(name, t, torch.int32, n)
    n_out = b_row.numel() if b_row is not None else rows
    for name, t in (("b_row", b_row), ("a_row", a_row)):
        if t is not None:
            _need_size(name, t, torch.int32, n_out)
    out = torch.empty(n_out, dtype=torch.float64, device=p_b.device) if out is None else out
    _need_size("out", out, torch.float64, n_out)
    rc = _lib().kascade_similarity_rows(_ptr(p_b), int(rows), int(ld), _ptr(row_len), _ptr(row_k),
                                        _ptr(idx_a), _ptr(idx_b), int(k_max), int(n_out),
                                        _ptr(b_row), _ptr(a_row), _ptr(out), _stream())
    check(rc, "kascade_similarity_rows")
    return out


def _pad4(p):
    """Rows padded to a multiple of 4 floats (the 16-byte row stride the kernels
    require); the padding lies beyond every row's length and is never read."""
    n = p.shape[-1]
    if n % 4 == 0 and p.is_contiguous():
        return p
    out = torch.zeros(*p.shape[:-1], (n + 3) // 4 * 4, dtype=p.dtype, device=p.device)
    out[..., :n] = p
    return out


def _row_sets(p, k, n):
    """Top-k sets of every row of p [rows, >= n] over its first n entries."""
    rows = p.shape[0]
    row_len = torch.full((rows,), n, dtype=torch.int32, device=p.device)
    row_k = torch.full((rows,), k, dtype=torch.int32, device=p.device)
    return topk(p, row_len, row_k, k), row_len, row_k


def similarity_mean(p_b, row_len, row_k, idx_a, idx_b, out=None, ws=None):
    """sim(a, b) on the device (kascade_similarity_mean): fp64 [1], the mean over
    rows of the per-row ratios of similarity_rows with identity row maps."""
    _need_cuda("p_b", p_b, torch.float32)
    ld = p_b.shape[-1]
    rows = p_b.numel() // ld if ld else 0
    k_max = idx_a.shape[-1]
    for name, t, n in (("row_len", row_len, rows), ("row_k", row_k, rows),
                       ("idx_a", idx_a, rows * k_max), ("idx_b", idx_b, rows * k_max)):
        _need_size(name, t, torch.int32, n)
    out = torch.empty(1, dtype=torch.float64, device=p_b.device) if out is None else out
    _need_size("out", out, torch.float64, 1)
    need = _lib().kascade_similarity_mean_workspace_bytes(int(rows))
    ws = workspace(need, p_b.device) if ws is None else ws
    rc = _lib().kascade_similarity_mean(_ptr(p_b), int(rows), int(ld), _ptr(row_len), _ptr(row_k),
                                        _ptr(idx_a), _ptr(idx_b), int(k_max), _ptr(out), _ptr(ws),
                                        _ws_bytes(ws), _stream())
    check(rc, "kascade_similarity_mean")
    return out


def similarity(p_a, p_b, k: int) -> float:
    """sim(a, b) of two layers: the mean over rows (queries, or pooled rows) of
    the share of b's Top-k mass that a's Top-k indices recover."""
    n = p_a.shape[-1]
    p_a, p_b = _pad4(p_a), _pad4(p_b)
    ia, row_len, row_k = _row_sets(p_a, k, n)
    ib, _, _ = _row_sets(p_b, k, n)
    return float(similarity_mean(p_b, row_len, row_k, ia, ib).item())


def similarity_matrix(p_layers, k: int):
    """L x L host fp64 matrix of sim(a, b) for a <= b (0 below the diagonal), from
    per-layer distributions p_layers [L, rows, n] (one Top-k pass per layer)."""
    L, n = p_layers.shape[0], p_layers.shape[-1]
    p_layers = _pad4(p_layers)
    dev = p_layers.device
    sets = [_row_sets(p_layers[l], k, n) for l in range(L)]
    sim = torch.zeros(L, L, dtype=torch.float64, device=dev)
    ws = workspace(_lib().kascade_similarity_mean_workspace_bytes(int(p_layers.shape[1])), dev)
    for a in range(L):
        for b in range(a, L):
            ib, row_len, row_k = sets[b]
            similarity_mean(p_layers[b], row_len, row_k, sets[a][0], ib, out=sim[a, b:b + 1], ws=ws)
    return sim.cpu().numpy()


def head_remap(p_anchor, p_reuse, k: int, sim=None):
    """Reuse-layer KV head -> anchor KV head with the highest similarity
    (kascade_head_remap; ties go to the lower anchor head).

    p_anchor / p_reuse: [Hkv, Q, n] distributions.  Returns int32 [Hkv] on the
    device; ``sim`` (fp64 [Hkv, Hkv] on the device), when given, receives the
    mean similarity of every (reuse head, anchor head) pair.
    """
    Hkv, Q, n = p_anchor.shape
    p_anchor, p_reuse = _pad4(p_anchor), _pad4(p_reuse)
    ld = p_anchor.shape[-1]
    ia, row_len, row_k = _row_sets(p_anchor.reshape(Hkv * Q, ld), k, n)
    ib, _, _ = _row_sets(p_reuse.reshape(Hkv * Q, ld), k, n)
    dev = p_anchor.device
    if sim is not None:
        _need_size("sim", sim, torch.float64, Hkv * Hkv)
    head_map = torch.empty(Hkv, dtype=torch.int32, device=dev)
    ws = workspace(_lib().kascade_head_remap_workspace_bytes(int(Hkv), int(Q)), dev)
    rc = _lib().kascade_head_remap(_ptr(p_reuse.reshape(Hkv * Q, ld)), int(Hkv), int(Q), int(ld),
                                   _ptr(row_len), _ptr(row_k), _ptr(ia), _ptr(ib), int(k),
                                   _ptr(sim), _ptr(head_map), _ptr(ws), _ws_bytes(ws), _stream())
    check(rc, "kascade_head_remap")
    return head_map


def select_anchors(S, M: int):
    """Anchor layers by the dynamic program (kascade_select_anchors, host code).

    S: the L x L weighted similarity matrix (array-like, fp64).  Returns
    (best covered similarity, ascending list of M anchor layers).
    """
    import ctypes
    import numpy as np

    S = np.ascontiguousarray(S, dtype=np.float64)
    L = S.shape[0]
    anchors = np.zeros(max(M, 1), dtype=np.int32)
    best = ctypes.c_double(0.0)
    rc = _lib().kascade_select_anchors(S.ctypes.data, int(L), int(M), anchors.ctypes.data,
                                       ctypes.addressof(best))
    check(rc, "kascade_select_anchors")
    return best.value, [int(x) for x in anchors[:M]]


def default_scale(d: int = HEAD_DIM) -> float:
    return 1.0 / math.sqrt(d)
