"""Paged KV cache: packing per-sequence caches into fixed-size pages.

A page store is bf16 [num_pages, Hkv, page_size, 128]; ``block_table[b, j]``
names the page that holds tokens j*page_size .. j*page_size + page_size - 1 of
sequence b (the layout kascade_decode_anchor_paged / kascade_decode_reuse_paged
read).  Pages are handed out in a seeded random order, as a serving engine's
allocator would after some churn.
"""
from __future__ import annotations

from typing import List, Optional

import torch


def to_paged(ks: List[torch.Tensor], vs: List[torch.Tensor], page_size: int,
             seed: int = 0, spare_pages: int = 0):
    """Pack per-sequence caches ks[b], vs[b] ([Hkv, T_b, d]) into a page store.

    Returns (k_pages, v_pages, block_table int32 [B, max_pages], num_pages).
    Unused tail slots of a sequence's last page are zero; unused block-table
    entries are -1.
    """
    if page_size < 16 or page_size % 16:
        raise ValueError("page_size must be a positive multiple of 16")
    B = len(ks)
    Hkv, _, d = ks[0].shape
    dev = ks[0].device
    n_pages = [(k.shape[1] + page_size - 1) // page_size for k in ks]
    max_pages = max(1, max(n_pages))
    num_pages = sum(n_pages) + spare_pages
    num_pages = max(num_pages, 1)
    g = torch.Generator(device="cpu").manual_seed(seed)
    order = torch.randperm(num_pages, generator=g).tolist()
    k_pages = torch.zeros(num_pages, Hkv, page_size, d, dtype=ks[0].dtype, device=dev)
    v_pages = torch.zeros_like(k_pages)
    table = torch.full((B, max_pages), -1, dtype=torch.int32)
    nxt = 0
    for b in range(B):
        T = ks[b].shape[1]
        for j in range(n_pages[b]):
            p = order[nxt]
            nxt += 1
            table[b, j] = p
            lo, hi = j * page_size, min(T, (j + 1) * page_size)
            k_pages[p, :, : hi - lo] = ks[b][:, lo:hi]
            v_pages[p, :, : hi - lo] = vs[b][:, lo:hi]
    return k_pages, v_pages, table.to(dev), num_pages
