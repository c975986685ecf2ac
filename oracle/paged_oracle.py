"""fp64 CPU oracle for MLA attention over a paged latent cache.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path may import or call this
module: only the tests and the benchmark's CPU leg use it.  It shares no code,
table or helper with the CUDA path.

What it computes.  "What is DeepSeek Sparse Attention (DSA)? A clear, modern
explainer" (sider.ai), section "How DSA works (conceptual)", its part on
efficient batching and memory: the serving runtime keeps the KV cache in
pages (paged attention) so that sequences of a continuous batch grow without
moving their cache.  The page fixes no page format; the reading taken here
(listed with the other readings in the design notes) is the usual block table:

    key j of sequence b sits in row  block_table[b, j // page_size] * page_size
                                     + j % page_size
    of kv_cache [num_pages * page_size, C] and pe_cache [num_pages * page_size, R].

Only the cache addressing changes: attention over a paged cache is attention
over the rows gathered in key order, so ``gather_paged`` builds the packed
cache and ``mla_naive_paged`` hands it to the packed oracle (mla_oracle).
Entries past a sequence's last page are never read; an entry that should hold
keys but lies outside the cache is an error.
"""
from __future__ import annotations

import numpy as np

from .mla_oracle import mla_naive


def gather_paged(kv_cache, pe_cache, block_table, seqlens_k, page_size: int):
    """Packed (kv [sum_t, C], pe [sum_t, R], cu_seqlens_k [batch+1]) of a paged cache."""
    if page_size <= 0:
        raise ValueError("page_size must be positive")
    kv_cache, pe_cache = np.asarray(kv_cache), np.asarray(pe_cache)
    table = np.asarray(block_table)
    rows = kv_cache.shape[0]
    num_pages = rows // page_size
    kv_parts, pe_parts, lens = [], [], []
    for b, t in enumerate(seqlens_k):
        t = int(t)
        idx = np.empty(t, dtype=np.int64)
        for j in range(t):
            page = int(table[b, j // page_size])
            if not 0 <= page < num_pages:
                raise ValueError(f"sequence {b}: block-table entry {page} for key {j} is outside the cache")
            idx[j] = page * page_size + j % page_size
        kv_parts.append(kv_cache[idx])
        pe_parts.append(pe_cache[idx])
        lens.append(t)
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
    c, r = kv_cache.shape[1], pe_cache.shape[1]
    kv = np.concatenate(kv_parts) if kv_parts else np.zeros((0, c), kv_cache.dtype)
    pe = np.concatenate(pe_parts) if pe_parts else np.zeros((0, r), pe_cache.dtype)
    return kv, pe, cu


def mla_naive_paged(q, kv_cache, pe_cache, block_table, seqlens_k, page_size, wkv_b, cu_seqlens_q, heads,
                    qk_nope, qk_rope, v_head, scale, pairs=None):
    """mla_naive over the keys a paged cache holds (see the module docstring)."""
    kv, pe, cu_k = gather_paged(kv_cache, pe_cache, block_table, seqlens_k, page_size)
    return mla_naive(q, kv, pe, wkv_b, cu_seqlens_q, cu_k, heads, qk_nope, qk_rope, v_head, scale, pairs=pairs)
