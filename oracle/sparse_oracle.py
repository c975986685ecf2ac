"""fp64 CPU oracle for token-granular sparse latent attention.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path may import or call this
module: only the tests and the benchmark's CPU leg use it.  It shares no code,
table or helper with the CUDA path.

What it computes.  "What is DeepSeek Sparse Attention (DSA)? A clear, modern
explainer" (sider.ai), section "How DSA works (conceptual)": a fast
pre-selector shortlists, per query, the tokens worth attending to, and exact
attention then runs over the shortlisted tokens only.  The page gives no
definition of the selector, so the selection is an input.  The reading taken
here (listed with the other readings in the design notes):

* a decode step (one query per sequence) attends to the cache rows
  indices[b, 0 .. counts[b]-1] of the packed latent cache, in any order; the
  list is a multiset of keys (an entry that appears twice counts twice);
* entries past counts[b] are never read; an entry among the first counts[b]
  that lies outside the cache is an error;
* the attention over the selected rows is the dense decode attention
  (mla_oracle) over those rows, so ``gather_selected`` builds the packed rows
  and ``mla_naive_sparse`` hands them to the packed oracle.

Everything is computed in float64; the gather is numpy indexing.
"""
from __future__ import annotations

import numpy as np

from .mla_oracle import mla_naive


def gather_selected(kv_cache, pe_cache, indices, counts):
    """Packed (kv [sum_n, C], pe [sum_n, R], cu_seqlens_k [batch+1]) of the selected rows."""
    kv_cache, pe_cache = np.asarray(kv_cache), np.asarray(pe_cache)
    idx = np.asarray(indices)
    rows = kv_cache.shape[0]
    kv_parts, pe_parts, lens = [], [], []
    for b, n in enumerate(counts):
        n = int(n)
        if n < 0 or n > idx.shape[1]:
            raise ValueError(f"sequence {b}: count {n} outside 0..{idx.shape[1]}")
        sel = idx[b, :n].astype(np.int64)
        bad = (sel < 0) | (sel >= rows)
        if np.any(bad):
            raise ValueError(f"sequence {b}: selected row {int(sel[np.argmax(bad)])} is outside the cache")
        kv_parts.append(kv_cache[sel])
        pe_parts.append(pe_cache[sel])
        lens.append(n)
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
    c, r = kv_cache.shape[1], pe_cache.shape[1]
    kv = np.concatenate(kv_parts) if kv_parts else np.zeros((0, c), kv_cache.dtype)
    pe = np.concatenate(pe_parts) if pe_parts else np.zeros((0, r), pe_cache.dtype)
    return kv, pe, cu


def mla_naive_sparse(q, kv_cache, pe_cache, indices, counts, wkv_b, heads, qk_nope, qk_rope, v_head, scale,
                     pairs=None):
    """Decode (one query per sequence, no mask) over the selected rows only: out [batch, H, Dv]."""
    kv, pe, cu_k = gather_selected(kv_cache, pe_cache, indices, counts)
    cu_q = np.arange(len(counts) + 1, dtype=np.int64)
    return mla_naive(q, kv, pe, wkv_b, cu_q, cu_k, heads, qk_nope, qk_rope, v_head, scale, pairs=pairs)
