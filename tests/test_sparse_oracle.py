"""Block-sparse decode as attention over selected pages: the fine-grained sparse attention step
of DeepSeek Sparse Attention ("What is DeepSeek Sparse Attention (DSA)?", section "How DSA works
(conceptual)": exact attention over the shortlisted spans only), at the granularity of cache
pages.  The cited page defines no indexer, so the selection is an input; a selection is a block table
listing the chosen pages, and mla_attn_paged computes it.  These pins hold the oracle's reading
to dense attention."""
import numpy as np

import oracle
from deepseek_mla_latent_b200 import workloads as wl


def _naive(w, kv, pe, cu_k):
    d = w.dims
    return oracle.mla_naive(w.q, kv, pe, w.wkv_b, w.cu_seqlens_q, cu_k, d.heads, d.qk_nope, d.qk_rope, d.v_head,
                            d.scale)


def _sparse(w, pc, table, seqlens):
    d = w.dims
    return oracle.mla_naive_paged(w.q, pc.kv_cache, pc.pe_cache, table, seqlens, pc.page_size, w.wkv_b,
                                  w.cu_seqlens_q, d.heads, d.qk_nope, d.qk_rope, d.v_head, d.scale)


def test_selecting_every_page_in_any_order_is_dense_attention():
    """Top-k = all: decode has no mask, so any order of all pages gives the dense result."""
    w = wl.make_workload("sp", wl.TINY, [1, 1], [128, 64], seed=21)
    pc = wl.paged_cache(w, 16, seed=1, spare_pages=2)
    rng = np.random.default_rng(0)
    table = pc.block_table.copy()
    for b, t in enumerate(w.seqlens_k):
        table[b, :t // 16] = rng.permutation(table[b, :t // 16])
    got = _sparse(w, pc, table, pc.seqlens_k)
    assert np.allclose(got, oracle.workload_naive(w), rtol=1e-12, atol=1e-13)


def test_selected_pages_equal_dense_attention_over_their_tokens():
    """A selection of pages 5, 1, 6 of a sequence equals dense attention over exactly those
    tokens (cut straight from the packed cache here)."""
    w = wl.make_workload("sp", wl.TINY, [1], [128], seed=22)
    pc = wl.paged_cache(w, 16, seed=2)
    pick = [5, 1, 6]
    table = np.array([[pc.block_table[0, p] for p in pick]], dtype=np.int32)
    got = _sparse(w, pc, table, [16 * len(pick)])
    kv = np.concatenate([w.kv[16 * p:16 * p + 16] for p in pick])
    pe = np.concatenate([w.pe[16 * p:16 * p + 16] for p in pick])
    ref = _naive(w, kv, pe, np.array([0, 48]))
    assert np.array_equal(got, ref)
