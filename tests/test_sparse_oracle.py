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


# ---- token-granular selection (oracle.mla_naive_sparse): any list of cache rows per sequence

def _sparse_tokens(w, indices, counts, kv=None, pe=None):
    d = w.dims
    return oracle.mla_naive_sparse(w.q, w.kv if kv is None else kv, w.pe if pe is None else pe, indices, counts,
                                   w.wkv_b, d.heads, d.qk_nope, d.qk_rope, d.v_head, d.scale)


def test_gather_selected_hand_example():
    """Rows numbered by their index: sequence 0 selects rows 4, 0, 4 (a repeated entry counts
    twice), sequence 1 selects nothing, sequence 2 row 5; entries past the counts (-1, 99) are
    never read."""
    kv = np.arange(6, dtype=np.float64)[:, None] * np.ones((1, 3))
    pe = 10 + np.arange(6, dtype=np.float64)[:, None] * np.ones((1, 2))
    idx = np.array([[4, 0, 4, -1], [99, -1, -1, -1], [5, 99, -1, -1]])
    g_kv, g_pe, cu = oracle.gather_selected(kv, pe, idx, [3, 0, 1])
    assert g_kv[:, 0].tolist() == [4, 0, 4, 5] and g_pe[:, 0].tolist() == [14, 10, 14, 15]
    assert cu.tolist() == [0, 3, 3, 4]


def test_selected_row_outside_the_cache_is_an_error():
    kv, pe = np.zeros((6, 3)), np.zeros((6, 2))
    for bad in (6, -1):
        try:
            oracle.gather_selected(kv, pe, np.array([[0, bad]]), [2])
        except ValueError:
            continue
        raise AssertionError(f"row {bad} was accepted")


def test_selecting_every_token_in_any_order_is_dense_decode():
    """Top-k = all: a permutation of all of a sequence's rows gives the dense decode result."""
    w = wl.make_workload("st", wl.TINY, [1, 1, 1], [128, 77, 1], seed=31)
    rng = np.random.default_rng(3)
    cu = w.cu_seqlens_k
    topk = max(w.seqlens_k)
    idx = np.full((w.batch, topk), -1, dtype=np.int64)
    for b in range(w.batch):
        idx[b, :w.seqlens_k[b]] = cu[b] + rng.permutation(w.seqlens_k[b])
    got = _sparse_tokens(w, idx, w.seqlens_k)
    assert np.allclose(got, oracle.workload_naive(w), rtol=1e-12, atol=1e-13)


def test_one_selected_token_returns_its_projected_value():
    """A single selected row j: the softmax over one key is 1, so out[b, h] = W_v[h] . kv[j]
    whatever the query (closed form)."""
    w = wl.make_workload("st1", wl.TINY, [1, 1], [50, 70], seed=32)
    d = w.dims
    idx = np.array([[17], [50 + 69]])
    got = _sparse_tokens(w, idx, [1, 1])
    _, wv = oracle.head_view(w.wkv_b, d.heads, d.qk_nope, d.v_head)
    for b, j in enumerate(idx[:, 0]):
        for h in range(d.heads):
            assert np.allclose(got[b, h], wv[h].astype(np.float64) @ w.kv[j].astype(np.float64), rtol=1e-12,
                               atol=1e-12)


def test_selection_is_attention_over_those_tokens_only():
    """Rows outside the selection have no influence (overwriting them changes nothing), and a
    selection of rows from another sequence's part of the cache is allowed (rows are global)."""
    w = wl.make_workload("st2", wl.TINY, [1, 1], [100, 60], seed=33)
    idx = np.array([[3, 90, 120, 7], [0, 1, 159, -1]])
    counts = [4, 3]
    got = _sparse_tokens(w, idx, counts)
    kv, pe = w.kv.copy(), w.pe.copy()
    keep = set(idx[0, :4]) | set(idx[1, :3])
    for r in range(kv.shape[0]):
        if r not in keep:
            kv[r] = 1e3
            pe[r] = -1e3
    assert np.array_equal(got, _sparse_tokens(w, idx, counts, kv, pe))
    d = w.dims
    sel = [3, 90, 120, 7]
    ref0 = oracle.mla_naive(w.q[:1], w.kv[sel], w.pe[sel], w.wkv_b, np.array([0, 1]), np.array([0, 4]), d.heads,
                            d.qk_nope, d.qk_rope, d.v_head, d.scale)
    assert np.allclose(got[0], ref0[0], rtol=1e-12, atol=1e-13)
