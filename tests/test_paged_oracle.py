"""Pins of the paged-cache oracle (oracle.paged_oracle) against facts fixed by the
block-table definition, independent of the oracle's own code."""
import numpy as np
import pytest

import oracle
from deepseek_mla_latent_b200 import workloads as wl


def test_gather_hand_example():
    """Page size 2, six cache rows whose values are their row numbers.  Sequence 0 (3 keys)
    lives in pages 2 then 0, sequence 1 (2 keys) in page 1; the trailing entries are unused
    padding (-1 and an out-of-range 7) and must not be read."""
    kv = np.arange(6, dtype=np.float64).reshape(6, 1) * np.array([[1.0, 10.0]])
    pe = np.arange(6, dtype=np.float64).reshape(6, 1) + 100.0
    table = np.array([[2, 0, 7], [1, -1, -1]])
    g_kv, g_pe, cu = oracle.gather_paged(kv, pe, table, [3, 2], 2)
    assert cu.tolist() == [0, 3, 5]
    assert g_kv[:, 0].tolist() == [4, 5, 0, 2, 3]
    assert g_kv[:, 1].tolist() == [40, 50, 0, 20, 30]
    assert g_pe[:, 0].tolist() == [104, 105, 100, 102, 103]


def test_gather_rejects_an_entry_outside_the_cache_that_holds_keys():
    kv, pe = np.zeros((4, 2)), np.zeros((4, 1))
    with pytest.raises(ValueError):
        oracle.gather_paged(kv, pe, np.array([[0, 2]]), [3], 2)   # key 2 would sit in page 2 of 2
    with pytest.raises(ValueError):
        oracle.gather_paged(kv, pe, np.array([[-1]]), [1], 2)


def test_gather_identity_table_is_the_packed_cache():
    """Pages 0, 1, 2, ... in order for one sequence give the cache rows in order."""
    rng = np.random.default_rng(0)
    kv, pe = rng.standard_normal((12, 3)), rng.standard_normal((12, 2))
    g_kv, g_pe, _ = oracle.gather_paged(kv, pe, np.array([[0, 1, 2]]), [11], 4)
    assert np.array_equal(g_kv, kv[:11]) and np.array_equal(g_pe, pe[:11])


@pytest.mark.parametrize("page", [1, 3, 64])
def test_gather_inverts_a_token_by_token_scatter(page):
    """Scatter a packed cache into randomly placed pages one token at a time (written here,
    not with the generator) and gather it back bit for bit."""
    rng = np.random.default_rng(page)
    lens = [0, 1, page, 2 * page + 1, 5]
    total = sum(lens)
    kv, pe = rng.standard_normal((total, 4)), rng.standard_normal((total, 2))
    need = [-(-t // page) for t in lens]
    perm = rng.permutation(sum(need) + 3)
    table = np.full((len(lens), max(need) + 2), -1)
    kv_c = np.full((len(perm) * page, 4), np.nan)
    pe_c = np.full((len(perm) * page, 2), np.nan)
    k, used = 0, 0
    for b, t in enumerate(lens):
        for p_ in range(need[b]):
            table[b, p_] = perm[used]
            used += 1
        for j in range(t):
            row = table[b, j // page] * page + j % page
            kv_c[row], pe_c[row] = kv[k], pe[k]
            k += 1
    g_kv, g_pe, cu = oracle.gather_paged(kv_c, pe_c, table, lens, page)
    assert np.array_equal(g_kv, kv) and np.array_equal(g_pe, pe)
    assert cu.tolist() == np.concatenate([[0], np.cumsum(lens)]).tolist()


@pytest.mark.parametrize("page", [1, 2, 64])
def test_paged_attention_equals_packed_attention(page):
    """The same keys in any page layout give the packed oracle's result exactly (the gather
    moves rows, it does not touch values), for decode and for a causal chunk."""
    w = wl.make_workload("pg", wl.TINY, [1, 3, 2], [5, 70, 2], seed=3)
    pc = wl.paged_cache(w, page, seed=page, spare_pages=2, extra_columns=1)
    d = w.dims
    ref = oracle.workload_naive(w)
    got = oracle.mla_naive_paged(w.q, pc.kv_cache, pc.pe_cache, pc.block_table, pc.seqlens_k, page, w.wkv_b,
                                 w.cu_seqlens_q, d.heads, d.qk_nope, d.qk_rope, d.v_head, d.scale)
    assert np.array_equal(got, ref)
    assert np.all(np.isfinite(got))   # the unused rows hold NaN and are never read


def test_generator_layout():
    """The page generator puts key j of sequence b where the block-table definition says and
    fills every other row."""
    w = wl.make_workload("pg", wl.TINY, [1, 1], [7, 0], seed=4)
    pc = wl.paged_cache(w, 4, seed=1, spare_pages=1)
    assert pc.block_table.shape == (2, 2) and np.all(pc.block_table[1] == -1)
    assert sorted(pc.block_table[0].tolist()) != [-1, -1]
    for j in range(7):
        row = pc.block_table[0, j // 4] * 4 + j % 4
        assert np.array_equal(pc.kv_cache[row], w.kv[j])
    assert np.isnan(pc.kv_cache).sum() == (3 * 4 - 7) * w.kv.shape[1]
