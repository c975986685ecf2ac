"""GPU parity of attention over a paged latent cache (mla_attn_paged) against the fp64
oracle, on seeded workloads scattered into randomly placed pages whose unused rows hold NaN."""
import numpy as np
import pytest
import torch

import oracle
from deepseek_mla_latent_b200 import workloads as wl

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    from deepseek_mla_latent_b200 import mla
    from gpu_util import assert_close, is_decode, run_path, to_dev

V3 = wl.V3


def _paged_dev(w, pc):
    dt = torch.bfloat16 if w.dims.dtype == "bf16" else torch.float32
    t = lambda a, ty=dt: torch.from_numpy(np.ascontiguousarray(a)).to(device="cuda", dtype=ty)
    return dict(kv=t(pc.kv_cache), pe=t(pc.pe_cache), table=t(pc.block_table, torch.int32),
                seqlens=t(pc.seqlens_k, torch.int32))


def _run_paged(w, pc, num_splits=0):
    """absorb_q -> mla_attn_paged -> out_proj; host float64 (o_lat, out)."""
    d = mla.dims_from(w.dims)
    dev = to_dev(w)
    pg = _paged_dev(w, pc)
    q_abs = mla.absorb_q(d, dev["q"], dev["wkv_b"])
    cu_q = None if is_decode(w) else dev["cu_q"]
    o_lat = mla.attn_paged(d, q_abs, dev["q"], pg["seqlens"], dev["max_k"], pg["kv"], pg["pe"], pg["table"],
                           pc.page_size, cu_seqlens_q=cu_q, num_splits=num_splits)
    out = mla.out_proj(d, o_lat, dev["wkv_b"])
    mla.device_status()
    f = lambda x: x.float().cpu().numpy().astype(np.float64)
    return f(o_lat), f(out)


def _oracle_paged(w, pc, pairs=None):
    d = w.dims
    return oracle.mla_naive_paged(w.q, pc.kv_cache, pc.pe_cache, pc.block_table, pc.seqlens_k, pc.page_size,
                                  w.wkv_b, w.cu_seqlens_q, d.heads, d.qk_nope, d.qk_rope, d.v_head, d.scale,
                                  pairs=pairs)


@pytest.mark.parametrize("page", [64, 128, 192, 256])
def test_v3_paged_decode_matches_oracle_and_packed(page):
    """Ragged decode over 1..4096 keys: the oracle within tolerance, and bit for bit the packed
    path (the same keys reach the same shared-memory layout; only the rows copied differ)."""
    w = wl.make_workload("v3pg", V3, [1] * 5, [1, 200, 777, 4096, 33], seed=11)
    pc = wl.paged_cache(w, page, seed=page, spare_pages=3, extra_columns=2)
    o_lat, out = _run_paged(w, pc)
    assert_close(out, _oracle_paged(w, pc), "bf16", f"paged out, page {page}")
    packed = run_path(w)
    assert np.array_equal(o_lat, packed["o_lat"])


@pytest.mark.parametrize("splits", [1, 7, 64])
def test_v3_paged_splits(splits):
    w = wl.make_workload("v3pgs", V3, [1, 1], [1000, 260], seed=12)
    pc = wl.paged_cache(w, 64, seed=splits, spare_pages=1)
    _, out = _run_paged(w, pc, splits)
    assert_close(out, _oracle_paged(w, pc), "bf16", f"splits {splits}")


def test_v3_paged_empty_sequences_give_zeros():
    w = wl.make_workload("v3pge", V3, [1, 1, 1], [0, 70, 0], seed=13)
    pc = wl.paged_cache(w, 64, seed=2, spare_pages=2, extra_columns=1)
    _, out = _run_paged(w, pc)
    assert np.all(out[0] == 0) and np.all(out[2] == 0)
    assert_close(out, _oracle_paged(w, pc), "bf16", "out")


@pytest.mark.parametrize("page", [64, 128])
def test_v3_paged_prefill_causal(page):
    w = wl.make_workload("v3pgp", V3, [5, 130, 1], [300, 700, 64], seed=14)
    pc = wl.paged_cache(w, page, seed=3, spare_pages=2)
    o_lat, out = _run_paged(w, pc)
    assert_close(out, _oracle_paged(w, pc), "bf16", f"paged prefill, page {page}")
    assert np.array_equal(o_lat, run_path(w)["o_lat"])


@pytest.mark.parametrize("page", [1, 3, 64])
def test_fp32_paged(page):
    """The CUDA-core kernels (fp32) take any page size."""
    w = wl.make_workload("f32pg", wl.TINY, [1, 1, 1], [1, 300, 129], seed=15)
    pc = wl.paged_cache(w, page, seed=4, spare_pages=2, extra_columns=1)
    _, out = _run_paged(w, pc, 3)
    assert_close(out, _oracle_paged(w, pc), "f32", f"fp32 paged, page {page}")


def test_fp32_paged_prefill():
    w = wl.make_workload("f32pgp", wl.TINY, [4, 9], [4, 200], seed=16)
    pc = wl.paged_cache(w, 16, seed=5)
    _, out = _run_paged(w, pc)
    assert_close(out, _oracle_paged(w, pc), "f32", "fp32 paged prefill")


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_entry_outside_the_cache_is_reported(dtype):
    """A table entry past the cache reads as zeros and sets the page bit of the device error
    word; the other sequences are unaffected and nothing faults."""
    dims = V3 if dtype == "bf16" else wl.TINY
    w = wl.make_workload("pgbad", dims, [1, 1], [300, 150], seed=17)
    pc = wl.paged_cache(w, 64, seed=6)
    bad = pc.block_table.copy()
    bad[1, 1] = pc.num_pages + 5
    pc_bad = wl.PagedCache(pc.page_size, pc.kv_cache, pc.pe_cache, bad, pc.seqlens_k)
    d = mla.dims_from(w.dims)
    dev = to_dev(w)
    pg = _paged_dev(w, pc_bad)
    q_abs = mla.absorb_q(d, dev["q"], dev["wkv_b"])
    o_lat = mla.attn_paged(d, q_abs, dev["q"], pg["seqlens"], dev["max_k"], pg["kv"], pg["pe"], pg["table"], 64)
    out = mla.out_proj(d, o_lat, dev["wkv_b"])
    with pytest.raises(mla.MlaError) as e:
        mla.device_status()
    assert "0x80" in str(e.value)
    assert mla.device_status() == 0   # the word was cleared
    got = out.float().cpu().numpy().astype(np.float64)
    ref = _oracle_paged(w, pc, pairs=[(0, h) for h in range(dims.heads)])
    for (b, h), r in ref.items():
        assert_close(got[b:b + 1, h, :], r, dims.dtype, f"seq {b} head {h}")
    assert np.all(np.isfinite(got[1]))


def test_full_v3_decode_paged_sampled():
    """Batch 8 x 4096 keys in 64-key pages (the benchmark's paged configuration), checked on
    (sequence, head) pairs the oracle computes one by one, and bit for bit against the packed path."""
    w = wl.workload(1)
    pc = wl.paged_cache(w, 64, seed=0, spare_pages=16)
    o_lat, out = _run_paged(w, pc)
    ref = _oracle_paged(w, pc, pairs=[(0, 0), (4, 77), (7, 127)])
    for (b, h), r in ref.items():
        assert_close(out[b:b + 1, h, :], r, "bf16", f"seq {b} head {h}")
    assert np.array_equal(o_lat, run_path(w)["o_lat"])


def test_v3_block_sparse_decode_selection():
    """Block-sparse decode: each sequence attends to 20 of its pages, chosen at random and
    listed in random order (a selection like a sparse-attention indexer's), given to
    mla_attn_paged as the block table; against the oracle over the same selection.  The
    split plan is made for the full length (4096), so most splits are empty."""
    w = wl.make_workload("v3sp", V3, [1, 1], [4096, 2048], seed=18)
    pc = wl.paged_cache(w, 64, seed=7)
    rng = np.random.default_rng(1)
    sel = np.full((2, 20), -1, dtype=np.int32)
    for b, t in enumerate(w.seqlens_k):
        sel[b] = pc.block_table[b, rng.choice(t // 64, size=20, replace=False)]
    sp = wl.PagedCache(64, pc.kv_cache, pc.pe_cache, sel, np.full(2, 20 * 64, dtype=np.int32))
    _, out = _run_paged(w, sp)
    assert_close(out, _oracle_paged(w, sp), "bf16", "block-sparse decode")
