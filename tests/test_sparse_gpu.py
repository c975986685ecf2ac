"""GPU parity of token-granular sparse decode (mla_attn_sparse_decode): attention over a selected
list of cache rows per sequence, against the fp64 oracle of the same selection."""
import numpy as np
import pytest
import torch

import oracle
from deepseek_mla_latent_b200 import workloads as wl

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    from deepseek_mla_latent_b200 import mla
    from gpu_util import assert_close, to_dev


def _run(w, idx, counts, num_splits=0, dev=None):
    d = mla.dims_from(w.dims)
    dev = dev or to_dev(w)
    q_abs = mla.absorb_q(d, dev["q"], dev["wkv_b"])
    ti = torch.from_numpy(np.ascontiguousarray(idx, dtype=np.int32)).cuda()
    tc = torch.from_numpy(np.ascontiguousarray(counts, dtype=np.int32)).cuda()
    o_lat = mla.attn_sparse_decode(d, q_abs, dev["q"], dev["kv"], dev["pe"], ti, tc, num_splits=num_splits)
    out = mla.out_proj(d, o_lat, dev["wkv_b"])
    mla.device_status()
    return out.float().cpu().numpy().astype(np.float64)


def _ref(w, idx, counts, pairs=None):
    d = w.dims
    return oracle.mla_naive_sparse(w.q, w.kv, w.pe, idx, counts, w.wkv_b, d.heads, d.qk_nope, d.qk_rope, d.v_head,
                                   d.scale, pairs=pairs)


def _random_selection(w, topk, seed, any_row=False):
    """Per sequence, `topk` distinct rows of its own keys (or of the whole cache) in random order;
    the count is min(topk, keys).  Unused entries are -1."""
    rng = np.random.default_rng(seed)
    idx = np.full((w.batch, topk), -1, dtype=np.int64)
    counts = []
    cu = w.cu_seqlens_k
    total = int(cu[-1])
    for b in range(w.batch):
        pool = np.arange(total) if any_row else np.arange(cu[b], cu[b + 1])
        n = min(topk, len(pool))
        idx[b, :n] = rng.choice(pool, size=n, replace=False)
        counts.append(n)
    return idx, counts


@pytest.mark.parametrize("dims,seqlens,topk", [("v3", [1000, 260, 70], 300), ("v3", [4096, 129], 2048),
                                                ("v3", [50, 5000], 1), ("tiny", [300, 5], 64)])
def test_sparse_decode_random_selection(dims, seqlens, topk):
    """Random selections of a sequence's own rows (several 128-key tiles, ragged counts, a
    single key), bf16 tensor-core path and fp32 CUDA-core path."""
    w = wl.make_workload("sp", wl.V3 if dims == "v3" else wl.TINY, [1] * len(seqlens), seqlens, seed=41)
    idx, counts = _random_selection(w, topk, seed=1)
    assert_close(_run(w, idx, counts), _ref(w, idx, counts), w.dims.dtype, "out")


def test_sparse_decode_rows_from_anywhere_and_repeats():
    """Rows may come from anywhere in the cache, a repeated row counts twice, and a sequence
    may select nothing (zeros)."""
    w = wl.make_workload("spx", wl.V3, [1, 1, 1], [700, 300, 10], seed=42)
    idx, counts = _random_selection(w, 200, seed=2, any_row=True)
    idx[0, 5] = idx[0, 6]
    counts[2] = 0
    got = _run(w, idx, counts)
    assert np.all(got[2] == 0)
    assert_close(got, _ref(w, idx, counts), "bf16", "out")


@pytest.mark.parametrize("splits", [1, 3])
def test_sparse_decode_all_rows_in_order_equals_dense_bit_for_bit(splits):
    """Top-k = all, in cache order: the gathered rows are the packed cache itself, so the result
    equals mla_attn_decode with the same split plan bit for bit."""
    w = wl.make_workload("spd", wl.V3, [1, 1], [1000, 260], seed=43)
    dev = to_dev(w)
    d = mla.dims_from(w.dims)
    cu = w.cu_seqlens_k
    topk = max(w.seqlens_k)
    idx = np.full((w.batch, topk), -1, dtype=np.int64)
    for b in range(w.batch):
        idx[b, :w.seqlens_k[b]] = np.arange(cu[b], cu[b + 1])
    got = _run(w, idx, w.seqlens_k, num_splits=splits, dev=dev)
    q_abs = mla.absorb_q(d, dev["q"], dev["wkv_b"])
    o = mla.attn_decode(d, q_abs, dev["q"], dev["kv"], dev["pe"], dev["cu_k"], dev["max_k"], num_splits=splits)
    dense = mla.out_proj(d, o, dev["wkv_b"]).float().cpu().numpy().astype(np.float64)
    mla.device_status()
    assert np.array_equal(got, dense)


def test_sparse_decode_row_outside_the_cache_is_reported():
    """A used entry outside the cache reads as zeros and raises bit 1<<7 of the device error word;
    the next call runs clean."""
    w = wl.make_workload("spe", wl.V3, [1, 1], [300, 200], seed=44)
    dev = to_dev(w)
    d = mla.dims_from(w.dims)
    q_abs = mla.absorb_q(d, dev["q"], dev["wkv_b"])
    idx = np.array([[0, 1, 10 ** 6], [300, 301, -1]], dtype=np.int32)
    ti, tc = torch.from_numpy(idx).cuda(), torch.tensor([3, 2], dtype=torch.int32).cuda()
    mla.attn_sparse_decode(d, q_abs, dev["q"], dev["kv"], dev["pe"], ti, tc)
    from deepseek_mla_latent_b200 import _lib
    with pytest.raises(_lib.MlaError) as e:
        mla.device_status()
    assert e.value.status == _lib.MLA_ERR_DEVICE_TIMEOUT
    tc2 = torch.tensor([2, 2], dtype=torch.int32).cuda()
    o = mla.attn_sparse_decode(d, q_abs, dev["q"], dev["kv"], dev["pe"], ti, tc2)
    out = mla.out_proj(d, o, dev["wkv_b"]).float().cpu().numpy().astype(np.float64)
    mla.device_status()
    assert_close(out, _ref(w, idx, [2, 2]), "bf16", "out")


def test_full_sparse_decode_sampled():
    """The DeepSeek-V3 decode workload (8 x 4096 keys) with 2048 selected rows per sequence, in
    the benchmark's launch configuration, checked on one head of every sequence and heads 0, 63,
    64, 127 of one."""
    w = wl.workload(1)
    idx, counts = _random_selection(w, 2048, seed=3)
    got = _run(w, idx, counts)
    rng = np.random.default_rng(45)
    pairs = sorted({(b, int(rng.integers(0, 128))) for b in range(8)} | {(6, h) for h in (0, 63, 64, 127)})
    ref = _ref(w, idx, counts, pairs=pairs)
    for (b, h), r in ref.items():
        assert_close(got[b:b + 1, h, :], r, "bf16", f"seq {b} head {h}")
