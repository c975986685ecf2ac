"""Host logic of sequence-parallel decode (deepseek_mla_latent_b200.seqpar) without a GPU: the
token ranges the ranks take, and the gather of the ranks' partials over two gloo ranks on CPU,
merged here with the log-sum-exp rule and compared with softmax attention over the whole cache."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from deepseek_mla_latent_b200 import seqpar


@pytest.mark.parametrize("lens,world", [([5, 0, 7, 1], 2), ([130, 1000, 3], 3), ([8], 8), ([3], 5)])
def test_shard_bounds_tile_every_sequence(lens, world):
    cu = np.concatenate([[0], np.cumsum(lens)])
    los, his = zip(*(seqpar.shard_bounds(cu, world, r) for r in range(world)))
    for b, t in enumerate(lens):
        # consecutive, non-overlapping, covering [cu[b], cu[b+1]), sizes within one of each other
        assert los[0][b] == cu[b] and his[-1][b] == cu[b + 1]
        for r in range(world - 1):
            assert his[r][b] == los[r + 1][b]
        sizes = [his[r][b] - los[r][b] for r in range(world)]
        assert min(sizes) >= 0 and max(sizes) - min(sizes) <= 1 and sum(sizes) == t


def _inputs(seed=0, B=3, H=2, C=8, lens=(9, 4, 13)):
    rng = np.random.default_rng(seed)
    cu = np.concatenate([[0], np.cumsum(lens)])
    q = rng.normal(size=(B, H, C))
    kv = rng.normal(size=(cu[-1], C))
    return q, kv, cu


def _partials(q, kv, cu, lo, hi, splits):
    """(O [S, B, H, C], (m, l) [S, B, H, 2]) over rows [lo[b], hi[b]) of each sequence, cut into
    `splits` consecutive pieces, in the layout the attention kernel writes (log2 units)."""
    B, H, C = q.shape
    o = np.zeros((splits, B, H, C))
    ml = np.zeros((splits, B, H, 2))
    ml[..., 0] = -np.inf
    for b in range(B):
        edges = np.linspace(lo[b], hi[b], splits + 1).astype(int)
        for s in range(splits):
            rows = kv[edges[s]:edges[s + 1]]
            if len(rows) == 0:
                continue
            x = (q[b] @ rows.T) * np.log2(np.e)          # [H, n]
            m = x.max(axis=1, keepdims=True)
            p = np.exp2(x - m)
            o[s, b] = p @ rows
            ml[s, b, :, 0], ml[s, b, :, 1] = m[:, 0], p.sum(axis=1)
    return o, ml


def _merge(o, ml):
    m = ml[..., 0]
    M = m.max(axis=0)
    w = np.where(np.isinf(m), 0.0, np.exp2(m - M))
    return (w[..., None] * o).sum(axis=0) / (w * ml[..., 1]).sum(axis=0)[..., None]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        q, kv, cu = _inputs()
        lo, hi = seqpar.shard_bounds(cu, world, rank)
        o, ml = _partials(q, kv, cu, lo, hi, splits=2)
        o_all, ml_all = seqpar.gather_partials(torch.from_numpy(o).float(), torch.from_numpy(ml).float())
        out[rank] = (o_all.double().numpy(), ml_all.double().numpy())
    finally:
        dist.destroy_process_group()


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_gathered_partials_merge_to_attention_over_the_whole_cache():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    out = ctx.Manager().dict()
    mp.start_processes(_worker, args=(world, port, out), nprocs=world, join=True, start_method="spawn")
    q, kv, cu = _inputs()
    # every rank holds the same stack: rank 0's two splits, then rank 1's
    for r in range(world):
        np.testing.assert_array_equal(out[r][0], out[0][0])
        np.testing.assert_array_equal(out[r][1], out[0][1])
    o_all, ml_all = out[0]
    for r in range(world):
        lo, hi = seqpar.shard_bounds(cu, world, r)
        o, ml = _partials(q, kv, cu, lo, hi, splits=2)
        np.testing.assert_allclose(o_all[2 * r:2 * r + 2], o, rtol=1e-6, atol=1e-6)
    got = _merge(o_all, ml_all)
    for b in range(len(cu) - 1):
        rows = kv[cu[b]:cu[b + 1]]
        s = q[b] @ rows.T
        p = np.exp(s - s.max(axis=1, keepdims=True))
        ref = (p / p.sum(axis=1, keepdims=True)) @ rows
        np.testing.assert_allclose(got[b], ref, rtol=1e-5, atol=1e-6)


def test_local_cache_takes_each_sequences_range_in_order():
    """local_cache packs rank r's rows of every sequence, in sequence order, with its cu_seqlens
    and longest range (CPU tensors: the index arithmetic is the same on any device)."""
    lens = [7, 0, 12, 3]
    cu = np.concatenate([[0], np.cumsum(lens)])
    kv = torch.arange(cu[-1] * 4, dtype=torch.float32).view(-1, 4)
    pe = torch.arange(cu[-1] * 2, dtype=torch.float32).view(-1, 2) + 1000
    world = 3
    for r in range(world):
        kv_r, pe_r, cu_r, max_r = seqpar.local_cache(kv, pe, cu, world, r)
        lo, hi = seqpar.shard_bounds(cu, world, r)
        rows = np.concatenate([np.arange(a, b) for a, b in zip(lo, hi)])
        assert torch.equal(kv_r, kv[rows]) and torch.equal(pe_r, pe[rows])
        assert cu_r.tolist() == [0] + np.cumsum(hi - lo).tolist()
        assert max_r == int((hi - lo).max())
