"""GPU parity of sequence-parallel decode: each sequence's cache cut into token ranges (as the
ranks of a group would hold them), the partial form over each range, the partials stacked along
the split axis and merged (mla_merge_partials, mla_merge_partials_out), against the fp64 oracle
over the whole cache; and the collective path itself over a one-rank NCCL group."""
import datetime
import socket

import numpy as np
import pytest
import torch

import oracle
from deepseek_mla_latent_b200 import workloads as wl

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    from deepseek_mla_latent_b200 import mla, seqpar
    from gpu_util import assert_close, to_dev


def _emulated_ranks(w, world, splits, fused):
    d = mla.dims_from(w.dims)
    dev = to_dev(w)
    q_abs = mla.absorb_q(d, dev["q"], dev["wkv_b"])
    os_, mls = [], []
    for r in range(world):
        kv_r, pe_r, cu_r, max_r = seqpar.local_cache(dev["kv"], dev["pe"], w.cu_seqlens_k, world, r)
        ws = mla.attn_decode_partials(d, q_abs, dev["q"], kv_r, pe_r, cu_r, max_r, num_splits=splits)
        o, ml = mla.split_partials(d, ws, w.batch, splits)
        os_.append(o.clone())
        mls.append(ml.clone())
    o_all, ml_all = torch.cat(os_), torch.cat(mls)
    if fused:
        out = mla.merge_partials_out(d, o_all, ml_all, dev["wkv_b"])
    else:
        out = mla.out_proj(d, mla.merge_partials(d, o_all, ml_all), dev["wkv_b"])
    mla.device_status()
    return out.float().cpu().numpy().astype(np.float64)


@pytest.mark.parametrize("world,splits,fused", [(2, 1, False), (3, 2, True), (4, 3, False), (8, 1, True)])
def test_ranges_merged_equal_attention_over_the_whole_cache(world, splits, fused):
    """Ragged sequences (one shorter than the number of ranges, so some ranges are empty) cut into
    `world` ranges of `splits` splits each."""
    w = wl.make_workload("sp", wl.V3, [1, 1, 1], [1000, 5, 300], seed=51)
    assert_close(_emulated_ranks(w, world, splits, fused), oracle.workload_naive(w), "bf16", "out")


def test_merge_of_nothing_is_zero_and_bad_split_counts_are_refused():
    """A row all of whose splits are empty (m = -inf, l = 0) gets zeros; 0 or 257 splits are refused."""
    d = mla.dims_from(wl.V3)
    o = torch.full((2, 1, 128, 512), float("nan"), dtype=torch.bfloat16, device="cuda")
    ml = torch.zeros(2, 1, 128, 2, dtype=torch.float32, device="cuda")
    ml[..., 0] = float("-inf")
    got = mla.merge_partials(d, o, ml)
    mla.device_status()
    assert torch.count_nonzero(got) == 0
    from deepseek_mla_latent_b200 import _lib
    import ctypes
    for s in (0, 257):
        st = _lib.LIB.mla_merge_partials(ctypes.byref(d), o.data_ptr(), ml.data_ptr(), s, 1, got.data_ptr(), None)
        assert st == _lib.MLA_ERR_INVALID_ARG


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_decode_sequence_parallel_over_a_one_rank_nccl_group():
    """The whole collective path (partials, NCCL all-gather, merge fused into the projection) on a
    group of one rank, against the oracle."""
    import torch.distributed as dist
    w = wl.make_workload("spn", wl.V3, [1, 1], [700, 129], seed=52)
    d = mla.dims_from(w.dims)
    dev = to_dev(w)
    q_abs = mla.absorb_q(d, dev["q"], dev["wkv_b"])
    kv_r, pe_r, cu_r, max_r = seqpar.local_cache(dev["kv"], dev["pe"], w.cu_seqlens_k, 1, 0)
    store = dist.TCPStore("127.0.0.1", _free_port(), 1, True, timeout=datetime.timedelta(seconds=30))
    dist.init_process_group("nccl", store=store, rank=0, world_size=1, timeout=datetime.timedelta(seconds=60))
    try:
        out = seqpar.decode_sequence_parallel(d, q_abs, dev["q"], kv_r, pe_r, cu_r, max_r, num_splits=3,
                                              wkv_b=dev["wkv_b"])
        o_lat = seqpar.decode_sequence_parallel(d, q_abs, dev["q"], kv_r, pe_r, cu_r, max_r, num_splits=3)
        torch.cuda.synchronize()
    finally:
        dist.destroy_process_group()
    mla.device_status()
    ref = oracle.workload_naive(w)
    assert_close(out.float().cpu().numpy().astype(np.float64), ref, "bf16", "out (fused merge)")
    assert_close(mla.out_proj(d, o_lat, dev["wkv_b"]).float().cpu().numpy().astype(np.float64), ref, "bf16",
                 "out (merge, then projection)")
