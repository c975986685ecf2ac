"""GPU parity: the library's CUDA path against the fp64 oracle on the same seeded inputs."""
import numpy as np
import pytest
import torch

import oracle
from deepseek_mla_latent_b200 import workloads as wl

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    from deepseek_mla_latent_b200 import mla
    from gpu_util import TOL, assert_close, run_path, to_dev


def _check_full(w, num_splits=0):
    got = run_path(w, num_splits=num_splits)
    q_abs, o_lat, _ = oracle.workload_absorb(w)
    ref = oracle.workload_naive(w)
    dt = w.dims.dtype
    assert_close(got["q_abs"], q_abs, dt, "q_abs")
    assert_close(got["o_lat"], o_lat, dt, "o_lat")
    return assert_close(got["out"], ref, dt, "out")


def test_tiny_fp32_workload():
    """Workload 0 in full: fp32 path within 1e-5 relative of the fp64 oracle."""
    _check_full(wl.workload(0))


@pytest.mark.parametrize("splits", [0, 1, 3])
def test_fp32_small_decode_and_splits(splits):
    w = wl.make_workload("f32", wl.TINY, [1, 1, 1], [1, 300, 129], seed=1)
    _check_full(w, splits)


def test_fp32_prefill():
    w = wl.make_workload("f32p", wl.TINY, [4, 9], [4, 200], seed=2)
    _check_full(w)


V3 = wl.V3


@pytest.mark.parametrize("seqlens", [[1, 200, 777], [129], [4096, 33]])
def test_v3_decode_ragged(seqlens):
    """DeepSeek-V3 shapes, several 128-key tiles with ragged tails, whole output compared."""
    w = wl.make_workload("v3d", V3, [1] * len(seqlens), seqlens, seed=3)
    _check_full(w)


@pytest.mark.parametrize("splits", [1, 2, 7, 64])
def test_v3_decode_split_invariance(splits):
    w = wl.make_workload("v3s", V3, [1, 1], [1000, 260], seed=4)
    _check_full(w, splits)


def test_v3_decode_more_splits_than_keys():
    w = wl.make_workload("v3k", V3, [1, 1, 1], [1, 2, 5], seed=5)
    _check_full(w, 8)


def test_v3_decode_empty_sequence_gives_zeros():
    w = wl.make_workload("v3e", V3, [1, 1, 1], [0, 70, 0], seed=6)
    got = run_path(w)
    assert np.all(got["out"][0] == 0) and np.all(got["out"][2] == 0)
    ref = oracle.workload_naive(w)
    assert_close(got["out"], ref, "bf16", "out")


@pytest.mark.parametrize("sq,sk", [([5, 130], [300, 700]), ([128], [128]), ([1, 257], [1, 1000]),
                                   ([3, 0, 64], [64, 10, 200])])
def test_v3_prefill_causal(sq, sk):
    w = wl.make_workload("v3p", V3, sq, sk, seed=7)
    _check_full(w)


def test_v3_prefill_equals_decode_for_single_query():
    w = wl.make_workload("v3pd", V3, [1, 1], [500, 77], seed=8)
    a = run_path(w, decode=True)["out"]
    b = run_path(w, decode=False)["out"]
    ref = oracle.workload_naive(w)
    assert_close(a, ref, "bf16", "decode")
    assert_close(b, ref, "bf16", "prefill")


def _sampled(index, pairs, num_splits=0):
    """A full-size workload run in the benchmark's launch configuration, checked
    on (sequence, head) pairs the oracle computes one by one."""
    w = wl.workload(index)
    got = run_path(w, num_splits=num_splits)["out"]
    ref = oracle.workload_naive(w, pairs=pairs)
    cq = w.cu_seqlens_q
    for (b, h), r in ref.items():
        assert_close(got[cq[b]:cq[b + 1], h, :], r, w.dims.dtype, f"workload {index} seq {b} head {h}")


def _cover_rows(n_seq, H, seed, row=0):
    """One head per sequence (spread over the heads by a seeded draw) plus heads 0, 63, 64 and
    127 of one sequence: every sequence, and with it every split unit of every row, is compared."""
    rng = np.random.default_rng(seed)
    pairs = {(b, int(rng.integers(0, H))) for b in range(n_seq)}
    pairs |= {(row, h) for h in (0, H // 2 - 1, H // 2, H - 1)}
    return sorted(pairs)


def test_full_v3_decode_sampled():
    _sampled(1, _cover_rows(8, 128, seed=11, row=3))


def test_full_ragged_sampled():
    _, _, _, sk = wl.workload_shape(2)
    longest, shortest = int(np.argmax(sk)), int(np.argmin(sk))
    pairs = set(_cover_rows(len(sk), 128, seed=12, row=longest)) | {(shortest, 100)}
    _sampled(2, sorted(pairs))


def test_full_long_context_sampled():
    _sampled(3, _cover_rows(2, 128, seed=13, row=1))


def test_full_prefill_sampled():
    """Every sequence of the chunked-prefill workload (all of its query rows, first and last
    included, are compared for each pair), heads 0, 63, 64 and 127 of one of them."""
    _sampled(4, _cover_rows(4, 128, seed=14, row=2))


def _decode_out(w, num_splits=0):
    d = mla.dims_from(w.dims)
    dev = to_dev(w)
    q_abs = mla.absorb_q(d, dev["q"], dev["wkv_b"])
    out = mla.attn_decode_out(d, q_abs, dev["q"], dev["kv"], dev["pe"], dev["cu_k"], dev["max_k"], dev["wkv_b"],
                              num_splits=num_splits)
    mla.device_status()
    return out.float().cpu().numpy().astype(np.float64)


@pytest.mark.parametrize("seqlens,splits", [([1, 200, 777], 0), ([4096, 33], 0), ([1000, 260], 7), ([0, 70, 0], 0)])
def test_v3_decode_out_matches_oracle_and_the_two_calls(seqlens, splits):
    """mla_attn_decode_out against the oracle, and bit for bit against mla_attn_decode + mla_out_proj
    (the same kernels on the same inputs)."""
    w = wl.make_workload("v3o", V3, [1] * len(seqlens), seqlens, seed=9)
    got = _decode_out(w, splits)
    assert_close(got, oracle.workload_naive(w), "bf16", "out")
    two = run_path(w, num_splits=splits)["out"]
    assert np.array_equal(got, two)


def test_fp32_decode_out():
    w = wl.make_workload("f32o", wl.TINY, [1, 1], [300, 5], seed=10)
    assert_close(_decode_out(w), oracle.workload_naive(w), "f32", "out")


def test_full_v3_decode_out_sampled():
    """The benchmark's launch configuration (mla_attn_decode_out at the full V3 decode size),
    checked on (sequence, head) pairs the oracle computes one by one: one head of every
    sequence and heads 0, 63, 64 and 127 of one."""
    w = wl.workload(1)
    got = _decode_out(w)
    ref = oracle.workload_naive(w, pairs=_cover_rows(8, 128, seed=15, row=5))
    for (b, h), r in ref.items():
        assert_close(got[b:b + 1, h, :], r, "bf16", f"seq {b} head {h}")


@pytest.mark.parametrize("seqlens,splits", [([1000, 260, 0], 7), ([4096, 33], 0), ([300, 5], 1)])
def test_v3_decode_partials_merge_to_the_decode_result(seqlens, splits):
    """mla_attn_decode_partials: the partial form, merged here by the log-sum-exp rule the header
    states, equals the oracle's o_lat; splits without keys carry m = -inf and l = 0."""
    w = wl.make_workload("v3part", V3, [1] * len(seqlens), seqlens, seed=16)
    d = mla.dims_from(w.dims)
    dev = to_dev(w)
    q_abs = mla.absorb_q(d, dev["q"], dev["wkv_b"])
    ws = mla.attn_decode_partials(d, q_abs, dev["q"], dev["kv"], dev["pe"], dev["cu_k"], dev["max_k"],
                                  num_splits=splits)
    mla.device_status()
    S = mla.decode_num_splits(d, w.batch, dev["max_k"], splits)
    o, ml = mla.split_partials(d, ws, w.batch, S)
    o = o.float().cpu().numpy().astype(np.float64)
    ml = ml.cpu().numpy().astype(np.float64)
    m, l = ml[..., 0], ml[..., 1]
    M = np.max(m, axis=0)
    wgt = np.where(np.isfinite(m), np.exp2(m - np.where(np.isfinite(M), M, 0.0)), 0.0)
    den = np.sum(wgt * l, axis=0)
    num = np.sum(wgt[..., None] * np.where(wgt[..., None] > 0, o, 0.0), axis=0)
    merged = np.where(den[..., None] > 0, num / np.where(den > 0, den, 1.0)[..., None], 0.0)
    _, o_lat, _ = oracle.workload_absorb(w)
    assert_close(merged, o_lat, "bf16", "merged partials")
    for b, t in enumerate(seqlens):
        if t == 0:
            assert np.all(np.isneginf(m[:, b])) and np.all(l[:, b] == 0)
