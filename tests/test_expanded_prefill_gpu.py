"""GPU parity of the naive-path chunked prefill: the latent KV expansion (mla_expand_kv) over the
packed cache, then per-head attention over the expanded keys and values
(mla_attn_prefill_expanded), against the fp64 naive-path oracle over the normalised cache."""
import numpy as np
import pytest
import torch

import oracle
from deepseek_mla_latent_b200 import workloads as wl

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    from deepseek_mla_latent_b200 import mla
    from gpu_util import assert_close, to_dev

EPS = 1e-6


def _naive_on_gpu(w, dev=None):
    """out [n_q, H, Dv] of the naive path on the GPU: the cache rows are the compressed KV that
    the expansion normalises (the workload's rows are already RMS-normalised; the oracle below
    normalises them again in the same way)."""
    d = mla.dims_from(w.dims)
    dev = dev or to_dev(w)
    T = dev["kv"].shape[0]
    k, v = mla.expand_kv(d, dev["kv"], dev["wkv_b"], 1, T, eps=EPS)
    out = mla.attn_prefill_expanded(d, dev["q"], k[0], v[0], dev["pe"], dev["cu_q"], dev["cu_k"], dev["max_q"])
    mla.device_status()
    return out.float().cpu().numpy().astype(np.float64)


def _oracle(w, pairs=None):
    kv = oracle.rms_norm(w.kv, None, EPS)
    dd = w.dims
    return oracle.mla_naive(w.q, kv, w.pe, w.wkv_b, w.cu_seqlens_q, w.cu_seqlens_k, dd.heads, dd.qk_nope,
                            dd.qk_rope, dd.v_head, dd.scale, pairs=pairs)


@pytest.mark.parametrize("sq,sk", [([5, 130], [300, 700]), ([128], [128]), ([1, 257], [1, 1000]),
                                   ([3, 0, 64], [64, 10, 200]), ([300], [300])])
def test_v3_expanded_prefill_causal(sq, sk):
    """Ragged chunks (several 128-row query tiles with a ragged last one, a chunk that is the
    whole cache, an empty chunk), whole output compared."""
    w = wl.make_workload("v3x", wl.V3, sq, sk, seed=21)
    assert_close(_naive_on_gpu(w), _oracle(w), "bf16", "out")


def test_v3_expanded_prefill_equals_absorb_path():
    """The two paths on the same cache agree (the pages: naive and absorb are mathematically
    identical); both against the oracle."""
    w = wl.make_workload("v3xa", wl.V3, [77, 200], [500, 256], seed=22)
    from gpu_util import run_path
    a = run_path(w)["out"]
    b = _naive_on_gpu(w)
    ref = _oracle(w)
    assert_close(a, ref, "bf16", "absorb path")
    assert_close(b, ref, "bf16", "naive path")


def test_v3_expanded_decode_rows():
    """One query per sequence (a decode step through the naive path)."""
    w = wl.make_workload("v3xd", wl.V3, [1, 1, 1], [1, 129, 1000], seed=23)
    assert_close(_naive_on_gpu(w), _oracle(w), "bf16", "out")


def test_full_expanded_prefill_sampled():
    """The chunked-prefill workload at full size (4 x 1024 queries after a 3072-token prefix), in
    the benchmark's launch configuration, checked on (sequence, head) pairs the oracle computes
    one by one: one head of every sequence (all its query rows) and heads 0, 63, 64, 127 of one."""
    w = wl.workload(4)
    got = _naive_on_gpu(w)
    rng = np.random.default_rng(24)
    pairs = sorted({(b, int(rng.integers(0, 128))) for b in range(4)} | {(1, h) for h in (0, 63, 64, 127)})
    ref = _oracle(w, pairs=pairs)
    cq = w.cu_seqlens_q
    for (b, h), r in ref.items():
        assert_close(got[cq[b]:cq[b + 1], h, :], r, "bf16", f"seq {b} head {h}")
