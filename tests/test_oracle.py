"""Pins for the fp64 oracle: each check rests on something other than the oracle itself
(a hand-worked example, closed forms, invariants, a library attention routine)."""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from oracle import mla_oracle
from deepseek_mla_latent_b200 import workloads as wl

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "two_head_worked_example.json")


def _golden():
    with open(GOLDEN) as f:
        g = json.load(f)
    a = {k: np.asarray(g[k], dtype=np.float64) for k in ("wkv_b", "kv", "pe")}
    return g, a


def _golden_outputs(fn_naive, fn_absorb):
    g, a = _golden()
    H, Dn, R, Dv = g["heads"], g["qk_nope"], g["qk_rope"], g["v_head"]
    scale = math.log(3.0)
    res = {}
    q = np.asarray(g["decode"]["q"], dtype=np.float64)
    cuq, cuk = np.array([0, 1]), np.array([0, 2])
    res["decode_naive"] = fn_naive(q, a["kv"], a["pe"], a["wkv_b"], cuq, cuk, H, Dn, R, Dv, scale)
    res["decode_absorb"] = fn_absorb(q, a["kv"], a["pe"], a["wkv_b"], cuq, cuk, H, Dn, R, Dv, scale)
    qp = np.asarray(g["prefill"]["q"], dtype=np.float64)
    res["prefill_naive"] = fn_naive(qp, a["kv"], a["pe"], a["wkv_b"], np.array([0, 2]), cuk, H, Dn, R, Dv, scale)
    return g, res


def _check_golden(g, res, tol=1e-12):
    np.testing.assert_allclose(res["decode_naive"], g["decode"]["out"], rtol=0, atol=tol)
    q_abs, o_lat, out = res["decode_absorb"]
    np.testing.assert_allclose(q_abs, g["decode"]["q_abs"], rtol=0, atol=tol)
    np.testing.assert_allclose(o_lat, g["decode"]["o_lat"], rtol=0, atol=tol)
    np.testing.assert_allclose(out, g["decode"]["out"], rtol=0, atol=tol)
    np.testing.assert_allclose(res["prefill_naive"], g["prefill"]["out"], rtol=0, atol=tol)


def test_golden_worked_example():
    g, res = _golden_outputs(oracle.mla_naive, oracle.mla_absorb)
    _check_golden(g, res)


# Planted mistakes: each is a plausible slip in the oracle; the hand-worked example must catch it.
def _mutants():
    orig_head_view = mla_oracle.head_view
    orig_naive_head = mla_oracle.naive_head
    orig_visible = mla_oracle.visible_keys

    def hv_swapped(w, H, Dn, Dv):
        wk, wv = orig_head_view(w, H, Dn, Dv)
        return wv, wk

    def hv_head_minor(w, H, Dn, Dv):  # wrong view order: [Dn+Dv, H, C]
        w = np.asarray(w, dtype=np.float64).reshape(Dn + Dv, H, -1).transpose(1, 0, 2)
        return w[:, :Dn], w[:, Dn:]

    def nh_no_pe(q, kv, pe, wk, wv, scale, return_probs=False):
        return orig_naive_head(q, kv, np.zeros_like(np.asarray(pe, dtype=np.float64)), wk, wv, scale, return_probs)

    def nh_no_scale(q, kv, pe, wk, wv, scale, return_probs=False):
        return orig_naive_head(q, kv, pe, wk, wv, 1.0, return_probs)

    def vis_top_left(t, s, i):
        return max(0, min(t, i + 1))

    def vis_no_mask(t, s, i):
        return t

    return [("head_view", hv_swapped), ("head_view", hv_head_minor), ("naive_head", nh_no_pe),
            ("naive_head", nh_no_scale), ("visible_keys", vis_top_left), ("visible_keys", vis_no_mask)]


@pytest.mark.parametrize("idx", range(6))
def test_golden_catches_planted_mistakes(monkeypatch, idx):
    name, fn = _mutants()[idx]
    monkeypatch.setattr(mla_oracle, name, fn)
    g, res = _golden_outputs(mla_oracle.mla_naive, mla_oracle.mla_absorb)
    with pytest.raises(AssertionError):
        _check_golden(g, res)


def _small(seed, sq, sk, dims=None, **kw):
    dims = dims or wl.Dims(heads=4, kv_lora_rank=32, qk_nope=16, qk_rope=8, v_head=16, dtype="bf16")
    return wl.make_workload("small", dims, sq, sk, seed=seed, **kw)


@pytest.mark.parametrize("seed,sq,sk", [(0, [1, 1, 1], [5, 17, 64]), (1, [3, 7], [3, 40]),
                                        (2, [1, 4, 0], [1, 9, 6]), (3, [16], [16])])
def test_naive_equals_absorb(seed, sq, sk):
    """The page's claim that both paths give the same output, held to fp64 rounding."""
    w = _small(seed, sq, sk)
    ref = oracle.workload_naive(w)
    _, _, out = oracle.workload_absorb(w)
    scale = np.max(np.abs(ref))
    assert np.max(np.abs(out - ref)) <= 1e-10 * scale


def test_naive_equals_absorb_v3_dims():
    w = wl.make_workload("v3small", wl.V3, [1, 2], [70, 33], seed=5)
    ref = oracle.workload_naive(w)
    _, _, out = oracle.workload_absorb(w)
    assert np.max(np.abs(out - ref)) <= 1e-10 * np.max(np.abs(ref))


def test_brute_force_scalar_expansion():
    """H=1, C=2, R=1, Dn=Dv=1, t=2, integer inputs, expanded by hand as scalar arithmetic."""
    wkv_b = np.array([[2.0, -1.0], [1.0, 3.0]])   # row 0 key, row 1 value
    kv = np.array([[1.0, 2.0], [-1.0, 1.0]])
    pe = np.array([[3.0], [-2.0]])
    q = np.array([[[1.0, 2.0]]])                  # q_nope = 1, q_pe = 2
    scale = 0.5
    k0 = 2 * 1 + (-1) * 2   # = 0
    k1 = 2 * (-1) + (-1) * 1  # = -3
    s0 = (1 * k0 + 2 * 3) * scale      # 3.0
    s1 = (1 * k1 + 2 * (-2)) * scale   # -3.5
    v0 = 1 * 1 + 3 * 2      # 7
    v1 = 1 * (-1) + 3 * 1   # 2
    e0, e1 = math.exp(s0 - s0), math.exp(s1 - s0)
    expect = (e0 * v0 + e1 * v1) / (e0 + e1)
    got = oracle.mla_naive(q, kv, pe, wkv_b, [0, 1], [0, 2], 1, 1, 1, 1, scale)
    assert abs(got[0, 0, 0] - expect) < 1e-14


def test_softmax_rows_sum_to_one():
    w = _small(7, [5], [23])
    d = w.dims
    wk, wv = oracle.head_view(w.wkv_b, d.heads, d.qk_nope, d.v_head)
    for h in range(d.heads):
        _, p = oracle.naive_head(w.q[:, h], w.kv, w.pe, wk[h], wv[h], d.scale, return_probs=True)
        assert np.all(p >= 0)
        np.testing.assert_allclose(p.sum(axis=1), 1.0, rtol=0, atol=1e-12)
        # causal, aligned to the end: query i of 5 sees 23 - 5 + i + 1 keys
        for i in range(5):
            assert np.all(p[i, 23 - 5 + i + 1:] == 0)
            assert p[i, 23 - 5 + i] > 0


def test_single_token_returns_projected_value():
    """t = 1: whatever q is, the output is W_v[h] . kv[0]."""
    w = _small(11, [1], [1])
    d = w.dims
    _, wv = oracle.head_view(w.wkv_b, d.heads, d.qk_nope, d.v_head)
    out = oracle.workload_naive(w)
    expect = np.einsum("hdc,c->hd", wv, w.kv[0].astype(np.float64))
    np.testing.assert_allclose(out[0], expect, rtol=1e-13, atol=1e-13)


def test_zero_scale_gives_mean_value():
    dims = wl.Dims(heads=3, kv_lora_rank=16, qk_nope=8, qk_rope=4, v_head=8, dtype="bf16", softmax_scale=0.0)
    w = wl.make_workload("s0", dims, [1], [37], seed=2)
    _, wv = oracle.head_view(w.wkv_b, dims.heads, dims.qk_nope, dims.v_head)
    out = oracle.workload_naive(w)
    expect = np.einsum("hdc,c->hd", wv, w.kv.astype(np.float64).mean(axis=0))
    np.testing.assert_allclose(out[0], expect, rtol=1e-12, atol=1e-13)


def test_constant_cache_is_query_independent():
    w = _small(4, [2, 1], [9, 12])
    w.kv[:] = w.kv[0]
    d = w.dims
    _, wv = oracle.head_view(w.wkv_b, d.heads, d.qk_nope, d.v_head)
    out = oracle.workload_naive(w)
    expect = np.einsum("hdc,c->hd", wv, w.kv[0].astype(np.float64))
    for n in range(out.shape[0]):
        np.testing.assert_allclose(out[n], expect, rtol=1e-12, atol=1e-13)


def test_decode_permutation_invariance():
    w = _small(9, [1], [50])
    ref = oracle.workload_naive(w)
    perm = np.random.default_rng(0).permutation(50)
    w.kv, w.pe = w.kv[perm], w.pe[perm]
    np.testing.assert_allclose(oracle.workload_naive(w), ref, rtol=1e-12, atol=1e-14)


def test_prefill_row_equals_decode_on_prefix():
    s, t = 6, 20
    w = _small(13, [s], [t])
    out = oracle.workload_naive(w)
    d = w.dims
    for i in range(s):
        n = t - s + i + 1
        dec = oracle.mla_naive(w.q[i:i + 1], w.kv[:n], w.pe[:n], w.wkv_b, [0, 1], [0, n], d.heads,
                               d.qk_nope, d.qk_rope, d.v_head, d.scale)
        np.testing.assert_allclose(out[i], dec[0], rtol=1e-12, atol=1e-14)


@pytest.mark.parametrize("sq,sk", [([1, 1], [31, 8]), ([5, 3], [12, 3])])
def test_latent_attention_matches_library_sdpa(sq, sk):
    """o_lat is multi-query attention with key [kv ; pe], value kv and query [q_abs ; q_pe];
    torch's scaled_dot_product_attention (fp64, CPU) with an explicit end-aligned mask must agree."""
    w = _small(21, sq, sk)
    d = w.dims
    q_abs, o_lat, _ = oracle.workload_absorb(w)
    cq, ck = w.cu_seqlens_q, w.cu_seqlens_k
    for b in range(w.batch):
        q0, q1, k0, k1 = cq[b], cq[b + 1], ck[b], ck[b + 1]
        s, t = q1 - q0, k1 - k0
        qq = torch.from_numpy(np.concatenate([q_abs[q0:q1], w.q[q0:q1, :, d.qk_nope:].astype(np.float64)], -1))
        kk = torch.from_numpy(np.concatenate([w.kv[k0:k1], w.pe[k0:k1]], -1).astype(np.float64))
        vv = torch.from_numpy(w.kv[k0:k1].astype(np.float64))
        mask = torch.tensor([[j <= t - s + i for j in range(t)] for i in range(s)])
        ref = torch.nn.functional.scaled_dot_product_attention(
            qq.permute(1, 0, 2), kk.expand(d.heads, t, -1), vv.expand(d.heads, t, -1),
            attn_mask=mask, scale=d.scale).permute(1, 0, 2).numpy()
        np.testing.assert_allclose(o_lat[q0:q1], ref, rtol=1e-10, atol=1e-12)


def test_empty_sequence_gives_zeros():
    """A decode query over an empty cache has no visible key: its output is zero, and the
    neighbouring sequence is unaffected."""
    w = _small(3, [1, 1], [0, 4])
    out = oracle.workload_naive(w)
    assert np.all(out[0] == 0)
    d = w.dims
    alone = oracle.mla_naive(w.q[1:2], w.kv, w.pe, w.wkv_b, [0, 1], [0, 4], d.heads, d.qk_nope,
                             d.qk_rope, d.v_head, d.scale)
    np.testing.assert_array_equal(out[1:2], alone)
