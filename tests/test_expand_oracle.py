"""Pins of the latent KV expansion oracle (oracle.expand_oracle) against a hand expansion,
the attention oracle it feeds, and properties the definition fixes."""
import math

import numpy as np
import pytest

import oracle
from deepseek_mla_latent_b200 import workloads as wl


def test_hand_example():
    """One token, C = 2, H = 1, Dn = Dv = 1, eps = 0: kv = (3, 4) has mean square 12.5, so the
    normalised row times gamma (1, 2) is (3, 8) / sqrt(12.5); W = [[1, 1], [2, -1]] gives
    K = 11 / sqrt(12.5) and V = -2 / sqrt(12.5)."""
    k, v = oracle.expand_kv(np.array([[3.0, 4.0]]), np.array([1.0, 2.0]), 0.0, np.array([[1.0, 1.0], [2.0, -1.0]]),
                            1, 1, 1, 1, 1)
    assert k.shape == (1, 1, 1, 1) and v.shape == (1, 1, 1, 1)
    assert abs(k[0, 0, 0, 0] - 11 / math.sqrt(12.5)) < 1e-14
    assert abs(v[0, 0, 0, 0] + 2 / math.sqrt(12.5)) < 1e-14


def test_layout_head_before_token_and_split():
    """K_nope[b, h, s, d] and V[b, h, s, d] come from token b*S + s and rows h*(Dn+Dv) + d and
    h*(Dn+Dv) + Dn + d of wkv_b (checked entry by entry on random indices)."""
    rng = np.random.default_rng(0)
    B, S, H, C, Dn, Dv = 2, 3, 4, 8, 3, 2
    kv = rng.standard_normal((B * S, C))
    w = rng.standard_normal((H * (Dn + Dv), C))
    g = rng.standard_normal(C)
    k, v = oracle.expand_kv(kv, g, 1e-6, w, H, Dn, Dv, B, S)
    assert k.shape == (B, H, S, Dn) and v.shape == (B, H, S, Dv)
    for _ in range(40):
        b, h, s = rng.integers(B), rng.integers(H), rng.integers(S)
        row = kv[b * S + s]
        x = row / math.sqrt(float(np.mean(row * row)) + 1e-6) * g
        d = rng.integers(Dn)
        assert abs(k[b, h, s, d] - float(x @ w[h * (Dn + Dv) + d])) < 1e-12
        d = rng.integers(Dv)
        assert abs(v[b, h, s, d] - float(x @ w[h * (Dn + Dv) + Dn + d])) < 1e-12


def test_scale_invariance_without_eps():
    rng = np.random.default_rng(1)
    kv, w = rng.standard_normal((6, 16)), rng.standard_normal((2 * 8, 16))
    a = oracle.expand_kv(kv, None, 0.0, w, 2, 4, 4, 1, 6)
    b = oracle.expand_kv(kv * 37.5, None, 0.0, w, 2, 4, 4, 1, 6)
    assert all(np.allclose(x, y, rtol=1e-12, atol=0) for x, y in zip(a, b))


def test_linear_in_the_weight():
    rng = np.random.default_rng(2)
    kv = rng.standard_normal((4, 16))
    w1, w2 = rng.standard_normal((24, 16)), rng.standard_normal((24, 16))
    s1, s2, s12 = (oracle.expand_kv(kv, None, 1e-6, w, 3, 5, 3, 2, 2) for w in (w1, w2, w1 + w2))
    for i in range(2):
        assert np.allclose(s12[i], s1[i] + s2[i], rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("sq,sk", [([1, 1], [7, 40]), ([3], [20])])
def test_expanded_keys_and_values_reproduce_the_attention_oracle(sq, sk):
    """Attention over the expanded per-head keys [K_nope ; pe] and values V equals the naive
    attention oracle over the normalised cache (which materialises k and v its own way)."""
    w = wl.make_workload("ex", wl.TINY, sq, sk, seed=5, v3_values=False)
    d = w.dims
    rng = np.random.default_rng(3)
    kv_c = rng.standard_normal(w.kv.shape) * 3.0
    gamma = 1.0 + 0.1 * rng.standard_normal(d.kv_lora_rank)
    kv_cache = oracle.rms_norm(kv_c, gamma, 1e-6)
    ref = oracle.mla_naive(w.q, kv_cache, w.pe, w.wkv_b, w.cu_seqlens_q, w.cu_seqlens_k, d.heads, d.qk_nope,
                           d.qk_rope, d.v_head, d.scale)
    cq, ck = w.cu_seqlens_q, w.cu_seqlens_k
    for b in range(w.batch):
        t, s = sk[b], sq[b]
        k_nope, v = oracle.expand_kv(kv_c[ck[b]:ck[b + 1]], gamma, 1e-6, w.wkv_b, d.heads, d.qk_nope, d.v_head, 1, t)
        for h in range(d.heads):
            q = w.q[cq[b]:cq[b + 1], h, :]
            keys = np.concatenate([k_nope[0, h], w.pe[ck[b]:ck[b + 1]]], axis=1)
            p = oracle.softmax_rows(q @ keys.T * d.scale, [oracle.visible_keys(t, s, i) for i in range(s)])
            assert np.allclose(p @ v[0, h], ref[cq[b]:cq[b + 1], h], rtol=1e-10, atol=1e-12)
