"""Pins of the latent-cache append oracle (CPU): closed forms, invariants and a second,
independent implementation (the seeded workload generator's own normalisation and rotation)."""
import numpy as np

import oracle
from deepseek_mla_latent_b200 import workloads as wl


def _rng(seed):
    return np.random.default_rng(seed)


def test_rms_norm_closed_forms():
    x = _rng(0).normal(size=(5, 512))
    y = oracle.rms_norm(x, None, 0.0)
    # unit root mean square with eps = 0
    assert np.allclose((y * y).mean(axis=1), 1.0, rtol=1e-13)
    # mean(y^2) = ms / (ms + eps) in general
    eps = 0.25
    ms = (x * x).mean(axis=1)
    assert np.allclose((oracle.rms_norm(x, None, eps) ** 2).mean(axis=1), ms / (ms + eps), rtol=1e-13)
    # a constant row c maps to sign(c) (eps = 0), scaled by gamma column-wise
    g = np.arange(1, 513, dtype=np.float64)
    z = oracle.rms_norm(np.full((1, 512), -3.0), g, 0.0)
    assert np.allclose(z, -g[None, :], rtol=1e-14)


def test_rms_norm_is_scale_invariant():
    x = _rng(1).normal(size=(3, 64))
    assert np.allclose(oracle.rms_norm(7.5 * x, None, 0.0), oracle.rms_norm(x, None, 0.0), rtol=1e-13)


def test_rope_closed_form_and_invariants():
    r = 64
    x = _rng(2).normal(size=(4, r))
    # position 0 is the identity
    assert np.array_equal(oracle.rope_interleaved(x, np.zeros(4), 10000.0), x)
    # one pair written out: pair i turns by p * base^(-2i/r)
    p, i = 5.0, 3
    th = p * 10000.0 ** (-2.0 * i / r)
    y = oracle.rope_interleaved(x[:1], np.array([p]), 10000.0)
    a, b = x[0, 2 * i], x[0, 2 * i + 1]
    assert np.isclose(y[0, 2 * i], a * np.cos(th) - b * np.sin(th), rtol=1e-14, atol=1e-15)
    assert np.isclose(y[0, 2 * i + 1], a * np.sin(th) + b * np.cos(th), rtol=1e-14, atol=1e-15)
    # pair norms are preserved
    pos = np.array([1.0, 17.0, 1000.0, 131071.0])
    y = oracle.rope_interleaved(x, pos, 10000.0)
    assert np.allclose(y[:, 0::2] ** 2 + y[:, 1::2] ** 2, x[:, 0::2] ** 2 + x[:, 1::2] ** 2, rtol=1e-12)
    # rotations compose
    y2 = oracle.rope_interleaved(oracle.rope_interleaved(x, pos, 10000.0), pos + 3.0, 10000.0)
    assert np.allclose(y2, oracle.rope_interleaved(x, 2 * pos + 3.0, 10000.0), rtol=1e-9, atol=1e-9)
    # the score of two rotated vectors depends only on the position difference
    q, k = x[0], x[1]
    s1 = oracle.rope_interleaved(q[None], np.array([40.0]), 10000.0) @ oracle.rope_interleaved(
        k[None], np.array([15.0]), 10000.0).T
    s2 = oracle.rope_interleaved(q[None], np.array([125.0]), 10000.0) @ oracle.rope_interleaved(
        k[None], np.array([100.0]), 10000.0).T
    assert np.isclose(s1, s2, rtol=1e-11)


def test_append_writes_only_its_slots():
    rng = _rng(3)
    rows, C, R, n = 40, 16, 8, 5
    kv_cache, pe_cache = rng.normal(size=(rows, C)), rng.normal(size=(rows, R))
    kv_new, pe_new = rng.normal(size=(n, C)), rng.normal(size=(n, R))
    slots = np.array([7, 0, 39, 40, -1])   # the last two are outside the cache
    pos = np.array([3, 0, 12, 5, 6])
    kv2, pe2 = oracle.append_latent(kv_new, pe_new, None, 1e-6, pos, slots, kv_cache, pe_cache)
    untouched = [r for r in range(rows) if r not in (7, 0, 39)]
    assert np.array_equal(kv2[untouched], kv_cache[untouched])
    assert np.array_equal(pe2[untouched], pe_cache[untouched])
    assert np.allclose(kv2[0], oracle.rms_norm(kv_new[1:2], None, 1e-6)[0])
    assert np.array_equal(pe2[0], pe_new[1])          # position 0: no rotation
    assert np.allclose(pe2[39], oracle.rope_interleaved(pe_new[2:3], np.array([12]), 10000.0)[0])


def test_append_agrees_with_the_workload_generator():
    """The generator normalises and rotates its cache rows with code of its own; feeding the
    oracle the same raw rows must give the same cache (to float32 rounding)."""
    rng = _rng(4)
    n, C, R = 33, 512, 64
    raw_kv = rng.normal(size=(n, C)).astype(np.float32)
    raw_pe = rng.normal(size=(n, R)).astype(np.float32)
    pos = np.arange(n) + 4000
    kv2, pe2 = oracle.append_latent(raw_kv, raw_pe, None, 1e-6, pos, np.arange(n),
                                    np.zeros((n, C)), np.zeros((n, R)))
    assert np.allclose(kv2, wl._rms_normalise(raw_kv), rtol=2e-6, atol=2e-6)
    assert np.allclose(pe2, wl._rope(raw_pe, pos), rtol=2e-5, atol=2e-5)
