"""The seeded generator: determinism, shapes, bf16 rounding and the value recipe."""
import numpy as np
import torch

from deepseek_mla_latent_b200 import workloads as wl


def test_bf16_rounding_matches_torch():
    x = np.random.default_rng(0).standard_normal(100000).astype(np.float32) * 37.0
    x[:4] = [1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -1.5 - 2 ** -9, 0.0]   # ties and exact values
    ours = wl.round_to_bf16(x)
    ref = torch.from_numpy(x).to(torch.bfloat16).float().numpy()
    np.testing.assert_array_equal(ours, ref)


def test_deterministic_and_stream_separated():
    a = wl.make_workload("a", wl.V3, [1, 1], [7, 9], seed=3)
    b = wl.make_workload("b", wl.V3, [1, 1], [7, 9], seed=3)
    for k in ("q", "kv", "pe", "wkv_b"):
        np.testing.assert_array_equal(getattr(a, k), getattr(b, k))
    c = wl.make_workload("c", wl.V3, [1, 1], [7, 9], seed=4)
    assert not np.array_equal(a.kv, c.kv)


def test_shapes_and_recipe():
    w = wl.make_workload("v3", wl.V3, [1, 2], [5, 6], seed=0)
    assert w.q.shape == (3, 128, 192) and w.kv.shape == (11, 512) and w.pe.shape == (11, 64)
    assert w.wkv_b.shape == (128 * 256, 512)
    assert list(w.cu_seqlens_k) == [0, 5, 11] and list(w.cu_seqlens_q) == [0, 1, 3]
    # kv rows are RMS-normalised before bf16 rounding
    ms = np.mean(w.kv.astype(np.float64) ** 2, axis=1)
    np.testing.assert_allclose(ms, 1.0, atol=2e-2)
    # every value is bf16-exact
    for k in ("q", "kv", "pe", "wkv_b"):
        a = getattr(w, k)
        np.testing.assert_array_equal(a, wl.round_to_bf16(a))
    assert abs(np.std(w.wkv_b) - 0.02) < 1e-3


def test_ragged_lengths_in_range():
    name, dims, sq, sk = wl.workload_shape(2)
    assert len(sk) == 64 and min(sk) >= 512 and max(sk) <= 8192
    assert sk == wl.workload_shape(2)[3]


def test_tiny_workload_is_fp32_unnormalised():
    w = wl.workload(0)
    assert w.dims.dtype == "f32" and w.q.shape == (1, 8, 48) and w.wkv_b.shape == (512, 64)
    assert not np.array_equal(w.kv, wl.round_to_bf16(w.kv))
    assert abs(np.std(w.wkv_b) - 0.125) < 0.01
