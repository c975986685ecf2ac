"""GPU parity of the latent KV expansion (mla_expand_kv) against the fp64 oracle."""
import numpy as np
import pytest
import torch

import oracle
from deepseek_mla_latent_b200 import workloads as wl

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    from deepseek_mla_latent_b200 import mla
    from gpu_util import assert_close


def _run(e: wl.ExpandInputs, with_gamma=True, eps=1e-6):
    d = mla.dims_from(e.dims)
    dt = torch.bfloat16 if e.dims.dtype == "bf16" else torch.float32
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(device="cuda", dtype=dt)
    k, v = mla.expand_kv(d, t(e.kv_c), t(e.wkv_b), e.batch, e.seq_len, gamma=t(e.gamma) if with_gamma else None,
                         eps=eps)
    mla.device_status()
    f = lambda x: x.float().cpu().numpy().astype(np.float64)
    return f(k), f(v)


def _check(e, with_gamma=True, eps=1e-6):
    k, v = _run(e, with_gamma, eps)
    dd = e.dims
    rk, rv = oracle.expand_kv(e.kv_c, e.gamma if with_gamma else None, eps, e.wkv_b, dd.heads, dd.qk_nope, dd.v_head,
                              e.batch, e.seq_len)
    assert_close(k, rk, dd.dtype, "k_nope")
    assert_close(v, rv, dd.dtype, "v")


@pytest.mark.parametrize("batch,seq", [(2, 300), (3, 128), (1, 1), (1, 129)])
def test_v3_expand(batch, seq):
    """DeepSeek-V3 shapes: several 128-token tiles with a ragged last tile, CTAs whose run of
    (tile, head) items crosses a tile boundary, and fewer items than SMs."""
    _check(wl.expand_inputs(wl.V3, batch, seq, seed=batch * 1000 + seq))


def test_v3_expand_without_gain():
    _check(wl.expand_inputs(wl.V3, 1, 200, seed=7), with_gamma=False)


def test_v3_expand_eps_zero_and_scale():
    """eps = 0 on rows whose scale spans 2^-2 .. 2^2: the RMS factor carries the scale."""
    _check(wl.expand_inputs(wl.V3, 2, 64, seed=8), eps=0.0)


@pytest.mark.parametrize("batch,seq", [(2, 5), (1, 1)])
def test_fp32_expand(batch, seq):
    _check(wl.expand_inputs(wl.TINY, batch, seq, seed=9))


def test_full_expand_sampled():
    """Batch 4 x 1024 tokens (the benchmark's expansion size), checked on sampled tokens of
    every (batch, head) against the oracle on those tokens."""
    e = wl.expand_inputs(wl.V3, 4, 1024, seed=0)
    k, v = _run(e)
    dd = e.dims
    rng = np.random.default_rng(0)
    for b in range(4):
        s_idx = np.sort(rng.choice(1024, size=6, replace=False))
        rows = e.kv_c[b * 1024 + s_idx]
        rk, rv = oracle.expand_kv(rows, e.gamma, 1e-6, e.wkv_b, dd.heads, dd.qk_nope, dd.v_head, 1, len(s_idx))
        assert_close(k[b][:, s_idx], rk[0], "bf16", f"k_nope batch {b}")
        assert_close(v[b][:, s_idx], rv[0], "bf16", f"v batch {b}")


def test_v3_expand_outputs_16_byte_aligned():
    """Outputs that are 16- but not 32-byte aligned take the 16-byte store path; same result."""
    e = wl.expand_inputs(wl.V3, 1, 130, seed=10)
    d = mla.dims_from(e.dims)
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(device="cuda", dtype=torch.bfloat16)
    n = 128 * 130 * 128
    kb = torch.empty(n + 8, dtype=torch.bfloat16, device="cuda")
    vb = torch.empty(n + 8, dtype=torch.bfloat16, device="cuda")
    k = kb[8:].view(1, 128, 130, 128)
    v = vb[8:].view(1, 128, 130, 128)
    assert k.data_ptr() % 32 == 16
    mla.expand_kv(d, t(e.kv_c), t(e.wkv_b), 1, 130, gamma=t(e.gamma), k_nope=k, v=v)
    k2, v2 = mla.expand_kv(d, t(e.kv_c), t(e.wkv_b), 1, 130, gamma=t(e.gamma))
    mla.device_status()
    assert torch.equal(k, k2) and torch.equal(v, v2)
    dd = e.dims
    rk, rv = oracle.expand_kv(e.kv_c, e.gamma, 1e-6, e.wkv_b, dd.heads, dd.qk_nope, dd.v_head, 1, 130)
    assert_close(k.float().cpu().numpy().astype(np.float64), rk, "bf16", "k_nope")
    assert_close(v.float().cpu().numpy().astype(np.float64), rv, "bf16", "v")
