"""GPU parity of the latent-cache append (mla_append_latent) against the fp64 oracle."""
import numpy as np
import pytest
import torch

import oracle
from deepseek_mla_latent_b200 import workloads as wl

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    from deepseek_mla_latent_b200 import mla
    from gpu_util import assert_close


def _case(dims, n, rows, seed, gamma=True, slots=None, positions=None):
    rng = np.random.default_rng(seed)
    dt = torch.bfloat16 if dims.dtype == "bf16" else torch.float32
    C, R = dims.kv_lora_rank, dims.qk_rope
    r = lambda *s: rng.normal(size=s).astype(np.float32)
    kv_new, pe_new = r(n, C) * 3.0, r(n, R)
    g = (1.0 + 0.1 * r(C)) if gamma else None
    cache_kv, cache_pe = r(rows, C), r(rows, R)
    if dims.dtype == "bf16":   # both sides see the bf16-rounded values
        kv_new, pe_new, cache_kv, cache_pe = map(wl.round_to_bf16, (kv_new, pe_new, cache_kv, cache_pe))
        g = wl.round_to_bf16(g) if g is not None else None
    if slots is None:
        slots = rng.permutation(rows)[:n]
    if positions is None:
        positions = rng.integers(0, 131072, size=n)
    T = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(device="cuda", dtype=dt)
    d = mla.dims_from(dims)
    kvc, pec = T(cache_kv), T(cache_pe)
    mla.append_latent(d, T(kv_new), T(pe_new), torch.from_numpy(np.asarray(positions, np.int32)).cuda(),
                      torch.from_numpy(np.asarray(slots, np.int64)).cuda(), kvc, pec,
                      T(g) if g is not None else None, eps=1e-6)
    mla.device_status()
    ref_kv, ref_pe = oracle.append_latent(kv_new, pe_new, g, 1e-6, positions, slots, cache_kv, cache_pe)
    got_kv = kvc.float().cpu().numpy().astype(np.float64)
    got_pe = pec.float().cpu().numpy().astype(np.float64)
    written = sorted({int(s) for s in slots if 0 <= s < rows})
    untouched = [i for i in range(rows) if i not in set(written)]
    # rows that were not written keep their exact bits
    assert np.array_equal(got_kv[untouched], ref_kv[untouched])
    assert np.array_equal(got_pe[untouched], ref_pe[untouched])
    if written:
        assert_close(got_kv[written], ref_kv[written], dims.dtype, "kv_cache")
        assert_close(got_pe[written], ref_pe[written], dims.dtype, "pe_cache")


@pytest.mark.parametrize("n,rows", [(8, 4096), (1, 10), (333, 2048), (4096, 4096)])
def test_append_v3_bf16(n, rows):
    _case(wl.V3, n, rows, seed=n)


def test_append_v3_bf16_without_gamma_and_edge_positions():
    n = 6
    _case(wl.V3, n, 64, seed=11, gamma=False, positions=[0, 1, 131071, 131072, 2 ** 20, 7])


def test_append_skips_slots_outside_the_cache():
    _case(wl.V3, 5, 32, seed=12, slots=[3, -1, 32, 31, 1 << 40])


def test_append_fp32_tiny_dims():
    _case(wl.TINY, 50, 200, seed=13)


def test_append_empty_is_a_no_op():
    d = mla.dims_from(wl.V3)
    kvc = torch.zeros(4, 512, dtype=torch.bfloat16, device="cuda")
    pec = torch.zeros(4, 64, dtype=torch.bfloat16, device="cuda")
    e = torch.empty(0, 512, dtype=torch.bfloat16, device="cuda")
    mla.append_latent(d, e, torch.empty(0, 64, dtype=torch.bfloat16, device="cuda"),
                      torch.empty(0, dtype=torch.int32, device="cuda"), torch.empty(0, dtype=torch.int64, device="cuda"),
                      kvc, pec)
    mla.device_status()
    assert int(kvc.abs().sum()) == 0 and int(pec.abs().sum()) == 0


def test_append_then_decode_without_a_kernel_between():
    """The attention reads the cache before it waits for the kernel before it on the stream;
    mla_append_latent makes its rows visible before it exits, so append -> decode on one stream
    (no kernel between) attends to the appended rows: against the oracle over the appended cache."""
    w = wl.make_workload("apd", wl.V3, [1, 1], [300, 700], seed=14)
    d = mla.dims_from(w.dims)
    rng = np.random.default_rng(15)
    C, R = w.dims.kv_lora_rank, w.dims.qk_rope
    cu = w.cu_seqlens_k
    slots = np.array([cu[1] - 1, cu[2] - 1], dtype=np.int64)      # the last key of each sequence
    positions = np.array([299, 699], dtype=np.int32)
    kv_new = wl.round_to_bf16(rng.normal(size=(2, C)).astype(np.float32) * 2.0)
    pe_new = wl.round_to_bf16(rng.normal(size=(2, R)).astype(np.float32))
    T = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(device="cuda", dtype=torch.bfloat16)
    q, wkv_b, kv, pe = T(w.q), T(w.wkv_b), T(w.kv), T(w.pe)
    cu_k = torch.from_numpy(cu).cuda()
    pos_d, slots_d = torch.from_numpy(positions).cuda(), torch.from_numpy(slots).cuda()
    kv_new_d, pe_new_d = T(kv_new), T(pe_new)
    q_abs = mla.absorb_q(d, q, wkv_b)
    mla.append_latent(d, kv_new_d, pe_new_d, pos_d, slots_d, kv, pe, eps=1e-6)
    o_lat = mla.attn_decode(d, q_abs, q, kv, pe, cu_k, max(w.seqlens_k))
    out = mla.out_proj(d, o_lat, wkv_b).float().cpu().numpy().astype(np.float64)
    mla.device_status()
    ref_kv, ref_pe = oracle.append_latent(kv_new, pe_new, None, 1e-6, positions, slots, w.kv, w.pe)
    dd = w.dims
    ref = oracle.mla_naive(w.q, ref_kv, ref_pe, w.wkv_b, w.cu_seqlens_q, cu, dd.heads, dd.qk_nope, dd.qk_rope,
                           dd.v_head, dd.scale)
    assert_close(out, ref, "bf16", "out")
