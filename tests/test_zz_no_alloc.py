"""mla_attn_decode_static_scratch: decode attention for callers that cannot allocate.

Some callers only get input and output buffers from a host framework and have
no allocator to call, or run where cudaMalloc is not allowed or would
synchronise the device.  The static-scratch entry point serves them with a
library-owned device array instead of a caller workspace.  These checks call it
through the C ABI and hold it to the workspace-taking entry point on the same
inputs, twice in a row (the array keeps the previous call's contents): the
same kernels run on the same inputs, so the results must agree bit for bit.
This file is collected last on purpose.
"""
import ctypes

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu


def _inputs(seqlens, seed):
    from deepseek_mla_latent_b200 import workloads as wl
    w = wl.make_workload("no_alloc", wl.V3, [1] * len(seqlens), seqlens, seed=seed)
    T = lambda a: torch.from_numpy(a).to(device="cuda", dtype=torch.bfloat16)
    return w, T(w.q), T(w.kv), T(w.pe), T(w.wkv_b), torch.from_numpy(w.cu_seqlens_k).cuda()


def _static_call(lib, d, q_abs, q, kv, pe, cu_k, max_k, o_lat, num_splits):
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return lib.LIB.mla_attn_decode_static_scratch(
        ctypes.byref(d), q_abs.data_ptr(), q.data_ptr(), q.stride(0), kv.data_ptr(), pe.data_ptr(), kv.shape[0],
        cu_k.data_ptr(), cu_k.numel() - 1, max_k, o_lat.data_ptr(), num_splits, stream)


@pytest.mark.parametrize("seqlens,num_splits", [([4096] * 8, 0), ([1000, 260, 3], 7), ([70, 5000], 0)])
def test_static_scratch_matches_workspace_entry_point(seqlens, num_splits):
    from deepseek_mla_latent_b200 import _lib as lib
    from deepseek_mla_latent_b200 import mla
    torch.cuda.set_device(0)
    w, q, kv, pe, wkv_b, cu_k = _inputs(seqlens, seed=31)
    d = mla.dims_from(w.dims)
    max_k = max(seqlens)
    q_abs = mla.absorb_q(d, q, wkv_b)
    ref = mla.attn_decode(d, q_abs, q, kv, pe, cu_k, max_k, num_splits=num_splits)
    mla.device_status()
    ref_h = ref.view(torch.int16).cpu().numpy()
    for call in range(2):
        got = torch.full_like(ref, float("nan"))
        st = _static_call(lib, d, q_abs, q, kv, pe, cu_k, max_k, got, num_splits)
        assert st == lib.MLA_OK, lib.LIB.mla_status_string(st).decode()
        mla.device_status()
        got_h = got.view(torch.int16).cpu().numpy()
        assert np.array_equal(got_h, ref_h), f"call {call}: {int(np.sum(got_h != ref_h))} entries differ"


def test_static_scratch_rejects_plans_beyond_its_size():
    from deepseek_mla_latent_b200 import _lib as lib
    from deepseek_mla_latent_b200 import mla
    torch.cuda.set_device(0)
    w, q, kv, pe, wkv_b, cu_k = _inputs([4096] * 8, seed=32)
    d = mla.dims_from(w.dims)
    # 64 splits x 8 rows x 128 heads x 512 bf16 partials are 64 MiB (plus the fp32 (m, l) pairs),
    # past the 32 MiB array
    assert 64 * 8 * 128 * 512 * 2 == 64 << 20
    assert mla.workspace_size(d, 8, 8, 4096, 64) > (32 << 20)
    q_abs = mla.absorb_q(d, q, wkv_b)
    out = torch.empty_like(q_abs)
    st = _static_call(lib, d, q_abs, q, kv, pe, cu_k, 4096, out, 64)
    assert st == lib.MLA_ERR_WORKSPACE
