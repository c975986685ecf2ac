"""The bounded device waits, exercised: the fault-injection build of the library (2 ms wait
limits, a host-set plan that drops one TMA copy) runs a decode whose first work unit never
receives the rotary keys of its first score tile.  The waits on that copy run out instead of
hanging, the device error word reports it (MLA_ERR_DEVICE_TIMEOUT, bit 0 = a consumer waited
too long for a TMA tile), and the next call in the same process, with the plan cleared, is
correct against the oracle.  No GPU fault is raised: every wait returns."""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from deepseek_mla_latent_b200 import workloads as wl

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def variant():
    from deepseek_mla_latent_b200 import _lib, build
    lib = _lib.load_library(build.build(variant="fault_inject"))
    lib.mla_test_set_fault_plan.restype = ctypes.c_int32
    lib.mla_test_set_fault_plan.argtypes = [ctypes.c_uint32]
    return lib


def _decode(lib, d, q_abs, dev, o_lat, ws, splits):
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return lib.mla_attn_decode(ctypes.byref(d), q_abs.data_ptr(), dev["q"].data_ptr(), dev["q"].stride(0),
                               dev["kv"].data_ptr(), dev["pe"].data_ptr(), dev["kv"].shape[0],
                               dev["cu_k"].data_ptr(), dev["cu_k"].numel() - 1, dev["max_k"], o_lat.data_ptr(),
                               ws.data_ptr(), ws.numel(), splits, stream)


def _status(lib):
    code = ctypes.c_uint32(0)
    st = lib.mla_device_status(ctypes.c_void_p(torch.cuda.current_stream().cuda_stream), ctypes.byref(code))
    return st, code.value


def test_a_dropped_copy_times_out_and_the_next_call_is_correct(variant):
    from deepseek_mla_latent_b200 import _lib, mla
    from gpu_util import assert_close, to_dev
    torch.cuda.set_device(0)
    w = wl.make_workload("fault", wl.V3, [1, 1], [1000, 300], seed=51)
    d = mla.dims_from(w.dims)
    dev = to_dev(w)
    q_abs = mla.absorb_q(d, dev["q"], dev["wkv_b"])
    mla.device_status()
    splits = 2
    ws = torch.empty(int(variant.mla_workspace_size(ctypes.byref(d), w.batch, w.batch, dev["max_k"], splits)) + 16,
                     dtype=torch.uint8, device="cuda")
    o_lat = torch.zeros((w.batch, 128, 512), dtype=torch.bfloat16, device="cuda")
    assert _status(variant) == (_lib.MLA_OK, 0)

    assert variant.mla_test_set_fault_plan(1) == _lib.MLA_OK
    assert _decode(variant, d, q_abs, dev, o_lat, ws, splits) == _lib.MLA_OK
    st, code = _status(variant)
    assert st == _lib.MLA_ERR_DEVICE_TIMEOUT
    assert code & 1, f"error word {code:#x} lacks the TMA-tile timeout bit"
    assert variant.mla_test_set_fault_plan(0) == _lib.MLA_OK

    # the context is usable and the next call is right; the error word was cleared by the read
    assert _decode(variant, d, q_abs, dev, o_lat, ws, splits) == _lib.MLA_OK
    assert _status(variant) == (_lib.MLA_OK, 0)
    got = o_lat.float().cpu().numpy().astype(np.float64)
    _, ref, _ = oracle.workload_absorb(w)
    assert_close(got, ref, "bf16", "o_lat after the fault")
