"""ctypes binding of libmla_b200.so (include/mla.h).

Argument marshalling only: tensors are checked for device, dtype and layout,
their device pointers and the current CUDA stream are handed to the C ABI,
and a non-OK status raises.  Every arithmetic step runs in the library's
CUDA kernels; if the library is missing the import fails.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libmla_b200.so")

MLA_OK, MLA_ERR_INVALID_ARG, MLA_ERR_UNSUPPORTED, MLA_ERR_WORKSPACE, MLA_ERR_CUDA, MLA_ERR_DEVICE_TIMEOUT = range(6)
MLA_DTYPE_BF16, MLA_DTYPE_F32 = 0, 1

# (name, restype, argtypes) of every entry point include/mla.h declares.
_P, _I32, _I64, _SZ = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t


class MlaDims(ctypes.Structure):
    _fields_ = [("num_heads", ctypes.c_int32), ("kv_lora_rank", ctypes.c_int32),
                ("qk_nope_head_dim", ctypes.c_int32), ("qk_rope_head_dim", ctypes.c_int32),
                ("v_head_dim", ctypes.c_int32), ("dtype", ctypes.c_int32), ("softmax_scale", ctypes.c_float)]


_DP = ctypes.POINTER(MlaDims)
SIGNATURES = {
    "mla_absorb_q": (_I32, [_DP, _P, _I64, _P, _P, _I64, _P]),
    "mla_workspace_size": (_SZ, [_DP, _I32, _I64, _I64, _I32]),
    "mla_attn_decode": (_I32, [_DP, _P, _P, _I64, _P, _P, _I64, _P, _I32, _I64, _P, _P, _SZ, _I32, _P]),
    "mla_attn_decode_static_scratch": (_I32, [_DP, _P, _P, _I64, _P, _P, _I64, _P, _I32, _I64, _P, _I32, _P]),
    "mla_decode_out_workspace_size": (_SZ, [_DP, _I32, _I64, _I32]),
    "mla_partials_workspace_size": (_SZ, [_DP, _I32, _I64, _I32]),
    "mla_decode_fused_workspace_size": (_SZ, [_DP, _I32, _I64, _I32]),
    "mla_attn_decode_fused": (_I32, [_DP, _P, _P, _I64, _P, _P, _I64, _P, _I32, _I64, _P, _P, _P, _SZ, _I32, _P]),
    "mla_attn_decode_partials": (_I32, [_DP, _P, _P, _I64, _P, _P, _I64, _P, _I32, _I64, _P, _SZ, _I32, _P]),
    "mla_merge_partials": (_I32, [_DP, _P, _P, _I32, _I64, _P, _P]),
    "mla_merge_partials_out": (_I32, [_DP, _P, _P, _I32, _I64, _P, _P, _P]),
    "mla_attn_decode_out": (_I32, [_DP, _P, _P, _I64, _P, _P, _I64, _P, _I32, _I64, _P, _P, _P, _SZ, _I32, _P]),
    "mla_attn_prefill_chunk": (_I32, [_DP, _P, _P, _I64, _P, _P, _I32, _I64, _I64, _I64, _P, _P, _I64, _P, _P, _SZ,
                                      _P]),
    "mla_attn_paged": (_I32, [_DP, _P, _P, _I64, _P, _I64, _P, _I32, _I64, _P, _P, _I64, _I32, _P, _I64, _P, _P,
                              _SZ, _I32, _P]),
    "mla_out_proj": (_I32, [_DP, _P, _P, _P, _I64, _P]),
    "mla_sparse_workspace_size": (_SZ, [_DP, _I32, _I32, _I32]),
    "mla_attn_sparse_decode": (_I32, [_DP, _P, _P, _I64, _P, _P, _I64, _P, _I64, _P, _I32, _I32, _P, _P, _SZ, _I32,
                                      _P]),
    "mla_attn_prefill_expanded": (_I32, [_DP, _P, _I64, _P, _P, _P, _I64, _P, _P, _I32, _I64, _I64, _P, _P]),
    "mla_expand_kv": (_I32, [_DP, _P, _P, ctypes.c_float, _P, _I64, _I64, _P, _P, _P]),
    "mla_append_latent": (_I32, [_DP, _P, _P, _P, ctypes.c_float, ctypes.c_float, _P, _P, _I64, _P, _P, _I64, _P]),
    "mla_status_string": (ctypes.c_char_p, [_I32]),
    "mla_device_status": (_I32, [_P, ctypes.POINTER(ctypes.c_uint32)]),
    "mla_kernel_family": (_I32, [_DP]),
    "mla_decode_num_splits": (_I32, [_DP, _I32, _I64, _I32]),
    "mla_api_version": (_I32, []),
}


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    if not os.path.exists(path):
        raise ImportError(f"{path} is missing: build it with `python -m deepseek_mla_latent_b200.build` "
                          "(or __graft_entry__.build()); there is no fallback implementation")
    lib = ctypes.CDLL(path)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype, fn.argtypes = res, args
    return lib


LIB = load_library()


class MlaError(RuntimeError):
    def __init__(self, status: int, where: str):
        msg = LIB.mla_status_string(status).decode()
        super().__init__(f"{where}: {msg} (status {status})")
        self.status = status


def _check(status: int, where: str) -> None:
    if status != MLA_OK:
        raise MlaError(status, where)


def make_dims(heads: int, kv_lora_rank: int, qk_nope: int, qk_rope: int, v_head: int, dtype: str,
              softmax_scale: float) -> MlaDims:
    return MlaDims(heads, kv_lora_rank, qk_nope, qk_rope, v_head,
                   MLA_DTYPE_BF16 if dtype == "bf16" else MLA_DTYPE_F32, float(softmax_scale))


def dims_from(d) -> MlaDims:
    """MlaDims from a workloads.Dims."""
    return make_dims(d.heads, d.kv_lora_rank, d.qk_nope, d.qk_rope, d.v_head, d.dtype, d.scale)
