"""Helpers shared by the GPU parity tests: run the library on a workload and
compare with the oracle under the tolerance of the path's dtype."""
from __future__ import annotations

import numpy as np
import torch

from deepseek_mla_latent_b200 import mla
from deepseek_mla_latent_b200 import workloads as wl

# max|gpu - oracle| <= TOL * max|oracle| over the compared entries: 2e-2 for
# bf16 operands with fp32 accumulation, 1e-5 for the fp32 path.
TOL = {"bf16": 2e-2, "f32": 1e-5}


def to_dev(w: wl.Workload, device="cuda"):
    dt = torch.bfloat16 if w.dims.dtype == "bf16" else torch.float32
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(device=device, dtype=dt)
    return dict(q=t(w.q), kv=t(w.kv), pe=t(w.pe), wkv_b=t(w.wkv_b),
                cu_q=torch.from_numpy(w.cu_seqlens_q).to(device),
                cu_k=torch.from_numpy(w.cu_seqlens_k).to(device),
                max_q=max(w.seqlens_q) if w.seqlens_q else 0,
                max_k=max(w.seqlens_k) if w.seqlens_k else 0)


def is_decode(w: wl.Workload) -> bool:
    return all(s == 1 for s in w.seqlens_q)


def run_path(w: wl.Workload, num_splits: int = 0, decode: bool = None, dev=None):
    """Run absorb_q -> attention -> out_proj; returns dict of host float64 arrays."""
    d = mla.dims_from(w.dims)
    dev = dev or to_dev(w)
    decode = is_decode(w) if decode is None else decode
    q_abs = mla.absorb_q(d, dev["q"], dev["wkv_b"])
    if decode:
        o_lat = mla.attn_decode(d, q_abs, dev["q"], dev["kv"], dev["pe"], dev["cu_k"], dev["max_k"],
                                num_splits=num_splits)
    else:
        o_lat = mla.attn_prefill_chunk(d, q_abs, dev["q"], dev["cu_q"], dev["cu_k"], dev["max_q"], dev["max_k"],
                                       dev["kv"], dev["pe"])
    out = mla.out_proj(d, o_lat, dev["wkv_b"])
    mla.device_status()
    f = lambda x: x.float().cpu().numpy().astype(np.float64)
    return dict(q_abs=f(q_abs), o_lat=f(o_lat), out=f(out))


def assert_close(got: np.ndarray, ref: np.ndarray, dtype: str, what: str = "") -> float:
    assert got.shape == ref.shape, (got.shape, ref.shape)
    assert np.all(np.isfinite(got)), f"{what}: non-finite values"
    scale = float(np.max(np.abs(ref))) if ref.size else 0.0
    err = float(np.max(np.abs(got - ref))) if ref.size else 0.0
    assert err <= TOL[dtype] * max(scale, 1e-30), f"{what}: max err {err:.3e} vs tol {TOL[dtype]} * {scale:.3e}"
    return err / max(scale, 1e-30)
