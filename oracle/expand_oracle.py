"""fp64 CPU oracle for the latent KV expansion (the naive path's materialisation).

TEST INFRASTRUCTURE ONLY.  Nothing on the product path may import or call this
module: only the tests and the benchmark's CPU leg use it.  It shares no code,
table or helper with the CUDA path.

What it computes.  "Latent KV expansion with split" (kernelindex.com), the
operation's description: the compressed KV (kv_lora_rank = 512 values per
token) is RMS-normalised, projected linearly to num_heads * (qk_nope_head_dim
+ v_head_dim) = 128 * 256 = 32768 values, reshaped per head, transposed so the
head axis comes before the token axis, and split into K_nope and V.  "Naive vs
Absorb Attention Implementations in DeepSeek-V3", section "Naive Path
Execution", consumes exactly these per-head keys and values.  Readings (listed
with the others in the design notes): the input is [batch, seq_len, C] (or
packed tokens with batch 1), the RMSNorm epsilon and gain are inputs, the
projection is wkv_b [H*(Dn+Dv), C] with per-head rows 0..Dn-1 giving K_nope and
rows Dn..Dn+Dv-1 giving V, and the outputs are [batch, H, seq_len, Dn] and
[batch, H, seq_len, Dv].

Everything is computed in float64 from the given inputs; the projection uses
numpy's matmul as a library primitive.
"""
from __future__ import annotations

import numpy as np

from .append_oracle import rms_norm


def expand_kv(kv_c, gamma, eps: float, wkv_b, heads: int, qk_nope: int, v_head: int, batch: int, seq_len: int):
    """(K_nope [B, H, S, Dn], V [B, H, S, Dv]) of compressed KV rows kv_c [B*S, C]."""
    kv_c = np.asarray(kv_c, dtype=np.float64)
    w = np.asarray(wkv_b, dtype=np.float64)
    if kv_c.shape[0] != batch * seq_len:
        raise ValueError("kv_c must have batch * seq_len rows")
    if w.shape != (heads * (qk_nope + v_head), kv_c.shape[1]):
        raise ValueError("wkv_b must be [heads * (qk_nope + v_head), C]")
    x = rms_norm(kv_c, gamma, eps)                                   # [B*S, C]
    y = x @ w.T                                                      # [B*S, H*(Dn+Dv)]
    y = y.reshape(batch, seq_len, heads, qk_nope + v_head).transpose(0, 2, 1, 3)   # [B, H, S, Dn+Dv]
    return np.ascontiguousarray(y[..., :qk_nope]), np.ascontiguousarray(y[..., qk_nope:])
