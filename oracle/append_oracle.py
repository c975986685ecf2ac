"""fp64 CPU oracle for the latent-cache append that precedes MLA attention.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path may import or call this
module: only the tests and the benchmark's CPU leg use it.  It shares no code,
table or helper with the CUDA path.

What it computes.  "Naive vs Absorb Attention Implementations in DeepSeek-V3",
section "Absorb Implementation Cache Design": the absorb path caches, per
token, the compressed key-value vector (kv_lora_rank values, kv_cache) and the
rotary key (qk_rope_head_dim values, pe_cache) separately.  "Latent KV
expansion with split" (kernelindex.com) states that the compressed KV is
RMS-normalised.  Appending one new token therefore writes
    kv_cache[slot] = kv / sqrt(mean(kv^2) + eps) * gamma
    pe_cache[slot] = RoPE(k_pe, position)
Readings where the cited pages are silent (each listed in the design notes): the
RMSNorm epsilon and gain are inputs (eps = 1e-6 and gamma = 1 in the
workloads); RoPE rotates interleaved pairs (x[2i], x[2i+1]) by the angle
position * base^(-2i/R) with base 10000; the position is the token's index in
its sequence; a slot outside the cache is not written.

Everything is computed in float64 from the given inputs.
"""
from __future__ import annotations

import numpy as np


def rms_norm(x: np.ndarray, gamma, eps: float) -> np.ndarray:
    """Each row of x divided by the root of (its mean square + eps), times gamma (per column)."""
    x = np.asarray(x, dtype=np.float64)
    g = np.ones(x.shape[-1]) if gamma is None else np.asarray(gamma, dtype=np.float64)
    ms = (x * x).mean(axis=-1, keepdims=True)
    return x / np.sqrt(ms + eps) * g


def rope_interleaved(x: np.ndarray, positions: np.ndarray, base: float) -> np.ndarray:
    """Rotate each pair (x[..., 2i], x[..., 2i+1]) of row n by positions[n] * base^(-2i/R)."""
    x = np.asarray(x, dtype=np.float64)
    r = x.shape[-1]
    out = np.empty_like(x)
    for i in range(r // 2):
        theta = np.asarray(positions, dtype=np.float64) * base ** (-2.0 * i / r)
        c, s = np.cos(theta), np.sin(theta)
        a, b = x[..., 2 * i], x[..., 2 * i + 1]
        out[..., 2 * i] = a * c - b * s
        out[..., 2 * i + 1] = a * s + b * c
    return out


def append_latent(kv_new, k_pe_new, gamma, eps, positions, slots, kv_cache, pe_cache, base=10000.0):
    """Write the normalised latents and rotated rotary keys of the new tokens into copies of the caches.

    kv_new [n, C], k_pe_new [n, R], gamma [C] or None, positions [n], slots [n] (row indices into the
    caches; entries outside [0, rows) are skipped), kv_cache [rows, C], pe_cache [rows, R].
    Returns (kv_cache', pe_cache') as float64 arrays; rows not written keep their values."""
    kv_out = np.array(kv_cache, dtype=np.float64, copy=True)
    pe_out = np.array(pe_cache, dtype=np.float64, copy=True)
    rows = kv_out.shape[0]
    kvn = rms_norm(kv_new, gamma, eps)
    per = rope_interleaved(k_pe_new, positions, base)
    for n, slot in enumerate(np.asarray(slots, dtype=np.int64)):
        if 0 <= slot < rows:
            kv_out[slot] = kvn[n]
            pe_out[slot] = per[n]
    return kv_out, pe_out
