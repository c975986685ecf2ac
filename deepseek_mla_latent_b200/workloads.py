"""Seeded synthetic workloads for MLA absorb attention.

This module only draws inputs: it holds none of the attention arithmetic.
Both the CUDA path (through the tests and the benchmark) and the fp64 oracle
consume exactly the arrays produced here.

Input recipe (shapes from "Naive vs Absorb Attention Implementations in
DeepSeek-V3", section "Memory Layout and Cache Structure"; DeepSeek-V3 head
sizes from "Latent KV expansion with split", workload line):

* ``q``      [N_q, H, Dn + R]   query, non-positional part first (dims 0..Dn-1),
                                 rotary part last (dims Dn..Dn+R-1)
* ``kv``     [sum_t, C]          compressed latent cache, sequences packed in
                                 batch order (cu_seqlens_k)
* ``pe``     [sum_t, R]          rotary key cache, same packing
* ``wkv_b``  [H * (Dn + Dv), C]  up-projection; per head rows 0..Dn-1 are the
                                 key part, rows Dn..Dn+Dv-1 the value part

Random numbers come from numpy's Philox4x32-10 counter-based generator keyed
by (seed, stream), one stream per tensor: q=1, kv=2, pe=3, wkv_b=4,
sequence lengths=5, page placement of a paged cache=6, RMSNorm gain of the
expansion inputs=7.  For the bf16 workloads every value is rounded to bf16
(round to nearest even) before either side sees it, so the oracle receives
the exact operand values the GPU does.

Value recipe for the DeepSeek-V3 workloads: kv rows are N(0,1) then RMS
normalised (x / sqrt(mean(x^2) + 1e-6), unit gain), pe rows are N(0,1) then
rotated by RoPE at their token position (interleaved pairs, base 10000),
q is N(0,1) with its rotary part rotated at the query's absolute position,
wkv_b is N(0, 0.02^2).  The tiny fp32 workload draws q, kv, pe ~ N(0,1) and
wkv_b ~ N(0, (1/8)^2) with no normalisation or rotation.
"""
from __future__ import annotations

import dataclasses
import math
from typing import List, Optional

import numpy as np

STREAM_Q, STREAM_KV, STREAM_PE, STREAM_W, STREAM_LEN, STREAM_PAGES, STREAM_GAMMA = 1, 2, 3, 4, 5, 6, 7


@dataclasses.dataclass(frozen=True)
class Dims:
    """Head geometry: H heads, latent rank C, nope/rope/value head dims."""
    heads: int = 128
    kv_lora_rank: int = 512
    qk_nope: int = 128
    qk_rope: int = 64
    v_head: int = 128
    dtype: str = "bf16"            # "bf16" or "f32": storage/compute type of the path
    softmax_scale: Optional[float] = None

    @property
    def scale(self) -> float:
        if self.softmax_scale is not None:
            return float(self.softmax_scale)
        return 1.0 / math.sqrt(self.qk_nope + self.qk_rope)


V3 = Dims()
TINY = Dims(heads=8, kv_lora_rank=64, qk_nope=32, qk_rope=16, v_head=32, dtype="f32")


@dataclasses.dataclass
class Workload:
    name: str
    dims: Dims
    seqlens_q: List[int]
    seqlens_k: List[int]
    q: np.ndarray          # float32 [N_q, H, Dn+R]   (bf16-exact values for bf16 workloads)
    kv: np.ndarray         # float32 [sum_t, C]
    pe: np.ndarray         # float32 [sum_t, R]
    wkv_b: np.ndarray      # float32 [H*(Dn+Dv), C]

    @property
    def batch(self) -> int:
        return len(self.seqlens_k)

    @property
    def cu_seqlens_q(self) -> np.ndarray:
        return np.concatenate([[0], np.cumsum(self.seqlens_q)]).astype(np.int32)

    @property
    def cu_seqlens_k(self) -> np.ndarray:
        return np.concatenate([[0], np.cumsum(self.seqlens_k)]).astype(np.int32)

    @property
    def n_q(self) -> int:
        return int(sum(self.seqlens_q))

    @property
    def total_k(self) -> int:
        return int(sum(self.seqlens_k))


def _rng(seed: int, stream: int) -> np.random.Generator:
    return np.random.Generator(np.random.Philox(key=[seed, stream]))


def round_to_bf16(x: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest bf16 (ties to even), kept as float32."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) & 0xFFFF0000
    return u.astype(np.uint32).view(np.float32)


def _rms_normalise(x: np.ndarray, eps: float = 1e-6) -> np.ndarray:
    ms = np.mean(x.astype(np.float64) ** 2, axis=-1, keepdims=True)
    return (x / np.sqrt(ms + eps)).astype(np.float32)


def _rope(x: np.ndarray, positions: np.ndarray, base: float = 10000.0) -> np.ndarray:
    """Rotate interleaved pairs (x[2i], x[2i+1]) by positions * base^(-2i/R)."""
    r = x.shape[-1]
    inv = base ** (-np.arange(0, r, 2, dtype=np.float64) / r)
    ang = positions.astype(np.float64)[:, None] * inv[None, :]
    shape = (positions.shape[0],) + (1,) * (x.ndim - 2) + (r // 2,)
    c, s = np.cos(ang).reshape(shape), np.sin(ang).reshape(shape)
    x0, x1 = x[..., 0::2].astype(np.float64), x[..., 1::2].astype(np.float64)
    out = np.empty(x.shape, dtype=np.float64)
    out[..., 0::2] = x0 * c - x1 * s
    out[..., 1::2] = x0 * s + x1 * c
    return out.astype(np.float32)


def make_workload(name: str, dims: Dims, seqlens_q: List[int], seqlens_k: List[int],
                  seed: int = 0, v3_values: Optional[bool] = None, w_std: Optional[float] = None) -> Workload:
    """Draw one workload.  ``v3_values`` selects the DeepSeek-V3 value recipe
    (RMS-normalised kv, RoPE-rotated pe/q_pe); it defaults to True for bf16."""
    if len(seqlens_q) != len(seqlens_k):
        raise ValueError("seqlens_q and seqlens_k differ in length")
    for sq, sk in zip(seqlens_q, seqlens_k):
        if sq < 0 or sk < 0:
            raise ValueError(f"negative sequence length: s={sq} t={sk}")
    if v3_values is None:
        v3_values = dims.dtype == "bf16"
    if w_std is None:
        w_std = 0.02 if v3_values else 1.0 / 8.0
    H, C, Dn, R, Dv = dims.heads, dims.kv_lora_rank, dims.qk_nope, dims.qk_rope, dims.v_head
    nq, tk = int(sum(seqlens_q)), int(sum(seqlens_k))

    q = _rng(seed, STREAM_Q).standard_normal((nq, H, Dn + R), dtype=np.float32)
    kv = _rng(seed, STREAM_KV).standard_normal((tk, C), dtype=np.float32)
    pe = _rng(seed, STREAM_PE).standard_normal((tk, R), dtype=np.float32)
    w = (_rng(seed, STREAM_W).standard_normal((H * (Dn + Dv), C), dtype=np.float32) * np.float32(w_std))

    if v3_values:
        kv = _rms_normalise(kv)
        kpos = np.concatenate([np.arange(t) for t in seqlens_k]) if tk else np.zeros(0)
        pe = _rope(pe, kpos)
        qpos = np.concatenate([np.arange(t - s, t) for s, t in zip(seqlens_q, seqlens_k)]) if nq else np.zeros(0)
        q = q.copy()
        q[:, :, Dn:] = _rope(q[:, :, Dn:], qpos)
    if dims.dtype == "bf16":
        q, kv, pe, w = (round_to_bf16(a) for a in (q, kv, pe, w))
    return Workload(name, dims, list(map(int, seqlens_q)), list(map(int, seqlens_k)),
                    np.ascontiguousarray(q), np.ascontiguousarray(kv),
                    np.ascontiguousarray(pe), np.ascontiguousarray(w))


def ragged_lengths(batch: int, lo: int, hi: int, seed: int = 0) -> List[int]:
    """Per-sequence cache lengths uniform on the integers lo..hi inclusive (stream 5)."""
    return [int(x) for x in _rng(seed, STREAM_LEN).integers(lo, hi + 1, size=batch)]


# The five workloads: index 0 is the tiny fp32 case, 1 the DeepSeek-V3 decode
# case the throughput metric is quoted on, 2 ragged batched decode, 3 long
# context decode, 4 chunked prefill.
WORKLOAD_NAMES = ["tiny_fp32", "v3_decode_b8_t4096", "v3_ragged_b64", "v3_long_b2_t131072",
                  "v3_prefill_b4_s1024_t4096"]


def workload_shape(index: int, seed: int = 0):
    """(name, dims, seqlens_q, seqlens_k) of workload ``index`` without drawing values."""
    if index == 0:
        return WORKLOAD_NAMES[0], TINY, [1], [128]
    if index == 1:
        return WORKLOAD_NAMES[1], V3, [1] * 8, [4096] * 8
    if index == 2:
        return WORKLOAD_NAMES[2], V3, [1] * 64, ragged_lengths(64, 512, 8192, seed)
    if index == 3:
        return WORKLOAD_NAMES[3], V3, [1] * 2, [131072] * 2
    if index == 4:
        return WORKLOAD_NAMES[4], V3, [1024] * 4, [4096] * 4
    raise IndexError(index)


def workload(index: int, seed: int = 0) -> Workload:
    name, dims, sq, sk = workload_shape(index, seed)
    return make_workload(name, dims, sq, sk, seed=seed)


@dataclasses.dataclass
class PagedCache:
    """A workload's cache laid out in pages (see ``paged_cache``)."""
    page_size: int
    kv_cache: np.ndarray     # float32 [num_pages * page_size, C]
    pe_cache: np.ndarray     # float32 [num_pages * page_size, R]
    block_table: np.ndarray  # int32 [batch, max_pages]; -1 past a sequence's last page
    seqlens_k: np.ndarray    # int32 [batch]

    @property
    def num_pages(self) -> int:
        return self.kv_cache.shape[0] // self.page_size


def paged_cache(w: Workload, page_size: int, seed: int = 0, spare_pages: int = 0, extra_columns: int = 0,
                fill: float = float("nan")) -> PagedCache:
    """Scatter a workload's packed cache into pages placed at random (stream 6).

    Sequence b's key j goes to row table[b, j // page_size] * page_size + j % page_size.  The
    pages of all sequences plus ``spare_pages`` unused ones are a random permutation of the
    page indices; rows no key occupies (the tail of each sequence's last page, spare pages)
    hold ``fill``.  The block table has ``extra_columns`` more columns than the longest
    sequence needs; every entry past a sequence's last page is -1.
    """
    if page_size <= 0:
        raise ValueError("page_size must be positive")
    need = [(t + page_size - 1) // page_size for t in w.seqlens_k]
    num_pages = sum(need) + spare_pages
    perm = _rng(seed, STREAM_PAGES).permutation(num_pages)
    C, R = w.kv.shape[1], w.pe.shape[1]
    kv = np.full((num_pages * page_size, C), fill, dtype=np.float32)
    pe = np.full((num_pages * page_size, R), fill, dtype=np.float32)
    table = np.full((w.batch, max(need + [0]) + extra_columns), -1, dtype=np.int32)
    cu = w.cu_seqlens_k
    nxt = 0
    for b, t in enumerate(w.seqlens_k):
        for pg in range(need[b]):
            phys = int(perm[nxt])
            nxt += 1
            table[b, pg] = phys
            j0, j1 = pg * page_size, min(t, (pg + 1) * page_size)
            kv[phys * page_size: phys * page_size + (j1 - j0)] = w.kv[cu[b] + j0: cu[b] + j1]
            pe[phys * page_size: phys * page_size + (j1 - j0)] = w.pe[cu[b] + j0: cu[b] + j1]
    return PagedCache(page_size, kv, pe, table, np.asarray(w.seqlens_k, dtype=np.int32))


@dataclasses.dataclass
class ExpandInputs:
    """Inputs of the latent KV expansion (see ``expand_inputs``)."""
    dims: Dims
    batch: int
    seq_len: int
    kv_c: np.ndarray       # float32 [batch * seq_len, C], before RMSNorm
    gamma: np.ndarray      # float32 [C]
    wkv_b: np.ndarray      # float32 [H * (Dn + Dv), C]


def expand_inputs(dims: Dims, batch: int, seq_len: int, seed: int = 0) -> ExpandInputs:
    """Compressed KV rows before normalisation: N(0,1) rows times a per-row scale 2^U(-2, 2)
    (so the RMSNorm matters), gain 1 + N(0, 0.1^2), wkv_b N(0, 0.02^2) (bf16-rounded for bf16)."""
    n, C = batch * seq_len, dims.kv_lora_rank
    rng = _rng(seed, STREAM_KV)
    kv = rng.standard_normal((n, C), dtype=np.float32) * np.exp2(rng.uniform(-2, 2, (n, 1))).astype(np.float32)
    gamma = (1.0 + 0.1 * _rng(seed, STREAM_GAMMA).standard_normal(C)).astype(np.float32)
    w = _rng(seed, STREAM_W).standard_normal((dims.heads * (dims.qk_nope + dims.v_head), C),
                                             dtype=np.float32) * np.float32(0.02)
    if dims.dtype == "bf16":
        kv, gamma, w = (round_to_bf16(a) for a in (kv, gamma, w))
    return ExpandInputs(dims, batch, seq_len, np.ascontiguousarray(kv), np.ascontiguousarray(gamma),
                        np.ascontiguousarray(w))
