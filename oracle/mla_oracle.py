"""fp64 CPU oracle for DeepSeek-V3 multi-head latent attention.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path may import or call this
module: only the tests, ``__graft_entry__.smoke()`` and the benchmark's CPU
baseline leg use it.  It shares no code, table or helper with the CUDA path.

Source: "Naive vs Absorb Attention Implementations in DeepSeek-V3"
(instagit.com), sections "Memory Layout and Cache Structure" (both cache
designs), "Naive Path Execution" (the two naive einsums) and "Absorb Path
Execution" (the per-head view of wkv_b and the four absorb einsums).  The page
states that both paths give the same result; this module writes both out and
the tests hold them to that.

Readings where the page is silent (each is listed in the design notes):
* a softmax over the key axis sits between the score einsum and the value
  einsum (the page shows ``scores`` fed straight into the value einsum);
* it is causal, aligned to the end of the cache: query i of a chunk of s new
  queries over a cache of t tokens sees keys j <= t - s + i (for s = 1 this is
  no mask at all);
* the naive key is [wkv_b_k . kv ; pe] (Dn + R dims, the rotary key shared by
  all heads because pe_cache has no head axis) and the naive value is
  wkv_b_v . kv (Dv dims);
* q = [q_nope (Dn) ; q_pe (R)], nope first;
* wkv_b viewed per head is [H, Dn + Dv, C]: rows 0..Dn-1 project keys, rows
  Dn..Dn+Dv-1 project values;
* a query row with no visible key (empty sequence) gives zeros.

Everything is computed in float64 from the (bf16-exact) float32 inputs.  The
matrix products use numpy's BLAS matmul as a library primitive; the softmax is
the plain two-pass definition (max, exponentials, sum, divide).
"""
from __future__ import annotations

from typing import Dict, Iterable, Optional, Sequence, Tuple

import numpy as np


def head_view(wkv_b: np.ndarray, heads: int, qk_nope: int, v_head: int):
    """wkv_b [H*(Dn+Dv), C] viewed as [H, Dn+Dv, C]; returns (W_k [H,Dn,C], W_v [H,Dv,C]).

    "Absorb Path Execution": the weight is viewed as (n_local_heads, -1,
    kv_lora_rank); its first qk_nope_head_dim rows per head act on q_nope and
    its last v_head_dim rows produce the output.
    """
    w = np.asarray(wkv_b, dtype=np.float64)
    c = w.shape[1]
    if w.shape[0] != heads * (qk_nope + v_head):
        raise ValueError("wkv_b rows must equal heads * (qk_nope + v_head)")
    w = w.reshape(heads, qk_nope + v_head, c)
    return w[:, :qk_nope, :], w[:, qk_nope:, :]


def visible_keys(t: int, s: int, i: int) -> int:
    """Number of keys query i (0-based) of s new queries sees in a cache of t tokens."""
    return max(0, min(t, t - s + i + 1))


def softmax_rows(scores: np.ndarray, n_visible: Sequence[int]) -> np.ndarray:
    """Two-pass softmax of each row over its first n_visible[i] entries; the rest are 0.

    Rows with no visible entry are all zero.
    """
    p = np.zeros_like(scores, dtype=np.float64)
    for i, n in enumerate(n_visible):
        if n <= 0:
            continue
        row = scores[i, :n]
        m = np.max(row)
        e = np.exp(row - m)
        p[i, :n] = e / np.sum(e)
    return p


def naive_head(q_bh: np.ndarray, kv_b: np.ndarray, pe_b: np.ndarray, wk_h: np.ndarray,
               wv_h: np.ndarray, scale: float, return_probs: bool = False):
    """Naive path for one (sequence, head): materialise k and v, then attend.

    q_bh [s, Dn+R], kv_b [t, C], pe_b [t, R], wk_h [Dn, C], wv_h [Dv, C].
    "Naive Path Execution": k and v are produced by wkv_b before caching,
    scores = q . k * softmax_scale, x = scores . v (with the softmax reading).
    """
    q_bh = np.asarray(q_bh, dtype=np.float64)
    kv_b = np.asarray(kv_b, dtype=np.float64)
    pe_b = np.asarray(pe_b, dtype=np.float64)
    s, t = q_bh.shape[0], kv_b.shape[0]
    k = np.concatenate([kv_b @ wk_h.T, pe_b], axis=1)          # [t, Dn+R]
    v = kv_b @ wv_h.T                                            # [t, Dv]
    scores = (q_bh @ k.T) * scale                                # [s, t]
    p = softmax_rows(scores, [visible_keys(t, s, i) for i in range(s)])
    out = p @ v                                                  # [s, Dv]
    return (out, p) if return_probs else out


def _seq_slices(cu: np.ndarray):
    return [(int(cu[b]), int(cu[b + 1])) for b in range(len(cu) - 1)]


def mla_naive(q, kv, pe, wkv_b, cu_seqlens_q, cu_seqlens_k, heads, qk_nope, qk_rope, v_head,
              scale, pairs: Optional[Iterable[Tuple[int, int]]] = None):
    """Naive-path MLA over packed sequences.

    q [N_q, H, Dn+R], kv [sum_t, C], pe [sum_t, R], wkv_b [H*(Dn+Dv), C].
    Returns out [N_q, H, Dv] in float64.  With ``pairs`` (a list of
    (sequence, head)) only those entries are computed and a dict
    {(b, h): out[s_b, Dv]} is returned.
    """
    wk, wv = head_view(wkv_b, heads, qk_nope, v_head)
    qs, ks = _seq_slices(np.asarray(cu_seqlens_q)), _seq_slices(np.asarray(cu_seqlens_k))
    if pairs is not None:
        res: Dict[Tuple[int, int], np.ndarray] = {}
        for b, h in pairs:
            (q0, q1), (k0, k1) = qs[b], ks[b]
            res[(b, h)] = naive_head(q[q0:q1, h, :], kv[k0:k1], pe[k0:k1], wk[h], wv[h], scale)
        return res
    out = np.zeros((q.shape[0], heads, v_head), dtype=np.float64)
    for b in range(len(qs)):
        (q0, q1), (k0, k1) = qs[b], ks[b]
        if q1 == q0:
            continue
        for h in range(heads):
            out[q0:q1, h, :] = naive_head(q[q0:q1, h, :], kv[k0:k1], pe[k0:k1], wk[h], wv[h], scale)
    return out


def mla_absorb(q, kv, pe, wkv_b, cu_seqlens_q, cu_seqlens_k, heads, qk_nope, qk_rope, v_head, scale):
    """Absorb-path MLA, the page's four einsums in float64, per packed sequence.

    Returns (q_abs [N_q,H,C], o_lat [N_q,H,C], out [N_q,H,Dv]):
      q_abs = einsum("shd,hdc->shc", q_nope, W_k)
      scores = (einsum("shc,tc->sht", q_abs, kv) + einsum("shr,tr->sht", q_pe, pe)) * scale
      o_lat  = einsum("sht,tc->shc", softmax_t(scores), kv)
      out    = einsum("shc,hdc->shd", o_lat, W_v)
    """
    wk, wv = head_view(wkv_b, heads, qk_nope, v_head)
    q = np.asarray(q, dtype=np.float64)
    kv = np.asarray(kv, dtype=np.float64)
    pe = np.asarray(pe, dtype=np.float64)
    q_nope, q_pe = q[:, :, :qk_nope], q[:, :, qk_nope:]
    q_abs = np.einsum("shd,hdc->shc", q_nope, wk)
    o_lat = np.zeros_like(q_abs)
    for (q0, q1), (k0, k1) in zip(_seq_slices(np.asarray(cu_seqlens_q)),
                                  _seq_slices(np.asarray(cu_seqlens_k))):
        s, t = q1 - q0, k1 - k0
        if s == 0:
            continue
        sc = (np.einsum("shc,tc->sht", q_abs[q0:q1], kv[k0:k1])
              + np.einsum("shr,tr->sht", q_pe[q0:q1], pe[k0:k1])) * scale
        nvis = [visible_keys(t, s, i) for i in range(s)]
        for h in range(heads):
            p = softmax_rows(sc[:, h, :], nvis)                  # [s, t]
            o_lat[q0:q1, h, :] = p @ kv[k0:k1]
    out = np.einsum("shc,hdc->shd", o_lat, wv)
    return q_abs, o_lat, out


def workload_naive(w, pairs=None):
    """mla_naive on a workload object (anything with the workload fields)."""
    d = w.dims
    return mla_naive(w.q, w.kv, w.pe, w.wkv_b, w.cu_seqlens_q, w.cu_seqlens_k, d.heads,
                     d.qk_nope, d.qk_rope, d.v_head, d.scale, pairs=pairs)


def workload_absorb(w):
    """mla_absorb on a workload object."""
    d = w.dims
    return mla_absorb(w.q, w.kv, w.pe, w.wkv_b, w.cu_seqlens_q, w.cu_seqlens_k, d.heads,
                      d.qk_nope, d.qk_rope, d.v_head, d.scale)
