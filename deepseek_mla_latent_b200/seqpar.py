"""Decode with every sequence's cache split along the token axis over the ranks of a process group.

Rank r of W holds tokens [floor(r t / W), floor((r + 1) t / W)) of each sequence of t tokens (its
own packed cache and cu_seqlens) and every rank holds the same queries.  Softmax attention over
the whole cache is the log-sum-exp combination of softmax attention over disjoint key ranges
("Naive vs Absorb Attention Implementations in DeepSeek-V3", section "Absorb Path Execution": the
score and latent value einsums run over the ranges), so each rank attends to its own range
(mla_attn_decode_partials: per split O relative to the split's reference m, and (m, l)), the
ranks all-gather those partials along the split axis (one collective for O, one for (m, l)),
and every rank merges them (mla_merge_partials, or mla_merge_partials_out fused into the output
projection).  The exchange per step is splits * rows * H * (C * 2 + 8) bytes from each rank.

Every arithmetic step runs in the library's CUDA kernels; this module only cuts the ranges,
moves the partials and calls the library.
"""
from __future__ import annotations

from typing import Optional, Tuple

import numpy as np
import torch
import torch.distributed as dist

from . import mla


def shard_bounds(cu_seqlens_k: np.ndarray, world: int, rank: int) -> Tuple[np.ndarray, np.ndarray]:
    """First and one-past-last cache row of rank `rank`'s token range of every sequence (rows of the
    packed cache described by cu_seqlens_k [batch + 1]); the ranges of the ranks tile each sequence."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError("need 0 <= rank < world")
    cu = np.asarray(cu_seqlens_k, dtype=np.int64)
    t = cu[1:] - cu[:-1]
    return cu[:-1] + (rank * t) // world, cu[:-1] + ((rank + 1) * t) // world


def local_cache(kv: torch.Tensor, pe: torch.Tensor, cu_seqlens_k: np.ndarray, world: int, rank: int):
    """This rank's part of a packed cache: (kv [T_r, C], pe [T_r, R], cu_seqlens [batch + 1] int32 on
    kv's device, longest range).  The rows are copied in sequence order."""
    lo, hi = shard_bounds(cu_seqlens_k, world, rank)
    rows = np.concatenate([np.arange(a, b) for a, b in zip(lo, hi)]) if len(lo) else np.zeros(0, np.int64)
    idx = torch.from_numpy(rows).to(kv.device)
    lens = hi - lo
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    return (kv.index_select(0, idx), pe.index_select(0, idx), torch.from_numpy(cu).to(kv.device),
            int(lens.max()) if len(lens) else 0)


def gather_partials(o: torch.Tensor, ml: torch.Tensor, group=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """All ranks' partials stacked along the split axis in rank order: O [W * S, n, H, C] and
    (m, l) [W * S, n, H, 2] from this rank's O [S, n, H, C] and (m, l) [S, n, H, 2].  Every rank
    must pass the same S (the same num_splits)."""
    world = dist.get_world_size(group)
    o, ml = o.contiguous(), ml.contiguous()
    o_all = o.new_empty((world * o.shape[0],) + tuple(o.shape[1:]))
    ml_all = ml.new_empty((world * ml.shape[0],) + tuple(ml.shape[1:]))
    if dist.get_backend(group) == "nccl":
        dist.all_gather_into_tensor(o_all, o, group=group)
        dist.all_gather_into_tensor(ml_all, ml, group=group)
    else:
        dist.all_gather(list(o_all.chunk(world)), o, group=group)
        dist.all_gather(list(ml_all.chunk(world)), ml, group=group)
    return o_all, ml_all


def decode_sequence_parallel(d: mla.MlaDims, q_abs: torch.Tensor, q: torch.Tensor, kv_local: torch.Tensor,
                             pe_local: torch.Tensor, cu_seqlens_k_local: torch.Tensor, max_seqlen_k_local: int,
                             num_splits: int, wkv_b: Optional[torch.Tensor] = None, group=None) -> torch.Tensor:
    """Decode of `batch` sequences whose caches are spread over the group's ranks (this rank's part:
    kv_local, pe_local, cu_seqlens_k_local, see local_cache).  Returns o_lat [batch, H, C], or
    out [batch, H, Dv] when wkv_b is given (merge fused into the output projection), on every rank.
    num_splits (>= 1) splits per rank; the same on every rank."""
    if num_splits < 1:
        raise ValueError("num_splits must be >= 1 and the same on every rank")
    batch = cu_seqlens_k_local.numel() - 1
    ws = mla.partials_workspace(d, batch, max_seqlen_k_local, num_splits, device=q_abs.device)
    mla.attn_decode_partials(d, q_abs, q, kv_local, pe_local, cu_seqlens_k_local, max_seqlen_k_local, ws, num_splits)
    o, ml = mla.split_partials(d, ws, batch, num_splits)
    o_all, ml_all = gather_partials(o, ml, group)
    if wkv_b is None:
        return mla.merge_partials(d, o_all, ml_all)
    return mla.merge_partials_out(d, o_all, ml_all, wkv_b)
