"""Torch-facing wrappers of the C ABI (same names as include/mla.h, without the prefix).

PyTorch only supplies device memory and the current stream; each wrapper checks
shapes and dtypes, allocates outputs when the caller gives none, and calls the
library.  Layouts are those of include/mla.h:

  q      [N_q, H, Dn+R] (rows may be strided), q_abs / o_lat [N_q, H, C],
  kv     [sum_t, C], pe [sum_t, R], wkv_b [H*(Dn+Dv), C], out [N_q, H, Dv],
  cu_seqlens_* int32 [batch+1] on the device.
"""
from __future__ import annotations

import ctypes
from typing import Optional

import torch

from ._lib import LIB, MLA_DTYPE_BF16, MLA_ERR_UNSUPPORTED, MlaDims, MlaError, _check, dims_from, make_dims  # noqa: F401


def _dtype(d: MlaDims) -> torch.dtype:
    return torch.bfloat16 if d.dtype == MLA_DTYPE_BF16 else torch.float32


def _stream(stream) -> ctypes.c_void_p:
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _need(t: torch.Tensor, name: str, dtype: torch.dtype, shape=None, contiguous=True) -> None:
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    if contiguous and not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _q_row_stride(q: torch.Tensor, d: MlaDims) -> int:
    H, W = d.num_heads, d.qk_nope_head_dim + d.qk_rope_head_dim
    if q.dim() != 3 or q.shape[1] != H or q.shape[2] != W or q.stride(2) != 1 or q.stride(1) != W:
        raise ValueError(f"q must be [N, {H}, {W}] with contiguous heads (row stride free)")
    return q.stride(0) if q.shape[0] > 1 else H * W


def kernel_family(d: MlaDims) -> int:
    return LIB.mla_kernel_family(ctypes.byref(d))


def decode_num_splits(d: MlaDims, batch: int, max_seqlen_k: int, num_splits: int = 0) -> int:
    return int(LIB.mla_decode_num_splits(ctypes.byref(d), batch, max_seqlen_k, num_splits))


def absorb_q(d: MlaDims, q: torch.Tensor, wkv_b: torch.Tensor, q_abs: Optional[torch.Tensor] = None,
             stream=None) -> torch.Tensor:
    dt = _dtype(d)
    n = q.shape[0]
    rs = _q_row_stride(q, d)
    _need(q, "q", dt, contiguous=False)
    _need(wkv_b, "wkv_b", dt, (d.num_heads * (d.qk_nope_head_dim + d.v_head_dim), d.kv_lora_rank))
    if q_abs is None:
        q_abs = torch.empty((n, d.num_heads, d.kv_lora_rank), dtype=dt, device=q.device)
    _need(q_abs, "q_abs", dt, (n, d.num_heads, d.kv_lora_rank))
    _check(LIB.mla_absorb_q(ctypes.byref(d), _ptr(q), rs, _ptr(wkv_b), _ptr(q_abs), n, _stream(stream)),
           "mla_absorb_q")
    return q_abs


def workspace_size(d: MlaDims, batch: int, n_q_rows: int, max_seqlen_k: int, num_splits: int = 0) -> int:
    return int(LIB.mla_workspace_size(ctypes.byref(d), batch, n_q_rows, max_seqlen_k, num_splits))


def workspace(d: MlaDims, batch: int, n_q_rows: int, max_seqlen_k: int, num_splits: int = 0,
              device="cuda") -> Optional[torch.Tensor]:
    nbytes = workspace_size(d, batch, n_q_rows, max_seqlen_k, num_splits)
    return torch.empty(max(nbytes, 16), dtype=torch.uint8, device=device) if nbytes else None


def attn_decode(d: MlaDims, q_abs: torch.Tensor, q: torch.Tensor, kv: torch.Tensor, pe: torch.Tensor,
                cu_seqlens_k: torch.Tensor, max_seqlen_k: int, o_lat: Optional[torch.Tensor] = None,
                ws: Optional[torch.Tensor] = None, num_splits: int = 0, stream=None) -> torch.Tensor:
    dt = _dtype(d)
    batch = cu_seqlens_k.numel() - 1
    H, C, R = d.num_heads, d.kv_lora_rank, d.qk_rope_head_dim
    rs = _q_row_stride(q, d)
    _need(q_abs, "q_abs", dt, (batch, H, C))
    _need(q, "q", dt, contiguous=False)
    _need(kv, "kv", dt)
    _need(pe, "pe", dt)
    _need(cu_seqlens_k, "cu_seqlens_k", torch.int32)
    if kv.dim() != 2 or kv.shape[1] != C or pe.dim() != 2 or pe.shape[1] != R or pe.shape[0] != kv.shape[0]:
        raise ValueError("kv must be [T, C] and pe [T, R]")
    if o_lat is None:
        o_lat = torch.empty((batch, H, C), dtype=dt, device=q_abs.device)
    _need(o_lat, "o_lat", dt, (batch, H, C))
    if ws is None:
        ws = workspace(d, batch, batch, max_seqlen_k, num_splits, device=q_abs.device)
    wsb = ws.numel() if ws is not None else 0
    _check(LIB.mla_attn_decode(ctypes.byref(d), _ptr(q_abs), _ptr(q), rs, _ptr(kv), _ptr(pe), kv.shape[0],
                               _ptr(cu_seqlens_k),
                               batch, int(max_seqlen_k), _ptr(o_lat), _ptr(ws), wsb, num_splits, _stream(stream)),
           "mla_attn_decode")
    return o_lat


def partials_workspace(d: MlaDims, batch: int, max_seqlen_k: int, num_splits: int = 0,
                       device="cuda") -> torch.Tensor:
    nbytes = int(LIB.mla_partials_workspace_size(ctypes.byref(d), batch, max_seqlen_k, num_splits))
    if nbytes == 0:
        raise MlaError(MLA_ERR_UNSUPPORTED, "mla_partials_workspace_size: dims without the partial form")
    return torch.empty(nbytes, dtype=torch.uint8, device=device)


def attn_decode_partials(d: MlaDims, q_abs: torch.Tensor, q: torch.Tensor, kv: torch.Tensor, pe: torch.Tensor,
                         cu_seqlens_k: torch.Tensor, max_seqlen_k: int, ws: Optional[torch.Tensor] = None,
                         num_splits: int = 0, stream=None) -> torch.Tensor:
    """Decode attention leaving the split partials in the workspace (mla_attn_decode_partials);
    returns the workspace (split_partials views it)."""
    dt = _dtype(d)
    batch = cu_seqlens_k.numel() - 1
    H, C, R = d.num_heads, d.kv_lora_rank, d.qk_rope_head_dim
    rs = _q_row_stride(q, d)
    _need(q_abs, "q_abs", dt, (batch, H, C))
    _need(q, "q", dt, contiguous=False)
    _need(kv, "kv", dt)
    _need(pe, "pe", dt)
    _need(cu_seqlens_k, "cu_seqlens_k", torch.int32)
    if kv.dim() != 2 or kv.shape[1] != C or pe.dim() != 2 or pe.shape[1] != R or pe.shape[0] != kv.shape[0]:
        raise ValueError("kv must be [T, C] and pe [T, R]")
    if ws is None:
        ws = partials_workspace(d, batch, max_seqlen_k, num_splits, device=q_abs.device)
    _need(ws, "workspace", torch.uint8)
    _check(LIB.mla_attn_decode_partials(ctypes.byref(d), _ptr(q_abs), _ptr(q), rs, _ptr(kv), _ptr(pe), kv.shape[0],
                                        _ptr(cu_seqlens_k), batch, int(max_seqlen_k), _ptr(ws), ws.numel(),
                                        num_splits, _stream(stream)),
           "mla_attn_decode_partials")
    return ws


def split_partials(d: MlaDims, ws: torch.Tensor, batch: int, splits: int):
    """Views of the partial form mla_attn_decode_partials leaves in `ws`: O [splits, batch, H, C]
    (bf16) and (m, l) [splits, batch, H, 2] (fp32), as include/mla.h lays them out."""
    H, C = d.num_heads, d.kv_lora_rank
    o_bytes = splits * batch * H * C * 2
    off = (o_bytes + 255) // 256 * 256
    o = ws[:o_bytes].view(torch.bfloat16).view(splits, batch, H, C)
    ml = ws[off:off + splits * batch * H * 8].view(torch.float32).view(splits, batch, H, 2)
    return o, ml


def merge_partials(d: MlaDims, part_o: torch.Tensor, part_ml: torch.Tensor, o_lat: Optional[torch.Tensor] = None,
                   stream=None) -> torch.Tensor:
    """o_lat [n, H, C] from split partials O [S, n, H, C] (bf16) and (m, l) [S, n, H, 2] (fp32), e.g.
    several attn_decode_partials results stacked along the split axis (mla_merge_partials)."""
    S, n, H, C = part_o.shape
    _need(part_o, "part_o", torch.bfloat16, (S, n, d.num_heads, d.kv_lora_rank))
    _need(part_ml, "part_ml", torch.float32, (S, n, d.num_heads, 2))
    if o_lat is None:
        o_lat = torch.empty((n, H, C), dtype=torch.bfloat16, device=part_o.device)
    _need(o_lat, "o_lat", torch.bfloat16, (n, H, C))
    _check(LIB.mla_merge_partials(ctypes.byref(d), _ptr(part_o), _ptr(part_ml), S, n, _ptr(o_lat), _stream(stream)),
           "mla_merge_partials")
    return o_lat


def merge_partials_out(d: MlaDims, part_o: torch.Tensor, part_ml: torch.Tensor, wkv_b: torch.Tensor,
                       out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """out [n, H, Dv]: the merge of merge_partials fused into the output projection (mla_merge_partials_out)."""
    S, n, H, C = part_o.shape
    _need(part_o, "part_o", torch.bfloat16, (S, n, d.num_heads, d.kv_lora_rank))
    _need(part_ml, "part_ml", torch.float32, (S, n, d.num_heads, 2))
    _need(wkv_b, "wkv_b", torch.bfloat16, (H * (d.qk_nope_head_dim + d.v_head_dim), C))
    if out is None:
        out = torch.empty((n, H, d.v_head_dim), dtype=torch.bfloat16, device=part_o.device)
    _need(out, "out", torch.bfloat16, (n, H, d.v_head_dim))
    _check(LIB.mla_merge_partials_out(ctypes.byref(d), _ptr(part_o), _ptr(part_ml), S, n, _ptr(wkv_b), _ptr(out),
                                      _stream(stream)), "mla_merge_partials_out")
    return out


def decode_out_workspace(d: MlaDims, batch: int, max_seqlen_k: int, num_splits: int = 0,
                         device="cuda") -> torch.Tensor:
    nbytes = int(LIB.mla_decode_out_workspace_size(ctypes.byref(d), batch, max_seqlen_k, num_splits))
    return torch.empty(max(nbytes, 16), dtype=torch.uint8, device=device)


def attn_decode_out(d: MlaDims, q_abs: torch.Tensor, q: torch.Tensor, kv: torch.Tensor, pe: torch.Tensor,
                    cu_seqlens_k: torch.Tensor, max_seqlen_k: int, wkv_b: torch.Tensor,
                    out: Optional[torch.Tensor] = None, ws: Optional[torch.Tensor] = None, num_splits: int = 0,
                    stream=None) -> torch.Tensor:
    """Decode attention and the output projection in one call (mla_attn_decode_out)."""
    dt = _dtype(d)
    batch = cu_seqlens_k.numel() - 1
    H, C, R = d.num_heads, d.kv_lora_rank, d.qk_rope_head_dim
    rs = _q_row_stride(q, d)
    _need(q_abs, "q_abs", dt, (batch, H, C))
    _need(q, "q", dt, contiguous=False)
    _need(kv, "kv", dt)
    _need(pe, "pe", dt)
    _need(cu_seqlens_k, "cu_seqlens_k", torch.int32)
    _need(wkv_b, "wkv_b", dt, (H * (d.qk_nope_head_dim + d.v_head_dim), C))
    if kv.dim() != 2 or kv.shape[1] != C or pe.dim() != 2 or pe.shape[1] != R or pe.shape[0] != kv.shape[0]:
        raise ValueError("kv must be [T, C] and pe [T, R]")
    if out is None:
        out = torch.empty((batch, H, d.v_head_dim), dtype=dt, device=q_abs.device)
    _need(out, "out", dt, (batch, H, d.v_head_dim))
    if ws is None:
        ws = decode_out_workspace(d, batch, max_seqlen_k, num_splits, device=q_abs.device)
    _check(LIB.mla_attn_decode_out(ctypes.byref(d), _ptr(q_abs), _ptr(q), rs, _ptr(kv), _ptr(pe), kv.shape[0],
                                   _ptr(cu_seqlens_k), batch, int(max_seqlen_k), _ptr(wkv_b), _ptr(out), _ptr(ws),
                                   ws.numel(), num_splits, _stream(stream)),
           "mla_attn_decode_out")
    return out


def decode_fused_workspace(d: MlaDims, batch: int, max_seqlen_k: int, num_splits: int = 0,
                           device="cuda") -> torch.Tensor:
    """Workspace of mla_attn_decode_fused, zero-filled (its control words must start at zero)."""
    nbytes = int(LIB.mla_decode_fused_workspace_size(ctypes.byref(d), batch, max_seqlen_k, num_splits))
    return torch.zeros(max(nbytes, 16), dtype=torch.uint8, device=device)


def attn_decode_fused(d: MlaDims, q_abs: torch.Tensor, q: torch.Tensor, kv: torch.Tensor, pe: torch.Tensor,
                      cu_seqlens_k: torch.Tensor, max_seqlen_k: int, wkv_b: torch.Tensor,
                      out: Optional[torch.Tensor] = None, ws: Optional[torch.Tensor] = None, num_splits: int = 0,
                      stream=None) -> torch.Tensor:
    """Decode attention, split merge and output projection, in one kernel where it fits
    (mla_attn_decode_fused).  ws must come from decode_fused_workspace (or be zero-filled)."""
    dt = _dtype(d)
    batch = cu_seqlens_k.numel() - 1
    H, C, R, Dn, Dv = d.num_heads, d.kv_lora_rank, d.qk_rope_head_dim, d.qk_nope_head_dim, d.v_head_dim
    rs = _q_row_stride(q, d)
    _need(q_abs, "q_abs", dt, (batch, H, C))
    _need(q, "q", dt, contiguous=False)
    _need(kv, "kv", dt)
    _need(pe, "pe", dt)
    _need(wkv_b, "wkv_b", dt, (H * (Dn + Dv), C))
    _need(cu_seqlens_k, "cu_seqlens_k", torch.int32)
    if kv.dim() != 2 or kv.shape[1] != C or pe.dim() != 2 or pe.shape[1] != R or pe.shape[0] != kv.shape[0]:
        raise ValueError("kv must be [T, C] and pe [T, R]")
    if out is None:
        out = torch.empty((batch, H, Dv), dtype=dt, device=q_abs.device)
    _need(out, "out", dt, (batch, H, Dv))
    if ws is None:
        ws = decode_fused_workspace(d, batch, max_seqlen_k, num_splits, device=q_abs.device)
    _need(ws, "workspace", torch.uint8)
    _check(LIB.mla_attn_decode_fused(ctypes.byref(d), _ptr(q_abs), _ptr(q), rs, _ptr(kv), _ptr(pe), kv.shape[0],
                                     _ptr(cu_seqlens_k), batch, int(max_seqlen_k), _ptr(wkv_b), _ptr(out), _ptr(ws),
                                     ws.numel(), num_splits, _stream(stream)), "mla_attn_decode_fused")
    return out


def attn_prefill_chunk(d: MlaDims, q_abs: torch.Tensor, q: torch.Tensor, cu_seqlens_q: torch.Tensor,
                       cu_seqlens_k: torch.Tensor, max_seqlen_q: int, max_seqlen_k: int, kv: torch.Tensor,
                       pe: torch.Tensor, o_lat: Optional[torch.Tensor] = None, ws: Optional[torch.Tensor] = None,
                       stream=None) -> torch.Tensor:
    dt = _dtype(d)
    batch = cu_seqlens_k.numel() - 1
    n = q_abs.shape[0]
    H, C, R = d.num_heads, d.kv_lora_rank, d.qk_rope_head_dim
    rs = _q_row_stride(q, d)
    _need(q_abs, "q_abs", dt, (n, H, C))
    _need(q, "q", dt, contiguous=False)
    _need(kv, "kv", dt)
    _need(pe, "pe", dt)
    _need(cu_seqlens_q, "cu_seqlens_q", torch.int32, (batch + 1,))
    _need(cu_seqlens_k, "cu_seqlens_k", torch.int32)
    if kv.dim() != 2 or kv.shape[1] != C or pe.dim() != 2 or pe.shape[1] != R or pe.shape[0] != kv.shape[0]:
        raise ValueError("kv must be [T, C] and pe [T, R]")
    if o_lat is None:
        o_lat = torch.empty((n, H, C), dtype=dt, device=q_abs.device)
    _need(o_lat, "o_lat", dt, (n, H, C))
    if ws is None:
        ws = workspace(d, batch, n, max_seqlen_k, 0, device=q_abs.device)
    wsb = ws.numel() if ws is not None else 0
    _check(LIB.mla_attn_prefill_chunk(ctypes.byref(d), _ptr(q_abs), _ptr(q), rs, _ptr(cu_seqlens_q),
                                      _ptr(cu_seqlens_k), batch, n, int(max_seqlen_q), int(max_seqlen_k), _ptr(kv),
                                      _ptr(pe), kv.shape[0], _ptr(o_lat), _ptr(ws), wsb, _stream(stream)),
           "mla_attn_prefill_chunk")
    return o_lat


def attn_paged(d: MlaDims, q_abs: torch.Tensor, q: torch.Tensor, seqlens_k: torch.Tensor, max_seqlen_k: int,
               kv_cache: torch.Tensor, pe_cache: torch.Tensor, block_table: torch.Tensor, page_size: int,
               cu_seqlens_q: Optional[torch.Tensor] = None, o_lat: Optional[torch.Tensor] = None,
               ws: Optional[torch.Tensor] = None, num_splits: int = 0, stream=None) -> torch.Tensor:
    """Attention over a paged cache (mla_attn_paged): decode when cu_seqlens_q is None, else a
    chunked prefill.  kv_cache [num_pages * page_size, C], pe_cache [num_pages * page_size, R],
    block_table int32 [batch, max_pages_per_seq], seqlens_k int32 [batch]."""
    dt = _dtype(d)
    batch = seqlens_k.numel()
    n = q_abs.shape[0]
    H, C, R = d.num_heads, d.kv_lora_rank, d.qk_rope_head_dim
    rs = _q_row_stride(q, d)
    _need(q_abs, "q_abs", dt, (n, H, C))
    _need(q, "q", dt, contiguous=False)
    _need(kv_cache, "kv_cache", dt)
    _need(pe_cache, "pe_cache", dt)
    _need(seqlens_k, "seqlens_k", torch.int32, (batch,))
    _need(block_table, "block_table", torch.int32)
    if cu_seqlens_q is not None:
        _need(cu_seqlens_q, "cu_seqlens_q", torch.int32, (batch + 1,))
    if block_table.dim() != 2 or block_table.shape[0] != batch:
        raise ValueError("block_table must be [batch, max_pages_per_seq]")
    if (kv_cache.dim() != 2 or kv_cache.shape[1] != C or pe_cache.dim() != 2 or pe_cache.shape[1] != R
            or pe_cache.shape[0] != kv_cache.shape[0] or page_size <= 0 or kv_cache.shape[0] % page_size != 0):
        raise ValueError("kv_cache must be [num_pages * page_size, C] and pe_cache [num_pages * page_size, R]")
    if o_lat is None:
        o_lat = torch.empty((n, H, C), dtype=dt, device=q_abs.device)
    _need(o_lat, "o_lat", dt, (n, H, C))
    if ws is None:
        ws = workspace(d, batch, n, max_seqlen_k, num_splits, device=q_abs.device)
    wsb = ws.numel() if ws is not None else 0
    _check(LIB.mla_attn_paged(ctypes.byref(d), _ptr(q_abs), _ptr(q), rs, _ptr(cu_seqlens_q), n, _ptr(seqlens_k),
                              batch, int(max_seqlen_k), _ptr(kv_cache), _ptr(pe_cache),
                              kv_cache.shape[0] // page_size, int(page_size), _ptr(block_table),
                              block_table.shape[1], _ptr(o_lat), _ptr(ws), wsb, num_splits, _stream(stream)),
           "mla_attn_paged")
    return o_lat


def out_proj(d: MlaDims, o_lat: torch.Tensor, wkv_b: torch.Tensor, out: Optional[torch.Tensor] = None,
             stream=None) -> torch.Tensor:
    dt = _dtype(d)
    n = o_lat.shape[0]
    _need(o_lat, "o_lat", dt, (n, d.num_heads, d.kv_lora_rank))
    _need(wkv_b, "wkv_b", dt, (d.num_heads * (d.qk_nope_head_dim + d.v_head_dim), d.kv_lora_rank))
    if out is None:
        out = torch.empty((n, d.num_heads, d.v_head_dim), dtype=dt, device=o_lat.device)
    _need(out, "out", dt, (n, d.num_heads, d.v_head_dim))
    _check(LIB.mla_out_proj(ctypes.byref(d), _ptr(o_lat), _ptr(wkv_b), _ptr(out), n, _stream(stream)),
           "mla_out_proj")
    return out


def expand_kv(d: MlaDims, kv_c: torch.Tensor, wkv_b: torch.Tensor, batch: int, seq_len: int,
              gamma: Optional[torch.Tensor] = None, eps: float = 1e-6, k_nope: Optional[torch.Tensor] = None,
              v: Optional[torch.Tensor] = None, stream=None):
    """Latent KV expansion (mla_expand_kv): K_nope [batch, H, seq_len, Dn] and V [batch, H, seq_len, Dv]
    from the compressed rows kv_c [batch * seq_len, C]."""
    dt = _dtype(d)
    H, C, Dn, Dv = d.num_heads, d.kv_lora_rank, d.qk_nope_head_dim, d.v_head_dim
    _need(kv_c, "kv_c", dt, (batch * seq_len, C))
    _need(wkv_b, "wkv_b", dt, (H * (Dn + Dv), C))
    if gamma is not None:
        _need(gamma, "gamma", dt, (C,))
    if k_nope is None:
        k_nope = torch.empty((batch, H, seq_len, Dn), dtype=dt, device=kv_c.device)
    if v is None:
        v = torch.empty((batch, H, seq_len, Dv), dtype=dt, device=kv_c.device)
    _need(k_nope, "k_nope", dt, (batch, H, seq_len, Dn))
    _need(v, "v", dt, (batch, H, seq_len, Dv))
    _check(LIB.mla_expand_kv(ctypes.byref(d), _ptr(kv_c), _ptr(gamma), float(eps), _ptr(wkv_b), batch, seq_len,
                             _ptr(k_nope), _ptr(v), _stream(stream)), "mla_expand_kv")
    return k_nope, v


def attn_prefill_expanded(d: MlaDims, q: torch.Tensor, k_nope: torch.Tensor, v: torch.Tensor, pe: torch.Tensor,
                          cu_seqlens_q: torch.Tensor, cu_seqlens_k: torch.Tensor, max_seqlen_q: int,
                          out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """Chunked-prefill attention on the naive path (mla_attn_prefill_expanded): out [n_q, H, Dv] from
    q [n_q, H, Dn+R], K_nope [H, T, Dn] and V [H, T, Dv] (mla_expand_kv with batch 1 over the T
    cache rows, viewed without the batch axis) and pe [T, R]."""
    dt = _dtype(d)
    H, Dn, R, Dv = d.num_heads, d.qk_nope_head_dim, d.qk_rope_head_dim, d.v_head_dim
    rs = _q_row_stride(q, d)
    n = q.shape[0]
    T = pe.shape[0]
    _need(q, "q", dt, contiguous=False)
    _need(k_nope, "k_nope", dt, (H, T, Dn))
    _need(v, "v", dt, (H, T, Dv))
    _need(pe, "pe", dt, (T, R))
    _need(cu_seqlens_q, "cu_seqlens_q", torch.int32)
    _need(cu_seqlens_k, "cu_seqlens_k", torch.int32)
    batch = cu_seqlens_q.numel() - 1
    if cu_seqlens_k.numel() != batch + 1:
        raise ValueError("cu_seqlens_q and cu_seqlens_k must have the same length")
    if out is None:
        out = torch.empty((n, H, Dv), dtype=dt, device=q.device)
    _need(out, "out", dt, (n, H, Dv))
    _check(LIB.mla_attn_prefill_expanded(ctypes.byref(d), _ptr(q), rs, _ptr(k_nope), _ptr(v), _ptr(pe), T,
                                         _ptr(cu_seqlens_q), _ptr(cu_seqlens_k), batch, n, int(max_seqlen_q),
                                         _ptr(out), _stream(stream)), "mla_attn_prefill_expanded")
    return out


def attn_sparse_decode(d: MlaDims, q_abs: torch.Tensor, q: torch.Tensor, kv: torch.Tensor, pe: torch.Tensor,
                       indices: torch.Tensor, counts: torch.Tensor, o_lat: Optional[torch.Tensor] = None,
                       ws: Optional[torch.Tensor] = None, num_splits: int = 0, stream=None) -> torch.Tensor:
    """Decode over a selected list of cache rows per sequence (mla_attn_sparse_decode): indices
    [batch, max_topk] int32 (row b: the cache rows sequence b attends to), counts [batch] int32."""
    dt = _dtype(d)
    batch, max_topk = indices.shape
    H, C, R = d.num_heads, d.kv_lora_rank, d.qk_rope_head_dim
    rs = _q_row_stride(q, d)
    _need(q_abs, "q_abs", dt, (batch, H, C))
    _need(q, "q", dt, contiguous=False)
    _need(kv, "kv", dt)
    _need(pe, "pe", dt)
    _need(indices, "indices", torch.int32, (batch, max_topk))
    _need(counts, "counts", torch.int32, (batch,))
    if kv.dim() != 2 or kv.shape[1] != C or pe.dim() != 2 or pe.shape[1] != R or pe.shape[0] != kv.shape[0]:
        raise ValueError("kv must be [T, C] and pe [T, R]")
    if o_lat is None:
        o_lat = torch.empty((batch, H, C), dtype=dt, device=q_abs.device)
    _need(o_lat, "o_lat", dt, (batch, H, C))
    if ws is None:
        nbytes = int(LIB.mla_sparse_workspace_size(ctypes.byref(d), batch, max_topk, num_splits))
        ws = torch.empty(max(nbytes, 16), dtype=torch.uint8, device=q_abs.device)
    _check(LIB.mla_attn_sparse_decode(ctypes.byref(d), _ptr(q_abs), _ptr(q), rs, _ptr(kv), _ptr(pe), kv.shape[0],
                                      _ptr(indices), max_topk, _ptr(counts), batch, max_topk, _ptr(o_lat), _ptr(ws),
                                      ws.numel(), num_splits, _stream(stream)), "mla_attn_sparse_decode")
    return o_lat


def append_latent(d: MlaDims, kv_new: torch.Tensor, k_pe_new: torch.Tensor, positions: torch.Tensor,
                  slots: torch.Tensor, kv_cache: torch.Tensor, pe_cache: torch.Tensor,
                  gamma: Optional[torch.Tensor] = None, eps: float = 1e-6, rope_base: float = 10000.0,
                  stream=None) -> None:
    """Write normalised latents and rotated rotary keys of new tokens into the caches (mla_append_latent)."""
    dt = _dtype(d)
    n = kv_new.shape[0]
    C, R = d.kv_lora_rank, d.qk_rope_head_dim
    _need(kv_new, "kv_new", dt, (n, C))
    _need(k_pe_new, "k_pe_new", dt, (n, R))
    _need(positions, "positions", torch.int32, (n,))
    _need(slots, "slots", torch.int64, (n,))
    _need(kv_cache, "kv_cache", dt)
    _need(pe_cache, "pe_cache", dt)
    if kv_cache.dim() != 2 or kv_cache.shape[1] != C or pe_cache.dim() != 2 or pe_cache.shape[1] != R or \
            pe_cache.shape[0] != kv_cache.shape[0]:
        raise ValueError("kv_cache must be [T, C] and pe_cache [T, R]")
    if gamma is not None:
        _need(gamma, "gamma", dt, (C,))
    _check(LIB.mla_append_latent(ctypes.byref(d), _ptr(kv_new), _ptr(k_pe_new), _ptr(gamma), float(eps),
                                 float(rope_base), _ptr(positions), _ptr(slots), n, _ptr(kv_cache), _ptr(pe_cache),
                                 kv_cache.shape[0], _stream(stream)),
           "mla_append_latent")


def device_status(stream=None) -> int:
    """Synchronise the stream and raise MlaError if a device wait ran out; returns the error word."""
    word = ctypes.c_uint32(0)
    st = LIB.mla_device_status(_stream(stream), ctypes.byref(word))
    _check(st, f"mla_device_status (device word {word.value:#x})")
    return word.value


def decode_step(d: MlaDims, q: torch.Tensor, wkv_b: torch.Tensor, kv: torch.Tensor, pe: torch.Tensor,
                cu_seqlens_k: torch.Tensor, max_seqlen_k: int, num_splits: int = 0, bufs: Optional[dict] = None,
                stream=None) -> torch.Tensor:
    """The whole absorb decode path: mla_absorb_q -> mla_attn_decode_out (attention, then the
    output projection, with the projection's weights staged into L2 during the attention tail).

    ``bufs`` may hold preallocated "q_abs", "out" and "ws_out" (mla_decode_out_workspace_size
    bytes) tensors."""
    bufs = bufs or {}
    q_abs = absorb_q(d, q, wkv_b, bufs.get("q_abs"), stream)
    return attn_decode_out(d, q_abs, q, kv, pe, cu_seqlens_k, max_seqlen_k, wkv_b, bufs.get("out"),
                           bufs.get("ws_out"), num_splits, stream)


def prefill_step(d: MlaDims, q: torch.Tensor, wkv_b: torch.Tensor, kv: torch.Tensor, pe: torch.Tensor,
                 cu_seqlens_q: torch.Tensor, cu_seqlens_k: torch.Tensor, max_seqlen_q: int, max_seqlen_k: int,
                 bufs: Optional[dict] = None, stream=None) -> torch.Tensor:
    """The whole chunked-prefill path: mla_absorb_q -> mla_attn_prefill_chunk -> mla_out_proj."""
    bufs = bufs or {}
    q_abs = absorb_q(d, q, wkv_b, bufs.get("q_abs"), stream)
    o_lat = attn_prefill_chunk(d, q_abs, q, cu_seqlens_q, cu_seqlens_k, max_seqlen_q, max_seqlen_k, kv, pe,
                               bufs.get("o_lat"), bufs.get("ws"), stream)
    return out_proj(d, o_lat, wkv_b, bufs.get("out"), stream)
