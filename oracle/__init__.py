"""fp64 CPU oracle for MLA attention (test infrastructure only; see mla_oracle)."""
from .mla_oracle import (head_view, visible_keys, softmax_rows, naive_head, mla_naive, mla_absorb,
                         workload_naive, workload_absorb)
from .append_oracle import rms_norm, rope_interleaved, append_latent
from .paged_oracle import gather_paged, mla_naive_paged
from .expand_oracle import expand_kv
from .sparse_oracle import gather_selected, mla_naive_sparse

__all__ = ["head_view", "visible_keys", "softmax_rows", "naive_head", "mla_naive", "mla_absorb",
           "workload_naive", "workload_absorb", "rms_norm", "rope_interleaved", "append_latent",
           "gather_paged", "mla_naive_paged", "expand_kv", "gather_selected", "mla_naive_sparse"]
