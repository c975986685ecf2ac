"""B200 (sm_100a) multi-head latent attention in absorb form over a compressed latent cache.

The compute path is the C-ABI library libmla_b200.so (include/mla.h), whose
hot path is hand-written CUDA for sm_100a.  ``deepseek_mla_latent_b200.mla``
holds thin torch-facing wrappers of its calls (importing it loads the
library) and ``workloads`` the seeded synthetic inputs.
"""
from . import workloads  # noqa: F401

__all__ = ["workloads"]
