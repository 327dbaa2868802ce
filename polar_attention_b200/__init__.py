"""B200 (sm_100a) Polar Attention: fused causal prefill, GQA paged decode and
the gated-delta memory channel.

The computation lives in libpolar_attn.so (hand-written CUDA for sm_100a behind
the C ABI of include/polar_attn.h and include/polar_gdelta.h); ``native`` is its thin ctypes binding and
``workloads`` the seeded synthetic inputs.  The library is loaded on first use,
and a missing build raises: there is no CPU or PyTorch fallback.
"""
from .native import (bwd, bwd_from_state, bwd_workspace_size,  # noqa: F401
                     decode_chunk_workspace_size,
                     decode_paged, decode_paged_chunk,
                     decode_paged_host, decode_staging_size,
                     decode_workspace_size, fwd, fwd_host, fwd_staging_size,
                     fwd_state_size, fwd_train, fwd_workspace_size, gdelta_prefill, gdelta_step,
                     gdelta_workspace_size, get_status,
                     launch_count, PolarError)

__all__ = ["fwd", "bwd", "bwd_workspace_size", "fwd_train", "bwd_from_state", "fwd_state_size",
           "fwd_host", "fwd_staging_size", "fwd_workspace_size", "decode_paged",
           "decode_paged_chunk", "decode_chunk_workspace_size", "decode_paged_host",
           "decode_staging_size", "decode_workspace_size", "gdelta_prefill", "gdelta_step",
           "gdelta_workspace_size", "get_status", "launch_count",
           "PolarError"]
