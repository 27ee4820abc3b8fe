"""B200 (sm_100a) exact attention: tiled online-softmax forward, recompute
backward, GQA, split-KV paged decode, behind the C ABI of include/fa.h.

Importing the package does not load libfa.so; the first call does, and fails
loudly if it has not been built.
"""
from .api import (  # noqa: F401
    fa_bwd,
    fa_bwd_workspace_size,
    fa_fwd,
    fa_fwd_kvcache,
    fa_kvcache_workspace_size,
    fa_last_device_status,
    fa_last_launch_count,
    fa_set_fwd_kernel,
    fa_status_string,
)
