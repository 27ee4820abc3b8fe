"""Float64 CPU oracle (test infrastructure only; see attn64 for the header)."""
from .attn64 import (  # noqa: F401
    attn_bwd,
    attn_bwd_varlen,
    attn_fwd,
    attn_fwd_varlen,
    attn_fwd_rows,
    attn_fwd_online,
    attn_partial,
    attn_with_kvcache,
    combine_splits,
    effective_window,
    gather_cache,
    kvcache_append,
    rotary,
    split_token_ranges,
    visible,
    visible_rows,
)
