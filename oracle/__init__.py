"""Float64 CPU oracle (test infrastructure only; see attn_oracle's header)."""
from .attn_oracle import (  # noqa: F401
    KV_TILE, Q_TILE, attention_rows, blasst_walk, causal_visible, decode_paged,
    decode_paged_blasst, gather_pages, kv_head_of, prefill, prefill_blasst,
)
