"""Exact attention forward with online softmax on B200 (sm_100a).

The kernels and the C ABI live in ``csrc/`` and are built into
``libattn_b200.so`` next to this file; :mod:`.binding` is a thin ctypes layer
over that ABI (argument marshalling only) and :mod:`.inputs` draws the seeded
synthetic workloads.
"""

from .binding import (  # noqa: F401
    AttnError, decode_paged, decode_paged_blasst, decode_workspace_bytes, lib_path,
    decode_paged_fp8, kv_append, load_library, prefill, prefill_blasst, prefill_paged,
)
