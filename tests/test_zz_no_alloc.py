"""The decode entry point that allocates nothing, against the one that takes a
caller workspace.

attn_decode_paged_noalloc serves callers that cannot allocate device memory
while they decode (their memory is reserved up front for the KV-cache pool,
or their thread must not call cudaMalloc, which may synchronise the device);
its split partials live in the library's fixed 16 MiB device scratch. This
file is collected last so that a run stopping at the first failure has run
every other test already; it also passes on its own in a fresh process.
"""

import ctypes

import numpy as np
import pytest
import torch

from attention_online_softmax_fwd_b200 import binding
from attention_online_softmax_fwd_b200 import inputs as gen

pytestmark = pytest.mark.gpu


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else None


def _noalloc_call(lib, cache, dev, split, o, lse):
    """Call the C ABI entry point directly (no Python-side workspace exists)."""
    q, kp, vp, bt, sl = (t.to(dev) for t in (cache.q, cache.k_pages, cache.v_pages, cache.block_table,
                                             cache.seq_lens))
    N, Hq, D = q.shape
    st = lib.attn_decode_paged_noalloc(
        _ptr(q), _ptr(kp), _ptr(vp), _ptr(bt), _ptr(sl), N, Hq, kp.shape[2], D, cache.page_size,
        bt.shape[1], kp.shape[0], gen.attn_scale(D), 0.0, split, _ptr(o), _ptr(lse), None, None,
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    return st


def _workspace_call(cache, dev, split):
    o, lse = binding.decode_paged(cache.q.to(dev), cache.k_pages.to(dev), cache.v_pages.to(dev),
                                  cache.block_table.to(dev), cache.seq_lens.to(dev),
                                  scale=gen.attn_scale(cache.q.shape[-1]), split_tokens=split)
    return o, lse


def test_noalloc_decode_matches_workspace_decode_twice(cuda_device):
    lib = binding.load_library()
    # two different workloads in a row: the second runs on the scratch the first left behind
    cases = [
        (gen.paged_decode_inputs(16, 32, 8, 128, 16, 64, 3000, seed=4100), 256),
        (gen.paged_decode_inputs(8, 16, 2, 64, 64, 1, 2500, seed=4101), 128),
    ]
    for cache, split in cases:
        N, Hq, D = cache.q.shape
        o = torch.empty((N, Hq, D), dtype=torch.bfloat16, device=cuda_device)
        lse = torch.empty((N, Hq), dtype=torch.float32, device=cuda_device)
        assert _noalloc_call(lib, cache, cuda_device, split, o, lse) == 0
        o_ref, lse_ref = _workspace_call(cache, cuda_device, split)
        torch.cuda.synchronize()
        # the same kernels on the same inputs, in a fixed order: the results agree bit for bit
        assert torch.equal(o, o_ref) and torch.equal(lse, lse_ref), f"noalloc split={split}"
        assert torch.isfinite(o.float()).all()


def test_noalloc_rejects_a_call_beyond_its_scratch(cuda_device):
    lib = binding.load_library()
    # 4096 sequences x 64 splits x 32 heads x 128 x 4 B is far above 16 MiB
    need = lib.attn_decode_workspace_bytes(4096, 32, 128, 4096, 16, 1024)
    assert need > binding.NOALLOC_SCRATCH_BYTES
    f = ctypes.c_void_p(1 << 20)
    st = lib.attn_decode_paged_noalloc(f, f, f, f, f, 4096, 32, 8, 128, 16, 4096, 1024, 0.088, 0.0, 1024, f,
                                       None, None, None, None)
    assert st == 1                       # ATTN_ERR_INVALID_ARG, nothing enqueued
