"""The entry points enqueue on the caller's stream without allocating or
synchronising, so a CUDA graph can capture them: replaying a graph of prefill,
decode and FP8 decode gives the eager results bit for bit, also after the
inputs are overwritten in place."""

import pytest
import torch

import attention_online_softmax_fwd_b200 as ab
from attention_online_softmax_fwd_b200 import inputs as gen

pytestmark = pytest.mark.gpu


def test_graph_replay_matches_eager(cuda_device):
    dev = cuda_device
    q, k, v = [t.to(dev) for t in gen.prefill_inputs(1, 8, 2, 1000, 128, seed=3100)]
    cache = gen.paged_decode_inputs(8, 32, 8, 128, 16, 100, 2000, seed=3101)
    kc, ks = gen.quantize_pool_e4m3(cache.k_pages)
    vc, vs = gen.quantize_pool_e4m3(cache.v_pages)
    dq, kp, vp, bt, sl = [t.to(dev) for t in (cache.q, cache.k_pages, cache.v_pages, cache.block_table,
                                              cache.seq_lens)]
    kcd, vcd = kc.to(dev), vc.to(dev)
    split = 256
    ws = torch.empty(ab.decode_workspace_bytes(8, 32, 128, cache.max_pages, 16, split), dtype=torch.uint8,
                     device=dev)
    ws8 = torch.empty_like(ws)
    po, plse = torch.empty_like(q), torch.empty((1, 8, 1000), dtype=torch.float32, device=dev)
    do, dlse = torch.empty_like(dq), torch.empty((8, 32), dtype=torch.float32, device=dev)
    fo, flse = torch.empty_like(dq), torch.empty((8, 32), dtype=torch.float32, device=dev)

    def step():
        ab.prefill(q, k, v, causal=True, out=po, lse=plse)
        ab.decode_paged(dq, kp, vp, bt, sl, split_tokens=split, out=do, lse=dlse, workspace=ws)
        ab.decode_paged_fp8(dq, kcd, vcd, ks, vs, bt, sl, split_tokens=split, out=fo, lse=flse, workspace=ws8)

    def eager_copy():
        step()
        torch.cuda.synchronize()
        return [t.clone() for t in (po, plse, do, dlse, fo, flse)]

    ref1 = eager_copy()
    side = torch.cuda.Stream(device=dev)
    side.wait_stream(torch.cuda.current_stream(dev))
    with torch.cuda.stream(side):
        step()
    torch.cuda.current_stream(dev).wait_stream(side)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        step()
    for t in (po, plse, do, dlse, fo, flse):
        t.zero_()
    graph.replay()
    torch.cuda.synchronize()
    for got, want in zip((po, plse, do, dlse, fo, flse), ref1):
        assert torch.equal(got, want)

    # new inputs in the same buffers: the replay follows them
    g = torch.Generator().manual_seed(3102)
    q.copy_(torch.randn(q.shape, generator=g).to(torch.bfloat16))
    dq.copy_(torch.randn(dq.shape, generator=g).to(torch.bfloat16))
    ref2 = eager_copy()
    assert not torch.equal(ref2[0], ref1[0]) and not torch.equal(ref2[2], ref1[2])
    for t in (po, plse, do, dlse, fo, flse):
        t.zero_()
    graph.replay()
    torch.cuda.synchronize()
    for got, want in zip((po, plse, do, dlse, fo, flse), ref2):
        assert torch.equal(got, want)
