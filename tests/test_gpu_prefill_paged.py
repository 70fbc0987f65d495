"""Chunked prefill over a paged KV cache on the GPU, through the C ABI, against
the float64 oracle (the chunk's queries at the end of each sequence, causal)."""

import numpy as np
import pytest
import torch

import attention_online_softmax_fwd_b200 as ab
from attention_online_softmax_fwd_b200 import inputs as gen
from oracle import attn_oracle as orc
from parity_util import compare_output

pytestmark = pytest.mark.gpu


def _run(c, dev, status=None):
    args = [t.to(dev) for t in (c.q, c.k_pages, c.v_pages, c.block_table, c.seq_lens)]
    scale = gen.attn_scale(c.q.shape[-1])
    o, lse = ab.prefill_paged(*args, scale=scale, device_status=status)
    torch.cuda.synchronize()
    return o, lse, scale


@pytest.mark.parametrize("B,Sq,Hq,Hkv,D,ps,lens", [
    (3, 100, 8, 2, 128, 16, [100, 357, 1000]),       # first chunk, mid, long prefix; ragged tails
    (2, 300, 4, 4, 64, 64, [300, 777]),               # D 64, 64-token pages, two query blocks
    (2, 129, 8, 1, 128, 256, [129, 1111]),            # MQA, pages longer than a K/V tile
    (1, 1, 8, 2, 128, 32, [613]),                     # a single query
    (2, 513, 16, 4, 128, 16, [513, 2049]),            # several 256-row blocks, ragged ends
    (4, 17, 8, 8, 64, 128, [17, 18, 145, 400]),       # MHA, short chunks
])
def test_prefill_paged_matches_oracle(cuda_device, B, Sq, Hq, Hkv, D, ps, lens):
    c = gen.paged_prefill_inputs(B, Sq, Hq, Hkv, D, ps, lens, seed=4000 + Sq + ps)
    st = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    o, lse, scale = _run(c, cuda_device, st)
    assert int(st.item()) == 0
    o_ref, lse_ref = orc.prefill_paged(c.q, c.k_pages, c.v_pages, c.block_table, c.seq_lens, ps, scale)
    compare_output(o, o_ref, lse, lse_ref, label=f"paged prefill Sq={Sq} ps={ps}")


def test_prefill_paged_whole_sequence_equals_prefill(cuda_device):
    # Sq = L: the chunk is the whole sequence, which the contiguous prefill kernel also computes
    L = 1000
    c = gen.paged_prefill_inputs(1, L, 8, 2, 128, 16, [L], seed=4100)
    o, lse, scale = _run(c, cuda_device)
    od, ld = ab.prefill(c.q.to(cuda_device), c.k_seqs[0][None].to(cuda_device), c.v_seqs[0][None].to(cuda_device),
                        causal=True, scale=scale)
    torch.cuda.synchronize()
    compare_output(o, od.float().cpu().double().numpy(), lse, ld.cpu().double().numpy(),
                   label="paged whole sequence vs contiguous prefill")


def test_prefill_paged_full_size_sampled(cuda_device):
    # a serving-sized chunk: 4 sequences, 2048 new tokens each after prefixes of 0..6144
    B, Sq, Hq, Hkv, D, ps = 4, 2048, 32, 8, 128, 16
    lens = [2048, 4096, 6144, 8192]
    c = gen.paged_prefill_inputs(B, Sq, Hq, Hkv, D, ps, lens, seed=4200)
    o, lse, scale = _run(c, cuda_device)
    heads = [0, 13, 31]
    o_ref, lse_ref = orc.prefill_paged(c.q, c.k_pages, c.v_pages, c.block_table, c.seq_lens, ps, scale,
                                       heads=heads)
    og, lg = o.cpu(), lse.cpu()
    for h in heads:
        compare_output(og[:, :, h], o_ref[:, :, h], lg[:, h], lse_ref[:, h], label=f"head {h}")


def test_prefill_paged_bad_page_raises_device_status(cuda_device):
    c = gen.paged_prefill_inputs(2, 40, 8, 2, 128, 16, [40, 90], seed=4300)
    c.block_table[1, 2] = 10_000                      # a page the pool does not hold
    st = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    o, lse, _ = _run(c, cuda_device, st)
    assert int(st.item()) == 4                        # ATTN_ERR_DEVICE_BOUNDS
    assert torch.isfinite(o.float()).all()
