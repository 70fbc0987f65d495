"""Writing new tokens' K/V into the paged cache on the GPU, against the oracle
(a copy: bit-exact), and the decode that follows it."""

import numpy as np
import pytest
import torch

import attention_online_softmax_fwd_b200 as ab
from attention_online_softmax_fwd_b200 import inputs as gen
from oracle import attn_oracle as orc
from parity_util import compare_output

pytestmark = pytest.mark.gpu


def _with_room(c, T, page_size):
    """The cache of ``c`` with block tables extended by fresh pages for T more tokens."""
    lens = [int(x) for x in c.seq_lens]
    N = len(lens)
    need = [-(-(L + T) // page_size) for L in lens]
    have = [-(-L // page_size) for L in lens]
    extra = sum(n - h for n, h in zip(need, have))
    shape = (extra,) + tuple(c.k_pages.shape[1:])
    kp = torch.cat([c.k_pages, torch.full(shape, float("nan"), dtype=torch.bfloat16)])
    vp = torch.cat([c.v_pages, torch.full(shape, float("nan"), dtype=torch.bfloat16)])
    bt = torch.full((N, max(need)), -1, dtype=torch.int32)
    nxt = c.k_pages.shape[0]
    for b in range(N):
        bt[b, :have[b]] = c.block_table[b, :have[b]]
        for j in range(have[b], need[b]):
            bt[b, j] = nxt
            nxt += 1
    return kp, vp, bt, torch.tensor(lens, dtype=torch.int32)


def _same(a, b):
    a, b = np.asarray(a, dtype=np.float64), np.asarray(b, dtype=np.float64)
    return np.array_equal(np.isnan(a), np.isnan(b)) and np.array_equal(a[~np.isnan(a)], b[~np.isnan(b)])


@pytest.mark.parametrize("T,ps,D", [(1, 16, 128), (7, 16, 64), (300, 64, 128), (33, 256, 128)])
def test_kv_append_matches_oracle(cuda_device, T, ps, D):
    c = gen.paged_decode_inputs(5, 32, 8, D, ps, 1, 700, seed=4500 + T)
    kp, vp, bt, start = _with_room(c, T, ps)
    g = torch.Generator().manual_seed(4600 + T)
    kn = torch.randn(5, T, 8, D, generator=g).to(torch.bfloat16)
    vn = torch.randn(5, T, 8, D, generator=g).to(torch.bfloat16)
    kd, vd = kp.to(cuda_device), vp.to(cuda_device)
    st = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    ab.kv_append(kn.to(cuda_device), vn.to(cuda_device), kd, vd, bt.to(cuda_device), start.to(cuda_device),
                 device_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    k_ref, v_ref = orc.kv_append(kp, vp, bt, start, kn, vn, ps)
    assert _same(kd.float().cpu().numpy(), k_ref)
    assert _same(vd.float().cpu().numpy(), v_ref)


def test_append_then_decode(cuda_device):
    # one decode step of a serving loop: append the new token, then attend over the grown cache
    c = gen.paged_decode_inputs(16, 32, 8, 128, 16, 100, 3000, seed=4700)
    kp, vp, bt, start = _with_room(c, 1, 16)
    g = torch.Generator().manual_seed(4701)
    kn = torch.randn(16, 1, 8, 128, generator=g).to(torch.bfloat16)
    vn = torch.randn(16, 1, 8, 128, generator=g).to(torch.bfloat16)
    kd, vd, btd = kp.to(cuda_device), vp.to(cuda_device), bt.to(cuda_device)
    ab.kv_append(kn.to(cuda_device), vn.to(cuda_device), kd, vd, btd, start.to(cuda_device))
    lens = (start + 1).to(cuda_device)
    o, lse = ab.decode_paged(c.q.to(cuda_device), kd, vd, btd, lens, scale=gen.attn_scale(128), split_tokens=512)
    torch.cuda.synchronize()
    k_ref, v_ref = orc.kv_append(kp, vp, bt, start, kn, vn, 16)
    o_ref, lse_ref = orc.decode_paged(c.q, k_ref, v_ref, bt, start + 1, 16, gen.attn_scale(128))
    compare_output(o, o_ref, lse, lse_ref, label="append then decode")


def test_kv_append_bad_page_raises_device_status(cuda_device):
    c = gen.paged_decode_inputs(2, 8, 2, 64, 16, 20, 40, seed=4800)
    kp, vp, bt, start = _with_room(c, 3, 16)
    bt[1, -1] = 10_000
    kd, vd = kp.to(cuda_device), vp.to(cuda_device)
    st = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    kn = torch.zeros(2, 3, 2, 64, dtype=torch.bfloat16, device=cuda_device)
    start_far = start.clone()
    start_far[1] = int(bt.shape[1]) * 16 - 1        # the new tokens run past the table's last page
    ab.kv_append(kn, kn, kd, vd, bt.to(cuda_device), start_far.to(cuda_device), device_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 4                       # ATTN_ERR_DEVICE_BOUNDS
