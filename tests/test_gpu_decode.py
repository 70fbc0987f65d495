"""Paged decode on the GPU, through the C ABI, against the float64 oracle."""

import numpy as np
import pytest
import torch

import attention_online_softmax_fwd_b200 as ab
from attention_online_softmax_fwd_b200 import inputs as gen
from oracle import attn_oracle as orc
from parity_util import assert_rounding_limited, compare_blasst, compare_output, compare_skip

pytestmark = pytest.mark.gpu


def _to(cache, dev):
    return [t.to(dev) for t in (cache.q, cache.k_pages, cache.v_pages, cache.block_table, cache.seq_lens)]


def _run(cache, dev, split, lam=None):
    q, kp, vp, bt, sl = _to(cache, dev)
    scale = gen.attn_scale(q.shape[-1])
    if lam is None:
        o, lse = ab.decode_paged(q, kp, vp, bt, sl, scale=scale, split_tokens=split)
        mask = None
    else:
        o, lse, mask = ab.decode_paged_blasst(q, kp, vp, bt, sl, lam, scale=scale, split_tokens=split)
    torch.cuda.synchronize()
    return o, lse, mask, scale


@pytest.mark.parametrize("Hq,Hkv,D", [(8, 2, 128), (8, 8, 64), (16, 1, 128), (4, 2, 64), (32, 16, 128),
                                      (16, 2, 128), (24, 12, 128), (48, 12, 64), (128, 8, 128), (64, 4, 64)])
@pytest.mark.parametrize("page_size", [16, 64, 256])
def test_decode_small(cuda_device, Hq, Hkv, D, page_size):
    lens = [1, 63, 64, 65, 700, 2049, 0, 130]
    cache = gen.paged_decode_inputs(len(lens), Hq, Hkv, D, page_size, 0, 0, seed=2000 + Hq + D + page_size,
                                    lens=lens)
    for split in (64, 128, 1024):
        o, lse, _, scale = _run(cache, cuda_device, split)
        o_ref, lse_ref = orc.decode_paged(cache.q, cache.k_pages, cache.v_pages, cache.block_table,
                                          cache.seq_lens, page_size, scale)
        o_ref[6], lse_ref[6] = 0.0, -np.inf
        compare_output(o, o_ref, lse, lse_ref, label=f"decode split={split}")


@pytest.fixture(scope="module")
def full_size_decode():
    c = gen.CONFIGS["paged_gqa_decode"]
    cache = gen.paged_decode_inputs(c["N"], c["Hq"], c["Hkv"], c["D"], c["page_size"], c["len_lo"], c["len_hi"],
                                    seed=c["seed"])
    scale = gen.attn_scale(c["D"])
    o_ref, lse_ref = orc.decode_paged(cache.q, cache.k_pages, cache.v_pages, cache.block_table, cache.seq_lens,
                                      c["page_size"], scale)
    return cache, o_ref, lse_ref


@pytest.mark.parametrize("split", [256, 1024])
def test_decode_paged_gqa_full_size(cuda_device, full_size_decode, split):
    """64 sequences, lengths uniform in [512, 8192], Hq=32, Hkv=8, D=128, page 16; split 256 is the
    launch configuration the benchmark times (about 1,150 split items over a grid of 444 CTAs)."""
    cache, o_ref, lse_ref = full_size_decode
    o, lse, _, _ = _run(cache, cuda_device, split)
    stats = compare_output(o, o_ref, lse, lse_ref, label=f"paged_gqa_decode split={split}")
    print("paged_gqa_decode", split, stats)


def test_decode_deterministic(cuda_device):
    cache = gen.paged_decode_inputs(16, 32, 8, 128, 16, 100, 3000, seed=2100)
    o1, l1, _, _ = _run(cache, cuda_device, 256)
    o2, l2, _, _ = _run(cache, cuda_device, 256)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def _with_mask(cache, scale, rows_per_unit="group"):
    """The oracle's formula on a given decision mask (for decisions inside the tie band)."""
    return lambda mask: orc.decode_paged_with_skip_mask(cache.q, cache.k_pages, cache.v_pages, cache.block_table,
                                                        cache.seq_lens, cache.page_size, scale, mask,
                                                        rows_per_unit=rows_per_unit)


@pytest.mark.parametrize("split", [256, 2048])
@pytest.mark.parametrize("lam", [0.1, 0.3])
def test_decode_blasst_matches_oracle(cuda_device, split, lam):
    S, Hq, Hkv, D = 4096, 32, 8, 128
    # a peaked key opens every split, so later tiles of a split fall below its running max
    q, k, v = gen.peaked_prefill_inputs(1, Hq, Hkv, S, D, seed=2200, amp=8.0, period=split)
    cache = gen.paged_from_contiguous(q[:, S - 1], k, v, page_size=16, seed=2201)
    o, lse, mask, scale = _run(cache, cuda_device, split, lam)
    o_ref, lse_ref, m_ref, margin = orc.decode_paged_blasst(cache.q, cache.k_pages, cache.v_pages,
                                                            cache.block_table, cache.seq_lens, 16, scale, lam,
                                                            split)
    st = compare_blasst(o, lse, mask, o_ref, lse_ref, m_ref, margin, _with_mask(cache, scale),
                        label=f"decode blasst lam={lam}")
    assert st["skipped"] > 0


@pytest.mark.parametrize("Hq,Hkv", [(32, 8), (8, 2)])
def test_decode_dominant_key_normalisation(cuda_device, Hq, Hkv):
    # a dominant key at 0 and a stronger one at 200 (P = 2^7.3 under the lagging
    # reference): the output must stay within rounding of the exact value
    S, D = 3000, 128
    q, k, v = gen.peaked_prefill_inputs(1, Hq, Hkv, S, D, seed=2250, amp=12.0, period=1 << 30)
    k[:, 200] = (k[:, 0].float() * 1.4).to(torch.bfloat16)
    cache = gen.paged_from_contiguous(q[:, S - 1], k, v, page_size=16, seed=2251)
    for split in (256, 4096):
        o, lse, _, scale = _run(cache, cuda_device, split)
        o_ref, lse_ref = orc.decode_paged(cache.q, cache.k_pages, cache.v_pages, cache.block_table, cache.seq_lens,
                                          16, scale)
        # outputs are close to one row of V: the element bound below is the sharper check
        assert np.abs(lse.cpu().double().numpy() - np.asarray(lse_ref)).max() <= 1e-3
        assert_rounding_limited(o, o_ref, label=f"dominant key split={split}")
        compare_output(o, o_ref, lse, lse_ref, label=f"dominant key split={split}")
        o, lse, _, _ = _run(cache, cuda_device, split, 0.0)   # the per-KV-head kernel
        assert_rounding_limited(o, o_ref, label=f"dominant key lambda 0 split={split}")


def test_decode_lambda_zero_mask_is_dense(cuda_device):
    # lambda = 0 with a decision mask runs the per-KV-head kernel; the dense call
    # runs the head-group kernel: same result up to summation order, nothing skipped
    cache = gen.paged_decode_inputs(8, 32, 8, 128, 16, 64, 2000, seed=2300)
    o0, l0, _, scale = _run(cache, cuda_device, 512)
    o1, l1, mask, _ = _run(cache, cuda_device, 512, 0.0)
    o_ref, l_ref, m_ref, margin = orc.decode_paged_blasst(cache.q, cache.k_pages, cache.v_pages, cache.block_table,
                                                          cache.seq_lens, 16, scale, 0.0, 512)
    compare_output(o0, o_ref, l0, l_ref, label="dense")
    compare_output(o1, o_ref, l1, l_ref, label="lambda 0")
    compare_skip(mask, m_ref, margin)
    assert not (mask == 1).any()


def test_decode_bad_page_raises_device_status(cuda_device):
    cache = gen.paged_decode_inputs(4, 8, 2, 128, 16, 100, 300, seed=2400)
    cache.block_table[1, 2] = cache.num_pages + 5      # out of range: never dereferenced
    cache.block_table[2, 0] = -7
    q, kp, vp, bt, sl = _to(cache, cuda_device)
    status = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    ab.binding.set_library_status(True)
    ab.binding.read_device_status(clear=True)
    o, lse = ab.decode_paged(q, kp, vp, bt, sl, split_tokens=64, device_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 4                        # ATTN_ERR_DEVICE_BOUNDS
    assert ab.binding.read_device_status(clear=True) == 4
    ab.binding.set_library_status(False)
    # sequences with valid tables are unaffected
    o_ref, lse_ref = orc.decode_paged(cache.q, cache.k_pages, cache.v_pages, cache.block_table, cache.seq_lens,
                                      16, gen.attn_scale(128), seqs=[0, 3])
    compare_output(o[[0, 3]], o_ref[[0, 3]], lse[[0, 3]], lse_ref[[0, 3]])


@pytest.mark.parametrize("split", [256, 2048])
@pytest.mark.parametrize("lam", [0.1, 0.3])
def test_decode_blasst_per_head_matches_oracle(cuda_device, split, lam):
    S, Hq, Hkv, D = 4096, 32, 8, 128
    q, k, v = gen.peaked_prefill_inputs(1, Hq, Hkv, S, D, seed=2400, amp=8.0, period=split)
    cache = gen.paged_from_contiguous(q[:, S - 1], k, v, page_size=16, seed=2401)
    args = [t.to(cuda_device) for t in (cache.q, cache.k_pages, cache.v_pages, cache.block_table, cache.seq_lens)]
    scale = gen.attn_scale(D)
    o, lse, mask = ab.decode_paged_blasst(*args, lam, scale=scale, split_tokens=split, rows_per_unit="head")
    torch.cuda.synchronize()
    assert mask.shape[1] == Hq
    o_ref, lse_ref, m_ref, margin = orc.decode_paged_blasst(cache.q, cache.k_pages, cache.v_pages,
                                                            cache.block_table, cache.seq_lens, 16, scale, lam,
                                                            split, rows_per_unit="head")
    st = compare_blasst(o, lse, mask, o_ref, lse_ref, m_ref, margin, _with_mask(cache, scale, "head"),
                        label=f"per-head blasst lam={lam}")
    assert st["skipped"] > 0
    # a head-level unit drops at least what its group drops
    _, _, mg, _ = orc.decode_paged_blasst(cache.q, cache.k_pages, cache.v_pages, cache.block_table,
                                          cache.seq_lens, 16, scale, lam, split)
    assert (m_ref == 1).sum() >= (mg == 1).sum() * (Hq // Hkv)


def test_decode_blasst_per_head_lambda_zero_is_dense(cuda_device):
    cache = gen.paged_decode_inputs(6, 32, 8, 128, 16, 64, 1500, seed=2450)
    o0, l0, _, scale = _run(cache, cuda_device, 512)
    args = [t.to(cuda_device) for t in (cache.q, cache.k_pages, cache.v_pages, cache.block_table, cache.seq_lens)]
    o1, l1, mask = ab.decode_paged_blasst(*args, 0.0, scale=scale, split_tokens=512, rows_per_unit="head")
    torch.cuda.synchronize()
    assert not (mask == 1).any()
    o_ref, l_ref = orc.decode_paged(cache.q, cache.k_pages, cache.v_pages, cache.block_table, cache.seq_lens, 16,
                                    scale)
    compare_output(o1, o_ref, l1, l_ref, label="per-head lambda 0")
