"""Paged decode over an FP8 E4M3 cache on the GPU, through the C ABI, against
the float64 oracle on the same codes (one scale per pool)."""

import numpy as np
import pytest
import torch

import attention_online_softmax_fwd_b200 as ab
from attention_online_softmax_fwd_b200 import inputs as gen
from oracle import attn_oracle as orc
from parity_util import compare_output

pytestmark = pytest.mark.gpu


def _quantized(cache):
    kc, ks = gen.quantize_pool_e4m3(cache.k_pages)
    vc, vs = gen.quantize_pool_e4m3(cache.v_pages)
    return kc, ks, vc, vs


def _run(cache, kc, ks, vc, vs, dev, split, status=None):
    scale = gen.attn_scale(cache.q.shape[-1])
    o, lse = ab.decode_paged_fp8(cache.q.to(dev), kc.to(dev), vc.to(dev), ks, vs, cache.block_table.to(dev),
                                 cache.seq_lens.to(dev), scale=scale, split_tokens=split, device_status=status)
    torch.cuda.synchronize()
    return o, lse, scale


@pytest.mark.parametrize("Hq,Hkv", [(8, 4), (32, 8), (16, 16), (64, 8), (128, 8), (4, 4), (24, 12), (64, 4)])
@pytest.mark.parametrize("page_size", [16, 64, 256])
def test_decode_fp8_small(cuda_device, Hq, Hkv, page_size):
    lens = [1, 15, 16, 17, 63, 700, 2049, 0, 130]
    cache = gen.paged_decode_inputs(len(lens), Hq, Hkv, 128, page_size, 0, 0, seed=2600 + Hq + Hkv + page_size,
                                    lens=lens)
    kc, ks, vc, vs = _quantized(cache)
    for split in (64, 1024):
        o, lse, scale = _run(cache, kc, ks, vc, vs, cuda_device, split)
        o_ref, lse_ref = orc.decode_paged_fp8(cache.q, kc, vc, ks, vs, cache.block_table, cache.seq_lens,
                                              page_size, scale)
        o_ref[7], lse_ref[7] = 0.0, -np.inf
        compare_output(o, o_ref, lse, lse_ref, label=f"fp8 decode Hq={Hq} Hkv={Hkv} split={split}")


def test_decode_fp8_poisoned_slots_are_nan_codes():
    """The fixture above only means something if the unused slots of a page
    hold NaN codes that the kernel must never multiply into O."""
    cache = gen.paged_decode_inputs(3, 8, 4, 128, 64, 0, 0, seed=2650, lens=[17, 100, 5])
    kc, _, vc, _ = _quantized(cache)
    assert ((kc & 0x7F) == 0x7F).any() and ((vc & 0x7F) == 0x7F).any()


def test_decode_fp8_full_size(cuda_device):
    """64 sequences, lengths uniform in [512, 8192], Hq=32, Hkv=8, D=128, page 16, split 256, FP8 codes."""
    c = gen.CONFIGS["paged_gqa_decode"]
    cache = gen.paged_decode_inputs(c["N"], c["Hq"], c["Hkv"], c["D"], c["page_size"], c["len_lo"], c["len_hi"],
                                    seed=c["seed"])
    kc, ks, vc, vs = _quantized(cache)
    o, lse, scale = _run(cache, kc, ks, vc, vs, cuda_device, 256)
    o_ref, lse_ref = orc.decode_paged_fp8(cache.q, kc, vc, ks, vs, cache.block_table, cache.seq_lens,
                                          c["page_size"], scale)
    print("fp8 paged_gqa_decode", compare_output(o, o_ref, lse, lse_ref, label="fp8 paged_gqa_decode"))


@pytest.mark.parametrize("Hq,Hkv", [(32, 8), (16, 4)])
def test_decode_fp8_dominant_key(cuda_device, Hq, Hkv):
    """One key far above the rest (P of the others ~e^-40): the normaliser and the
    f16 rounding of P must not let the dominant key's weight drift."""
    S = 3000
    q, k, v = gen.peaked_prefill_inputs(1, Hq, Hkv, S, 128, seed=2700 + Hq, amp=12.0, period=S)
    cache = gen.paged_from_contiguous(q[:, S - 1], k, v, page_size=16, seed=2701)
    kc, ks, vc, vs = _quantized(cache)
    for split in (256, 4096):
        o, lse, scale = _run(cache, kc, ks, vc, vs, cuda_device, split)
        o_ref, lse_ref = orc.decode_paged_fp8(cache.q, kc, vc, ks, vs, cache.block_table, cache.seq_lens, 16,
                                              scale)
        compare_output(o, o_ref, lse, lse_ref, label=f"fp8 dominant split={split}")


def test_decode_fp8_scales_enter_linearly(cuda_device):
    """Halving k_scale halves every score (so it equals the call with half the
    softmax scale); doubling v_scale doubles O and leaves the LSE alone."""
    cache = gen.paged_decode_inputs(6, 32, 8, 128, 16, 50, 900, seed=2750)
    kc, ks, vc, vs = _quantized(cache)
    dev = cuda_device
    args = [t.to(dev) for t in (cache.q, kc, vc)]
    bt, sl = cache.block_table.to(dev), cache.seq_lens.to(dev)
    s = gen.attn_scale(128)
    o1, l1 = ab.decode_paged_fp8(args[0], args[1], args[2], ks * 0.5, vs, bt, sl, scale=s, split_tokens=256)
    o2, l2 = ab.decode_paged_fp8(args[0], args[1], args[2], ks, vs * 2.0, bt, sl, scale=s * 0.5, split_tokens=256)
    torch.cuda.synchronize()
    o_ref, l_ref = orc.decode_paged_fp8(cache.q, kc, vc, ks * 0.5, vs, cache.block_table, cache.seq_lens, 16, s)
    compare_output(o1, o_ref, l1, l_ref, label="k_scale / 2")
    compare_output(o2, 2.0 * o_ref, l2, l_ref, label="v_scale * 2, scale / 2")


def test_decode_fp8_deterministic(cuda_device):
    cache = gen.paged_decode_inputs(16, 32, 8, 128, 16, 100, 3000, seed=2800)
    kc, ks, vc, vs = _quantized(cache)
    o1, l1, _ = _run(cache, kc, ks, vc, vs, cuda_device, 256)
    o2, l2, _ = _run(cache, kc, ks, vc, vs, cuda_device, 256)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_decode_fp8_bad_page_raises_device_status(cuda_device):
    cache = gen.paged_decode_inputs(4, 16, 4, 128, 16, 100, 300, seed=2850)
    cache.block_table[1, 2] = cache.num_pages + 5      # out of range: never dereferenced
    cache.block_table[2, 0] = -7
    kc, ks, vc, vs = _quantized(cache)
    status = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    ab.binding.set_library_status(True)
    ab.binding.read_device_status(clear=True)
    o, lse, scale = _run(cache, kc, ks, vc, vs, cuda_device, 64, status=status)
    assert int(status.item()) == 4                        # ATTN_ERR_DEVICE_BOUNDS
    assert ab.binding.read_device_status(clear=True) == 4
    ab.binding.set_library_status(False)
    o_ref, lse_ref = orc.decode_paged_fp8(cache.q, kc, vc, ks, vs, cache.block_table, cache.seq_lens, 16, scale,
                                          seqs=[0, 3])
    compare_output(o[[0, 3]], o_ref[[0, 3]], lse[[0, 3]], lse_ref[[0, 3]])


def test_decode_fp8_rejects_unsupported_shapes(cuda_device):
    cache = gen.paged_decode_inputs(2, 8, 2, 128, 16, 10, 40, seed=2900)
    kc, ks, vc, vs = _quantized(cache)
    with pytest.raises(ab.AttnError):
        _run(cache, kc, ks, vc, vs, cuda_device, 64)     # Hkv = 2
