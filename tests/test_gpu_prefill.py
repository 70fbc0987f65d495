"""Prefill on the GPU, through the C ABI, against the float64 oracle."""

import numpy as np
import pytest
import torch

import attention_online_softmax_fwd_b200 as ab
from attention_online_softmax_fwd_b200 import inputs as gen
from oracle import attn_oracle as orc
from parity_util import assert_rounding_limited, compare_blasst, compare_output, compare_skip

pytestmark = pytest.mark.gpu


def _run(q, k, v, causal, dev, lam=None):
    qd, kd, vd = q.to(dev), k.to(dev), v.to(dev)
    scale = gen.attn_scale(q.shape[-1])
    if lam is None:
        o, lse = ab.prefill(qd, kd, vd, causal=causal, scale=scale)
        mask = None
    else:
        o, lse, mask = ab.prefill_blasst(qd, kd, vd, lam, causal=causal, scale=scale)
    torch.cuda.synchronize()
    return o, lse, mask, scale


def test_tiny_gqa_prefill(cuda_device):
    c = gen.CONFIGS["tiny_gqa_prefill"]
    q, k, v = gen.prefill_inputs(c["B"], c["Hq"], c["Hkv"], c["S"], c["D"], c["seed"])
    o, lse, _, scale = _run(q, k, v, True, cuda_device)
    o_ref, lse_ref = orc.prefill(q, k, v, True, scale)
    print("tiny", compare_output(o, o_ref, lse, lse_ref, label="tiny"))


@pytest.mark.parametrize("B,Hq,Hkv,S,D", [(2, 8, 2, 700, 128), (1, 4, 4, 300, 64), (1, 8, 1, 513, 128),
                                          (1, 2, 1, 1, 128), (1, 2, 2, 129, 64), (2, 4, 2, 255, 128),
                                          (1, 4, 2, 257, 128), (1, 2, 1, 1024, 64)])
@pytest.mark.parametrize("causal", [True, False])
def test_prefill_small(cuda_device, B, Hq, Hkv, S, D, causal):
    q, k, v = gen.prefill_inputs(B, Hq, Hkv, S, D, seed=3000 + S + D)
    o, lse, _, scale = _run(q, k, v, causal, cuda_device)
    o_ref, lse_ref = orc.prefill(q, k, v, causal, scale)
    compare_output(o, o_ref, lse, lse_ref, label=f"S={S} D={D} causal={causal}")


def _sample_rows(S, rng):
    rows = set(range(0, 64)) | set(range(S - 64, S))
    for t in (127, 128, 255, 256, 511, 512, 1023, 1024):
        if t < S:
            rows |= {t - 1, t, min(t + 1, S - 1)}
    rows |= set(rng.integers(0, S, 64).tolist())
    return sorted(rows)


@pytest.mark.parametrize("name", ["mha_prefill_llama2_7b", "gqa_prefill_llama3_8b"])
def test_prefill_full_size_sampled(cuda_device, name):
    c = gen.CONFIGS[name]
    q, k, v = gen.prefill_inputs(c["B"], c["Hq"], c["Hkv"], c["S"], c["D"], c["seed"])
    o, lse, _, scale = _run(q, k, v, True, cuda_device)
    rng = np.random.default_rng(7)
    heads = [(0, 0), (0, c["Hq"] - 1), (c["B"] - 1, 5), (c["B"] - 1, c["Hq"] // 2), (0, 9), (c["B"] - 1, 30)]
    rows = _sample_rows(c["S"], rng)
    o_ref, lse_ref = orc.prefill(q, k, v, True, scale, heads=heads, rows=rows)
    og, lg = o.cpu(), lse.cpu()
    for b, h in heads:
        stats = compare_output(og[b, rows, h], o_ref[b, rows, h], lg[b, h, rows], lse_ref[b, h, rows],
                               label=f"{name} b={b} h={h}")
    print(name, stats)
    assert torch.isfinite(o.float()).all()


def test_prefill_deterministic(cuda_device):
    q, k, v = gen.prefill_inputs(2, 8, 2, 1000, 128, seed=3100)
    o1, l1, _, _ = _run(q, k, v, True, cuda_device)
    o2, l2, _, _ = _run(q, k, v, True, cuda_device)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def _with_mask(q, k, v, causal, scale):
    """The oracle's formula on a given decision mask (for decisions inside the tie band)."""
    return lambda mask: orc.prefill_with_skip_mask(q, k, v, causal, scale, mask)


@pytest.mark.parametrize("causal", [True, False])
def test_prefill_blasst_matches_oracle(cuda_device, causal):
    # single peaked key: later tiles fall below the running max for all 128 rows
    q, k, v = gen.peaked_prefill_inputs(1, 4, 2, 1100, 128, seed=3200, amp=8.0, period=1 << 30)
    for lam in (0.05, 0.3, 0.7):
        o, lse, mask, scale = _run(q, k, v, causal, cuda_device, lam)
        o_ref, lse_ref, m_ref, margin = orc.prefill_blasst(q, k, v, causal, scale, lam)
        st = compare_blasst(o, lse, mask, o_ref, lse_ref, m_ref, margin, _with_mask(q, k, v, causal, scale),
                            label=f"prefill blasst lam={lam}")
    assert st["skipped"] > 0


def _later_peak_inputs():
    # one dominant key at 0 and a stronger one at 200: under the lagging reference
    # maximum the second has P = 2^7.3, which bf16 rounds by up to 2^-8 relative
    q, k, v = gen.peaked_prefill_inputs(1, 4, 2, 777, 128, seed=3250, amp=12.0, period=1 << 30)
    k[:, 200] = (k[:, 0].float() * 1.4).to(torch.bfloat16)
    return q, k, v


@pytest.mark.parametrize("causal", [True, False])
def test_prefill_dominant_key_normalisation(cuda_device, causal):
    q, k, v = _later_peak_inputs()
    o, lse, _, scale = _run(q, k, v, causal, cuda_device)
    o_ref, lse_ref = orc.prefill(q, k, v, causal, scale)
    assert_rounding_limited(o, o_ref, label=f"dominant key causal={causal}")
    o, lse, _, scale = _run(q, k, v, causal, cuda_device, 0.01)
    o_ref, lse_ref, _, _ = orc.prefill_blasst(q, k, v, causal, scale, 0.01)
    assert_rounding_limited(o, o_ref, label=f"dominant key blasst causal={causal}")


@pytest.mark.parametrize("causal", [True, False])
def test_prefill_blasst_later_peak(cuda_device, causal):
    # a stronger key at 200 (second half of K/V tile 1) after the peak at key 0:
    # tile 1 keeps its second 64-key half and drops its first, and the running
    # maximum rises past the first peak
    q, k, v = _later_peak_inputs()
    kept_second_half_only = 0
    for lam in (0.01, 0.2):
        o, lse, mask, scale = _run(q, k, v, causal, cuda_device, lam)
        o_ref, lse_ref, m_ref, margin = orc.prefill_blasst(q, k, v, causal, scale, lam)
        compare_blasst(o, lse, mask, o_ref, lse_ref, m_ref, margin, _with_mask(q, k, v, causal, scale),
                       label=f"prefill blasst later peak lam={lam}")
        m = mask.cpu().numpy()
        kept_second_half_only += int(((m[..., 2] == 1) & (m[..., 3] == 0)).sum())
    assert kept_second_half_only > 0


def test_prefill_lambda_zero_is_dense(cuda_device):
    q, k, v = gen.peaked_prefill_inputs(1, 4, 2, 700, 128, seed=3300, amp=4.0)
    o0, l0, _, scale = _run(q, k, v, True, cuda_device)
    o1, l1, mask, _ = _run(q, k, v, True, cuda_device, 0.0)
    assert torch.equal(o0, o1) and torch.equal(l0, l1)
    _, _, m_ref, margin = orc.prefill_blasst(q, k, v, True, scale, 0.0)
    compare_skip(mask, m_ref, margin)


def test_decode_equals_prefill_last_row(cuda_device):
    S, Hq, Hkv, D = 3000, 32, 8, 128
    q, k, v = gen.peaked_prefill_inputs(1, Hq, Hkv, S, D, seed=3400, amp=4.0)
    o, lse, _, scale = _run(q, k, v, True, cuda_device)
    cache = gen.paged_from_contiguous(q[:, S - 1], k, v, page_size=16, seed=3401)
    dev = cuda_device
    od, ld = ab.decode_paged(cache.q.to(dev), cache.k_pages.to(dev), cache.v_pages.to(dev),
                             cache.block_table.to(dev), cache.seq_lens.to(dev), scale=scale, split_tokens=512)
    torch.cuda.synchronize()
    compare_output(od[0], o[0, S - 1].float().cpu().double().numpy(), ld[0], lse[0, :, S - 1].cpu().numpy())
