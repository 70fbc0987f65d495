"""CPU checks of the parity helpers themselves.

The GPU side is stood in for by the oracle: a result the GPU could return is
the oracle's output rounded to bf16, and a decision the GPU could take
differently is planted in the oracle's mask, on the CPU.
"""

import numpy as np
import pytest
import torch

from attention_online_softmax_fwd_b200 import inputs as gen
from oracle import attn_oracle as orc
from parity_util import bf16_round, bf16_ulp, compare_blasst, compare_output


def test_bf16_round_matches_torch():
    rng = np.random.default_rng(5)
    x = np.concatenate([rng.standard_normal(20000) * 10.0 ** rng.integers(-6, 6, 20000),
                        [0.0, 1.0, -1.0, 1.00390625, 1.005859375, 255.5, 3e38 / 4]])
    x32 = x.astype(np.float32).astype(np.float64)          # exactly representable in fp32: no double rounding
    want = torch.from_numpy(x32).float().to(torch.bfloat16).double().numpy()
    np.testing.assert_array_equal(bf16_round(x32), want)
    assert (np.abs(bf16_round(x32) - x32) <= 0.5 * bf16_ulp(x32)).all()


def test_mean_is_taken_against_the_rounded_reference():
    rng = np.random.default_rng(6)
    ref = rng.standard_normal(10000) * 3.0
    gpu = torch.from_numpy(ref).float().to(torch.bfloat16)   # the best a bf16 kernel can return
    st = compare_output(gpu, ref)
    assert st["mean_abs"] == 0.0 and st["mean_abs_vs_f64"] > 5e-4
    bad = gpu.double() + 3e-3                                # a real bias of the kernel
    with pytest.raises(AssertionError):
        compare_output(bad, ref)


def _blasst_case():
    q, k, v = gen.peaked_prefill_inputs(1, 2, 1, 400, 16, seed=91, amp=8.0, period=1 << 20)
    o, lse, skip, margin = orc.prefill_blasst(q, k, v, True, 0.25, 0.3)
    return q, k, v, o, lse, skip, margin


def test_a_flipped_tie_is_checked_on_the_gpu_decisions():
    q, k, v, o, lse, skip, margin = _blasst_case()
    kept = np.argwhere(skip == 0)
    kept = kept[kept[:, 3] > 0]                    # not the first tile of a unit
    b, h, qt, t = kept[-1]
    margin = margin.copy()
    margin[b, h, qt, t] = 0.0                      # planted: this decision sits on the threshold
    flipped = skip.copy()
    flipped[b, h, qt, t] = 1                       # and the "GPU" took it the other way
    o_gpu, lse_gpu = orc.prefill_with_skip_mask(q, k, v, True, 0.25, flipped)
    o_gpu = torch.from_numpy(o_gpu).float().to(torch.bfloat16)

    def with_mask(m):
        return orc.prefill_with_skip_mask(q, k, v, True, 0.25, m)

    st = compare_blasst(o_gpu, lse_gpu, torch.from_numpy(flipped), o, lse, skip, margin, with_mask)
    assert st["tie_mismatches"] == 1 and st["reference"].startswith("oracle formula")
    # the walk's own output differs on the rows of the flipped tile: compared with it, the planted
    # decision would have to be absorbed by the tolerance
    rows = slice(qt * 128, qt * 128 + 128)
    assert np.abs(o[b, rows, h] - with_mask(flipped)[0][b, rows, h]).max() > 0


def test_a_flipped_decision_outside_the_tie_band_fails():
    q, k, v, o, lse, skip, margin = _blasst_case()
    kept = np.argwhere((skip == 0) & (margin > 1e-3))
    kept = kept[kept[:, 3] > 0]
    flipped = skip.copy()
    flipped[tuple(kept[-1])] = 1
    o_gpu, lse_gpu = orc.prefill_with_skip_mask(q, k, v, True, 0.25, flipped)
    with pytest.raises(AssertionError):
        compare_blasst(torch.from_numpy(o_gpu), lse_gpu, torch.from_numpy(flipped), o, lse, skip, margin,
                       lambda m: orc.prefill_with_skip_mask(q, k, v, True, 0.25, m))
