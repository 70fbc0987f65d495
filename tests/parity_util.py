"""Comparison helpers for the GPU-vs-oracle parity tests.

Tolerances (bf16 inputs and outputs, fp32 accumulation):
  output O : max |O - O_ref| <= 1e-2 and mean |O - O_ref| <= 1e-3,
  LSE      : max |LSE - LSE_ref| <= 1e-3 (natural log).
An output element above 1e-2 is accepted only as a rounding-limited case: it
must lie within one bf16 ulp of the float64 reference (for |O| >= 4 the bf16
half-ulp alone exceeds 1e-2). Such elements are counted and reported.
Skip decisions must match exactly, except decisions whose distance from the
threshold (|exp(r - m) - lambda| over the unit's rows) is within 1e-6.
"""

from __future__ import annotations

import numpy as np
import torch

O_MAX_ABS = 1e-2
O_MEAN_ABS = 1e-3
LSE_MAX_ABS = 1e-3
TIE_WIDTH = 1e-6


def bf16_ulp(x):
    """Spacing of bf16 numbers at |x| (8 significant bits)."""
    a = np.abs(np.asarray(x, dtype=np.float64))
    a = np.where(a < 2.0 ** -126, 2.0 ** -126, a)
    e = np.floor(np.log2(a))
    return 2.0 ** (e - 7)


def compare_output(o_gpu, o_ref, lse_gpu=None, lse_ref=None, mask=None, label=""):
    """Element-wise comparison; ``mask`` (bool, o's shape) selects the elements checked."""
    og = o_gpu.detach().float().cpu().double().numpy() if isinstance(o_gpu, torch.Tensor) else np.asarray(o_gpu)
    orf = np.asarray(o_ref, dtype=np.float64)
    if mask is not None:
        og, orf = og[mask], orf[mask]
    assert np.isfinite(og).all(), f"{label}: non-finite GPU output"
    assert np.isfinite(orf).all(), f"{label}: reference not computed for every checked element"
    err = np.abs(og - orf)
    over = err > O_MAX_ABS
    rounding_limited = over & (err <= bf16_ulp(orf))
    hard = over & ~rounding_limited
    stats = {"max_abs": float(err.max(initial=0.0)), "mean_abs": float(err.mean()) if err.size else 0.0,
             "n": int(err.size), "rounding_limited": int(rounding_limited.sum())}
    assert not hard.any(), f"{label}: {int(hard.sum())} elements beyond 1e-2 and 1 bf16 ulp (max {stats['max_abs']:.3g})"
    assert stats["mean_abs"] <= O_MEAN_ABS, f"{label}: mean abs error {stats['mean_abs']:.3g}"
    if lse_gpu is not None:
        lg = lse_gpu.detach().cpu().double().numpy() if isinstance(lse_gpu, torch.Tensor) else np.asarray(lse_gpu)
        lr = np.asarray(lse_ref, dtype=np.float64)
        sel = np.isfinite(lr)
        lerr = np.abs(lg[sel] - lr[sel])
        stats["lse_max_abs"] = float(lerr.max(initial=0.0))
        assert stats["lse_max_abs"] <= LSE_MAX_ABS, f"{label}: LSE error {stats['lse_max_abs']:.3g}"
        assert np.array_equal(np.isneginf(lg[~sel]), np.isneginf(lr[~sel])), f"{label}: -inf LSE mismatch"
    return stats


def compare_skip(mask_gpu, mask_ref, margin_ref, label=""):
    """Skip decisions: exact outside the tie band; visited/unvisited sets identical."""
    mg = mask_gpu.cpu().numpy() if isinstance(mask_gpu, torch.Tensor) else np.asarray(mask_gpu)
    mr = np.asarray(mask_ref)
    assert mg.shape == mr.shape, f"{label}: mask shape {mg.shape} vs {mr.shape}"
    visited_ref = mr != 2
    assert np.array_equal(mg != 2, visited_ref), f"{label}: visited tiles differ"
    diff = (mg != mr) & visited_ref
    ties = np.asarray(margin_ref) <= TIE_WIDTH
    hard = diff & ~ties
    assert not hard.any(), f"{label}: {int(hard.sum())} skip decisions differ outside the tie band"
    return {"decisions": int(visited_ref.sum()), "skipped": int((mr == 1).sum()),
            "tie_mismatches": int((diff & ties).sum())}


def assert_rounding_limited(o_gpu, o_ref, ulps=0.6, floor=1e-3, label=""):
    """Every element within ``ulps`` bf16 spacings of the exact value (plus ``floor``).

    Rounding the exact result to bf16 costs at most half a spacing; ``floor``
    covers the bf16 rounding of P where two keys share a row's mass (a weight
    of 0.05 next to 0.93 moves by ~1e-4 of |v|). An error in the normalisation
    of a row (such as the bf16 rounding of one dominant probability left out of
    l) scales the whole row by up to 2^-8 and exceeds this on outputs of order
    one, where the absolute 1e-2 bound with its one-spacing allowance does not
    see it.
    """
    og = o_gpu.detach().float().cpu().double().numpy() if isinstance(o_gpu, torch.Tensor) else np.asarray(o_gpu)
    orf = np.asarray(o_ref, dtype=np.float64)
    err = np.abs(og - orf)
    bound = ulps * bf16_ulp(orf) + floor
    bad = err > bound
    assert not bad.any(), (f"{label}: {int(bad.sum())} elements beyond {ulps} bf16 spacing "
                           f"(worst {float((err / bf16_ulp(orf)).max()):.2f} spacings)")
