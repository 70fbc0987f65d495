"""Comparison helpers for the GPU-vs-oracle parity tests.

Tolerances (bf16 inputs and outputs, fp32 accumulation):
  output O : max |O - O_ref| <= 1e-2 and mean |O - O_ref| <= 1e-3,
  LSE      : max |LSE - LSE_ref| <= 1e-3 (natural log).

Reading of the output tolerance. The kernels return O in bf16, so the best any
kernel can return is bf16(O_ref), the float64 reference rounded to the nearest
bf16 value. Both bounds are therefore taken against bf16(O_ref):
  * the mean |O - bf16(O_ref)| must stay <= 1e-3 (on outputs of order one the
    rounding to bf16 alone costs about 5e-4 on average, half the budget, and is
    not an error of the kernel);
  * an element with |O - bf16(O_ref)| > 1e-2 passes only when it lies within
    one bf16 spacing of bf16(O_ref) (for |O| >= 4 half a spacing alone exceeds
    1e-2); such elements are counted and reported.
The mean and maximum against the unrounded reference are reported beside them.

Skip decisions must match exactly, except decisions whose distance from the
threshold (|exp(r - m) - lambda| over the unit's rows) is within 1e-6. Where
such a tie went the other way on the GPU, the outputs are compared with the
oracle's formula evaluated on the GPU's own decisions.
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


def bf16_round(x):
    """float64 -> nearest bf16 value (ties to even), returned as float64."""
    x = np.asarray(x, dtype=np.float64)
    u = bf16_ulp(x)
    return np.rint(x / u) * u          # rint rounds halves to even; x / u is exact (power-of-two u)


def _np(t):
    if isinstance(t, torch.Tensor):
        return t.detach().float().cpu().double().numpy()
    return np.asarray(t, dtype=np.float64)


def compare_output(o_gpu, o_ref, lse_gpu=None, lse_ref=None, mask=None, label=""):
    """Element-wise comparison; ``mask`` (bool, o's shape) selects the elements checked."""
    og = _np(o_gpu)
    orf = np.asarray(o_ref, dtype=np.float64)
    if mask is not None:
        og, orf = og[mask], orf[mask]
    assert np.isfinite(og).all(), f"{label}: non-finite GPU output"
    assert np.isfinite(orf).all(), f"{label}: reference not computed for every checked element"
    ob = bf16_round(orf)
    err = np.abs(og - ob)
    over = err > O_MAX_ABS
    rounding_limited = over & (err <= bf16_ulp(ob))
    hard = over & ~rounding_limited
    raw = np.abs(og - orf)
    stats = {"max_abs": float(err.max(initial=0.0)), "mean_abs": float(err.mean()) if err.size else 0.0,
             "max_abs_vs_f64": float(raw.max(initial=0.0)),
             "mean_abs_vs_f64": float(raw.mean()) if raw.size else 0.0,
             "n": int(err.size), "rounding_limited": int(rounding_limited.sum())}
    assert not hard.any(), f"{label}: {int(hard.sum())} elements beyond 1e-2 and 1 bf16 ulp (max {stats['max_abs']:.3g})"
    assert stats["mean_abs"] <= O_MEAN_ABS, f"{label}: mean abs error {stats['mean_abs']:.3g} against bf16(oracle)"
    if lse_gpu is not None:
        lg = _np(lse_gpu)
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
            "skipped_gpu": int(((mg == 1) & visited_ref).sum()),
            "ties": int((ties & visited_ref).sum()), "tie_mismatches": int((diff & ties).sum())}


def compare_blasst(o_gpu, lse_gpu, mask_gpu, o_ref, lse_ref, mask_ref, margin_ref, with_gpu_mask, label="",
                   select=None):
    """Decisions, then outputs, of one BLASST run.

    The decisions are compared first (compare_skip). When none of them differs,
    the outputs are compared with the oracle walk's (o_ref, lse_ref). When
    decisions inside the tie band differ, ``with_gpu_mask(mask)`` must return the
    oracle's (o, lse) evaluated on the GPU's decisions, and the outputs are
    compared with that instead. ``select`` maps a full (o, lse) pair to the
    checked part (for sampled heads and rows); identity by default.
    Returns the decision statistics with the output statistics under "output".
    """
    sel = select if select is not None else (lambda o, l: (o, l))
    st = compare_skip(mask_gpu, mask_ref, margin_ref, label=label)
    if st["tie_mismatches"]:
        mg = mask_gpu.cpu().numpy() if isinstance(mask_gpu, torch.Tensor) else np.asarray(mask_gpu)
        o_ref, lse_ref = with_gpu_mask(mg)
        st["reference"] = "oracle formula on the GPU's decisions"
    else:
        st["reference"] = "oracle walk"
    og, lg = sel(o_gpu, lse_gpu)
    orf, lrf = sel(o_ref, lse_ref)
    st["output"] = compare_output(og, orf, lg, lrf, label=label)
    return st


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
    og = _np(o_gpu)
    orf = np.asarray(o_ref, dtype=np.float64)
    err = np.abs(og - orf)
    bound = ulps * bf16_ulp(orf) + floor
    bad = err > bound
    assert not bad.any(), (f"{label}: {int(bad.sum())} elements beyond {ulps} bf16 spacing "
                           f"(worst {float((err / bf16_ulp(orf)).max()):.2f} spacings)")
