"""Pins for the float64 oracle, independent of the oracle's own code.

Every check here compares the oracle with something other than itself:
scalar brute force, torch's float64 SDPA (a library routine), closed forms of
softmax attention, invariants of the definition, and a brute-force restatement
of the BLASST rule. All run on the CPU (``-m "not gpu"``).
"""

import math

import numpy as np
import pytest
import torch

from oracle import attn_oracle as orc
from attention_online_softmax_fwd_b200 import inputs as gen


def _rand(shape, seed, dtype=np.float64):
    return np.random.default_rng(seed).standard_normal(shape).astype(dtype)


# ---------------------------------------------------------------- brute force

def brute_prefill(q, k, v, causal, scale):
    """Scalar loops straight from the definition (no max subtraction)."""
    B, S, Hq, D = q.shape
    Hkv = k.shape[2]
    G = Hq // Hkv
    o = np.zeros((B, S, Hq, D))
    lse = np.zeros((B, Hq, S))
    for b in range(B):
        for h in range(Hq):
            kv = h // G
            for i in range(S):
                w = []
                for j in range(S):
                    if causal and j > i:
                        continue
                    s = sum(q[b, i, h, d] * k[b, j, kv, d] for d in range(D)) * scale
                    w.append((j, math.exp(s)))
                z = sum(e for _, e in w)
                for d in range(D):
                    o[b, i, h, d] = sum(e * v[b, j, kv, d] for j, e in w) / z
                lse[b, h, i] = math.log(z)
    return o, lse


@pytest.mark.parametrize("B,Hq,Hkv,S,D", [(1, 2, 2, 5, 3), (2, 4, 2, 7, 4), (1, 3, 1, 6, 8),
                                          (2, 4, 4, 9, 2), (1, 8, 2, 4, 5)])
@pytest.mark.parametrize("causal", [True, False])
def test_prefill_matches_brute_force(B, Hq, Hkv, S, D, causal):
    q, k, v = _rand((B, S, Hq, D), 1), _rand((B, S, Hkv, D), 2), _rand((B, S, Hkv, D), 3)
    scale = 1 / math.sqrt(D)
    o, lse = orc.prefill(q, k, v, causal, scale)
    ob, lb = brute_prefill(q, k, v, causal, scale)
    np.testing.assert_allclose(o, ob, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, lb, rtol=0, atol=1e-12)


def test_decode_matches_brute_force():
    rng = np.random.default_rng(7)
    N, Hq, Hkv, D, ps = 3, 4, 2, 5, 4
    lens = [1, 6, 11]
    P = 12
    kp, vp = rng.standard_normal((P, ps, Hkv, D)), rng.standard_normal((P, ps, Hkv, D))
    q = rng.standard_normal((N, Hq, D))
    bt = np.array([[5, -1, -1], [0, 9, -1], [3, 2, 11]])
    o, lse = orc.decode_paged(q, kp, vp, bt, lens, ps, 0.5)
    for b in range(N):
        for h in range(Hq):
            kv = h // 2
            ws = []
            for p in range(lens[b]):
                page, slot = bt[b, p // ps], p % ps
                s = sum(q[b, h, d] * kp[page, slot, kv, d] for d in range(D)) * 0.5
                ws.append((page, slot, math.exp(s)))
            z = sum(e for *_, e in ws)
            for d in range(D):
                ref = sum(e * vp[pg, sl, kv, d] for pg, sl, e in ws) / z
                assert abs(o[b, h, d] - ref) < 1e-12
            assert abs(lse[b, h] - math.log(z)) < 1e-12


# ---------------------------------------------------------------- library routine

@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("Hq,Hkv", [(8, 2), (8, 8), (8, 1)])
def test_prefill_matches_torch_sdpa_f64(causal, Hq, Hkv):
    B, S, D = 2, 37, 16
    q, k, v = _rand((B, S, Hq, D), 11), _rand((B, S, Hkv, D), 12), _rand((B, S, Hkv, D), 13)
    scale = 0.3
    o, _ = orc.prefill(q, k, v, causal, scale)
    t = lambda x: torch.from_numpy(x).permute(0, 2, 1, 3)
    ref = torch.nn.functional.scaled_dot_product_attention(
        t(q), t(k), t(v), is_causal=causal, scale=scale, enable_gqa=True)
    np.testing.assert_allclose(o, ref.permute(0, 2, 1, 3).numpy(), rtol=0, atol=1e-12)


# ---------------------------------------------------------------- closed forms

def test_zero_query_causal_is_running_mean():
    B, S, H, D = 1, 20, 2, 4
    q = np.zeros((B, S, H, D))
    k, v = _rand((B, S, H, D), 21), _rand((B, S, H, D), 22)
    o, lse = orc.prefill(q, k, v, True, 1.0)
    for i in range(S):
        np.testing.assert_allclose(o[0, i], v[0, : i + 1].mean(axis=0), atol=1e-13)
        np.testing.assert_allclose(lse[0, :, i], math.log(i + 1), atol=1e-13)


def test_single_key():
    q, k, v = _rand((1, 1, 2, 6), 31), _rand((1, 1, 2, 6), 32), _rand((1, 1, 2, 6), 33)
    o, lse = orc.prefill(q, k, v, True, 0.7)
    np.testing.assert_allclose(o, v, atol=1e-14)
    np.testing.assert_allclose(lse[0, :, 0], (q[0, 0] * k[0, 0]).sum(-1) * 0.7, atol=1e-13)


def test_dominant_key_selects_its_value():
    S, D = 9, 8
    k, v = _rand((1, S, 1, D), 41), _rand((1, S, 1, D), 42)
    j = 5
    q = np.zeros((1, S, 1, D))
    q[0, :, 0] = 60.0 * k[0, j, 0] / np.linalg.norm(k[0, j, 0])
    o, _ = orc.prefill(q, k, v, False, 1.0)
    # every other key's score is lower by a wide margin for these draws
    s = q[0, 0, 0] @ k[0, :, 0].T
    assert np.sort(s)[-1] - np.sort(s)[-2] > 40
    np.testing.assert_allclose(o[0, :, 0], np.broadcast_to(v[0, j, 0], (S, D)), atol=1e-12)


def test_softmax_rows_sum_to_one_and_causal_zeros():
    # With V = identity, O is the probability matrix itself.
    S = D = 12
    q, k = _rand((1, S, 1, D), 51), _rand((1, S, 1, D), 52)
    v = np.eye(S)[None, :, None, :]
    for causal in (True, False):
        o, _ = orc.prefill(q, k, v, causal, 0.5)
        P = o[0, :, 0, :]
        np.testing.assert_allclose(P.sum(axis=1), 1.0, atol=1e-13)
        assert (P >= 0).all()
        if causal:
            assert np.all(P[np.triu_indices(S, 1)] == 0.0)


# ---------------------------------------------------------------- invariants

def test_constant_v_returns_v():
    q, k = _rand((2, 30, 4, 8), 61), _rand((2, 30, 2, 8), 62)
    v = np.broadcast_to(_rand((1, 1, 2, 8), 63), (2, 30, 2, 8)).copy()
    for causal in (True, False):
        o, _ = orc.prefill(q, k, v, causal, 0.4)
        np.testing.assert_allclose(o, v[:, :, [0, 0, 1, 1], :], atol=1e-13)


def test_noncausal_invariant_under_key_permutation():
    q, k, v = _rand((1, 25, 2, 8), 71), _rand((1, 25, 2, 8), 72), _rand((1, 25, 2, 8), 73)
    perm = np.random.default_rng(74).permutation(25)
    o1, l1 = orc.prefill(q, k, v, False, 0.5)
    o2, l2 = orc.prefill(q, k[:, perm], v[:, perm], False, 0.5)
    np.testing.assert_allclose(o1, o2, atol=1e-13)
    np.testing.assert_allclose(l1, l2, atol=1e-13)


def test_gqa_equals_mha_with_repeated_kv():
    Hq, Hkv, G = 8, 2, 4
    q, k, v = _rand((2, 19, Hq, 8), 81), _rand((2, 19, Hkv, 8), 82), _rand((2, 19, Hkv, 8), 83)
    k_rep = np.repeat(k, G, axis=2)      # each KV head copied G times, in order
    v_rep = np.repeat(v, G, axis=2)
    for causal in (True, False):
        o1, l1 = orc.prefill(q, k, v, causal, 0.5)
        o2, l2 = orc.prefill(q, k_rep, v_rep, causal, 0.5)
        np.testing.assert_array_equal(o1, o2)
        np.testing.assert_array_equal(l1, l2)


def test_score_shift_moves_lse_not_o():
    # Append one dimension: q' = [q, c], k' = [k, 1] adds c to every score of a row.
    q, k, v = _rand((1, 15, 1, 6), 91), _rand((1, 15, 1, 6), 92), _rand((1, 15, 1, 6), 93)
    c = 3.25
    q2 = np.concatenate([q, np.full((1, 15, 1, 1), c)], axis=-1)
    k2 = np.concatenate([k, np.ones((1, 15, 1, 1))], axis=-1)
    o1, l1 = orc.prefill(q, k, v, True, 1.0)
    o2, l2 = orc.prefill(q2, k2, v, True, 1.0)
    np.testing.assert_allclose(o1, o2, atol=1e-13)
    np.testing.assert_allclose(l2, l1 + c, atol=1e-12)


def test_row_blocking_and_row_sampling_do_not_change_results():
    q, k, v = _rand((1, 50, 2, 4), 95), _rand((1, 50, 1, 4), 96), _rand((1, 50, 1, 4), 97)
    o1, l1 = orc.prefill(q, k, v, True, 0.5)
    o2, l2 = orc.prefill(q, k, v, True, 0.5, row_block=7)
    o3, l3 = orc.prefill(q, k, v, True, 0.5, heads=[(0, 1)], rows=[0, 13, 49])
    np.testing.assert_allclose(o1, o2, rtol=0, atol=1e-14)     # BLAS blocking: rounding order only
    np.testing.assert_allclose(l1, l2, rtol=0, atol=1e-14)
    np.testing.assert_allclose(o3[0, [0, 13, 49], 1], o1[0, [0, 13, 49], 1], rtol=0, atol=1e-14)
    assert np.isnan(o3[0, 1, 1]).all() and np.isnan(o3[0, 0, 0]).all()


# ---------------------------------------------------------------- online softmax recurrence

def online_softmax_walk(q, k, v, scale, tile):
    """Running max m, running sum l, rescaled accumulator O over key tiles."""
    R, D = q.shape
    m = np.full(R, -np.inf)
    l = np.zeros(R)
    acc = np.zeros((R, v.shape[1]))
    for c0 in range(0, k.shape[0], tile):
        s = (q @ k[c0:c0 + tile].T) * scale
        m_new = np.maximum(m, s.max(axis=1))
        alpha = np.exp(m - m_new)
        p = np.exp(s - m_new[:, None])
        l = alpha * l + p.sum(axis=1)
        acc = alpha[:, None] * acc + p @ v[c0:c0 + tile]
        m = m_new
    return acc / l[:, None], m + np.log(l)


@pytest.mark.parametrize("tile", [1, 3, 16, 64])
def test_online_recurrence_equals_definition(tile):
    q, k, v = _rand((1, 70, 1, 8), 101), _rand((1, 70, 1, 8), 102), _rand((1, 70, 1, 8), 103)
    o, lse = orc.prefill(q, k, v, False, 0.6)
    ow, lw = online_softmax_walk(q[0, :, 0], k[0, :, 0], v[0, :, 0], 0.6, tile)
    np.testing.assert_allclose(ow, o[0, :, 0], atol=1e-12)
    np.testing.assert_allclose(lw, lse[0, 0], atol=1e-12)


def test_split_merge_algebra():
    """Partial (O_s, lse_s) over disjoint key ranges merge to the full result:
    L = ln sum exp(lse_s), O = sum exp(lse_s - L) O_s."""
    q, k, v = _rand((1, 1, 1, 8), 111), _rand((1, 200, 1, 8), 112), _rand((1, 200, 1, 8), 113)
    o_full, l_full = orc.attention_rows(q[0, :, 0], k[0, :, 0], v[0, :, 0], 0.5)
    parts = [orc.attention_rows(q[0, :, 0], k[0, a:b, 0], v[0, a:b, 0], 0.5)
             for a, b in [(0, 64), (64, 150), (150, 200)]]
    lses = np.array([p[1][0] for p in parts])
    L = np.log(np.exp(lses - lses.max()).sum()) + lses.max()
    O = sum(np.exp(p[1][0] - L) * p[0][0] for p in parts)
    np.testing.assert_allclose(O, o_full[0], atol=1e-13)
    assert abs(L - l_full[0]) < 1e-12


# ---------------------------------------------------------------- paged gather

def test_paged_decode_equals_contiguous_and_prefill_last_row():
    B, S, Hq, Hkv, D = 1, 77, 4, 2, 8
    q, k, v = gen.prefill_inputs(B, Hq, Hkv, S, D, seed=5)
    cache = gen.paged_from_contiguous(q[:, S - 1], k, v, page_size=16, seed=6)
    assert torch.isnan(cache.k_pages.float()).any()          # poisoned slots exist
    od, ld = orc.decode_paged(cache.q, cache.k_pages, cache.v_pages, cache.block_table,
                              cache.seq_lens, 16, 0.25)
    op, lp = orc.prefill(q, k, v, True, 0.25, rows=[S - 1])
    np.testing.assert_allclose(od[0], op[0, S - 1], atol=1e-13)
    np.testing.assert_allclose(ld[0], lp[0, :, S - 1], atol=1e-13)
    assert np.isfinite(od).all()


def test_identity_block_table_is_a_reshape():
    rng = np.random.default_rng(121)
    ps, Hkv, D, L = 8, 2, 4, 40
    kc, vc = rng.standard_normal((L, Hkv, D)), rng.standard_normal((L, Hkv, D))
    kp, vp = kc.reshape(L // ps, ps, Hkv, D), vc.reshape(L // ps, ps, Hkv, D)
    bt = np.arange(L // ps)[None, :]
    np.testing.assert_array_equal(orc.gather_pages(kp, bt[0], L, ps), kc)
    q = rng.standard_normal((1, 4, D))
    o, lse = orc.decode_paged(q, kp, vp, bt, [L], ps, 0.5)
    for h in range(4):
        oc, lc = orc.attention_rows(q[0, h][None], kc[:, h // 2], vc[:, h // 2], 0.5)
        np.testing.assert_array_equal(o[0, h], oc[0])


def test_aliased_pages_give_identical_rows():
    c = gen.paged_decode_inputs(2, 4, 2, 8, 16, 40, 40, seed=9)
    bt = c.block_table.clone()
    bt[1] = bt[0]                                  # second sequence shares the first one's pages
    q = c.q.clone()
    q[1] = q[0]
    o, lse = orc.decode_paged(q, c.k_pages, c.v_pages, bt, c.seq_lens, 16, 0.3)
    np.testing.assert_array_equal(o[0], o[1])
    np.testing.assert_array_equal(lse[0], lse[1])


def test_empty_sequence():
    c = gen.paged_decode_inputs(3, 4, 2, 8, 16, 0, 0, seed=10, lens=[5, 0, 17])
    o, lse, skip, _ = orc.decode_paged_blasst(c.q, c.k_pages, c.v_pages, c.block_table,
                                              c.seq_lens, 16, 0.3, 0.0, 64)
    assert (o[1] == 0).all() and np.isneginf(lse[1]).all()
    assert np.isfinite(o).all()


def test_decode_generator_lengths_and_poison():
    c = gen.paged_decode_inputs(64, 32, 8, 128, 16, 512, 8192, seed=1004)
    lens = c.seq_lens.tolist()
    assert min(lens) >= 512 and max(lens) <= 8192 and len(set(lens)) > 50
    used = c.block_table[c.block_table >= 0]
    assert len(set(used.tolist())) == used.numel()        # every page used once
    assert c.num_pages > used.numel()                      # spare pages exist
    spare = sorted(set(range(c.num_pages)) - set(used.tolist()))
    assert torch.isnan(c.k_pages[spare].float()).all()


# ---------------------------------------------------------------- BLASST walk

def brute_blasst_prefill_decisions(q, k, causal, scale, lam):
    """Rule restated from the full score matrix: tile t of a unit is skipped
    iff every row with a visible key in t has exp(r_t - M_t) < lam, where M_t is
    the max over ALL visible scores of the tiles before t (kept or not), and no
    row with a visible key in t has M_t = -inf."""
    B, S, Hq, D = q.shape
    G = Hq // k.shape[2]
    n_qt, n_kt = -(-S // 128), -(-S // 64)
    out = np.full((B, Hq, n_qt, n_kt), 2, np.uint8)
    for b in range(B):
        for h in range(Hq):
            s_full = (q[b, :, h] @ k[b, :, h // G].T) * scale
            for qt in range(n_qt):
                r0, r1 = qt * 128, min(qt * 128 + 128, S)
                n_vis = ((r1 - 1) // 64 + 1) if causal else n_kt
                for t in range(n_vis):
                    verdict = lam > 0
                    for i in range(r0, r1):
                        vis = [j for j in range(t * 64, min(t * 64 + 64, S)) if not causal or j <= i]
                        if not vis:
                            continue
                        r = max(s_full[i, j] for j in vis)
                        prev = [j for j in range(0, t * 64) if not causal or j <= i]
                        if not prev:
                            verdict = False
                            continue
                        M = max(s_full[i, j] for j in prev)
                        if not math.exp(r - M) < lam:
                            verdict = False
                    out[b, h, qt, t] = 1 if verdict else 0
    return out


def _peaked(B, Hq, Hkv, S, D, seed, amp, period=64):
    q, k, v = gen.peaked_prefill_inputs(B, Hq, Hkv, S, D, seed, amp=amp, period=period)
    return q.double().numpy(), k.double().numpy(), v.double().numpy()


@pytest.mark.parametrize("causal", [True, False])
def test_blasst_prefill_decisions_match_brute_force(causal):
    q, k, v = _peaked(1, 2, 1, 300, 16, 131, amp=8.0, period=1 << 20)  # only key 0 peaked
    scale = 1 / 4
    for lam in (0.05, 0.3, 0.7):
        _, _, skip, _ = orc.prefill_blasst(q, k, v, causal, scale, lam)
        ref = brute_blasst_prefill_decisions(q, k, causal, scale, lam)
        np.testing.assert_array_equal(skip, ref)
    assert (skip == 1).any(), "the stress input should produce skips"


def test_blasst_lambda_zero_is_dense():
    q, k, v = _peaked(1, 4, 2, 260, 16, 141, amp=6.0)
    for causal in (True, False):
        o, lse, skip, _ = orc.prefill_blasst(q, k, v, causal, 0.25, 0.0)
        od, ld = orc.prefill(q, k, v, causal, 0.25)
        assert not (skip == 1).any()
        np.testing.assert_allclose(o, od, atol=1e-12)
        np.testing.assert_allclose(lse, ld, atol=1e-12)


def test_blasst_skip_sets_monotone_in_lambda_and_error_bounded():
    q, k, v = _peaked(1, 2, 1, 512, 16, 151, amp=8.0, period=1 << 20)
    scale = 0.25
    od, ld = orc.prefill(q, k, v, True, scale)
    prev = None
    for lam in (0.01, 0.1, 0.3, 0.6, 0.9):
        o, lse, skip, _ = orc.prefill_blasst(q, k, v, True, scale, lam)
        cur = skip == 1
        if prev is not None:
            assert not (prev & ~cur).any(), "a tile skipped at a smaller lambda must stay skipped"
        prev = cur
        # dropped mass bound per row: weights relative to the row's dense max
        for h in range(2):
            s = (q[0, :, h] @ k[0, :, 0].T) * scale
            s = np.where(np.tri(512, dtype=bool), s, -np.inf)
            M = s.max(axis=1)
            w = np.exp(s - M[:, None])
            vis_skip = np.zeros_like(w, dtype=bool)
            for qt in range(4):
                for t in range(8):
                    if skip[0, h, qt, t] == 1:
                        vis_skip[qt * 128:qt * 128 + 128, t * 64:t * 64 + 64] = True
            vis_skip &= np.isfinite(s)
            d = np.where(vis_skip, w, 0).sum(axis=1)
            l_kept = np.where(~vis_skip, w, 0).sum(axis=1)
            assert (d <= vis_skip.sum(axis=1) * lam + 1e-12).all()
            vmax = np.abs(v[0, :, 0]).max()
            err = np.abs(o[0, :, h] - od[0, :, h]).max(axis=1)
            assert (err <= 2 * vmax * d / (l_kept + d) + 1e-12).all()
            # LSE excludes the skipped mass
            np.testing.assert_allclose(lse[0, h], M + np.log(l_kept), atol=1e-10)


def test_blasst_decode_decisions_and_splits():
    B, S, Hq, Hkv, D = 1, 1000, 8, 2, 16
    q, k, v = gen.peaked_prefill_inputs(B, Hq, Hkv, S, D, seed=161, amp=6.0)
    cache = gen.paged_from_contiguous(q[:, S - 1], k, v, page_size=16, seed=162)
    scale = 0.25
    od, ld = orc.decode_paged(cache.q, cache.k_pages, cache.v_pages, cache.block_table,
                              cache.seq_lens, 16, scale)
    for split in (64, 256, 1024):
        o0, l0, s0, _ = orc.decode_paged_blasst(cache.q, cache.k_pages, cache.v_pages,
                                                cache.block_table, cache.seq_lens, 16, scale,
                                                0.0, split)
        np.testing.assert_allclose(o0, od, atol=1e-12)        # lambda 0: independent of splits
        np.testing.assert_allclose(l0, ld, atol=1e-12)
        assert not (s0 == 1).any()
    # brute-force decisions for lambda 0.3, split 256, group rows
    lam, split = 0.3, 256
    _, _, skip, _ = orc.decode_paged_blasst(cache.q, cache.k_pages, cache.v_pages,
                                            cache.block_table, cache.seq_lens, 16, scale, lam, split)
    qd, kd = cache.q.double().numpy(), k[0].double().numpy()
    G = Hq // Hkv
    n_skip = 0
    for kv in range(Hkv):
        s = (qd[0, kv * G:kv * G + G] @ kd[:, kv].T) * scale
        for t in range(-(-S // 64)):
            sp0 = (t * 64 // split) * split
            if t * 64 == sp0:
                assert skip[0, kv, t] == 0
                continue
            M = s[:, sp0:t * 64].max(axis=1)
            r = s[:, t * 64:min(t * 64 + 64, S)].max(axis=1)
            want = bool((np.exp(r - M) < lam).all())
            assert skip[0, kv, t] == int(want)
            n_skip += want
        assert (skip[0, kv, -(-S // 64):] == 2).all()
    assert n_skip > 0
    # per-head rows skip at least as often as group rows
    _, _, skip_h, _ = orc.decode_paged_blasst(cache.q, cache.k_pages, cache.v_pages,
                                              cache.block_table, cache.seq_lens, 16, scale, lam,
                                              split, rows_per_unit="head")
    for kv in range(Hkv):
        grp = skip[0, kv] == 1
        for h in range(kv * G, kv * G + G):
            assert not (grp & ~(skip_h[0, h] == 1)).any()


# ---------------------------------------------------------------- chunked prefill over pages

def test_prefill_paged_matches_brute_force():
    rng = np.random.default_rng(31)
    B, Sq, Hq, Hkv, D, ps = 2, 3, 4, 2, 3, 4
    lens = [5, 9]
    P = 8
    kp, vp = rng.standard_normal((P, ps, Hkv, D)), rng.standard_normal((P, ps, Hkv, D))
    q = rng.standard_normal((B, Sq, Hq, D))
    bt = np.array([[6, 1, -1], [0, 7, 3]])
    o, lse = orc.prefill_paged(q, kp, vp, bt, lens, ps, 0.5)
    for b in range(B):
        for h in range(Hq):
            kv = h // 2
            for i in range(Sq):
                pos = lens[b] - Sq + i
                ws = []
                for j in range(pos + 1):
                    page, slot = bt[b, j // ps], j % ps
                    s_ = sum(q[b, i, h, d] * kp[page, slot, kv, d] for d in range(D)) * 0.5
                    ws.append((page, slot, math.exp(s_)))
                z = sum(e for *_, e in ws)
                for d in range(D):
                    ref = sum(e * vp[pg, sl, kv, d] for pg, sl, e in ws) / z
                    assert abs(o[b, i, h, d] - ref) < 1e-12
                assert abs(lse[b, h, i] - math.log(z)) < 1e-12


def test_prefill_paged_whole_sequence_is_causal_prefill():
    c = gen.paged_prefill_inputs(1, 50, 4, 2, 8, 16, [50], seed=32)
    o, lse = orc.prefill_paged(c.q, c.k_pages, c.v_pages, c.block_table, c.seq_lens, 16, 0.3)
    op, lp = orc.prefill(c.q, c.k_seqs[0][None], c.v_seqs[0][None], True, 0.3)
    np.testing.assert_allclose(o, op, rtol=0, atol=1e-13)
    np.testing.assert_allclose(lse, lp, rtol=0, atol=1e-13)


def test_prefill_paged_single_query_is_decode():
    c = gen.paged_prefill_inputs(3, 1, 8, 2, 8, 16, [1, 17, 60], seed=33)
    o, lse = orc.prefill_paged(c.q, c.k_pages, c.v_pages, c.block_table, c.seq_lens, 16, 0.4)
    od, ld = orc.decode_paged(c.q[:, 0], c.k_pages, c.v_pages, c.block_table, c.seq_lens, 16, 0.4)
    np.testing.assert_allclose(o[:, 0], od, rtol=0, atol=1e-13)
    np.testing.assert_allclose(lse[:, :, 0], ld, rtol=0, atol=1e-13)


def test_prefill_paged_chunks_compose():
    # the last Sq1 + Sq2 tokens as one chunk equal two chunks: the first Sq1 of
    # them against the cache up to their own end, then the last Sq2
    c = gen.paged_prefill_inputs(2, 12, 4, 2, 8, 16, [40, 12], seed=34)
    o, lse = orc.prefill_paged(c.q, c.k_pages, c.v_pages, c.block_table, c.seq_lens, 16, 0.3)
    Sq1 = 5
    lens1 = c.seq_lens - (12 - Sq1)
    o1, l1 = orc.prefill_paged(c.q[:, :Sq1], c.k_pages, c.v_pages, c.block_table, lens1, 16, 0.3)
    o2, l2 = orc.prefill_paged(c.q[:, Sq1:], c.k_pages, c.v_pages, c.block_table, c.seq_lens, 16, 0.3)
    np.testing.assert_allclose(o[:, :Sq1], o1, rtol=0, atol=1e-13)
    np.testing.assert_allclose(o[:, Sq1:], o2, rtol=0, atol=1e-13)
    np.testing.assert_allclose(lse[:, :, :Sq1], l1, rtol=0, atol=1e-13)
    np.testing.assert_allclose(lse[:, :, Sq1:], l2, rtol=0, atol=1e-13)


def test_prefill_paged_matches_torch_sdpa_with_end_aligned_mask():
    c = gen.paged_prefill_inputs(2, 9, 8, 2, 16, 16, [33, 9], seed=35, poison=False)
    o, _ = orc.prefill_paged(c.q, c.k_pages, c.v_pages, c.block_table, c.seq_lens, 16, 0.25)
    for b in range(2):
        L = int(c.seq_lens[b])
        qb = c.q[b].double().permute(1, 0, 2)[None]                  # [1, Hq, Sq, D]
        kb = c.k_seqs[b].double().permute(1, 0, 2)[None]             # [1, Hkv, L, D]
        vb = c.v_seqs[b].double().permute(1, 0, 2)[None]
        mask = torch.arange(L)[None, :] <= (torch.arange(9)[:, None] + (L - 9))
        ref = torch.nn.functional.scaled_dot_product_attention(qb, kb, vb, attn_mask=mask, scale=0.25,
                                                               enable_gqa=True)
        np.testing.assert_allclose(o[b], ref[0].permute(1, 0, 2).numpy(), rtol=0, atol=1e-12)


def test_prefill_paged_rejects_short_cache():
    c = gen.paged_prefill_inputs(1, 4, 2, 1, 8, 16, [4], seed=36)
    with pytest.raises(ValueError):
        orc.prefill_paged(c.q, c.k_pages, c.v_pages, c.block_table, torch.tensor([3]), 16, 0.3)


# ---------------------------------------------------------------- KV append

def test_kv_append_then_gather_is_concatenation():
    c = gen.paged_prefill_inputs(3, 1, 4, 2, 8, 16, [5, 16, 33], seed=37, poison=False)
    g = torch.Generator().manual_seed(38)
    T = 20
    lens = [int(x) for x in c.seq_lens]
    # room for T more tokens: extend the block tables with fresh pages
    need = [-(-(L + T) // 16) for L in lens]
    P0 = c.k_pages.shape[0]
    extra = sum(max(0, n - -(-L // 16)) for n, L in zip(need, lens))
    kp = torch.cat([c.k_pages, torch.zeros(extra, 16, 2, 8, dtype=torch.bfloat16)])
    vp = torch.cat([c.v_pages, torch.zeros(extra, 16, 2, 8, dtype=torch.bfloat16)])
    bt = torch.full((3, max(need)), -1, dtype=torch.int32)
    nxt = P0
    for b in range(3):
        have = -(-lens[b] // 16)
        bt[b, :have] = c.block_table[b, :have]
        for j in range(have, need[b]):
            bt[b, j] = nxt
            nxt += 1
    kn = torch.randn(3, T, 2, 8, generator=g).to(torch.bfloat16)
    vn = torch.randn(3, T, 2, 8, generator=g).to(torch.bfloat16)
    kp2, vp2 = orc.kv_append(kp, vp, bt, lens, kn, vn, 16)
    for b in range(3):
        kk = orc.gather_pages(kp2, bt[b].numpy(), lens[b] + T, 16)
        vv = orc.gather_pages(vp2, bt[b].numpy(), lens[b] + T, 16)
        np.testing.assert_array_equal(kk[:lens[b]], c.k_seqs[b].double().numpy())
        np.testing.assert_array_equal(kk[lens[b]:], kn[b].double().numpy())
        np.testing.assert_array_equal(vv[lens[b]:], vn[b].double().numpy())
    # slots nobody wrote are unchanged
    written = np.zeros(kp.shape[:2], dtype=bool)
    for b in range(3):
        for pos in range(lens[b] + T):
            written[int(bt[b, pos // 16]), pos % 16] = True
    np.testing.assert_array_equal(kp2[~written], kp.float().numpy()[~written])


def test_kv_append_rejects_positions_past_the_table():
    kp = np.zeros((4, 16, 1, 8))
    bt = np.array([[0, 1]])
    with pytest.raises(IndexError):
        orc.kv_append(kp, kp, bt, [30], np.zeros((1, 3, 1, 8)), np.zeros((1, 3, 1, 8)), 16)


# ---------------------------------------------------------------- FP8 cache

def test_e4m3_decoding_matches_torch_for_every_code():
    codes = np.arange(256, dtype=np.uint8)
    ours = orc.e4m3_to_float(codes)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).double().numpy()
    assert np.array_equal(np.isnan(ours), np.isnan(ref))
    np.testing.assert_array_equal(ours[~np.isnan(ours)], ref[~np.isnan(ref)])
    assert np.nanmax(ours) == 448.0 and np.nanmin(ours[ours > 0]) == 2.0 ** -9


def test_quantised_pool_within_half_an_e4m3_step():
    c = gen.paged_decode_inputs(4, 8, 2, 64, 16, 30, 90, seed=39, poison=False)
    codes, s = gen.quantize_pool_e4m3(c.k_pages)
    x = c.k_pages.double().numpy()
    deq = orc.e4m3_to_float(codes.numpy()) * s
    # round to nearest: |error| <= 2^-4 |x| for normals, <= 2^-10 * s for subnormals
    assert (np.abs(deq - x) <= np.maximum(np.abs(x) * 2.0 ** -4, s * 2.0 ** -10) + 1e-12).all()


def test_fp8_decode_is_decode_of_the_dequantised_cache():
    c = gen.paged_decode_inputs(3, 8, 2, 64, 16, 20, 200, seed=40)
    kc, ks = gen.quantize_pool_e4m3(c.k_pages)
    vc, vs = gen.quantize_pool_e4m3(c.v_pages)
    o, lse = orc.decode_paged_fp8(c.q, kc, vc, ks, vs, c.block_table, c.seq_lens, 16, 0.3)
    kd = orc.e4m3_to_float(kc.numpy()) * ks
    vd = orc.e4m3_to_float(vc.numpy()) * vs
    od, ld = orc.decode_paged(c.q, kd, vd, c.block_table, c.seq_lens, 16, 0.3)
    np.testing.assert_array_equal(o, od)
    np.testing.assert_array_equal(lse, ld)
    assert np.isfinite(o).all()                   # poisoned (NaN) slots are never read



# ---------------------------------------------------------------- the formula on a given decision mask

def brute_prefill_masked(q, k, v, causal, scale, skip_mask):
    """Scalar loops: row i of head h sees key j iff j is visible and the 64-key
    tile of j is not marked skipped (1) for the 128-row tile of i."""
    B, S, Hq, D = q.shape
    G = Hq // k.shape[2]
    o = np.zeros((B, S, Hq, D))
    lse = np.zeros((B, Hq, S))
    for b in range(B):
        for h in range(Hq):
            for i in range(S):
                w = []
                for j in range(S):
                    if (causal and j > i) or skip_mask[b, h, i // 128, j // 64] == 1:
                        continue
                    s = sum(q[b, i, h, d] * k[b, j, h // G, d] for d in range(D)) * scale
                    w.append((j, math.exp(s)))
                z = sum(e for _, e in w)
                for d in range(D):
                    o[b, i, h, d] = sum(e * v[b, j, h // G, d] for j, e in w) / z
                lse[b, h, i] = math.log(z)
    return o, lse


@pytest.mark.parametrize("causal", [True, False])
def test_prefill_with_skip_mask_matches_brute_force(causal):
    B, Hq, Hkv, S, D = 1, 2, 1, 150, 3
    q, k, v = _rand((B, S, Hq, D), 71), _rand((B, S, Hkv, D), 72), _rand((B, S, Hkv, D), 73)
    rng = np.random.default_rng(74)
    mask = rng.integers(0, 2, (B, Hq, 2, 3)).astype(np.uint8)
    mask[..., 0] = 0            # every row keeps a key of its first tile
    o, lse = orc.prefill_with_skip_mask(q, k, v, causal, 0.5, mask)
    ob, lb = brute_prefill_masked(q, k, v, causal, 0.5, mask)
    np.testing.assert_allclose(o, ob, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, lb, rtol=0, atol=1e-12)


def test_prefill_with_skip_mask_keep_all_is_dense_and_walk_mask_is_walk():
    q, k, v = _peaked(1, 4, 2, 300, 16, 171, amp=8.0, period=1 << 20)
    for causal in (True, False):
        keep = np.zeros((1, 4, 3, 5), np.uint8)
        o, lse = orc.prefill_with_skip_mask(q, k, v, causal, 0.25, keep)
        od, ld = orc.prefill(q, k, v, causal, 0.25)
        np.testing.assert_allclose(o, od, atol=1e-12)
        np.testing.assert_allclose(lse, ld, atol=1e-12)
        ow, lw, skip, _ = orc.prefill_blasst(q, k, v, causal, 0.25, 0.3)
        assert skip.shape == keep.shape and (skip == 1).any()
        om, lm = orc.prefill_with_skip_mask(q, k, v, causal, 0.25, skip)
        np.testing.assert_allclose(om, ow, atol=1e-12)
        np.testing.assert_allclose(lm, lw, atol=1e-12)


def test_decode_with_skip_mask_matches_brute_force():
    S, Hq, Hkv, D = 300, 4, 2, 8
    q, k, v = gen.peaked_prefill_inputs(1, Hq, Hkv, S, D, seed=181, amp=6.0)
    cache = gen.paged_from_contiguous(q[:, S - 1], k, v, page_size=16, seed=182)
    rng = np.random.default_rng(183)
    n_tiles = -(-cache.max_pages * 16 // 64)
    scale = 0.3
    qd, kd, vd = cache.q.double().numpy(), k[0].double().numpy(), v[0].double().numpy()
    for unit_rows, n_units in (("group", Hkv), ("head", Hq)):
        mask = rng.integers(0, 2, (1, n_units, n_tiles)).astype(np.uint8)
        mask[..., 0] = 0
        o, lse = orc.decode_paged_with_skip_mask(cache.q, cache.k_pages, cache.v_pages, cache.block_table,
                                                 cache.seq_lens, 16, scale, mask, rows_per_unit=unit_rows)
        for h in range(Hq):
            kv = h // (Hq // Hkv)
            unit = kv if unit_rows == "group" else h
            w = [(j, math.exp(scale * sum(qd[0, h, d] * kd[j, kv, d] for d in range(D))))
                 for j in range(S) if mask[0, unit, j // 64] != 1]
            z = sum(e for _, e in w)
            for d in range(D):
                assert abs(o[0, h, d] - sum(e * vd[j, kv, d] for j, e in w) / z) < 1e-12
            assert abs(lse[0, h] - math.log(z)) < 1e-12
    keep = np.zeros((1, Hkv, n_tiles), np.uint8)
    o, lse = orc.decode_paged_with_skip_mask(cache.q, cache.k_pages, cache.v_pages, cache.block_table,
                                             cache.seq_lens, 16, scale, keep)
    od, ld = orc.decode_paged(cache.q, cache.k_pages, cache.v_pages, cache.block_table, cache.seq_lens, 16, scale)
    np.testing.assert_allclose(o, od, atol=1e-12)
    np.testing.assert_allclose(lse, ld, atol=1e-12)


def test_oracle_reproduces_its_golden_fixtures():
    """tests/golden/oracle_fixtures.json holds the oracle's answers for two small
    seeded cases (written by tests/golden/make_fixtures.py): recomputing them must
    give the same values, so any change to the oracle's arithmetic is visible."""
    import importlib.util
    import json
    import os
    here = os.path.join(os.path.dirname(__file__), "golden")
    spec = importlib.util.spec_from_file_location("make_fixtures", os.path.join(here, "make_fixtures.py"))
    mf = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mf)
    stored = json.load(open(os.path.join(here, "oracle_fixtures.json")))
    fresh = mf.build()
    for case in ("tiny_gqa_prefill", "blasst_paged_decode"):
        for key, val in stored[case].items():
            got = fresh[case][key]
            if isinstance(val, list) and val and isinstance(val[0], (float, int, str)):
                a = np.array([float(x) for x in val])
                b = np.array([float(x) for x in got])
                assert a.shape == b.shape, (case, key)
                fin = np.isfinite(a)
                assert np.array_equal(fin, np.isfinite(b)) and np.array_equal(a[~fin], b[~fin]), (case, key)
                assert np.allclose(a[fin], b[fin], rtol=2e-7, atol=1e-12), (case, key)
            else:
                assert val == got, (case, key)
