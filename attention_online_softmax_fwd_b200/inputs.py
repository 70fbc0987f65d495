"""Seeded synthetic inputs shared by the tests, the bench and the oracle checks.

This module only draws numbers and lays them out; it holds none of the
attention arithmetic. Every tensor is produced on the CPU from a
``torch.Generator`` (fp32 N(0, 1) draws rounded to bf16, round-to-nearest-even),
so both sides of a parity check see the same bytes.

Layouts (row-major, contiguous):
  q, k, v (prefill)     [B][S][H][D]  bf16
  q (decode)            [N][Hq][D]    bf16
  k_pages, v_pages      [P][page_size][Hkv][D] bf16
  block_table           [N][max_pages] int32, -1 past the last page
  seq_lens              [N] int32
"""

from __future__ import annotations

import math
from dataclasses import dataclass

import torch


def attn_scale(D: int) -> float:
    """Softmax scale 1/sqrt(D) rounded to fp32 (the value the kernels receive)."""
    return float(torch.tensor(1.0 / math.sqrt(D), dtype=torch.float32))


def _randn(gen, shape):
    return torch.randn(shape, generator=gen, dtype=torch.float32)


def prefill_inputs(B, Hq, Hkv, S, D, seed):
    g = torch.Generator().manual_seed(seed)
    q = _randn(g, (B, S, Hq, D)).to(torch.bfloat16)
    k = _randn(g, (B, S, Hkv, D)).to(torch.bfloat16)
    v = _randn(g, (B, S, Hkv, D)).to(torch.bfloat16)
    return q, k, v


def peaked_prefill_inputs(B, Hq, Hkv, S, D, seed, amp=4.0, period=64):
    """Peaked scores: amp*u added to every ``period``-th key and to all queries.

    u is one seeded unit vector shared by all heads; the sums are formed in
    fp32 before rounding to bf16. V ~ N(0, 1).
    """
    g = torch.Generator().manual_seed(seed)
    u = _randn(g, (D,))
    u = u / u.norm()
    q = _randn(g, (B, S, Hq, D)) + amp * u
    k = _randn(g, (B, S, Hkv, D))
    k[:, ::period] += amp * u
    v = _randn(g, (B, S, Hkv, D))
    return q.to(torch.bfloat16), k.to(torch.bfloat16), v.to(torch.bfloat16)


@dataclass
class PagedCache:
    q: torch.Tensor            # [N, Hq, D] bf16
    k_pages: torch.Tensor      # [P, page_size, Hkv, D] bf16
    v_pages: torch.Tensor
    block_table: torch.Tensor  # [N, max_pages] int32
    seq_lens: torch.Tensor     # [N] int32
    page_size: int

    @property
    def num_pages(self):
        return self.k_pages.shape[0]

    @property
    def max_pages(self):
        return self.block_table.shape[1]


def page_sequences(k_seqs, v_seqs, page_size, gen, extra_frac=0.1, poison=True, max_pages=None):
    """Scatter per-sequence K/V [L_b, Hkv, D] into a shared page pool.

    Physical page ids are a seeded random permutation of the pool, handed out
    in sequence order. The pool has ``extra_frac`` unused pages; unused pages
    and the slots past L in each last page are NaN when ``poison``.
    """
    lens = [int(kk.shape[0]) for kk in k_seqs]
    Hkv, D = k_seqs[0].shape[1], k_seqs[0].shape[2]
    need = [-(-L // page_size) for L in lens]
    used = sum(need)
    P = used + max(1, int(math.ceil(extra_frac * used)))
    fill = float("nan") if poison else 0.0
    k_pool = torch.full((P, page_size, Hkv, D), fill, dtype=torch.bfloat16)
    v_pool = torch.full((P, page_size, Hkv, D), fill, dtype=torch.bfloat16)
    perm = torch.randperm(P, generator=gen)
    mp = max(need) if max_pages is None else max_pages
    mp = max(mp, 1)
    bt = torch.full((len(lens), mp), -1, dtype=torch.int32)
    nxt = 0
    for b, L in enumerate(lens):
        for j in range(need[b]):
            page = int(perm[nxt]); nxt += 1
            bt[b, j] = page
            t0, t1 = j * page_size, min(j * page_size + page_size, L)
            k_pool[page, : t1 - t0] = k_seqs[b][t0:t1]
            v_pool[page, : t1 - t0] = v_seqs[b][t0:t1]
    return k_pool, v_pool, bt


def paged_decode_inputs(num_seqs, Hq, Hkv, D, page_size, len_lo, len_hi, seed,
                        extra_frac=0.1, poison=True, lens=None, max_pages=None):
    """Decode workload: lengths uniform in [len_lo, len_hi] (inclusive) unless given."""
    g = torch.Generator().manual_seed(seed)
    if lens is None:
        lens = torch.randint(len_lo, len_hi + 1, (num_seqs,), generator=g).tolist()
    q = _randn(g, (num_seqs, Hq, D)).to(torch.bfloat16)
    k_seqs = [_randn(g, (L, Hkv, D)).to(torch.bfloat16) for L in lens]
    v_seqs = [_randn(g, (L, Hkv, D)).to(torch.bfloat16) for L in lens]
    if max_pages is None:
        max_pages = max(1, -(-max(lens) // page_size)) if lens else 1
    k_pool, v_pool, bt = page_sequences(k_seqs, v_seqs, page_size, g, extra_frac, poison,
                                        max_pages=max_pages) if any(lens) else _empty_pool(
        len(lens), Hkv, D, page_size, max_pages)
    return PagedCache(q, k_pool, v_pool, bt, torch.tensor(lens, dtype=torch.int32), page_size)


def _empty_pool(N, Hkv, D, page_size, max_pages):
    kp = torch.full((1, page_size, Hkv, D), float("nan"), dtype=torch.bfloat16)
    return kp, kp.clone(), torch.full((N, max_pages), -1, dtype=torch.int32)


def paged_from_contiguous(q_last, k, v, page_size, seed, poison=True):
    """Decode over a prefill's K/V: the query is ``q_last`` [1, Hq, D] and the
    cache holds k/v [1, S, Hkv, D] paged by a seeded random permutation."""
    g = torch.Generator().manual_seed(seed)
    k_pool, v_pool, bt = page_sequences([k[0]], [v[0]], page_size, g, 0.1, poison)
    return PagedCache(q_last.contiguous(), k_pool, v_pool, bt,
                      torch.tensor([k.shape[1]], dtype=torch.int32), page_size)


def peaked_decode_batch(num_seqs, Hq, Hkv, L, D, seed, amp=12.0, period=None, page_size=16, poison=False):
    """A decode batch of ``num_seqs`` sequences of L tokens whose scores are
    peaked like peaked_prefill_inputs: one seeded unit vector u, amp*u added to
    every ``period``-th key of each sequence (key 0 only when period is None) and
    to every query. K/V ~ N(0, 1) otherwise; paged by a seeded permutation."""
    g = torch.Generator().manual_seed(seed)
    u = _randn(g, (D,))
    u = u / u.norm()
    q = (_randn(g, (num_seqs, Hq, D)) + amp * u).to(torch.bfloat16)
    step = L if period is None else period
    k_seqs, v_seqs = [], []
    for _ in range(num_seqs):
        k = _randn(g, (L, Hkv, D))
        k[::step] += amp * u
        k_seqs.append(k.to(torch.bfloat16))
        v_seqs.append(_randn(g, (L, Hkv, D)).to(torch.bfloat16))
    k_pool, v_pool, bt = page_sequences(k_seqs, v_seqs, page_size, g, 0.1, poison)
    return PagedCache(q, k_pool, v_pool, bt, torch.tensor([L] * num_seqs, dtype=torch.int32), page_size)


@dataclass
class PagedPrefill:
    q: torch.Tensor            # [B, Sq, Hq, D] bf16: queries of the Sq newest tokens
    k_pages: torch.Tensor      # [P, page_size, Hkv, D] bf16, the new tokens' K/V included
    v_pages: torch.Tensor
    block_table: torch.Tensor  # [B, max_pages] int32
    seq_lens: torch.Tensor     # [B] int32, total tokens per sequence (>= Sq)
    k_seqs: list               # per sequence [L_b, Hkv, D] bf16 (contiguous copy)
    v_seqs: list
    page_size: int


def paged_prefill_inputs(B, Sq, Hq, Hkv, D, page_size, lens, seed, poison=True, extra_frac=0.1):
    """Chunked-prefill workload: each sequence b holds lens[b] >= Sq tokens of
    K/V ~ N(0, 1) in a shared page pool (seeded permutation, NaN-poisoned spare
    pages and tail slots); q ~ N(0, 1) for its Sq newest tokens."""
    g = torch.Generator().manual_seed(seed)
    q = _randn(g, (B, Sq, Hq, D)).to(torch.bfloat16)
    k_seqs = [_randn(g, (int(L), Hkv, D)).to(torch.bfloat16) for L in lens]
    v_seqs = [_randn(g, (int(L), Hkv, D)).to(torch.bfloat16) for L in lens]
    k_pool, v_pool, bt = page_sequences(k_seqs, v_seqs, page_size, g, extra_frac, poison)
    return PagedPrefill(q, k_pool, v_pool, bt, torch.tensor([int(L) for L in lens], dtype=torch.int32),
                        k_seqs, v_seqs, page_size)


def quantize_pool_e4m3(pool):
    """FP8 E4M3 codes (uint8, same shape) and the scale of a bf16 page pool:
    scale = max|finite x| / 448, codes = e4m3(x / scale) rounded to nearest
    (NaN stays NaN)."""
    x = pool.float()
    finite = torch.isfinite(x)
    amax = float(x[finite].abs().max()) if finite.any() else 1.0
    scale = max(amax, 1e-30) / 448.0
    codes = (x / scale).to(torch.float8_e4m3fn).view(torch.uint8)
    return codes, scale


# The workloads the library is measured and checked on (sizes as named).
CONFIGS = {
    "tiny_gqa_prefill": dict(kind="prefill", B=1, Hq=4, Hkv=2, S=128, D=64, causal=True, seed=1001),
    "mha_prefill_llama2_7b": dict(kind="prefill", B=4, Hq=32, Hkv=32, S=2048, D=128, causal=True, seed=1002),
    "gqa_prefill_llama3_8b": dict(kind="prefill", B=2, Hq=32, Hkv=8, S=8192, D=128, causal=True, seed=1003),
    "paged_gqa_decode": dict(kind="decode", N=64, Hq=32, Hkv=8, D=128, page_size=16,
                             len_lo=512, len_hi=8192, seed=1004),
    "blasst_long_context": dict(kind="blasst", B=1, Hq=32, Hkv=8, S=32768, D=128, causal=True,
                                lambdas=(0.0, 0.1, 0.3), page_size=16, seed=1005),
}
