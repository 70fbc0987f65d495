"""Float64 CPU oracle for exact scaled-dot-product attention with online softmax.

TEST INFRASTRUCTURE. Only the tests, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` import this module. The product path (the
CUDA library and its Python binding) never calls it, and it calls nothing of
the product path: it shares no code, table or constant with the kernels.

What it computes, and the passages it follows:

* Exact attention O = softmax(Q K^T * scale + mask) V, materialised. The
  method is exact, not an approximation ("flash-attention与TensorRT-LLM集成",
  section 背景与痛点分析, which names the paper "FlashAttention: Fast and
  Memory-Efficient Exact Attention with IO-Awareness"; "LLM推理优化技术综述",
  PART04). The log-sum-exp LSE = max + ln(sum exp(s - max)) is returned beside
  O in natural-log units.
* Grouped-query head mapping: query head h reads KV head floor(h / G) with
  G = Hq / Hkv, the mapping that duplicating each KV head G times produces
  ("TensorRT对Grouped Query Attention的支持进展", sections 技术演进背景 and
  图优化与算子融合; "LLM推理优化技术综述", PART03). MHA is G = 1, MQA is Hkv = 1.
* Causal mask: key j is visible to query i iff j <= i (autoregressive
  generation, "LLM推理优化技术综述", PART01). Queries and keys share positions.
* Paged KV cache: token p of a sequence lives in physical page
  block_table[p // page_size], slot p % page_size ("LLM推理优化技术综述",
  PART02: a block table maps contiguous logical blocks to non-contiguous
  physical ones; "Optimizing Inference on LLMs with TensorRT-LLM", PagedAttention
  section). The oracle gathers the pages and applies the dense formula.
* BLASST tile skip ("高效部署稀疏注意力加速方案：BLASST方法详解与实践指南",
  section 架构与组件: keep a running maximum of the attention scores during the
  blockwise online softmax and compare against a threshold lambda; a negligible
  block skips its exponentials, its Value load and its matrix product). The
  pages do not print the inequality. The reading used here: a KV tile of 64
  keys is skipped iff lambda > 0 and, for every row of the decision unit,
  exp(tile_rowmax - running_max) < lambda (strict), on scaled natural-log
  scores, where running_max is the maximum over the tiles of the unit already
  kept. A row that sees no key of the tile is vacuously below the threshold;
  a row whose running maximum is still -inf is not. The walk visits the tiles
  of a unit in ascending key order; the result is the exact formula
  restricted to the kept keys.

* Chunked prefill over the paged cache (prefill_paged): the reading of
  "chunked prefill" stated in its docstring.
* Writing new tokens' K/V into the paged cache (kv_append).
* FP8 E4M3 paged cache with one scale per pool (decode_paged_fp8): the
  reading stated in its docstring; E4M3 decoded from its bit layout.
* The exact formula restricted to the tiles that a given decision mask keeps
  (prefill_with_skip_mask, decode_paged_with_skip_mask), for decision sets
  that differ from the walk's only where a decision sits within the tie band.

Parity status: dense prefill, paged decode, chunked paged prefill and the
gather are pinned by the
CPU tests (brute force, torch's float64 SDPA, closed forms, invariants). The
BLASST walk is pinned against a brute-force recomputation of the rule from the
full score matrix and against its invariants; the rule itself is a reading of
the pages ("parity unpinned" against the pages, which never print it).
"""

from __future__ import annotations

import math

import numpy as np

NEG_INF = -np.inf
KV_TILE = 64          # keys per BLASST decision tile (block_size 64 in the BLASST guide's config)
Q_TILE = 128          # query rows per prefill decision unit


def _f64(x):
    """Widen a tensor or array (bf16 torch tensors included) to float64 numpy."""
    if hasattr(x, "detach"):
        return x.detach().to("cpu").double().numpy()
    return np.asarray(x, dtype=np.float64)


def kv_head_of(hq: int, Hq: int, Hkv: int) -> int:
    """Query head hq reads KV head floor(hq / (Hq / Hkv))."""
    if Hq % Hkv != 0:
        raise ValueError("Hq must be a multiple of Hkv")
    return hq // (Hq // Hkv)


def attention_rows(q, k, v, scale, visible=None):
    """Exact attention for one head.

    q [R, D], k [N, D], v [N, D] (float64); visible: bool [R, N] or None (all
    keys visible). Returns (o [R, D], lse [R]). A row that sees no key gets
    o = 0 and lse = -inf.
    """
    s = (q @ k.T) * scale
    if visible is not None:
        s = np.where(visible, s, NEG_INF)
    m = s.max(axis=1) if s.shape[1] else np.full(s.shape[0], NEG_INF)
    empty = ~np.isfinite(m)
    m_safe = np.where(empty, 0.0, m)
    p = np.exp(s - m_safe[:, None])                    # exp(-inf) = 0 for hidden keys
    l = p.sum(axis=1)
    l_safe = np.where(empty, 1.0, l)
    o = (p @ v) / l_safe[:, None]
    o[empty] = 0.0
    lse = np.where(empty, NEG_INF, m_safe + np.log(l_safe))
    return o, lse


def causal_visible(rows, n_keys):
    """bool [len(rows), n_keys]: key j visible to query row i iff j <= i."""
    rows = np.asarray(rows)
    return np.arange(n_keys)[None, :] <= rows[:, None]


def prefill(q, k, v, causal: bool, scale: float, row_block: int = 2048,
            heads=None, rows=None):
    """Dense prefill attention.

    q [B, S, Hq, D], k/v [B, S, Hkv, D] (any dtype; widened to float64).
    Returns o [B, S, Hq, D] and lse [B, Hq, S] (float64). ``heads`` (list of
    (b, hq)) and ``rows`` (list of query positions) restrict the work to a
    sample; entries outside the sample are NaN. Row blocking only bounds
    memory: every row still sees its full key range.
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, S, Hq, _ = q.shape
    Hkv = k.shape[2]
    o = np.full((B, S, Hq, v.shape[-1]), np.nan)   # value width may differ from the key width
    lse = np.full((B, Hq, S), np.nan)
    if heads is None:
        heads = [(b, h) for b in range(B) for h in range(Hq)]
    row_list = np.arange(S) if rows is None else np.asarray(sorted(set(int(r) for r in rows)))
    for b, hq in heads:
        kv = kv_head_of(hq, Hq, Hkv)
        for i0 in range(0, len(row_list), row_block):
            rr = row_list[i0:i0 + row_block]
            vis = causal_visible(rr, S) if causal else None
            ob, lb = attention_rows(q[b, rr, hq, :], k[b, :, kv, :], v[b, :, kv, :], scale, vis)
            o[b, rr, hq, :] = ob
            lse[b, hq, rr] = lb
    return o, lse


def gather_pages(pages, block_table_row, seq_len: int, page_size: int):
    """Contiguous [seq_len, Hkv, D] float64 view of one sequence's paged K or V.

    pages [P, page_size, Hkv, D]; token p is pages[block_table_row[p // page_size], p % page_size].
    Only the pages the sequence uses are read (and widened).
    """
    n_pages = -(-seq_len // page_size)
    ids = [int(x) for x in block_table_row[:n_pages]]
    n_pool = pages.shape[0]
    for j, page in enumerate(ids):
        if page < 0 or page >= n_pool:
            raise IndexError(f"block_table entry {page} out of range for logical page {j}")
    if n_pages == 0:
        return np.empty((0,) + tuple(pages.shape[2:]))
    picked = _f64(pages[ids])                           # [n_pages, page_size, Hkv, D]
    return picked.reshape((n_pages * page_size,) + picked.shape[2:])[:seq_len]


def decode_paged(q, k_pages, v_pages, block_table, seq_lens, page_size: int, scale: float,
                 seqs=None):
    """Single-token decode over a paged KV cache (dense, no skip).

    q [N, Hq, D]; k_pages/v_pages [P, page_size, Hkv, D]; block_table [N, max_pages]
    int; seq_lens [N] int. The new query sees all seq_len cached keys.
    Returns o [N, Hq, D] and lse [N, Hq] (float64); a sequence of length 0
    gives o = 0 and lse = -inf.
    """
    q = _f64(q)
    bt = np.asarray(block_table)
    lens = np.asarray(seq_lens)
    N, Hq, D = q.shape
    Hkv = k_pages.shape[2]
    o = np.full((N, Hq, D), np.nan)
    lse = np.full((N, Hq), np.nan)
    for b in (range(N) if seqs is None else seqs):
        L = int(lens[b])
        kb = gather_pages(k_pages, bt[b], L, page_size)
        vb = gather_pages(v_pages, bt[b], L, page_size)
        for hq in range(Hq):
            kv = kv_head_of(hq, Hq, Hkv)
            ob, lb = attention_rows(q[b, hq][None, :], kb[:, kv, :], vb[:, kv, :], scale)
            o[b, hq], lse[b, hq] = ob[0], lb[0]
    return o, lse


def kv_append(k_pages, v_pages, block_table, start_pos, k_new, v_new, page_size: int):
    """Write the keys and values of new tokens into the paged cache.

    The cache keeps the K/V of past tokens so that each new token only adds
    its own ("TensorRT-LLM：大模型推理优化利器", section 4 on the KV cache; "LLM推理
    优化技术综述", PART01), in fixed-size pages addressed through a block table
    ("TensorRT对Grouped Query Attention的支持进展", section 动态形状与KV Cache管理).
    Token t of sequence b goes to position p = start_pos[b] + t, that is to
    physical page block_table[b][p // page_size], slot p % page_size.

    k_pages/v_pages [P, page_size, Hkv, D]; k_new/v_new [N, T, Hkv, D]. Returns
    new (k_pages, v_pages) numpy arrays in the input dtype's values (copies;
    every other slot unchanged). Raises IndexError for a position past the
    table or a page outside the pool.
    """
    def host(x):
        return x.detach().cpu().float().numpy().copy() if hasattr(x, "detach") else np.array(x, copy=True)
    kp, vp, kn, vn = host(k_pages), host(v_pages), host(k_new), host(v_new)
    bt = np.asarray(block_table)
    starts = np.asarray(start_pos)
    N, T = kn.shape[0], kn.shape[1]
    for b in range(N):
        for t in range(T):
            pos = int(starts[b]) + t
            lp = pos // page_size
            if lp >= bt.shape[1]:
                raise IndexError(f"sequence {b}: position {pos} past the block table")
            page = int(bt[b, lp])
            if page < 0 or page >= kp.shape[0]:
                raise IndexError(f"sequence {b}: block_table entry {page} out of range")
            kp[page, pos % page_size] = kn[b, t]
            vp[page, pos % page_size] = vn[b, t]
    return kp, vp


def prefill_paged(q, k_pages, v_pages, block_table, seq_lens, page_size: int, scale: float,
                  seqs=None, heads=None):
    """Chunked (append) prefill over a paged KV cache.

    The GQA page ("TensorRT对Grouped Query Attention的支持进展", section
    与动态批处理协同) recommends chunked prefill and prefix caching for batches of
    mixed lengths; the integration page ("flash-attention与TensorRT-LLM集成")
    runs attention against a KV cache (flash_attn_with_kvcache). Neither spells
    out the masking; the plainest reading, used here: the queries are the Sq
    newest tokens of each sequence, whose keys and values are already in the
    cache, and query row i of sequence b sits at position L_b - Sq + i and sees
    the cached keys 0 .. L_b - Sq + i (causal, aligned at the end of the
    sequence; L_b = seq_lens[b] >= Sq).

    q [B, Sq, Hq, D]; k_pages/v_pages [P, page_size, Hkv, D]; block_table
    [B, max_pages]; seq_lens [B]. Returns o [B, Sq, Hq, D] and lse [B, Hq, Sq]
    (float64). ``seqs`` / ``heads`` (lists of b / hq) restrict the work to a
    sample; entries outside it are NaN.
    """
    q = _f64(q)
    bt = np.asarray(block_table)
    lens = np.asarray(seq_lens)
    B, Sq, Hq, D = q.shape
    Hkv = k_pages.shape[2]
    o = np.full((B, Sq, Hq, v_pages.shape[-1]), np.nan)
    lse = np.full((B, Hq, Sq), np.nan)
    for b in (range(B) if seqs is None else seqs):
        L = int(lens[b])
        if L < Sq:
            raise ValueError(f"sequence {b}: {L} cached tokens for {Sq} queries")
        kb = gather_pages(k_pages, bt[b], L, page_size)
        vb = gather_pages(v_pages, bt[b], L, page_size)
        vis = causal_visible(np.arange(Sq) + (L - Sq), L)
        for hq in (range(Hq) if heads is None else heads):
            kv = kv_head_of(hq, Hq, Hkv)
            ob, lb = attention_rows(q[b, :, hq, :], kb[:, kv, :], vb[:, kv, :], scale, vis)
            o[b, :, hq, :] = ob
            lse[b, hq, :] = lb
    return o, lse


def e4m3_to_float(codes):
    """Float64 values of FP8 E4M3 codes (uint8): 1 sign bit, 4 exponent bits with
    bias 7, 3 mantissa bits; exponent 0 holds the subnormals m/8 * 2^-6; no
    infinities, and S.1111.111 is NaN (so the largest finite value is 448)."""
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = (c & 0x7).astype(np.float64)
    val = np.where(e == 0, m / 8.0 * 2.0 ** -6, (1.0 + m / 8.0) * 2.0 ** (e - 7.0))
    val = sign * val
    return np.where((c & 0x7F) == 0x7F, np.nan, val)


def decode_paged_fp8(q, k_codes, v_codes, k_scale: float, v_scale: float, block_table, seq_lens,
                     page_size: int, scale: float, seqs=None):
    """Single-token decode over a paged cache stored as FP8 E4M3.

    The TensorRT-LLM page ("TensorRT-LLM：大模型推理优化利器", 量化) lists FP8
    among the low-precision formats for cutting memory and bandwidth, and the
    integration page ("flash-attention与TensorRT-LLM集成") stores in FP8. The
    scale convention is not given; the reading used: one scale per pool,
    K = k_scale * e4m3(k_codes) and V = v_scale * e4m3(v_codes). The oracle
    dequantises the codes it gathers and applies the dense decode.

    k_codes/v_codes [P, page_size, Hkv, D] uint8; other arguments as decode_paged.
    """
    k = e4m3_to_float(np.asarray(k_codes.cpu() if hasattr(k_codes, "cpu") else k_codes)) * float(k_scale)
    v = e4m3_to_float(np.asarray(v_codes.cpu() if hasattr(v_codes, "cpu") else v_codes)) * float(v_scale)
    return decode_paged(q, k, v, block_table, seq_lens, page_size, scale, seqs=seqs)


# ----------------------------------------------------------------------------
# BLASST walk
# ----------------------------------------------------------------------------

def blasst_walk(s, visible, tiles, lam: float):
    """Run the skip decisions of one decision unit.

    s [R, N] scaled scores of the unit's rows against the keys it may visit;
    visible bool [R, N]; tiles: list of key-index ranges (start, stop) in
    visiting order. Returns (kept bool [R, N], skipped list[bool] per tile,
    margin list[float] per tile). ``margin`` is the smallest
    |exp(r - m) - lam| over the rows where both r and m are finite (inf when
    no row has both), the distance of the decision from a tie.
    """
    R = s.shape[0]
    m = np.full(R, NEG_INF)
    kept = np.zeros_like(visible)
    skipped, margins = [], []
    for (c0, c1) in tiles:
        vis_t = visible[:, c0:c1]
        any_vis = vis_t.any(axis=1)
        r = np.where(any_vis, np.where(vis_t, s[:, c0:c1], NEG_INF).max(axis=1, initial=NEG_INF), NEG_INF)
        both = np.isfinite(r) & np.isfinite(m)
        ratio = np.exp(np.where(both, r - np.where(both, m, 0.0), 0.0))
        row_ok = np.where(~np.isfinite(r), True,
                          np.where(~np.isfinite(m), False, ratio < lam))
        skip = bool(lam > 0.0 and row_ok.all())
        margins.append(float(np.abs(ratio[both] - lam).min()) if both.any() else math.inf)
        skipped.append(skip)
        if not skip:
            m = np.maximum(m, r)
            kept[:, c0:c1] = vis_t
    return kept, skipped, margins


def _attention_kept(s, kept, v):
    """Exact formula restricted to the kept keys (scores already scaled)."""
    s = np.where(kept, s, NEG_INF)
    m = s.max(axis=1)
    p = np.exp(s - m[:, None])
    l = p.sum(axis=1)
    return (p @ v) / l[:, None], m + np.log(l)


def prefill_blasst(q, k, v, causal: bool, scale: float, lam: float, heads=None, q_tiles=None):
    """Prefill with the BLASST tile skip.

    Decision unit: (b, hq, q tile of 128 rows [128 qt, min(128 qt + 128, S))).
    Its tiles are the 64-key tiles t = 0, 1, ... in ascending order; causal
    units visit only tiles with 64 t <= last row of the q tile.
    Returns o [B,S,Hq,D], lse [B,Hq,S], skip [B,Hq,n_qt,n_kt] uint8
    (1 skipped, 0 kept, 2 not visited) and margin [B,Hq,n_qt,n_kt] float64
    (inf where not visited). ``heads``/``q_tiles`` restrict the work to a sample.
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, S, Hq, D = q.shape
    Hkv = k.shape[2]
    n_qt = -(-S // Q_TILE)
    n_kt = -(-S // KV_TILE)
    o = np.full((B, S, Hq, D), np.nan)
    lse = np.full((B, Hq, S), np.nan)
    skip = np.full((B, Hq, n_qt, n_kt), 2, dtype=np.uint8)
    margin = np.full((B, Hq, n_qt, n_kt), np.inf)
    if heads is None:
        heads = [(b, h) for b in range(B) for h in range(Hq)]
    for b, hq in heads:
        kv = kv_head_of(hq, Hq, Hkv)
        for qt in (range(n_qt) if q_tiles is None else q_tiles):
            rows = np.arange(qt * Q_TILE, min(qt * Q_TILE + Q_TILE, S))
            last = rows[-1]
            n_vis_tiles = (last // KV_TILE + 1) if causal else n_kt
            n_keys = min(n_vis_tiles * KV_TILE, S)
            s = (q[b, rows, hq, :] @ k[b, :n_keys, kv, :].T) * scale
            vis = causal_visible(rows, n_keys) if causal else np.ones((len(rows), n_keys), bool)
            tiles = [(t * KV_TILE, min(t * KV_TILE + KV_TILE, n_keys)) for t in range(n_vis_tiles)]
            kept, skipped, margins = blasst_walk(s, vis, tiles, lam)
            ob, lb = _attention_kept(s, kept, v[b, :n_keys, kv, :])
            o[b, rows, hq, :] = ob
            lse[b, hq, rows] = lb
            skip[b, hq, qt, :n_vis_tiles] = np.asarray(skipped, dtype=np.uint8)
            margin[b, hq, qt, :n_vis_tiles] = margins
    return o, lse, skip, margin


def decode_paged_blasst(q, k_pages, v_pages, block_table, seq_lens, page_size: int,
                        scale: float, lam: float, split_tokens: int,
                        rows_per_unit: str = "group", seqs=None):
    """Paged decode with the BLASST tile skip.

    Decision unit: (sequence, KV head, split). A split covers tokens
    [sp * split_tokens, min((sp + 1) * split_tokens, L)); its tiles are its
    64-token tiles in ascending order and its running maximum starts at -inf.
    The unit's rows are the G query heads that share the KV head
    (rows_per_unit="group") or each query head alone (rows_per_unit="head").
    Returns o [N,Hq,D], lse [N,Hq], skip and margin indexed
    [N, Hkv, max_tiles] with max_tiles = ceil(max_pages * page_size / 64)
    (for "head": [N, Hq, max_tiles]); skip is 1 skipped, 0 kept, 2 not visited.
    """
    if split_tokens % KV_TILE != 0 or split_tokens <= 0:
        raise ValueError("split_tokens must be a positive multiple of 64")
    q = _f64(q)
    bt = np.asarray(block_table)
    lens = np.asarray(seq_lens)
    N, Hq, D = q.shape
    Hkv = k_pages.shape[2]
    G = Hq // Hkv
    max_tiles = -(-bt.shape[1] * page_size // KV_TILE)
    n_units = Hkv if rows_per_unit == "group" else Hq
    o = np.full((N, Hq, D), np.nan)
    lse = np.full((N, Hq), np.nan)
    skip = np.full((N, n_units, max_tiles), 2, dtype=np.uint8)
    margin = np.full((N, n_units, max_tiles), np.inf)
    for b in (range(N) if seqs is None else seqs):
        L = int(lens[b])
        if L == 0:
            o[b], lse[b] = 0.0, NEG_INF
            continue
        kb = gather_pages(k_pages, bt[b], L, page_size)
        vb = gather_pages(v_pages, bt[b], L, page_size)
        for kv in range(Hkv):
            heads = list(range(kv * G, kv * G + G))
            groups = [heads] if rows_per_unit == "group" else [[h] for h in heads]
            for rows in groups:
                s = (q[b, rows, :] @ kb[:, kv, :].T) * scale           # [R, L]
                kept = np.zeros(s.shape, dtype=bool)
                unit = kv if rows_per_unit == "group" else rows[0]
                for sp0 in range(0, L, split_tokens):
                    sp1 = min(sp0 + split_tokens, L)
                    tiles = [(t, min(t + KV_TILE, sp1)) for t in range(sp0, sp1, KV_TILE)]
                    vis = np.zeros(s.shape, dtype=bool)
                    vis[:, sp0:sp1] = True
                    kept_sp, skipped, margins = blasst_walk(s, vis, tiles, lam)
                    kept |= kept_sp
                    t0 = sp0 // KV_TILE
                    skip[b, unit, t0:t0 + len(skipped)] = np.asarray(skipped, dtype=np.uint8)
                    margin[b, unit, t0:t0 + len(margins)] = margins
                ob, lb = _attention_kept(s, kept, vb[:, kv, :])
                o[b, rows, :] = ob
                lse[b, rows] = lb
    return o, lse, skip, margin


def prefill_with_skip_mask(q, k, v, causal: bool, scale: float, skip_mask, heads=None, q_tiles=None):
    """Prefill restricted to the tiles a given decision mask keeps.

    The same decision units and tiles as prefill_blasst, but the decisions are
    read from ``skip_mask`` [B, Hq, ceil(S/128), ceil(S/64)] (1 skipped, 0 kept,
    2 not visited) instead of being walked: every visible key of a tile whose
    entry is not 1 takes part in the exact formula. This evaluates a decision
    set that differs from the walk's own inside the tie band of a decision.
    Returns o [B,S,Hq,D], lse [B,Hq,S] (NaN outside the sample).
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    mask = np.asarray(skip_mask.cpu() if hasattr(skip_mask, "cpu") else skip_mask)
    B, S, Hq, D = q.shape
    Hkv = k.shape[2]
    n_qt = -(-S // Q_TILE)
    o = np.full((B, S, Hq, v.shape[-1]), np.nan)
    lse = np.full((B, Hq, S), np.nan)
    if heads is None:
        heads = [(b, h) for b in range(B) for h in range(Hq)]
    for b, hq in heads:
        kv = kv_head_of(hq, Hq, Hkv)
        for qt in (range(n_qt) if q_tiles is None else q_tiles):
            rows = np.arange(qt * Q_TILE, min(qt * Q_TILE + Q_TILE, S))
            vis = causal_visible(rows, S) if causal else np.ones((len(rows), S), bool)
            key_tile = np.arange(S) // KV_TILE
            kept = vis & (mask[b, hq, qt, key_tile] != 1)[None, :]
            ob, lb = attention_rows(q[b, rows, hq, :], k[b, :, kv, :], v[b, :, kv, :], scale, kept)
            o[b, rows, hq, :] = ob
            lse[b, hq, rows] = lb
    return o, lse


def decode_paged_with_skip_mask(q, k_pages, v_pages, block_table, seq_lens, page_size: int, scale: float,
                                skip_mask, rows_per_unit: str = "group", seqs=None):
    """Paged decode restricted to the tiles a given decision mask keeps.

    ``skip_mask`` [N, Hkv, max_tiles] (rows_per_unit="group") or [N, Hq,
    max_tiles] ("head"), 1 skipped / 0 kept / 2 not visited, as returned by
    decode_paged_blasst: each query head attends to the tokens of the 64-token
    tiles its unit keeps. Returns o [N,Hq,D], lse [N,Hq].
    """
    q = _f64(q)
    mask = np.asarray(skip_mask.cpu() if hasattr(skip_mask, "cpu") else skip_mask)
    bt = np.asarray(block_table)
    lens = np.asarray(seq_lens)
    N, Hq, D = q.shape
    Hkv = k_pages.shape[2]
    o = np.full((N, Hq, D), np.nan)
    lse = np.full((N, Hq), np.nan)
    for b in (range(N) if seqs is None else seqs):
        L = int(lens[b])
        if L == 0:
            o[b], lse[b] = 0.0, NEG_INF
            continue
        kb = gather_pages(k_pages, bt[b], L, page_size)
        vb = gather_pages(v_pages, bt[b], L, page_size)
        tile = np.arange(L) // KV_TILE
        for hq in range(Hq):
            kv = kv_head_of(hq, Hq, Hkv)
            unit = kv if rows_per_unit == "group" else hq
            kept = (mask[b, unit, tile] != 1)[None, :]
            ob, lb = attention_rows(q[b, hq][None, :], kb[:, kv, :], vb[:, kv, :], scale, kept)
            o[b, hq], lse[b, hq] = ob[0], lb[0]
    return o, lse
