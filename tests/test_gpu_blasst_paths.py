"""Tile-skip paths on the GPU against the float64 oracle: the one-pass and the
two-pass decode over every head layout they serve (and the per-KV-head kernel
kept for 16 query heads per KV head), the skipped-decision counters, and the
library's status word being opt-in."""

import numpy as np
import pytest
import torch

import attention_online_softmax_fwd_b200 as ab
from attention_online_softmax_fwd_b200 import inputs as gen
from oracle import attn_oracle as orc
from parity_util import compare_blasst

pytestmark = pytest.mark.gpu

LENS = [0, 2049, 1, 63, 64, 65, 700, 1300]   # ragged, one empty sequence
ONE_PASS_MIN = 2048   # (sequence, KV head, split) triples from which the skip decode makes one pass over K


def _cache(Hq, Hkv, D, ps, seed, lens=LENS, max_pages=None):
    """Ragged sequences of N(0, 1) K/V; the queries are scaled by 3 so that scores
    spread and later tiles fall below their split's running maximum."""
    c = gen.paged_decode_inputs(len(lens), Hq, Hkv, D, ps, 0, 0, seed=seed, lens=lens, max_pages=max_pages)
    c.q = (c.q.float() * 3.0).to(torch.bfloat16)
    return c


def _widen(c, max_pages):
    """The same cache with a wider block table (unused entries -1): more splits per sequence."""
    n, mp = c.block_table.shape
    if max_pages > mp:
        c.block_table = torch.cat([c.block_table, torch.full((n, max_pages - mp), -1, dtype=torch.int32)], 1)
    return c


def _splits(max_pages, ps, split):
    return -(-max_pages * ps // split)


def _layout(passes, Hkv, ps, split, G=1):
    """Sequences and block-table width that put the skip decode on the requested path:
    one pass once the batch has ONE_PASS_MIN (sequence, KV head, split) triples (a wider
    table adds empty splits), two passes below (fewer sequences where needed). Sixteen
    query heads per KV head have the one-pass path only."""
    lens = list(LENS)
    mp = -(-max(lens) // ps)
    if G == 16:
        return lens, mp
    if passes == 1:
        need = -(-ONE_PASS_MIN // (len(lens) * Hkv))
        return lens, max(mp, -(-need * split // ps))
    while len(lens) * Hkv * _splits(mp, ps, split) >= ONE_PASS_MIN:
        lens = lens[:-1]
    return lens, mp


def _run(c, dev, lam, split, rows):
    args = [t.to(dev) for t in (c.q, c.k_pages, c.v_pages, c.block_table, c.seq_lens)]
    counter = torch.zeros(1, dtype=torch.int64, device=dev)
    scale = gen.attn_scale(c.q.shape[-1])
    o, lse, mask = ab.decode_paged_blasst(*args, lam, scale=scale, split_tokens=split, rows_per_unit=rows,
                                          skipped_tiles=counter)
    torch.cuda.synchronize()
    return o, lse, mask, int(counter.item()), scale


def _passes(c, split):
    N, Hq, _ = c.q.shape
    _, ps, Hkv, _ = c.k_pages.shape
    return ab.binding.decode_skip_passes(N, Hq, Hkv, c.block_table.shape[1], ps, split)


# (Hq, Hkv, D, page size): G = 1, 2, 4, 8 with even and odd numbers of KV heads (one- and
# two-head groups in one pass; groups of 4 KV heads, or single KV heads, in two); G = 16
# on the one-pass per-KV-head kernel
SHAPES = [(8, 2, 128, 16), (32, 8, 64, 64), (8, 8, 128, 256), (64, 8, 128, 16), (24, 12, 128, 64),
          (16, 8, 64, 16), (12, 3, 128, 16), (16, 1, 128, 16)]
CASES = [(shape, passes) for shape in SHAPES for passes in (1, 2) if not (shape[0] // shape[1] == 16 and passes == 2)]


@pytest.mark.parametrize("shape,passes", CASES, ids=[f"{s[0]}x{s[1]}-d{s[2]}-p{s[3]}-{n}pass" for s, n in CASES])
@pytest.mark.parametrize("split", [64, 320, 2048])
@pytest.mark.parametrize("rows", ["group", "head"])
def test_decode_blasst_layouts(cuda_device, shape, passes, split, rows):
    Hq, Hkv, D, ps = shape
    lens, mp = _layout(passes, Hkv, ps, split, G=Hq // Hkv)
    c = _cache(Hq, Hkv, D, ps, seed=5000 + Hq + D + ps, lens=lens, max_pages=mp)
    assert _passes(c, split) == passes
    o, lse, mask, counted, scale = _run(c, cuda_device, 0.5, split, rows)
    o_ref, lse_ref, m_ref, margin = orc.decode_paged_blasst(c.q, c.k_pages, c.v_pages, c.block_table, c.seq_lens,
                                                            ps, scale, 0.5, split, rows_per_unit=rows)

    def with_mask(m):
        return orc.decode_paged_with_skip_mask(c.q, c.k_pages, c.v_pages, c.block_table, c.seq_lens, ps, scale,
                                               m, rows_per_unit=rows)

    st = compare_blasst(o, lse, mask, o_ref, lse_ref, m_ref, margin, with_mask,
                        label=f"Hq={Hq} Hkv={Hkv} D={D} ps={ps} split={split} {rows} {passes} pass")
    assert counted == st["skipped_gpu"], "the counter adds one per skipped decision"
    if split > 64:
        assert st["skipped"] > 0


@pytest.mark.parametrize("passes", [1, 2])
def test_decode_blasst_lambda_zero_keeps_everything(cuda_device, passes):
    lens, mp = _layout(passes, 8, 16, 320)
    c = _cache(32, 8, 128, 16, seed=5100, lens=lens, max_pages=mp)
    assert _passes(c, 320) == passes
    o, lse, mask, counted, scale = _run(c, cuda_device, 0.0, 320, "group")
    o_ref, lse_ref = orc.decode_paged(c.q, c.k_pages, c.v_pages, c.block_table, c.seq_lens, 16, scale)
    o_ref[0], lse_ref[0] = 0.0, -np.inf
    assert counted == 0 and not (mask == 1).any()
    from parity_util import compare_output
    compare_output(o, o_ref, lse, lse_ref, label=f"lambda 0, {passes} pass")


@pytest.mark.parametrize("passes", [1, 2])
def test_decode_blasst_repeatable(cuda_device, passes):
    lens, mp = _layout(passes, 8, 16, 2048)
    c = _cache(32, 8, 128, 16, seed=5200, lens=lens, max_pages=mp)
    assert _passes(c, 2048) == passes
    a = _run(c, cuda_device, 0.5, 2048, "group")
    b = _run(c, cuda_device, 0.5, 2048, "group")
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1]) and torch.equal(a[2], b[2]) and a[3] == b[3]


def test_prefill_skipped_counter(cuda_device):
    q, k, v = gen.peaked_prefill_inputs(1, 4, 2, 1100, 128, seed=3200, amp=8.0, period=1 << 30)
    dev = cuda_device
    counter = torch.zeros(1, dtype=torch.int64, device=dev)
    o, lse, mask = ab.prefill_blasst(q.to(dev), k.to(dev), v.to(dev), 0.3, causal=True,
                                     scale=gen.attn_scale(128), skipped_tiles=counter)
    torch.cuda.synchronize()
    assert int(counter.item()) == int((mask == 1).sum().item()) > 0


def test_library_status_word_is_opt_in(cuda_device):
    c = gen.paged_decode_inputs(4, 8, 2, 128, 16, 100, 300, seed=5300)
    c.block_table[1, 2] = c.num_pages + 5      # out of range: never dereferenced, reported
    args = [t.to(cuda_device) for t in (c.q, c.k_pages, c.v_pages, c.block_table, c.seq_lens)]
    status = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    ab.binding.set_library_status(False)
    ab.binding.read_device_status(clear=True)
    ab.decode_paged(*args, split_tokens=64, device_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 4                               # the caller's own word
    assert ab.binding.read_device_status(clear=True) == 0        # the library's stays untouched
    ab.binding.set_library_status(True)
    try:
        ab.decode_paged(*args, split_tokens=64)
        assert ab.binding.read_device_status(clear=True) == 4
    finally:
        ab.binding.set_library_status(False)


@pytest.mark.parametrize("split,passes", [(2048, 2), (256, 1), (4096, 2)])
def test_decode_blasst_dominant_key_batch(cuda_device, split, passes):
    """A batch with one dominant key per sequence (the bench's bandwidth-bound skip
    workload, at reduced size): group and per-head decisions against the oracle, on
    either path, and with one split per sequence."""
    c = gen.peaked_decode_batch(3, 32, 8, 4096, 128, seed=5400, amp=12.0, page_size=16)
    if passes == 1:
        _widen(c, -(-ONE_PASS_MIN // (3 * 8)) * split // 16)
    assert _passes(c, split) == passes
    for rows in ("group", "head"):
        o, lse, mask, counted, scale = _run(c, cuda_device, 0.3, split, rows)
        o_ref, lse_ref, m_ref, margin = orc.decode_paged_blasst(c.q, c.k_pages, c.v_pages, c.block_table,
                                                                c.seq_lens, 16, scale, 0.3, split, rows_per_unit=rows)
        st = compare_blasst(o, lse, mask, o_ref, lse_ref, m_ref, margin,
                            lambda m: orc.decode_paged_with_skip_mask(c.q, c.k_pages, c.v_pages, c.block_table,
                                                                      c.seq_lens, 16, scale, m, rows_per_unit=rows),
                            label=f"dominant batch {rows} split {split}")
        assert st["skipped"] > 0 and counted == st["skipped_gpu"]


@pytest.mark.parametrize("passes", [1, 2])
@pytest.mark.parametrize("rows", ["group", "head"])
def test_decode_blasst_bad_page_raises_device_status(cuda_device, passes, rows):
    """Out-of-range block-table entries on either skip path are never dereferenced:
    the caller's status word reads ATTN_ERR_DEVICE_BOUNDS and the sequences whose
    tables are valid match the oracle."""
    lens = [300, 700, 1300, 2049]
    split = 256
    mp = -(-max(lens) // 16)
    if passes == 1:
        mp = max(mp, -(-ONE_PASS_MIN // (len(lens) * 2)) * split // 16)
    c = _cache(8, 2, 128, 16, seed=5500, lens=lens, max_pages=mp)
    c.block_table[1, 3] = c.num_pages + 5
    c.block_table[2, 0] = -7
    assert _passes(c, split) == passes
    args = [t.to(cuda_device) for t in (c.q, c.k_pages, c.v_pages, c.block_table, c.seq_lens)]
    status = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    scale = gen.attn_scale(128)
    o, lse, mask = ab.decode_paged_blasst(*args, 0.5, scale=scale, split_tokens=split, rows_per_unit=rows,
                                          device_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 4                        # ATTN_ERR_DEVICE_BOUNDS
    good = [0, 3]
    o_ref, lse_ref, m_ref, margin = orc.decode_paged_blasst(c.q, c.k_pages, c.v_pages, c.block_table, c.seq_lens,
                                                            16, scale, 0.5, split, rows_per_unit=rows, seqs=good)
    m_ref = m_ref[good]
    st = compare_blasst(o, lse, mask[good], o_ref, lse_ref, m_ref, margin[good],
                        lambda m: orc.decode_paged_with_skip_mask(c.q, c.k_pages, c.v_pages, c.block_table,
                                                                  c.seq_lens, 16, scale, _full_mask(m, mask, good),
                                                                  rows_per_unit=rows, seqs=good),
                        label=f"bad pages, {passes} pass, {rows}", select=lambda oo, ll: (oo[good], ll[good]))
    assert st["decisions"] > 0


def _full_mask(m_good, mask_gpu, good):
    """The GPU's mask with the rows of the checked sequences replaced by ``m_good``."""
    full = mask_gpu.cpu().numpy().copy()
    full[good] = m_good
    return full
