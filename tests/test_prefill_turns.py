"""Host model of the prefill kernel's MUFU turns (prefill.cuh; dense, paged and tile-skip kernels).

The two softmax warpgroups of a CTA (query tiles A and B of each 256-row block) take
turns for their exponentials on the K/V tiles both visit: tile A's exponentials of
common tile j follow tile B's of the previous common tile, and tile B's follow tile A's
of tile j. The hand-over runs through two mbarriers whose waits test a phase parity.
This model walks both groups over a CTA's items, in the kernel's item order (snake over
the grid, or cost-ranked pairs for the paged kernel), with the kernel's tile counts, and
checks, for every schedule the two groups can take:
  * no group waits for an arrival that never comes (every wait is eventually released);
  * when a group waits, the barrier has completed at most one phase it has not yet
    waited for, so a parity test can never mistake a later phase for the awaited one.
It needs no GPU and runs the model on the shapes of the GPU tests and the benchmarks.
"""

import random

import pytest

ROWS = 128   # rows per query tile
KEYS = 128   # keys per K/V tile
BLOCK = 256  # rows per work item (two query tiles)


def tile_rows(S, qb, x):
    return max(0, min(ROWS, S - qb * BLOCK - x * ROWS))


def tile_nkv(S, qb, x, rows, off, causal):
    if rows == 0:
        return 0
    if causal:
        return (off + qb * BLOCK + x * ROWS + rows - 1) // KEYS + 1
    return (S + KEYS - 1) // KEYS


def items_of_cta(n_items, grid, cta, snake=True):
    """Round r takes item r * grid + b, with b reversed on odd rounds (the snake)."""
    out, r = [], 0
    while True:
        b = grid - 1 - cta if (snake and r & 1) else cta
        item = r * grid + b
        if item >= n_items:
            return out
        out.append(item)
        r += 1


def common_counts(items, coords, S, offs, causal):
    """Per item: the number of K/V tiles both query tiles visit (0 when tile B has no rows)."""
    out = []
    for it in items:
        qb, b = coords(it)
        off = offs[b]
        n0 = tile_nkv(S, qb, 0, tile_rows(S, qb, 0), off, causal)
        n1 = tile_nkv(S, qb, 1, tile_rows(S, qb, 1), off, causal)
        out.append(min(n0, n1))
    return out


def run_turns(commons, rng):
    """Both groups walk the same common-tile counts; a random scheduler picks which group
    moves. Returns the number of turns taken per group; raises on a stuck wait or a
    parity alias."""
    total = sum(commons)
    arrivals = [0, 0]   # arrivals[x]: phases completed on the barrier group x waits on
    waited = [0, 0]     # phases group x has waited for
    done = [0, 0]       # common tiles whose exponentials group x has finished
    started_a = False
    steps = 0
    while done[0] < total or done[1] < total:
        movable = []
        for x in (0, 1):
            if done[x] == total:
                continue
            needs_wait = x == 1 or (x == 0 and (started_a or done[0] > 0))
            if not needs_wait or arrivals[x] > waited[x]:
                movable.append(x)
        if not movable:
            raise AssertionError(f"both groups wait forever after {done} of {total} common tiles")
        x = rng.choice(movable)
        needs_wait = x == 1 or (x == 0 and (started_a or done[0] > 0))
        if needs_wait:
            # a parity test is sound only if the barrier is at most one phase ahead
            assert arrivals[x] - waited[x] <= 1, "a barrier ran two phases ahead of its waiter"
            waited[x] += 1
        if x == 0:
            started_a = True
        done[x] += 1
        arrivals[1 - x] += 1   # hand the turn to the other group
        steps += 1
    # tile A waits once less than tile B arrives (its first common tile waits for nobody)
    assert waited[0] == total - 1 if total else waited[0] == 0
    assert waited[1] == total
    return steps


CASES = [
    # (B, Hq, S, causal, prefix lengths of the paged chunk or None)
    (2, 8, 700, True, None), (1, 4, 300, True, None), (1, 8, 513, True, None), (1, 2, 1, True, None),
    (1, 2, 129, True, None), (2, 4, 255, True, None), (1, 4, 257, True, None), (1, 2, 1024, False, None),
    (2, 8, 700, False, None), (4, 32, 2048, True, None), (2, 32, 8192, True, None),
    (3, 8, 100, True, [0, 257, 900]), (2, 4, 300, True, [0, 477]), (1, 8, 1, True, [612]),
    (2, 16, 513, True, [0, 1536]), (4, 8, 17, True, [0, 1, 128, 383]),
    (4, 32, 2048, True, [0, 2048, 4096, 6144]),
]


@pytest.mark.parametrize("B,Hq,S,causal,prefix", CASES)
def test_turns_never_stall_or_alias(B, Hq, S, causal, prefix):
    n_qblocks = (S + BLOCK - 1) // BLOCK
    n_items = n_qblocks * B * Hq
    grid = min(n_items, 148)
    offs = prefix if prefix is not None else [0] * B
    if prefix is not None:
        # paged: (sequence, query block) pairs ranked by both tiles' K/V tile counts, most first
        pairs = list(range(B * n_qblocks))

        def cost(i):
            b, qb = divmod(i, n_qblocks)
            return sum(tile_nkv(S, qb, x, tile_rows(S, qb, x), offs[b], causal) for x in (0, 1))

        order = sorted(pairs, key=lambda i: (-cost(i), i))

        def coords(it):
            b, qb = divmod(order[it // Hq], n_qblocks)
            return qb, b
    else:
        def coords(it):
            per = B * Hq
            return n_qblocks - 1 - it // per, (it % per) // Hq
    rng = random.Random(1234 + S + B)
    for cta in range(grid):
        commons = common_counts(items_of_cta(n_items, grid, cta), coords, S, offs, causal)
        for _ in range(3):
            run_turns(commons, rng)


def test_model_detects_a_missing_arrival():
    """The model is not vacuous: a protocol in which tile A also waits before its first
    common tile stalls at once."""
    rng = random.Random(7)
    commons = [3, 2]
    total = sum(commons)
    arrivals, waited, done = [0, 0], [0, 0], [0, 0]
    with pytest.raises(AssertionError):
        while done[0] < total or done[1] < total:
            movable = [x for x in (0, 1) if done[x] < total and arrivals[x] > waited[x]]
            if not movable:
                raise AssertionError("stall")
            x = rng.choice(movable)
            waited[x] += 1
            done[x] += 1
            arrivals[1 - x] += 1
