"""The split-KV work list, restated in Python from TileSplit in csrc/common.cuh
(device arithmetic mirrored: 32-bit unsigned products when they fit, else 64-bit),
and the properties the split kernels and the combine rely on.  CPU only.

  - every tile of the batch belongs to exactly one CTA, and cta_of inverts first;
  - every partial slot cta + b that the combine reads for sequence b (the CTAs from
    cta_of(first tile of b) to cta_of(last tile of b)) is written by exactly one CTA,
    and every slot index is below grid + B (the workspace's slot count);
  - a grid sized from an upper bound of the tokens can exceed the batch's tiles: the
    split then uses the first NT CTAs, and an equal cut over all CTAs would leave
    tile-less CTAs inside a sequence's run of slots (checked to fail below);
  - with NT >= grid the split is the plain equal cut floor(i * NT / grid).
"""
import random

import pytest

M32 = 0xFFFFFFFF


def used(NT, grid):
    return grid if grid < NT else (NT if NT > 0 else 1)


def narrow(NT, g):
    return NT <= 0x7FFFFFFF // g


def first(i, NT, grid):
    g = used(NT, grid)
    i = min(i, g)
    return ((i * NT) & M32) // g if narrow(NT, g) else i * NT // g


def cta_of(u, NT, grid):
    g = used(NT, grid)
    return (((u + 1) * g - 1) & M32) // NT if narrow(NT, g) else ((u + 1) * g - 1) // NT


def tile_prefix(lengths, tt):
    tp = [0]
    for L in lengths:
        tp.append(tp[-1] + (L + tt - 1) // tt)
    return tp


def check_split(lengths, grid, tt, first_fn=first, cta_of_fn=cta_of):
    tp = tile_prefix(lengths, tt)
    NT, B = tp[-1], len(lengths)
    owner = [None] * NT
    written = {}
    for i in range(grid):
        t0, t1 = first_fn(i, NT, grid), first_fn(i + 1, NT, grid)
        assert 0 <= t0 <= t1 <= NT
        for u in range(t0, t1):
            assert owner[u] is None
            owner[u] = i
            assert cta_of_fn(u, NT, grid) == i
        for b in range(B):
            if max(t0, tp[b]) < min(t1, tp[b + 1]):
                written[i + b] = written.get(i + b, 0) + 1
    assert None not in owner
    assert all(n == 1 for n in written.values())
    assert all(s < grid + B for s in written)
    for b in range(B):
        if tp[b + 1] == tp[b]:
            continue
        lo, hi = cta_of_fn(tp[b], NT, grid), cta_of_fn(tp[b + 1] - 1, NT, grid)
        for i in range(lo, hi + 1):
            assert written.get(i + b) == 1, f"slot {i + b} of sequence {b} is not written"


def batches(seed, n):
    rng = random.Random(seed)
    for _ in range(n):
        B = rng.randint(1, 70)
        grid = rng.choice([1, 2, 7, 148, 296, 444, 592])
        tt = rng.choice([16, 32, 64])
        mode = rng.random()
        if mode < 0.4:
            lengths = [rng.randint(0, 60) for _ in range(B)]              # fewer tiles than CTAs
        elif mode < 0.7:
            lengths = [rng.choice([0, 1, rng.randint(1, 40000)]) for _ in range(B)]
        else:
            lengths = [rng.randint(1000, 17000) for _ in range(B)]
        yield lengths, grid, tt


@pytest.mark.parametrize("seed", range(4))
def test_split_invariants(seed):
    for lengths, grid, tt in batches(seed, 150):
        check_split(lengths, grid, tt)


@pytest.mark.parametrize("L,B", [(1, 1), (33, 8), (4096, 8), (4097, 8), (32768, 4), (131072, 1)])
def test_split_invariants_benchmark_shapes(L, B):
    for grid in (148, 296):
        check_split([L] * B, grid, 32)
        check_split([L] * B, grid, 16)


def test_equal_cut_when_tiles_outnumber_ctas():
    for lengths, grid, tt in batches(7, 200):
        NT = tile_prefix(lengths, tt)[-1]
        if NT < grid:
            continue
        for i in range(grid + 1):
            assert first(i, NT, grid) == i * NT // grid


def test_cut_over_all_ctas_fails_with_few_tiles():
    """The equal cut over every launched CTA leaves unwritten slots inside a run."""
    def first_all(i, NT, grid):
        return i * NT // grid

    def cta_of_all(u, NT, grid):
        return ((u + 1) * grid - 1) // NT

    with pytest.raises(AssertionError):
        check_split([5, 40, 100, 0, 1], 296, 32, first_all, cta_of_all)
