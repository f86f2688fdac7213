"""The split-KV work list, restated in Python from TileSplit and pool_tiles in
csrc/common.cuh (device arithmetic mirrored: 32-bit unsigned products when they
fit, else 64-bit), and the properties the split kernels and the combine rely on.
CPU only.

  - the batch's NT tiles are cut into NS static tiles and a tail pool [NS, NT)
    (the last grid * pool_per_cta tiles when there are at least 4 tiles per CTA);
  - every static tile belongs to exactly one CTA, and cta_of inverts first;
  - every partial slot the combine reads for sequence b -- static slots cta + b for
    the CTAs from cta_of(first static tile of b) to cta_of(last static tile of b),
    then pool slots grid + B + (v - NS) for b's pool tiles v -- is written by
    exactly one piece, and every slot index is below grid * (1 + pool_per_cta) + B
    (the workspace's slot count);
  - a grid sized from an upper bound of the tokens can exceed the batch's tiles: the
    split then uses the first NS CTAs, and an equal cut over all CTAs would leave
    tile-less CTAs inside a sequence's run of slots (checked to fail below);
  - with NS >= grid the static split is the plain equal cut floor(i * NS / grid).
"""
import random

import pytest

M32 = 0xFFFFFFFF
POOL_MIN_TILES_PER_CTA = 4


def pool_tiles(NT, grid, per_cta):
    if per_cta <= 0 or NT < POOL_MIN_TILES_PER_CTA * grid:
        return 0
    return min(per_cta * grid, NT)


def used(NS, grid):
    return grid if grid < NS else (NS if NS > 0 else 1)


def narrow(NS, g):
    return NS <= 0x7FFFFFFF // g


def first(i, NS, grid):
    g = used(NS, grid)
    i = min(i, g)
    return ((i * NS) & M32) // g if narrow(NS, g) else i * NS // g


def cta_of(u, NS, grid):
    g = used(NS, grid)
    return (((u + 1) * g - 1) & M32) // NS if narrow(NS, g) else ((u + 1) * g - 1) // NS


def slots(b, t0, t1, B, NS, grid, cta_of_fn=cta_of):
    """TileSplit::slots: (first static slot, static count, first pool slot, pool count)."""
    sf = sc = pf = pc = 0
    s1 = min(t1, NS)
    if t0 < s1:
        f, l = cta_of_fn(t0, NS, grid), cta_of_fn(s1 - 1, NS, grid)
        sf, sc = f + b, l - f + 1
    u0 = max(t0, NS)
    if u0 < t1:
        pf, pc = grid + B + (u0 - NS), t1 - u0
    return sf, sc, pf, pc


def tile_prefix(lengths, tt):
    tp = [0]
    for L in lengths:
        tp.append(tp[-1] + (L + tt - 1) // tt)
    return tp


def check_split(lengths, grid, tt, pool_per_cta=1, first_fn=first, cta_of_fn=cta_of):
    tp = tile_prefix(lengths, tt)
    NT, B = tp[-1], len(lengths)
    NS = NT - pool_tiles(NT, grid, pool_per_cta)
    owner = [None] * NT
    written = {}
    for i in range(grid):
        t0, t1 = first_fn(i, NS, grid), first_fn(i + 1, NS, grid)
        assert 0 <= t0 <= t1 <= NS
        for u in range(t0, t1):
            assert owner[u] is None
            owner[u] = i
            assert cta_of_fn(u, NS, grid) == i
        for b in range(B):
            if max(t0, tp[b]) < min(t1, tp[b + 1]):
                written[i + b] = written.get(i + b, 0) + 1
    for v in range(NS, NT):                     # pool tiles: one piece each
        assert owner[v] is None
        owner[v] = "pool"
        s = grid + B + (v - NS)
        written[s] = written.get(s, 0) + 1
    assert None not in owner
    assert all(n == 1 for n in written.values())
    n_slots = grid * (1 + pool_per_cta) + B
    assert all(0 <= s < n_slots for s in written)
    read = set()
    for b in range(B):
        if tp[b + 1] == tp[b]:
            continue
        sf, sc, pf, pc = slots(b, tp[b], tp[b + 1], B, NS, grid, cta_of_fn)
        assert sc + pc >= 1
        for s in list(range(sf, sf + sc)) + list(range(pf, pf + pc)):
            assert written.get(s) == 1, f"slot {s} of sequence {b} is not written"
            assert s not in read
            read.add(s)
    assert read == set(written), "a written slot is read by no sequence"


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


@pytest.mark.parametrize("pool_per_cta", [0, 1, 2])
@pytest.mark.parametrize("seed", range(4))
def test_split_invariants(seed, pool_per_cta):
    for lengths, grid, tt in batches(seed, 150):
        check_split(lengths, grid, tt, pool_per_cta)


def launched_grids(max_total_tokens, tt, num_sms=148):
    """The grids mma_grid, tc_decode_grid and simt_grid launch on a 148-SM B200:
    num_sms x (1..4 CTAs per SM), capped at the tiles of the token bound."""
    want = max(1, -(-max_total_tokens // tt))
    return sorted({min(num_sms * per_sm, want) for per_sm in (1, 2, 3, 4)})


@pytest.mark.parametrize("L,B", [(1, 1), (33, 8), (4096, 8), (4097, 8), (32768, 4), (32769, 4),
                                 (131072, 1), (131073, 1), (8704, 64)])
def test_split_invariants_benchmark_shapes(L, B):
    for tt in (16, 32, 64):
        for bound in (L * B, L * B + B, 300000):        # exact, plus the step's tokens, a loose bound
            for grid in launched_grids(bound, tt):
                for pool in (0, 1):
                    check_split([L] * B, grid, tt, pool)


def test_ragged_benchmark_batch():
    """The ragged serving batch's lengths (64 draws from U{1024..16384})."""
    import numpy as np
    rng = np.random.default_rng(0)
    lengths = [int(x) + 1 for x in rng.integers(1024, 16384, size=64, endpoint=True)]
    for grid in launched_grids(sum(lengths), 32):
        check_split(lengths, grid, 32, 1)


def test_pool_only_with_enough_tiles():
    assert pool_tiles(4 * 296 - 1, 296, 1) == 0
    assert pool_tiles(4 * 296, 296, 1) == 296
    assert pool_tiles(4100, 296, 1) == 296
    assert pool_tiles(10 ** 6, 296, 0) == 0


def test_equal_cut_when_tiles_outnumber_ctas():
    for lengths, grid, tt in batches(7, 200):
        NT = tile_prefix(lengths, tt)[-1]
        NS = NT - pool_tiles(NT, grid, 1)
        if NS < grid:
            continue
        for i in range(grid + 1):
            assert first(i, NS, grid) == i * NS // grid


def test_cut_over_all_ctas_fails_with_few_tiles():
    """The equal cut over every launched CTA leaves unwritten slots inside a run."""
    def first_all(i, NS, grid):
        return i * NS // grid

    def cta_of_all(u, NS, grid):
        return ((u + 1) * grid - 1) // NS

    with pytest.raises(AssertionError):
        check_split([5, 40, 100, 0, 1], 296, 32, 1, first_all, cta_of_all)
