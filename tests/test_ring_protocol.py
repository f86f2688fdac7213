"""The stage-ring protocol of the tensor-core split kernel (csrc/decode_mma.cuh),
restated as a small model and run over random schedules.  CPU only.

One producer thread arms tiles 0, 1, ... of a CTA's range in order; tile k lands
in stage k % S.  Before its PDL wait it arms the first `prefetch` tiles (at most S)
with no check; after it, it arms tile k (k >= depth) only once tile k - depth has
been released by its owning warp of every group.  Each value group has W consumer
warps, warp w taking tiles w, w + W, ...; a warp consumes its tiles in order, each
only after it has been armed.  The invariant the kernel needs: when tile k is
armed, tile k - S, the previous occupant of the same stage, has been released
(otherwise the new copy could be armed on a barrier whose previous copy is still
landing).

The kernel uses depth = S - 1 for short ranges only with one warp per group, and
depth = S otherwise.  The model shows why: with W = 1 releases come in tile order,
so the release of k - depth implies that of k - S.  With W = 2 the first tile armed
after a full-ring prefetch, tile S, checks only tile 1 (the other warp's), while
tile 0 may still be held; without the prefetch the check of tile k - 1 - depth =
k - S at the previous step would have covered it.
"""
import random

import pytest


def kernel_depth(S, W, range_tiles, short_range_tiles=16):
    """The producer's depth rule of the split kernel."""
    if W == 1 and S >= 4 and range_tiles <= short_range_tiles:
        return S - 1
    return S


def run_schedule(n, S, W, groups, depth, rng, prefetch=0):
    """One random interleaving; returns the first violation (k, k - S) or None."""
    armed = min(prefetch, S, n)                 # tiles armed before the wait, unchecked
    nxt = [[w for w in range(W)] for _ in range(groups)]   # next tile of each warp
    released = [[False] * n for _ in range(groups)]
    done = lambda: armed == n and all(nxt[g][w] >= n for g in range(groups) for w in range(W))
    while not done():
        actors = []
        if armed < n:
            k = armed
            if k < depth or all(released[g][k - depth] for g in range(groups)):
                actors.append(("p", None, None))
        for g in range(groups):
            for w in range(W):
                t = nxt[g][w]
                if t < n and t < armed:
                    actors.append(("c", g, w))
        assert actors, "deadlock"
        kind, g, w = rng.choice(actors)
        if kind == "p":
            k = armed
            if k >= S and not all(released[gg][k - S] for gg in range(groups)):
                return (k, k - S)
            armed += 1
        else:
            released[g][nxt[g][w]] = True
            nxt[g][w] += W
    return None


@pytest.mark.parametrize("prefetch", [0, 2, 99], ids=["no-prefetch", "partial", "full-ring"])
@pytest.mark.parametrize("S,W,n", [(5, 1, 14), (5, 1, 4), (4, 1, 16), (6, 1, 40), (4, 2, 14),
                                   (6, 2, 30), (4, 2, 4), (6, 3, 18)])
def test_kernel_depth_rule_never_rearms_a_busy_stage(S, W, n, prefetch):
    rng = random.Random(S * 1000 + W * 100 + n + prefetch)
    depth = kernel_depth(S, W, n)
    for _ in range(300):
        assert run_schedule(n, S, W, 4, depth, rng, prefetch) is None


def test_one_stage_fewer_is_unsafe_with_two_warps_after_a_full_prefetch():
    """The counterexample behind the kernel's rule: with two warps per group, a
    full-ring prefetch and one stage fewer in flight, some schedule re-arms a
    stage whose tile is unreleased."""
    rng = random.Random(7)
    S, W, n = 4, 2, 14
    hits = [run_schedule(n, S, W, 4, S - 1, rng, prefetch=S) for _ in range(300)]
    assert any(h is not None for h in hits)


def test_one_stage_fewer_is_safe_with_one_warp_per_group():
    rng = random.Random(11)
    for S in (4, 5, 6):
        for prefetch in (0, S):
            for _ in range(300):
                assert run_schedule(14, S, 1, 4, S - 1, rng, prefetch) is None


def test_one_stage_fewer_without_prefetch_is_safe_for_any_warp_count():
    """Without the unchecked prefetch, arming tile k - 1 already required the
    release of k - S, so the ordering argument needs no in-order releases."""
    rng = random.Random(13)
    for W in (1, 2, 3):
        S = 6
        for _ in range(300):
            assert run_schedule(18, S, W, 4, S - 1, rng, prefetch=0) is None
