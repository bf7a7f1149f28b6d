"""The tail refresh of a kept pooled key cache, its work split modelled on the CPU: the launch
gives each sequence a window of (T - 1) // P + 2 groups starting at the group of the first
appended row, and each thread pools group lo // P + j when that group holds an appended row.
Over many (context, appended rows, factor, cache size) cases the threads pool exactly the groups
that hold a row appended inside the cache, each once, and never a group outside the cache."""
import random

import pytest


def window(T: int, P: int) -> int:
    return (T - 1) // P + 2   # as in the launch


def groups_pooled(ctx: int, T: int, P: int, S_max: int):
    """The groups one sequence's threads pool (the kernel's index arithmetic)."""
    out = []
    lo, hi = max(ctx - T, 0), min(ctx, S_max)
    if hi <= lo:
        return out
    for j in range(window(T, P)):
        g = lo // P + j
        if g > (hi - 1) // P:
            continue
        out.append(g)
    return out


@pytest.mark.parametrize("P", [2, 4, 8])
def test_tail_refresh_pools_exactly_the_touched_groups(P):
    rng = random.Random(P)
    for _ in range(4000):
        S_max = P * rng.randint(1, 64)
        T = rng.randint(1, 3 * P + 5)
        ctx = rng.randint(-3, S_max + 2 * P)
        got = groups_pooled(ctx, T, P, S_max)
        rows = [r for r in range(ctx - T, ctx) if 0 <= r < S_max]
        want = sorted({r // P for r in rows})
        assert got == want, (ctx, T, P, S_max)
        assert all(0 <= g < S_max // P for g in got)
