"""The decode kernel's split of the flat tile sequence over CTAs, restated on the
CPU: every CTA owns at least one tile, the CTAs covering a unit are consecutive,
the owner formula is right, and partial-slot ids are dense (the ticket-based
combine relies on all three)."""
import random


def cta_of_tile(t, N, C):
    c = ((t + 1) * C + N - 1) // N - 1
    return min(c, C - 1)


def _check(tiles, grid):
    N = sum(tiles)
    if N == 0:
        return
    C = min(grid, N)                      # effective grid
    ranges = [(c * N // C, (c + 1) * N // C) for c in range(C)]
    assert all(e > s for s, e in ranges)
    ts = sb = 0
    slots = set()
    for nt in tiles:
        if nt == 0:
            continue
        cf, cl = cta_of_tile(ts, N, C), cta_of_tile(ts + nt - 1, N, C)
        cover = [c for c, (s, e) in enumerate(ranges) if s < ts + nt and e > ts]
        assert cover == list(range(cf, cl + 1))
        slots.update(sb + c - cf for c in cover)
        for t in range(ts, ts + nt):
            s, e = ranges[cta_of_tile(t, N, C)]
            assert s <= t < e
        sb += cl - cf + 1
        ts += nt
    assert slots == set(range(sb))
    assert sb <= sum(1 for t in tiles if t) + C - 1      # workspace bound: units + CTAs


def test_schedule_random():
    rng = random.Random(0)
    for _ in range(5000):
        tiles = [rng.choice([0, 0, 1, 2, 3, 8, 65]) for _ in range(rng.randint(1, 12))]
        _check(tiles, rng.randint(1, 160))


def test_schedule_grid_larger_than_tiles():
    _check([8, 8, 1, 1, 0, 0, 5, 5], 64)
    _check([1], 148)
    _check([64] * 64, 148)
    _check([1024] * 8, 148)
