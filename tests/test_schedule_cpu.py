"""The decode kernels' split of the tile sequence over CTAs, restated on the
CPU.  Every non-empty unit (sequence, KV head) occupies W boundary positions
followed by P positions per tile in a flat sequence of positions; CTAs split
the positions evenly and own the tiles whose first position falls in their
range, so a CTA whose range crosses into a new unit (and pays a second
selection switch and segment merge) gets fewer tiles.  Checked here: the real
tiles of every CTA are contiguous and cover every tile exactly once, the CTAs
covering a unit are consecutive, the owner formula is right, and the partial
slots (unit u on CTA c takes slot u + c) are distinct, consecutive within a
unit and below the workspace bound (the ticket-based combine relies on all of
it)."""
import random

P = 4          # positions per tile (kTilePos in csrc/decode.cu)
W = 14         # boundary positions per unit (kBoundaryPos)


def cta_of_pos(p, NV, C):
    c = ((p + 1) * C + NV - 1) // NV - 1
    return min(c, C - 1)


LATE = 10      # kLatePos: positions fewer for each of the last n_late CTAs


def make_split(NV, grid, pt, n_late, late):
    """(C, c0, E): C CTAs, the first c0 share positions [0, E), the rest [E, NV)."""
    C = max(1, min(grid, NV // pt))     # every CTA's range spans at least one tile's positions
    c0, E = C, NV
    if 0 < n_late < C:
        c = C - n_late
        e = c * (NV + n_late * late) // C
        if e <= NV and e // c >= pt and (NV - e) // n_late >= pt:
            c0, E = c, e
    return C, c0, E


def split_start(c, NV, C, c0, E):
    return c * E // c0 if c <= c0 else E + (c - c0) * (NV - E) // (C - c0)


def cta_of_pos_even(p, N, C):
    c = ((p + 1) * C + N - 1) // N - 1
    return min(c, C - 1)


def cta_of_pos2(p, NV, C, c0, E):
    return cta_of_pos_even(p, E, c0) if p < E else c0 + cta_of_pos_even(p - E, NV - E, C - c0)


def split(tiles, grid, w=W, pt=P, n_late=0, late=LATE, full=False):
    """Real tile range [start, end) of every CTA, and the units' virtual starts.
    Tile j of a unit starting at position vs occupies positions from
    vs + w + j pt; a CTA owns the tiles whose first position is in its range."""
    vstart, vs = [], 0
    for nt in tiles:
        vstart.append(vs)
        vs += nt * pt + w if nt else 0
    NV = vs
    C, c0, E = make_split(NV, grid, pt, n_late, late)
    N = sum(tiles)

    def real_index(pos):
        # first real tile whose first position is >= pos (N past the end)
        r = 0
        for u, nt in enumerate(tiles):
            if nt == 0:
                continue
            first = vstart[u] + w
            for j in range(nt):
                if first + j * pt >= pos:
                    return r + j
            r += nt
        return N

    ranges = [(real_index(split_start(c, NV, C, c0, E)), real_index(split_start(c + 1, NV, C, c0, E)))
              for c in range(C)]
    if full:
        return ranges, vstart, NV, C, c0, E
    return ranges, vstart, NV, C


def _check(tiles, grid, w=W, pt=P, n_late=0, late=LATE):
    N = sum(tiles)
    if N == 0:
        return
    ranges, vstart, NV, C, c0, E = split(tiles, grid, w, pt, n_late, late, full=True)

    def cta_of_pos(p, NV_, C_):
        return cta_of_pos2(p, NV_, C_, c0, E)

    # the CTAs' real ranges tile [0, N) in order
    pos = 0
    for s, e in ranges:
        assert s == pos and e >= s
        pos = e
    assert pos == N
    ts = 0
    slots = []
    for u, nt in enumerate(tiles):
        if nt == 0:
            continue
        first, last = vstart[u] + w, vstart[u] + w + (nt - 1) * pt
        cf, cl = cta_of_pos(first, NV, C), cta_of_pos(last, NV, C)
        cover = [c for c, (s, e) in enumerate(ranges) if s < e and s < ts + nt and e > ts]   # CTAs owning tiles
        assert cover == list(range(cf, cl + 1))
        slots += [u + c for c in cover]                      # consecutive within the unit
        for j in range(nt):                                  # owner of every tile
            s, e = ranges[cta_of_pos(first + j * pt, NV, C)]
            assert s <= ts + j < e
        ts += nt
    assert len(set(slots)) == len(slots)                     # distinct across units
    assert max(slots) < len(tiles) + C - 1                   # workspace bound: units + CTAs


def test_schedule_random():
    rng = random.Random(0)
    for _ in range(4000):
        tiles = [rng.choice([0, 0, 1, 2, 3, 8, 65]) for _ in range(rng.randint(1, 12))]
        _check(tiles, rng.randint(1, 160), w=rng.choice([0, 1, 3, 14]), pt=rng.choice([1, 2, 4]),
               n_late=rng.choice([0, 0, 1, 5, 64, 200]), late=rng.choice([0, 3, 7, 20]))


def test_schedule_grid_larger_than_tiles():
    for w, pt in ((0, 1), (3, 1), (W, P)):
        for n_late in (0, 8, 64):
            _check([8, 8, 1, 1, 0, 0, 5, 5], 64, w, pt, n_late)
            _check([1], 148, w, pt, n_late)
            _check([64] * 64, 148, w, pt, n_late)
            _check([1024] * 8, 148, w, pt, n_late)


def test_late_ctas_get_fewer_positions():
    """At the Llama decode shape the 64 CTAs that start behind the projection
    kernel's CTAs get about kLatePos fewer positions than the other 84."""
    tiles = [65] * 64
    NV = 64 * (65 * P + W)
    C, c0, E = make_split(NV, 148, P, 64, LATE)
    assert (C, c0) == (148, 84)
    early = [split_start(c + 1, NV, C, c0, E) - split_start(c, NV, C, c0, E) for c in range(c0)]
    late = [split_start(c + 1, NV, C, c0, E) - split_start(c, NV, C, c0, E) for c in range(c0, C)]
    assert abs(sum(early) / len(early) - sum(late) / len(late) - LATE) < 1.0
    ranges, _, _, _ = split(tiles, 148, n_late=64)
    assert sum(e - s for s, e in ranges) == sum(tiles)


def test_boundary_positions_balance_the_split():
    """At the Llama decode shape (64 units of 65 tiles over 148 CTAs) the CTAs
    that cross into a second unit get fewer tiles than those that do not."""
    tiles = [65] * 64
    ranges, vstart, NV, C = split(tiles, 148)
    one, two = [], []
    starts = {sum(tiles[:u]) for u in range(64)}
    for s, e in ranges:
        crosses = any(s < b < e for b in starts)
        (two if crosses else one).append(e - s)
    assert two and one and max(two) < max(one)


def guess_first_tile(len0, len_add, Tcap, n_units, grid, n_late, c, TT=128):
    """The attention kernel's guess of CTA c's first tile for its L2 prefetch
    (prefetch_first_tiles_l2 in csrc/decode.cu): every sequence taken to have
    sequence 0's length.  Returns (unit, tile within the unit, tiles per unit)
    or None when the kernel prefetches nothing."""
    T = min(max(len0, 0) + len_add, Tcap)
    nt = (T + TT - 1) // TT
    if nt == 0:
        return None
    unitpos = nt * P + W
    NV = n_units * unitpos
    if NV > 0x7fffffff:
        return None
    C, c0, E = make_split(NV, grid, P, n_late, LATE)
    if c >= C:
        return None
    a = split_start(c, NV, C, c0, E)
    u = a // unitpos
    if u >= n_units:
        return None
    off = a - u * unitpos
    t = (off - W + P - 1) // P if off > W else 0
    return u, t, nt


def test_prefetch_guess_is_exact_for_equal_lengths():
    """With equal lengths the guessed first tile is the CTA's real first tile."""
    rng = random.Random(1)
    for _ in range(300):
        n_units = rng.choice([1, 2, 8, 64, 100, 256])
        T = rng.randint(1, 20000)
        grid, n_late = rng.choice([148, 64, 16]), rng.choice([0, n_units])
        nt = (T + 127) // 128
        ranges, _, _, C = split([nt] * n_units, grid, n_late=n_late)
        for c, (s, e) in enumerate(ranges):
            if s == e:
                continue
            g = guess_first_tile(T - 1, 1, 1 << 20, n_units, grid, n_late, c)
            assert g is not None
            u, t, _ = g
            assert u * nt + t == s, (n_units, T, grid, n_late, c)


def test_prefetch_addresses_stay_inside_the_unit():
    """Every byte range the guess prefetches (K~ row r of tiles t..t+2, and the
    tiles' V rows) lies inside the unit's slots, starts on a 16-byte boundary
    and has a positive multiple of 16 bytes, whatever the device length."""
    rng = random.Random(2)
    for _ in range(3000):
        Tcap = 16 * rng.randint(1, 400)
        len0 = rng.choice([-5, 0, 1, rng.randint(0, Tcap), Tcap, Tcap + 7, 10 ** 9])
        len_add = rng.choice([0, 1])
        n_units = rng.choice([1, 3, 8, 64, 256])
        d_store = rng.randint(1, 128)
        vcols = rng.choice([128, 16 * rng.randint(1, 8)])
        grid = rng.randint(1, 160)
        n_late = rng.choice([0, n_units])
        for c in range(grid):
            g = guess_first_tile(len0, len_add, Tcap, n_units, grid, n_late, c)
            if g is None:
                continue
            u, t, nt = g
            assert 0 <= u < n_units
            for j in range(3):
                if t + j >= nt:
                    continue
                t0 = (t + j) * 128
                ntok = min(128, Tcap - t0)
                assert 0 < ntok and t0 + ntok <= Tcap
                for r in range(d_store):
                    start = ((u * d_store + r) * Tcap + t0) * 2
                    size = ntok * 2
                    row0 = (u * d_store + r) * Tcap * 2
                    assert row0 <= start and start + size <= row0 + Tcap * 2
                    assert start % 16 == 0 and size % 16 == 0
                vstart = (u * Tcap + t0) * vcols * 2
                vsize = ntok * vcols * 2
                assert u * Tcap * vcols * 2 <= vstart and vstart + vsize <= (u + 1) * Tcap * vcols * 2
                assert vstart % 16 == 0 and vsize % 16 == 0
