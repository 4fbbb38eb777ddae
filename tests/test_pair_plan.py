"""The host-side plan of 128-row query blocks (CPU, no device work): with
tile volumes that are an odd multiple of 64 rows, w-adjacent tiles share
their blocks.  Checked through vattn_debug_query_blocks against the oracle's
window definitions: every tile-major row lies in exactly one block, a block
holds rows of one tile or straddles the last 64 rows of a tile and the first
64 of its w-neighbour in the same tile row, the two windows of a straddling
block start at most one tile apart (sliding) or coincide (partitions), and
pairing removes every half-empty block it can."""

import pytest

from oracle import vattn_oracle as O


@pytest.fixture(scope="module")
def V():
    import video_dit_local_b200 as V
    return V


def _w_window(mode, a, w, n):
    if mode == 0:
        return O.window_range(a, w, n)
    return O.partition_range(a, w, n, shifted=(mode == 2))


CASES = [
    # (grid, tile, window) with tile volumes 64, 192, 320 (paired) and 128, 384, 48 (never paired)
    ((3, 8, 72), (3, 8, 8), (1, 1, 3)),
    ((3, 16, 40), (3, 8, 8), (1, 3, 3)),
    ((3, 8, 64), (3, 8, 8), (1, 1, 5)),
    ((3, 8, 48), (3, 8, 8), (1, 2, 2)),
    ((3, 8, 56), (3, 8, 8), (1, 1, 1)),
    ((3, 8, 16), (3, 8, 8), (1, 1, 3)),
    ((3, 8, 8), (3, 8, 8), (1, 1, 3)),
    ((2, 16, 48), (1, 8, 8), (1, 1, 3)),
    ((5, 8, 40), (5, 8, 8), (1, 1, 4)),
    ((2, 8, 32), (2, 8, 8), (1, 1, 3)),
    ((6, 16, 32), (6, 8, 8), (1, 3, 3)),
    ((3, 20, 24), (3, 4, 4), (1, 3, 3)),
]


@pytest.mark.parametrize("mode", [0, 1, 2])
@pytest.mark.parametrize("grid,tile,window", CASES)
def test_query_block_plan(V, grid, tile, window, mode):
    g = V.make_geom(1, 1, 128, grid, tile, window)
    s = tile[0] * tile[1] * tile[2]
    nt, nh, nw = (a // b for a, b in zip(grid, tile))
    n = grid[0] * grid[1] * grid[2]
    plan = V.vattn_debug_query_blocks(g, mode).numpy()
    seen = [0] * n
    straddles = 0
    for row0, valid, straddle, t in plan.tolist():
        assert 0 < valid <= 128
        for r in range(row0, row0 + valid):
            seen[r] += 1
        if straddle:
            straddles += 1
            assert valid == 128 and s % 128 == 64
            assert row0 == t * s + s - 64, "a straddling block starts 64 rows before the next tile"
            assert t % nw != nw - 1, "the two tiles share a tile row"
            w0 = _w_window(mode, t % nw, window[2], nw)
            w1 = _w_window(mode, t % nw + 1, window[2], nw)
            if mode == 0:
                assert w1.start - w0.start in (0, 1) and len(w0) == len(w1) >= 2
            else:
                assert w0 == w1, "partition pairs keep their two tiles in one block"
        else:
            assert row0 // s == t and (row0 + valid - 1) // s == t, "a block inside one tile"
    assert seen == [1] * n, "every row in exactly one block"
    half = sum(1 for _, valid, _, _ in plan.tolist() if valid < 128)
    if s % 128 == 64:
        # tiles of a tile row left without a partner (each keeps a half-empty block)
        if nw < 2:
            singles = nw
        elif mode == 0:
            singles = nw % 2 if min(window[2], nw) >= 2 else nw
        else:  # greedy, left to right: a tile pairs with the next one when their windows coincide
            singles, a = 0, 0
            while a < nw:
                if a + 1 < nw and _w_window(mode, a, window[2], nw) == _w_window(mode, a + 1, window[2], nw):
                    a += 2
                else:
                    singles, a = singles + 1, a + 1
            if singles == nw:
                assert straddles == 0
        assert half == nt * nh * singles, (half, singles)
    else:
        assert straddles == 0
        assert half == (n // s) * (1 if s % 128 else 0)


def test_pairing_counts_at_the_benchmark_shapes(V):
    """1080p and 4K (192-row tiles): 1449 and 5670 query blocks per slice
    instead of 1890 and 7560 (every tile row of 15 / 30 tiles along w
    paired)."""
    for grid, window, expect in (((21, 72, 120), (3, 3, 3), 7 * 9 * 23), ((21, 144, 240), (3, 3, 5), 7 * 18 * 45)):
        g = V.make_geom(1, 1, 128, grid, (3, 8, 8), window)
        assert V.vattn_debug_query_blocks(g, 0).shape[0] == expect
