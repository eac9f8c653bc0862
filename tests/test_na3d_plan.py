"""ltxattn_na3d_plan (host only, no GPU): the blocking the 3-D neighbourhood kernel uses.

Pins, independent of the library's own arithmetic:
* the tile count it reports equals a brute-force count: for every query brick, the union
  of its queries' windows (each window taken from Neighborhood Attention's definition,
  query by query) is a box, covered by ceil(extent / tile) key tiles per axis;
* of the shape pairs the kernel is built for (the header lists the brick sizes and key
  tile sizes), the choice has the fewest key tiles, then the fewest keys;
* every window of every query lies inside its brick's key box, and the keys the tiles
  hold are at least the neighbourhood work (density <= 1);
* the grid and window rules of ltxattn_na3d_forward, without a device.
"""
import itertools

import numpy as np
import pytest

from joint_audio_video_flash_b200 import build, ltxattn

# the (query brick, key tile) pairs of the kernel's instantiations
PAIRS = [((2, 8, 8), (2, 8, 8)), ((2, 8, 8), (4, 2, 16)), ((1, 8, 16), (1, 8, 16)),
         ((1, 8, 16), (1, 16, 8)), ((4, 4, 8), (4, 4, 8)), ((4, 4, 8), (4, 2, 16)),
         ((2, 8, 8), (4, 2, 14))]


@pytest.fixture(scope="module", autouse=True)
def lib():
    build.build()
    ltxattn.load()


def window(i, k, n):
    """Neighborhood Attention's window along one axis: k positions from its start."""
    s = min(max(i - k // 2, 0), n - k)
    return s, s + k


def brute_tiles(grid, win, brick, tile):
    """Key tiles over all bricks, each brick's key box the union of its queries' windows."""
    total = 0
    starts = [range(0, grid[a], brick[a]) for a in range(3)]
    for b0 in itertools.product(*starts):
        lo = [None] * 3
        hi = [None] * 3
        for q in itertools.product(*(range(b0[a], min(b0[a] + brick[a], grid[a]))
                                     for a in range(3))):
            for a in range(3):
                s, e = window(q[a], win[a], grid[a])
                lo[a] = s if lo[a] is None else min(lo[a], s)
                hi[a] = e if hi[a] is None else max(hi[a], e)
        total += int(np.prod([-(-(hi[a] - lo[a]) // tile[a]) for a in range(3)]))
    return total


CASES = [((2, 8, 8), (1, 3, 3)), ((3, 10, 13), (3, 5, 7)), ((5, 12, 20), (3, 7, 7)),
         ((1, 24, 40), (1, 7, 9)), ((16, 8, 8), (7, 3, 3)), ((12, 6, 9), (5, 3, 5)),
         ((1, 5, 6), (1, 3, 5)), ((9, 4, 5), (5, 3, 3)), ((2, 3, 40), (1, 3, 9)),
         ((8, 12, 16), (3, 3, 9)), ((6, 12, 32), (3, 5, 9)), ((6, 13, 30), (3, 7, 7)),
         ((4, 14, 22), (3, 7, 7)), ((3, 9, 17), (3, 3, 9))]


@pytest.mark.parametrize("grid,win", CASES, ids=lambda x: "x".join(map(str, x)))
def test_plan_is_the_least_work_cover(grid, win):
    brick, tile, tiles = ltxattn.na3d_plan(grid, win)
    assert (brick, tile) in PAIRS
    assert tiles == brute_tiles(grid, win, brick, tile)
    best = min((brute_tiles(grid, win, b, t), brute_tiles(grid, win, b, t) * int(np.prod(t)))
               for b, t in PAIRS)
    assert (tiles, tiles * int(np.prod(tile))) == best
    # the tiles hold at least the neighbourhood's keys
    assert tiles * 128 * int(np.prod(tile)) >= int(np.prod(grid)) * int(np.prod(win))


def test_decoder_grid_takes_the_exact_cover():
    # a 2x8x8 brick's key box under a 3x7x7 window is 4x14x14: seven 4x2x14 tiles of 112 keys
    assert ltxattn.na3d_plan((16, 34, 60), (3, 7, 7)) == ((2, 8, 8), (4, 2, 14), 1984)


def test_plan_rejects_what_the_kernel_rejects():
    bad = [((4, 4, 4), (2, 3, 3)), ((4, 4, 4), (5, 3, 3)), ((0, 4, 4), (1, 3, 3)),
           ((4, 4, 4), (1, 3, -1)), ((4, 4, 4), (1, 0, 3))]
    for grid, win in bad:
        with pytest.raises(ltxattn.LtxAttnError):
            ltxattn.na3d_plan(grid, win)
