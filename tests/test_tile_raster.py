"""The persistent GEMM kernels' tile raster covers every output tile once.

The dense and the 2:4 sparse forward kernels walk tiles t = b, b + G,
b + 2G, ... (b the CTA or CTA pair, G the grid) and map each t to a (row
tile, column tile) pair in groups of 8 row tiles (the last group may be
shorter), so that consecutive tiles reuse the same column tile from L2.
This CPU restatement checks that the map is a bijection onto the tile grid
for every ragged tile count, and that the grid-strided walk visits each tile
exactly once for any grid size."""
import pytest

GROUP_M = 8


def tile_coords(tile, tiles_m, tiles_n):
    per_group = GROUP_M * tiles_n
    group = tile // per_group
    first_m = group * GROUP_M
    gm = min(tiles_m - first_m, GROUP_M)
    r = tile - group * per_group
    return first_m + r % gm, r // gm


@pytest.mark.parametrize("tiles_m", [1, 2, 7, 8, 9, 15, 16, 17, 33, 86])
@pytest.mark.parametrize("tiles_n", [1, 3, 8, 19, 32])
def test_raster_is_a_bijection(tiles_m, tiles_n):
    seen = [tile_coords(t, tiles_m, tiles_n) for t in range(tiles_m * tiles_n)]
    assert len(set(seen)) == len(seen)
    assert all(0 <= tm < tiles_m and 0 <= tn < tiles_n for tm, tn in seen)


@pytest.mark.parametrize("grid", [1, 74, 148, 1000])
def test_grid_strided_walk_visits_each_tile_once(grid):
    tiles_m, tiles_n = 32, 19          # 4096 x 4864 at 128 x 256 tiles
    num = tiles_m * tiles_n
    g = min(grid, num)                 # the launcher never starts more CTAs than tiles
    visits = [t for b in range(g) for t in range(b, num, g)]
    assert sorted(visits) == list(range(num))


def test_consecutive_tiles_share_a_column_tile_within_a_group():
    tiles_m, tiles_n = 32, 19
    for t in range(0, tiles_m * tiles_n - 1):
        (m0, n0), (m1, n1) = tile_coords(t, tiles_m, tiles_n), tile_coords(t + 1, tiles_m, tiles_n)
        if (t + 1) % GROUP_M:          # inside a run of 8 row tiles
            assert n0 == n1 and m1 == m0 + 1
