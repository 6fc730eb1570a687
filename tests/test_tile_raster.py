"""The persistent GEMM kernels' tile raster covers every output tile once (grouped launches included).

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


def group_of(tn0, count, tn):
    """The grouped launch's column tile -> (group, column tile inside it)."""
    gi = 0
    while gi + 1 < count and tn >= tn0[gi + 1]:
        gi += 1
    return gi, tn - tn0[gi]


@pytest.mark.parametrize("widths,bn", [((4864, 4864), 256), ((1536, 256, 256), 256), ((272, 1040, 48, 784), 128),
                                       ((16,), 128), ((8192, 8192, 8192, 4864), 256)])
@pytest.mark.parametrize("tokens,pair", [(4096, True), (1000, True), (100, False), (1, False)])
def test_grouped_raster_covers_every_output_tile_of_every_group_once(widths, bn, tokens, pair):
    """sbl_forward_group: the launch's column tiles are the groups' tiles in
    order (tn0 = prefix sums of ceil(width / BN)); every (group, row tile,
    column tile) is visited exactly once by the grid-strided walk over CTAs
    or CTA pairs, and no tile column lies past its group's width by a whole tile."""
    tn0 = [0]
    for w in widths:
        tn0.append(tn0[-1] + -(-w // bn))
    tile_m = 256 if pair else 128
    tiles_m, tiles_n = -(-tokens // tile_m), tn0[-1]
    num = tiles_m * tiles_n
    units = min(num, 74 if pair else 148)
    seen = []
    for u in range(units):
        for t in range(u, num, units):
            tm, tn = tile_coords(t, tiles_m, tiles_n)
            gi, tl = group_of(tn0, len(widths), tn)
            assert tl * bn < widths[gi]          # the tile starts inside its group's columns
            seen.append((gi, tm, tl))
    expected = {(gi, tm, tl) for gi, w in enumerate(widths) for tm in range(tiles_m) for tl in range(-(-w // bn))}
    assert len(seen) == len(expected) and set(seen) == expected


@pytest.mark.parametrize("M,N", [(4096, 4864), (1000, 9792), (16384, 2048), (300, 256)])
def test_pair_tiles_split_rows_and_b_rows_between_the_two_ctas(M, N):
    """CTA-pair form: tile (tm, tn) covers A rows [256 tm, 256 tm + 256) and B
    rows [256 tn, 256 tn + 256); CTA rank r of the pair loads A rows
    256 tm + 128 r .. + 127 and B rows 256 tn + 128 r .. + 127, and drains its
    own 128 accumulator rows over all 256 columns.  Over the grid the A rows
    and the output rows each come out exactly once per column tile."""
    tiles_m, tiles_n = -(-M // 256), -(-N // 256)
    a_rows, out_cells, b_rows = [], set(), []
    for t in range(tiles_m * tiles_n):
        tm, tn = tile_coords(t, tiles_m, tiles_n)
        for r in (0, 1):
            arow = tm * 256 + 128 * r
            brow = tn * 256 + 128 * r
            if tn == 0:
                a_rows.extend(range(arow, arow + 128))
            if tm == 0:
                b_rows.extend(range(brow, brow + 128))
            out_cells.add((arow, tn))      # 128 output rows x the tile's 256 columns
    assert sorted(a_rows) == list(range(tiles_m * 256))
    assert sorted(b_rows) == list(range(tiles_n * 256))
    assert out_cells == {(tm * 256 + 128 * r, tn) for tm in range(tiles_m) for r in (0, 1) for tn in range(tiles_n)}
