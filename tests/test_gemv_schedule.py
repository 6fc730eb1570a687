"""The streaming decode GEMV's work split, restated on the CPU.

A work item is a block of 16 << tl2 rows of one layer (tl2 = log2 of its
16-row tiles: 4 tiles when 64 rows of K/4 bytes fit a 54 KiB stage, else 2
when 32 do, else 1).  Sixteen consumer warps share an item: warp w owns tile
w & (tiles - 1) and takes that tile's 128-weight K slices w >> tl2,
w >> tl2 + 16 >> tl2, ...; full slices first, then, when K % 128 == 64, the
one ragged slice falls to whichever warp's sequence reaches it.  After the
item's barrier, output o = (15 - w) 32 + 512 i + lane (token o / rows, row
o % rows) is finished by lane `lane` of warp w.  These checks pin that every
(tile, slice) pair of an item is computed by exactly one warp, that the
ragged slice is taken exactly once, that every output is finished exactly
once, and that the item-height rule keeps an item inside one stage."""
import pytest

STAGE = 54 * 1024
SLICE = 128
WARPS = 16
MAX_K = 4 * STAGE // 16 // 64 * 64


def tiles_for(K):
    return 4 if 64 * (K // 4) <= STAGE else 2 if 32 * (K // 4) <= STAGE else 1


def warp_slices(w, tl2, K):
    """(full slices, ragged slice or None) that warp w computes for its tile."""
    slices, full = -(-K // SLICE), K // SLICE
    sl0, step = w >> tl2, WARPS >> tl2
    mine = list(range(sl0, full, step))
    sl = sl0 if sl0 >= full else sl0 + -(-(full - sl0) // step) * step  # first of its sequence past the full ones
    return mine, (sl if sl < slices else None)


@pytest.mark.parametrize("K", [64, 128, 192, 320, 896, 1536, 2560, 4864, 6912, 8960, 11008, 13824])
def test_every_tile_and_slice_of_an_item_is_computed_once(K):
    tiles = tiles_for(K)
    tl2 = tiles.bit_length() - 1
    assert tiles * 16 * (K // 4) <= STAGE        # an item fits one stage
    slices = -(-K // SLICE)
    seen = {}
    for w in range(WARPS):
        tile = w & (tiles - 1)
        full, ragged = warp_slices(w, tl2, K)
        for s in full + ([ragged] if ragged is not None else []):
            assert (tile, s) not in seen, (K, w, tile, s, seen.get((tile, s)))
            seen[(tile, s)] = w
    assert set(seen) == {(t, s) for t in range(tiles) for s in range(slices)}
    if K % SLICE:                                # the ragged slice: exactly one warp per tile
        assert sum(1 for (t, s) in seen if s == slices - 1) == tiles


def test_the_largest_supported_k_is_a_stage_of_16_rows():
    assert MAX_K == 13824 and 16 * (MAX_K // 4) <= STAGE < 16 * ((MAX_K + 64) // 4)
    assert tiles_for(2560) == 4 and tiles_for(6912) == 2 and tiles_for(13824) == 1


@pytest.mark.parametrize("T", [1, 3, 8, 9, 16])
@pytest.mark.parametrize("tiles", [1, 2, 4])
def test_every_output_of_an_item_is_finished_once(T, tiles):
    rows = 16 * tiles
    n_out = T * rows
    seen = []
    for w in range(WARPS):
        for o0 in range((WARPS - 1 - w) * 32, n_out, WARPS * 32):
            for lane in range(32):
                o = o0 + lane
                if o < n_out:
                    seen.append((o // rows, o % rows))
    assert sorted(seen) == [(t, r) for t in range(T) for r in range(rows)]
