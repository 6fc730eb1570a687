"""The N:M selection of the packing kernel equals the mask definition.

The packing kernel ("N:M Mask Generation", Sparse-BitNet summary section
3.4) picks each group's kept positions with a scan when at most two
positions are dropped or kept (7:8, 6:8, 3:4, 2:4, 2:8, 1:4, ...): it
removes the minimum twice (ties to the higher index) or takes the maximum
twice (ties to the lower index), on the fp32 bit patterns of |w|.  Other
patterns count ranks.  This CPU restatement of those steps is checked
against the oracle's mask on every group over small, tie-heavy alphabets
(every multiset order, so every tie pattern) and on random groups; the GPU
parity tests check the kernel itself bit for bit on seeded layers.
"""
import itertools
import random

import numpy as np
import pytest

import oracle


def keep_mask(key, n):
    """The kernel's keep mask of one group, from uint32 keys (|w| bits)."""
    m = len(key)
    full = (1 << m) - 1
    drop = m - n
    if drop <= 2 or n <= 2:
        by_drop = drop <= 2
        picks = drop if by_drop else n
        # keep: the complement 2^31 - 1 - key turns a maximum into a minimum
        k = [key[i] if by_drop else 0x7FFFFFFF - key[i] for i in range(m)]
        chosen = 0
        for p in range(2):
            if p >= picks:
                break
            best = m - 1 if by_drop else 0
            kb = k[best]
            for t in range(1, m):
                i = m - 1 - t if by_drop else t
                if k[i] < kb:
                    kb, best = k[i], i
            chosen |= 1 << best
            k[best] = 0xFFFFFFFF
        return full & ~chosen if by_drop else chosen
    rank = [0] * m
    for i in range(m):
        for j in range(i + 1, m):
            if key[j] > key[i]:
                rank[i] += 1
            else:
                rank[j] += 1
    return sum(1 << i for i in range(m) if rank[i] < n)


def masks_both_ways(rows, n, m):
    """(kernel restatement, oracle) keep bits for every row of |w| values."""
    w = np.asarray(rows, dtype=np.float32)
    keys = (np.abs(w).view(np.uint32)).tolist()
    got = np.array([keep_mask(k, n) for k in keys], dtype=np.int64)
    ref_mask = oracle.nm_mask(w, n, m)  # [R, m] of 0/1
    ref = (ref_mask.astype(np.int64) << np.arange(m)).sum(axis=1)
    return got, ref


@pytest.mark.parametrize("m,alphabet", [(4, [0.0, -0.0, 1.0, 2.0, 2.0000002]),
                                        (8, [0.0, 1.0, -1.0]),
                                        (8, [0.5, 0.25, 3.0])])
def test_every_tie_pattern_matches_the_definition(m, alphabet):
    rows = [list(t) for t in itertools.product(alphabet, repeat=m)]
    for n in range(1, m + 1):
        got, ref = masks_both_ways(rows, n, m)
        bad = np.nonzero(got != ref)[0]
        assert bad.size == 0, (n, rows[bad[0]] if bad.size else None)


def test_random_groups_match_the_definition():
    rnd = random.Random(5)
    vals = [0.0, -0.0, 1e-30, 0.02, -0.02, 0.0200001, 7.5, -7.5, 3.4e38]
    for m in (4, 8):
        rows = [[rnd.choice(vals) if rnd.random() < 0.5 else rnd.gauss(0, 0.02) for _ in range(m)]
                for _ in range(3000)]
        for n in range(1, m + 1):
            got, ref = masks_both_ways(rows, n, m)
            assert (got == ref).all(), n


def test_scan_and_rank_paths_are_both_exercised():
    """The scan serves n <= 2 or m - n <= 2; 4:8 and 5:8 (and m = 4 never)
    take the rank count."""
    scan = {(n, m) for m in (4, 8) for n in range(1, m + 1) if m - n <= 2 or n <= 2}
    assert {(n, 8) for n in range(1, 9)} - scan == {(3, 8), (4, 8), (5, 8)}
    assert all((n, 4) in scan for n in range(1, 5))
