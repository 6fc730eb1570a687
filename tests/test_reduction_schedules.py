"""The summation schedules of the GPU reductions equal the pairwise tree.

gamma (the absmean of "Step 1", Sparse-BitNet summary section 3.4) and the
RMSNorm sum of squares are fp64 sums over the tree that splits a range at its
largest power of two below the length.  After the final fp32 rounding almost
no input can tell two summation orders apart, so the bit-exact GPU parity
tests cannot check the order.  These CPU tests restate, lane by lane, the
schedules the kernels use (shuffle reduce-scatter over lanes, butterflies,
warp and slot combination) and check them against the tree on inputs where
the order changes the fp64 result (powers of two over a wide exponent range).
"""
import random

import pytest


def tree(v):
    n = len(v)
    if n == 0:
        return 0.0
    if n == 1:
        return v[0]
    h = 1
    while h * 2 < n:
        h *= 2
    return tree(v[:h]) + tree(v[h:])


def leaf8(s):
    return ((s[0] + s[1]) + (s[2] + s[3])) + ((s[4] + s[5]) + (s[6] + s[7]))


def reduce_scatter(vals):
    """vals[lane][q], q < 8: after xor 1, 2, 4 (keeping half, a quarter, one
    of the eight) and xor 8, 16, lane L holds the sum over all lanes of slot
    4 (L & 1) + 2 (L >> 1 & 1) + (L >> 2 & 1)."""
    r1 = [[None] * 4 for _ in range(32)]
    for L in range(32):
        P = L ^ 1
        for i in range(4):
            keep = vals[L][4 + i] if L & 1 else vals[L][i]
            give = vals[P][i] if P & 1 else vals[P][4 + i]
            r1[L][i] = keep + give
    r2 = [[None] * 2 for _ in range(32)]
    for L in range(32):
        P = L ^ 2
        for i in range(2):
            keep = r1[L][2 + i] if (L >> 1) & 1 else r1[L][i]
            give = r1[P][i] if (P >> 1) & 1 else r1[P][2 + i]
            r2[L][i] = keep + give
    r3 = []
    for L in range(32):
        P = L ^ 4
        keep = r2[L][1] if (L >> 2) & 1 else r2[L][0]
        give = r2[P][0] if (P >> 2) & 1 else r2[P][1]
        r3.append(keep + give)
    for off in (8, 16):
        r3 = [r3[L] + r3[L ^ off] for L in range(32)]
    return r3


def slot_of(L):
    return 4 * (L & 1) + 2 * ((L >> 1) & 1) + ((L >> 2) & 1)


def gamma_warp_schedule(w):
    """One warp of gamma_kernel: 1024 |w| as 8 chunks of 128, lane l holding
    leaves 128 q + 4 l .. + 3 of chunk q."""
    c = [[(abs(w[128 * q + 4 * l]) + abs(w[128 * q + 4 * l + 1])) +
          (abs(w[128 * q + 4 * l + 2]) + abs(w[128 * q + 4 * l + 3])) for q in range(8)] for l in range(32)]
    t = reduce_scatter(c)
    for off in (4, 2, 1):
        t = [t[L] + t[L ^ off] for L in range(32)]
    return t[0]


def norm_row_schedule(x2, K, RT):
    """act_norm_quant_kernel<RT>: thread lt holds chunks lt + c RT; per warp a
    reduce-scatter; the row's first warp adds (slot, warp) sums in lanes."""
    chunks, W = K // 8, RT // 32

    def chunk(ci):
        return leaf8(x2[8 * ci:8 * ci + 8]) if ci < chunks else 0.0

    wsum = {}
    for wr in range(W):
        r3 = reduce_scatter([[chunk(32 * wr + L + c * RT) for c in range(8)] for L in range(32)])
        for L in range(8):
            wsum[slot_of(L) * W + wr] = r3[L]
    H = (8 * W + 31) // 32
    x = [[wsum[h * 32 + l] if h * 32 + l < 8 * W else 0.0 for h in range(H)] for l in range(32)]
    off = 1
    while off < 32:
        x = [[x[l][h] + x[l ^ off][h] for h in range(H)] for l in range(32)]
        off *= 2
    xs, step = x[0][:], 1
    while step < H:
        for h in range(0, H, 2 * step):
            xs[h] = xs[h] + xs[h + step]
        step *= 2
    return xs[0]


def wide(rng, n, p_zero=0.4):
    return [0.0 if rng.random() < p_zero else rng.choice([-1.0, 1.0]) * 2.0 ** rng.randint(-80, 60)
            for _ in range(n)]


def test_gamma_warp_schedule_is_the_tree():
    rng = random.Random(1)
    for _ in range(100):
        w = wide(rng, 1024)
        assert gamma_warp_schedule(w) == tree([abs(v) for v in w])


def test_schedule_inputs_are_order_sensitive():
    """The inputs above do tell orders apart: a sequential sum differs from
    the tree on most of them."""
    rng = random.Random(1)
    differ = 0
    for _ in range(50):
        v = [abs(x) for x in wide(rng, 1024)]
        seq = 0.0
        for x in v:
            seq += x
        differ += seq != tree(v)
    assert differ > 25


@pytest.mark.parametrize("RT", [32, 64, 128, 256, 512, 1024])
def test_norm_row_schedule_is_the_tree(RT):
    rng = random.Random(RT)
    for _ in range(6 if RT >= 512 else 20):
        lo = max(2, RT * 4) if RT > 32 else 2  # the chunk counts the launcher maps to RT
        chunks = rng.randint(lo, RT * 8)
        chunks -= chunks % 2
        K = 8 * chunks
        x2 = [v * v for v in wide(rng, K)]
        assert norm_row_schedule(x2, K, RT) == tree(x2)
