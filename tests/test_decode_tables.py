"""The decode kernel's T24 expansion equals the oracle's packing.

The T24 decode ("Inference Implementation: GPU" of the BitNet b1.58 2B4T
summary gives the 2-bit packing; the 6-bit group code is this library's
denser form) turns each lane's 8 low-plane and 4 high-plane bytes of a
64-weight segment into the 16 PK2 bytes of the same weights, through a
4096-entry table indexed by a pair of group codes.  This CPU restatement of
the table construction and of the lane's indexing is checked against the
oracle: for every ordered pair of the 33 group states, the expansion of the
oracle's T24 planes must equal the oracle's PK2 bytes.  The GPU parity tests
check the kernel itself bit for bit.
"""
import itertools

import numpy as np

import oracle

PAIR_POSITIONS = 0x323121302010  # byte k: q << 4 | p for the k-th pair (p, q) of positions


def pk2_byte(c):
    """PK2 byte of one group from its 6-bit T24 code (the kernel's rule)."""
    b = 0x55
    if 1 <= c <= 8:
        p, neg = (c - 1) >> 1, (c - 1) & 1
        b = (b & ~(3 << (2 * p))) | ((0 if neg else 2) << (2 * p))
    elif 9 <= c <= 32:
        k, r = (c - 9) >> 2, (c - 9) & 3
        pq = (PAIR_POSITIONS >> (8 * k)) & 0xFF
        p, q = pq & 15, pq >> 4
        b = (b & ~(3 << (2 * p)) & ~(3 << (2 * q))) | ((0 if r & 2 else 2) << (2 * p)) | \
            ((0 if r & 1 else 2) << (2 * q))
    return b & 0xFF


def pair_entry(idx):
    """Table entry: the two PK2 bytes of a pair of groups from its 12-bit index."""
    lo, hi = idx & 0xFF, idx >> 8
    return pk2_byte((lo & 15) | ((hi & 3) << 4)) | (pk2_byte((lo >> 4) | ((hi >> 2) << 4)) << 8)


LUT = [pair_entry(i) for i in range(4096)]


def decode_segment(vx, vy, vz):
    """The lane's four PK2 words from its low-plane words (vx, vy) and its
    32 high-plane bits (vz): word j is pairs 2j and 2j + 1."""
    words = []
    for j in range(4):
        lo = vx if j < 2 else vy
        i0 = ((lo >> (16 * (j & 1))) & 0xFF) | (((vz >> (8 * j)) & 15) << 8)
        i1 = ((lo >> (16 * (j & 1) + 8)) & 0xFF) | (((vz >> (8 * j + 4)) & 15) << 8)
        words.append(LUT[i0] | (LUT[i1] << 16))
    return words


def groups_2of4():
    """The 33 ternary groups of four with at most two nonzeros."""
    out = []
    for g in itertools.product((-1, 0, 1), repeat=4):
        if sum(1 for v in g if v) <= 2:
            out.append(g)
    return out


def check_rows(weff):
    lo, hi = oracle.pack_t24(weff)
    pk = oracle.pack_pk2(weff)
    rows, k = weff.shape
    for r in range(rows):
        for s in range(k // 64):
            le = lambda a: int.from_bytes(bytes(a), "little")  # noqa: E731
            vx, vy = le(lo[r, 8 * s:8 * s + 4]), le(lo[r, 8 * s + 4:8 * s + 8])
            vz = le(hi[r, 4 * s:4 * s + 4])
            want = [le(pk[r, 16 * s + 4 * j:16 * s + 4 * j + 4]) for j in range(4)]
            assert decode_segment(vx, vy, vz) == want, (r, s)


def test_state_count():
    assert len(groups_2of4()) == 33


def test_every_pair_of_group_states_expands_to_the_pk2_bytes():
    gs = groups_2of4()
    seq = [v for a in gs for b in gs for v in a + b]          # all 33 x 33 ordered pairs, 8 weights each
    k = (len(seq) + 63) // 64 * 64
    row = np.zeros(k, dtype=np.int8)
    row[:len(seq)] = seq
    check_rows(row.reshape(1, k))


def test_seeded_layers_expand_to_the_pk2_bytes():
    from sparsity_sbl_quantize_b200 import workloads as wl
    for n, m, seed in [(2, 4, 1), (1, 4, 2), (2, 8, 3), (1, 8, 4)]:
        layer = oracle.Layer(wl.master_weights(16, 512, seed=seed), n, m)
        check_rows(layer.weff)
