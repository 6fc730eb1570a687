"""Pins of the CPU oracle against things other than itself.

The pages print no numeric worked example of the layer, so each oracle
function is pinned by a hand-derived case (tests/golden), closed forms,
invariants the definitions fix, special cases that reduce to an independent
library routine (numpy / torch CPU), and brute force on tiny inputs.  Each
test names the definition it pins: the Sparse-BitNet summary (arXiv
2603.05168), section 3.4, and the BitNet b1.58 2B4T summary (arXiv
2504.12285), section 3.4.
"""
import itertools
import math
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
from sparsity_sbl_quantize_b200 import workloads as wl
from conftest import load_golden


def _floats(vals):
    return np.array([float(v) for v in vals], dtype=np.float32)


def _ints(vals):
    return np.array([int(v, 0) for v in vals])


def test_rounding_mode_is_nearest():
    assert oracle.rounding_is_nearest()


# ------------------------------------------------------------------ worked example

def test_hand_row_6of8():
    """Hand-derived row: gamma ("Step 1"), RoundClip ("Step 2"), 6:8 mask,
    W_eff = W_q * M, 2-bit codes; see tests/golden/hand_row_6of8.txt."""
    g = load_golden("hand_row_6of8.txt")
    w = _floats(g["w"]).reshape(1, 8)
    n, m = int(g["n"][0]), int(g["m"][0])
    gam = oracle.gamma(w)
    exact = Fraction(0)
    for v in w.ravel():
        exact += abs(Fraction(float(v)))
    assert gam == np.float32(float(exact / 8))
    assert abs(float(gam) - float(g["gamma"][0])) < 1e-7
    wq = oracle.ternarize(w, gam)
    np.testing.assert_array_equal(wq.ravel(), _ints(g["wq"]))
    mask = oracle.nm_mask(w, n, m)
    np.testing.assert_array_equal(mask.ravel(), _ints(g["mask"]))
    weff = oracle.apply_mask(wq, mask)
    np.testing.assert_array_equal(weff.ravel(), _ints(g["weff"]))
    np.testing.assert_array_equal(oracle.pack_pk2(weff).ravel(), _ints(g["pk2"]))
    vals, bm = oracle.pack_nm(weff, mask, n, m)
    np.testing.assert_array_equal(vals.ravel(), _ints(g["nm_vals"]))
    np.testing.assert_array_equal(bm.ravel(), _ints(g["nm_bitmap"]))


# ------------------------------------------------------------------------ gamma

def test_abs_sum_pairwise_order():
    """Reading R1 (pairwise tree).  With a = 2**-53, 1 + a rounds back to 1
    (tie to even), so a left-to-right sum of [1, a, a, a] is 1.0 while the tree
    (1 + a) + (a + a) is 1 + 2**-52."""
    a = 2.0 ** -53
    assert oracle.abs_sum(np.array([1.0, a, a, a], dtype=np.float32)) == 1.0 + 2.0 ** -52
    # eight leaves: ((1+a)+(a+a)) + ((a+a)+(a+a)) = 1 + 2**-52 + 2**-51
    v = np.array([1.0] + [a] * 7, dtype=np.float32)
    assert oracle.abs_sum(v) == 1.0 + 3 * 2.0 ** -52
    # odd length: the tree over 3 leaves is (1 + a) + a = 1.0 (zero padding)
    assert oracle.abs_sum(np.array([1.0, a, a], dtype=np.float32)) == 1.0
    # five leaves split 4 + 1: ((a+a)+(a+a)) + 1 = 1 + 2**-51
    assert oracle.abs_sum(np.array([a, a, a, a, 1.0], dtype=np.float32)) == 1.0 + 2.0 ** -51
    # signs are dropped
    assert oracle.abs_sum(np.array([-1.5, 2.0, -0.25], dtype=np.float32)) == 3.75


def test_abs_sum_exact_for_dyadic_values():
    """Sums of small dyadic values are exact in fp64 whatever the order."""
    rng = np.random.default_rng(1)
    v = (rng.integers(-1000, 1000, size=12345) / 64.0).astype(np.float32)
    assert oracle.abs_sum(v) == sum(abs(Fraction(float(x))) for x in v)


@pytest.mark.parametrize("shape", [(128, 256), (1000, 64), (37, 48)])
def test_gamma_within_error_bound_of_exact_mean(shape):
    """gamma = mean |W| ("Step 1" equation): the exact rational mean rounded to
    fp32 and the oracle differ by at most one fp32 ulp (pairwise fp64 error is
    ~log2(n) * 2**-53, far below half an fp32 ulp except at a tie)."""
    w = wl.master_weights(*shape, seed=7)
    exact = math.fsum(abs(float(x)) for x in w.ravel()) / w.size
    gam = float(oracle.gamma(w))
    ulp = np.spacing(np.float32(exact))
    assert abs(gam - exact) <= float(ulp)
    assert oracle.gamma(w) == np.float32(exact) or abs(gam - exact) <= 0.5 * float(ulp) + 1e-300


def test_gamma_includes_masked_weights():
    """"Composition Order": gamma is taken over all weights, masked ones too,
    so it does not depend on n:m and equals the plain mean of |W|."""
    w = wl.master_weights(64, 128, seed=3)
    gam = oracle.gamma(w)
    assert gam == np.float32(np.abs(w.astype(np.float64)).mean()) or \
        abs(float(gam) - np.abs(w.astype(np.float64)).mean()) <= float(np.spacing(gam))


def test_gamma_zero_matrix():
    w = np.zeros((4, 16), dtype=np.float32)
    assert oracle.gamma(w) == 0.0
    assert not oracle.ternarize(w, 0.0).any()


# -------------------------------------------------------------------- ternarise

def test_ternarize_ties_and_clip():
    """RoundClip at the rounding ties: |W|/gamma = 0.5 -> 0 (half-even),
    1.5 -> 2 -> clip 1, 2.5 -> 2 -> clip 1; the row's mean |W| is exactly 1."""
    v = [0.5, -0.5, 1.5, -1.5, 2.5, -2.5] + [0.75] * 8 + [0.5, 0.5]
    w = np.array(v, dtype=np.float32).reshape(1, 16)
    gam = oracle.gamma(w)
    assert gam == 1.0
    expect = [0, 0, 1, -1, 1, -1] + [1] * 8 + [0, 0]
    np.testing.assert_array_equal(oracle.ternarize(w, gam).ravel(), expect)
    # just above and below the 0.5 boundary
    up = np.nextafter(np.float32(0.5), np.float32(1))
    dn = np.nextafter(np.float32(0.5), np.float32(0))
    np.testing.assert_array_equal(
        oracle.ternarize(np.array([up, -up, dn, -dn, 0.0, -0.0], dtype=np.float32), 1.0),
        [1, -1, 0, 0, 0, 0])


def test_ternarize_matches_numpy_library_rounding():
    """Special case reducing to library routines: numpy's IEEE float32 divide,
    rint (half-even) and clip give the same W_q."""
    w = wl.master_weights(300, 512, seed=11)
    gam = oracle.gamma(w)
    ref = np.clip(np.rint(w / np.float32(gam)), -1, 1).astype(np.int8)
    np.testing.assert_array_equal(oracle.ternarize(w, gam), ref)


def test_ternary_values_and_gaussian_zero_fraction():
    """W_q in {-1, 0, 1}; for Gaussian W the zero fraction is
    P(|Z| < 0.5 * sqrt(2/pi)) = erf(0.5/sqrt(pi)) ~= 0.3101 (closed form)."""
    w = wl.master_weights(1024, 1024, seed=5)
    wq = oracle.ternarize(w, oracle.gamma(w))
    assert set(np.unique(wq).tolist()) <= {-1, 0, 1}
    frac0 = float((wq == 0).mean())
    expect = math.erf(0.5 / math.sqrt(math.pi))
    assert abs(frac0 - expect) < 3e-3, (frac0, expect)


# ------------------------------------------------------------------------- mask

def _brute_mask_group(keys, n):
    """Top-n by (key desc, index asc) via an exhaustive search over subsets."""
    m = len(keys)
    best = None
    for subset in itertools.combinations(range(m), n):
        # a valid top-n set dominates every outsider under the (key, -index) order
        ok = all((keys[i], -i) > (keys[j], -j) for i in subset for j in range(m) if j not in subset)
        if ok:
            assert best is None
            best = subset
    out = np.zeros(m, dtype=np.uint8)
    out[list(best)] = 1
    return out


@pytest.mark.parametrize("n,m", [(6, 8), (2, 4), (1, 4), (3, 8), (7, 8), (2, 8), (4, 8)])
def test_mask_brute_force_tiny(n, m):
    """"N:M Mask Generation": per group of m along d_in keep the n largest |W|;
    brute force over subsets, with values drawn from a tiny set to force ties."""
    rng = np.random.default_rng(n * 10 + m)
    w = (rng.integers(-3, 4, size=(40, 4 * m)) * 0.25).astype(np.float32)
    mask = oracle.nm_mask(w, n, m)
    for r in range(w.shape[0]):
        for g in range(4):
            keys = [abs(float(x)) for x in w[r, g * m:(g + 1) * m]]
            np.testing.assert_array_equal(mask[r, g * m:(g + 1) * m], _brute_mask_group(keys, n))


@pytest.mark.parametrize("n,m", [(6, 8), (2, 4), (5, 8)])
def test_mask_exactly_n_and_matches_stable_sort(n, m):
    """Exactly n kept per group; equals numpy's stable argsort of -|W| (ties
    to the lower index, the reading for ties)."""
    w = wl.master_weights(200, 64 * m, seed=13)
    mask = oracle.nm_mask(w, n, m)
    groups = np.abs(w).reshape(-1, m)
    assert (mask.reshape(-1, m).sum(axis=1) == n).all()
    order = np.argsort(-groups, axis=1, kind="stable")
    ref = np.zeros_like(groups, dtype=np.uint8)
    np.put_along_axis(ref, order[:, :n], 1, axis=1)
    np.testing.assert_array_equal(mask.reshape(-1, m), ref)


def test_mask_degenerate_cases():
    # all keys equal (including -0 vs +0): the first n positions are kept
    w = np.array([[0.0, -0.0, 0.0, -0.0, 0.5, -0.5, 0.5, -0.5]], dtype=np.float32)
    np.testing.assert_array_equal(oracle.nm_mask(w, 2, 4).ravel(), [1, 1, 0, 0, 1, 1, 0, 0])
    # n == m keeps everything: the layer reduces to dense BitLinear
    w = wl.master_weights(8, 64, seed=2)
    assert oracle.nm_mask(w, 8, 8).all() and oracle.nm_mask(w, 4, 4).all()


def test_nm_equal_m_is_dense_bitlinear():
    """8:8 is dense BitLinear: W_eff == W_q."""
    w = wl.master_weights(32, 64, seed=9)
    layer = oracle.Layer(w, 8, 8)
    np.testing.assert_array_equal(layer.weff, layer.wq)


def test_mask_uses_master_not_quantized_weights():
    """The mask ranks |W| of the master weights, not |W_q|: two weights that
    both ternarise to +1 are still ordered by their master magnitude."""
    w = np.array([[0.9, 0.8, 0.7, 0.6, 0.1, 0.2, 0.3, 0.4]], dtype=np.float32)
    # all of the first four quantise to 1; 2:8 must keep the two largest masters
    np.testing.assert_array_equal(oracle.nm_mask(w, 2, 8).ravel(), [1, 1, 0, 0, 0, 0, 0, 0])


# ---------------------------------------------------------------------- packing

def _decode_pk2(packed, d_in):
    b = packed[:, : d_in // 4].astype(np.int16)
    codes = np.stack([(b >> (2 * j)) & 3 for j in range(4)], axis=-1).reshape(packed.shape[0], d_in)
    return (codes - 1).astype(np.int8)


def test_pk2_roundtrip_and_padding():
    w = wl.master_weights(16, 80, seed=4)  # 80/4 = 20 bytes -> padded to 32
    layer = oracle.Layer(w, 6, 8)
    pk = oracle.pack_pk2(layer.weff)
    assert pk.shape == (16, 32)
    np.testing.assert_array_equal(_decode_pk2(pk, 80), layer.weff)
    assert (pk[:, 20:] == 0x55).all()
    assert not ((pk[:, :20] >> 6) == 3).any()  # code 3 is never written


def test_nm_roundtrip():
    for n, m in [(6, 8), (2, 4), (3, 8)]:
        w = wl.master_weights(12, 96, seed=n + m)
        layer = oracle.Layer(w, n, m)
        vals, bm = oracle.pack_nm(layer.weff, layer.mask, n, m)
        for r in range(12):
            bits = np.array([(bm[r, k // 8] >> (k % 8)) & 1 for k in range(96)])
            np.testing.assert_array_equal(bits, layer.mask[r])
            kept = np.nonzero(bits)[0]
            codes = np.array([(vals[r, s // 4] >> (2 * (s % 4))) & 3 for s in range(len(kept))])
            dec = np.zeros(96, dtype=np.int8)
            dec[kept] = codes - 1
            np.testing.assert_array_equal(dec, layer.weff[r])


def _decode_sp24(vals, meta, d_in):
    """Independent decompression of the SP24 operand: group g's nibble gives
    the two positions of values 2g and 2g+1."""
    out = np.zeros((vals.shape[0], d_in), dtype=np.int8)
    for r in range(vals.shape[0]):
        for g in range(d_in // 4):
            nib = (int(meta[r, g // 2]) >> (4 * (g % 2))) & 0xF
            i0, i1 = nib & 3, nib >> 2
            assert i0 < i1, "positions must be distinct and ascending"
            out[r, 4 * g + i0] = vals[r, 2 * g]
            out[r, 4 * g + i1] = vals[r, 2 * g + 1]
    return out


def test_sp24_hand_example():
    """Two groups by hand: positions {1, 3} kept -> nibble 1 | 3 << 2 = 0xD;
    only position 2 kept -> completed with position 0 -> nibble 0 | 2 << 2 =
    0x8; metadata byte 0x8D; values [W1, W3, W4, W6]; zero padding."""
    weff = np.array([[0, 1, 0, -1, 0, 0, 1, 0] + [0] * 8], dtype=np.int8)
    mask = np.array([[0, 1, 0, 1, 0, 0, 1, 0] + [1, 1, 0, 0] * 2], dtype=np.uint8)
    vals, meta = oracle.pack_sp24(weff, mask)
    assert vals.shape == (1, 16) and meta.shape == (1, 16)
    np.testing.assert_array_equal(vals[0, :8], [1, -1, 0, 1, 0, 0, 0, 0])
    np.testing.assert_array_equal(meta[0, :2], [0x8D, 0x44])
    assert (vals[0, 8:] == 0).all() and (meta[0, 2:] == 0).all()


@pytest.mark.parametrize("n,m", [(2, 4), (1, 4), (2, 8), (1, 8)])
def test_sp24_roundtrip(n, m):
    """Every 2:4-compatible mask (n <= 2 of 4, n <= 2 of 8) round-trips: the
    decompressed operand equals W_eff, and each stored position is a kept
    one unless the group keeps fewer than two."""
    w = wl.master_weights(16, 96, seed=10 * n + m)
    layer = oracle.Layer(w, n, m)
    vals, meta = oracle.pack_sp24(layer.weff, layer.mask)
    assert vals.shape == (16, oracle.sp24_value_row_bytes(96)) == (16, 48)
    assert meta.shape == (16, oracle.sp24_meta_row_bytes(96)) == (16, 16)
    np.testing.assert_array_equal(_decode_sp24(vals, meta, 96), layer.weff)
    for r in range(16):
        for g in range(24):
            nib = (int(meta[r, g // 2]) >> (4 * (g % 2))) & 0xF
            chosen = {nib & 3, nib >> 2}
            kept = set(np.nonzero(layer.mask[r, 4 * g: 4 * g + 4])[0])
            assert kept <= chosen
            # completion uses the smallest positions not kept
            fill = sorted(chosen - kept)
            assert fill == sorted(set(range(4)) - kept)[: len(fill)]


def test_sp24_rejects_masks_that_are_not_2of4():
    w = wl.master_weights(16, 64, seed=3)
    layer = oracle.Layer(w, 6, 8)
    with pytest.raises(ValueError):
        oracle.pack_sp24(layer.weff, layer.mask)


# ------------------------------------------------------------------- T24

T24_PAIRS = [(0, 1), (0, 2), (0, 3), (1, 2), (1, 3), (2, 3)]


def _t24_group_of_code(c):
    """The group of four ternary weights a 6-bit T24 code stands for, read
    off the code's definition (not from the oracle)."""
    g = [0, 0, 0, 0]
    if c == 0:
        return g
    if c <= 8:
        p, neg = divmod(c - 1, 2)
        g[p] = -1 if neg else 1
        return g
    k, rest = divmod(c - 9, 4)
    p, q = T24_PAIRS[k]
    g[p] = -1 if rest & 2 else 1
    g[q] = -1 if rest & 1 else 1
    return g


def _t24_decode(lo, hi, d_in):
    d_out = lo.shape[0]
    w = np.zeros((d_out, d_in), dtype=np.int8)
    for o in range(d_out):
        for g in range(d_in // 4):
            c = ((int(lo[o, g // 2]) >> (4 * (g % 2))) & 15) | (((int(hi[o, g // 4]) >> (2 * (g % 4))) & 3) << 4)
            assert c <= 32, "codes above 32 are never written"
            w[o, 4 * g:4 * g + 4] = _t24_group_of_code(c)
    return w


def test_t24_hand_row():
    """Groups (0,0,0,0) (0,0,-1,0) (1,0,0,-1) (0,-1,1,0) have codes 0, 1 + 2*2
    + 1 = 6, 9 + 4*2 + 0 + 1 = 18 ((0,3) is pair 2), 9 + 4*3 + 2 + 0 = 23
    ((1,2) is pair 3): low plane bytes 0x60 0x72, high plane byte
    0 | 0 << 2 | 1 << 4 | 1 << 6 = 0x50; padding zero."""
    w = np.array([[0, 0, 0, 0, 0, 0, -1, 0, 1, 0, 0, -1, 0, -1, 1, 0]], dtype=np.int8)
    lo, hi = oracle.pack_t24(w)
    assert lo.shape == (1, 16) and hi.shape == (1, 16)
    assert list(lo[0, :2]) == [0x60, 0x72] and not lo[0, 2:].any()
    assert hi[0, 0] == 0x50 and not hi[0, 1:].any()


def test_t24_all_groups():
    """Every one of the 81 sign patterns of a group: the 33 with at most two
    nonzeros get 33 distinct codes in 0..32 that decode back to the group;
    the 48 others are refused."""
    seen = set()
    for digits in itertools.product([-1, 0, 1], repeat=4):
        w = np.zeros((1, 16), dtype=np.int8)
        w[0, 4:8] = digits  # group 1: low nibble 1 of byte 0, high bits 2..3
        if sum(1 for v in digits if v) > 2:
            with pytest.raises(ValueError):
                oracle.pack_t24(w)
            continue
        lo, hi = oracle.pack_t24(w)
        c = (int(lo[0, 0]) >> 4) | (((int(hi[0, 0]) >> 2) & 3) << 4)
        assert c <= 32 and c not in seen
        seen.add(c)
        assert _t24_group_of_code(c) == list(digits)
        assert lo[0, 0] & 15 == 0 and hi[0, 0] & 0xF3 == 0  # the zero groups stay zero
    assert seen == set(range(33))


@pytest.mark.parametrize("n,m", [(2, 4), (1, 4), (2, 8), (1, 8)])
def test_t24_roundtrip(n, m):
    """Layers with 2:4-compatible masks: an independent decoder of the two
    planes gives W_eff back; padding bytes are zero."""
    w = wl.master_weights(48, 272, seed=n * 10 + m)
    layer = oracle.Layer(w, n, m)
    lo, hi = oracle.pack_t24(layer.weff)
    np.testing.assert_array_equal(_t24_decode(lo, hi, 272), layer.weff)
    assert not lo[:, 272 // 8:].any() and not hi[:, 272 // 16:].any()


def test_t24_rejects_masks_that_are_not_2of4():
    w = wl.master_weights(16, 64, seed=5)
    with pytest.raises(ValueError):
        oracle.pack_t24(oracle.Layer(w, 6, 8).weff)


# ------------------------------------------------------ RMSNorm + act quant

def _np_rmsnorm_quant(xb, gb, eps):
    """The fused definition in numpy float32 steps, with the row's sum of
    squares taken exactly (math.fsum) -- the oracle's fp64 tree of exact
    squares rounds only at its additions."""
    x = (xb.astype(np.uint32) << 16).view(np.float32)
    g = None if gb is None else (gb.astype(np.uint32) << 16).view(np.float32)
    t, k = x.shape
    q = np.zeros((t, k), dtype=np.int8)
    d = np.zeros((t,), dtype=np.float32)
    for i in range(t):
        s = math.fsum(float(v) * float(v) for v in x[i])
        r = np.float32(1.0 / math.sqrt(s / k + float(np.float32(eps))))
        u = (x[i] * r).astype(np.float32)
        if g is not None:
            u = (u * g).astype(np.float32)
        a = np.float32(np.abs(u).max())
        if a == 0:
            continue
        rq = np.float32(np.float32(127) / a)
        q[i] = np.clip(np.rint((u * rq).astype(np.float32)), -128, 127).astype(np.int8)
        d[i] = np.float32(a / np.float32(127))
    return q, d


def test_rmsnorm_quant_matches_numpy_definition():
    """RMSNorm fused into the quantiser ("The Full Sparse-BitLinear Layer",
    forward step 1: x~ = Q_a(Norm(x))): the same float32 steps in numpy."""
    x = wl.activations(16, 896, seed=21, outlier_frac=0.01)
    x[3] = 0  # a zero row stays zero
    g = wl.activations(1, 896, seed=22)[0]
    for gb, eps in [(None, 1e-5), (g, 1e-6), (g, 0.0)]:
        q, d = oracle.rmsnorm_quantize_act(x, gb, eps)
        if eps == 0.0:
            continue  # the zero row has 0/0 without eps
        qn, dn = _np_rmsnorm_quant(x, gb, eps)
        np.testing.assert_array_equal(q, qn)
        np.testing.assert_array_equal(d, dn)
        assert (np.abs(q[np.arange(16) != 3]).max(axis=1) == 127).all() and not q[3].any() and d[3] == 0


def test_rmsnorm_quant_scale_invariance_and_torch():
    """With eps = 0 and no gains the normalised row does not depend on a
    power-of-two scale of x (every step scales exactly); the normalised
    values agree with torch's fp64 rms_norm to fp32 precision."""
    x = wl.activations(8, 512, seed=23)
    xf = (x.astype(np.uint32) << 16).view(np.float32)
    x4 = ((xf * np.float32(4.0)).view(np.uint32) >> 16).astype(np.uint16)  # exact in bf16
    q1, d1 = oracle.rmsnorm_quantize_act(x, None, 0.0)
    q4, d4 = oracle.rmsnorm_quantize_act(x4, None, 0.0)
    np.testing.assert_array_equal(q1, q4)
    np.testing.assert_array_equal(d1, d4)
    ref = torch.nn.functional.rms_norm(torch.from_numpy(xf.astype(np.float64)), (512,), eps=1e-5).numpy()
    _, d = oracle.rmsnorm_quantize_act(x, None, 1e-5)
    amax = np.abs(ref).max(axis=1)
    np.testing.assert_allclose(d * 127, amax, rtol=2e-7)


# --------------------------------------------------------------- epilogue

def test_epilogue_hand_values():
    """ReLU^2 ("Squared ReLU Activation": max(0, x)^2) then the residual:
    [-2, -0, 0.5, 3] -> [0, 0, 0.25, 9]; + 1 -> [1, 1, 1.25, 10] (exact),
    bf16 of 1.25 = 0x3FA0."""
    y = np.array([[-2.0, -0.0, 0.5, 3.0]], dtype=np.float32)
    out, _ = oracle.epilogue(y, relu2=True)
    np.testing.assert_array_equal(out, [[0.0, 0.0, 0.25, 9.0]])
    assert not np.signbit(out).any()
    one = np.full((1, 4), 0x3F80, dtype=np.uint16)
    out, ob = oracle.epilogue(y, relu2=True, residual_bf16_bits=one)
    np.testing.assert_array_equal(out, [[1.0, 1.0, 1.25, 10.0]])
    assert ob[0, 2] == 0x3FA0
    out, _ = oracle.epilogue(y, residual_bf16_bits=one)
    np.testing.assert_array_equal(out, [[-1.0, 1.0, 1.5, 4.0]])


def test_epilogue_matches_numpy_float32_and_torch_bf16():
    rng = np.random.default_rng(8)
    y = (rng.standard_normal((64, 96)) * 40).astype(np.float32)
    r = torch.from_numpy(rng.standard_normal((64, 96)).astype(np.float32)).to(torch.bfloat16)
    rb = r.view(torch.int16).numpy().view(np.uint16)
    out, ob = oracle.epilogue(y, relu2=True, residual_bf16_bits=rb)
    sq = np.where(y > 0, y * y, np.float32(0)).astype(np.float32)
    expect = (sq + r.to(torch.float32).numpy()).astype(np.float32)
    np.testing.assert_array_equal(out, expect)
    np.testing.assert_array_equal(ob, torch.from_numpy(expect).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16))


# ------------------------------------------------------- ablation variants

def test_gamma_survivors_hand_row_and_exact_mean():
    """Mask-then-quant ("Composition Order": gamma from only the Top-N active
    weights): the golden 1x8 row keeps 0.9, 0.7, 0.5, 0.3, 0.2, 0.1 at 6:8, so
    gamma = 2.7 / 6 (not / 8); on random layers gamma is within one fp32 ulp
    of the exact rational mean of the kept |W|, equals the plain gamma at
    n = m, and exceeds it otherwise (the survivors are the largest)."""
    row = np.array([[0.9, -0.1, 0.5, -0.7, 0.05, 0.3, -0.2, 0.0]], dtype=np.float32)
    mask = oracle.nm_mask(row, 6, 8)
    kept = [Fraction(float(abs(v))) for v, k in zip(row[0], mask[0]) if k]
    assert oracle.gamma_survivors(row, mask) == np.float32(float(sum(kept) / 6))
    for (n, m) in [(6, 8), (2, 4), (3, 8)]:
        w = wl.master_weights(48, 96, seed=n + m)
        mask = oracle.nm_mask(w, n, m)
        g = oracle.gamma_survivors(w, mask)
        exact = sum(Fraction(float(abs(v))) for v in w[mask == 1]) / int(mask.sum())
        assert abs(Fraction(float(g)) - exact) <= Fraction(float(np.spacing(g)))
        assert g > oracle.gamma(w)
    w = wl.master_weights(16, 64, seed=9)
    assert oracle.gamma_survivors(w, oracle.nm_mask(w, 8, 8)) == oracle.gamma(w)


def test_mask_from_quantized_hand_and_brute_force():
    """Mask from |W_q| ("Where the mask is computed"): W_q = [1,0,1,-1,0,1,-1,0]
    at 6:8 keeps the five nonzeros and then the lowest-index zero (position
    1); in general the top-n of a stable descending order of |W_q|."""
    wq = np.array([[1, 0, 1, -1, 0, 1, -1, 0]], dtype=np.int8)
    np.testing.assert_array_equal(oracle.nm_mask_quantized(wq, 6, 8)[0], [1, 1, 1, 1, 0, 1, 1, 0])
    rng = np.random.default_rng(4)
    for n, m in [(6, 8), (2, 4), (3, 8), (1, 4)]:
        q = rng.integers(-1, 2, size=(16, 64)).astype(np.int8)
        got = oracle.nm_mask_quantized(q, n, m)
        g = (q != 0).astype(np.int8).reshape(16, 64 // m, m)
        order = np.argsort(-g, axis=-1, kind="stable")
        expect = np.zeros_like(g)
        np.put_along_axis(expect, order[..., :n], 1, axis=-1)
        np.testing.assert_array_equal(got, expect.reshape(16, 64))


def test_layer_variants_invariants():
    """Layer options: mask-then-quant keeps exactly the master mask and zeroes
    every dropped position; the quantized-weight mask keeps every nonzero
    W_q it can (a group with at most n nonzeros keeps all of them)."""
    w = wl.master_weights(32, 64, seed=12)
    base = oracle.Layer(w, 6, 8)
    mtq = oracle.Layer(w, 6, 8, order="mask_then_quant")
    np.testing.assert_array_equal(mtq.mask, base.mask)
    assert not mtq.weff[mtq.mask == 0].any()
    qm = oracle.Layer(w, 6, 8, mask_source="quantized")
    nz = (qm.wq != 0).reshape(32, 8, 8).sum(-1)
    kept_nz = ((qm.wq != 0) & (qm.mask == 1)).reshape(32, 8, 8).sum(-1)
    np.testing.assert_array_equal(kept_nz, np.minimum(nz, 6))
    with pytest.raises(ValueError):
        oracle.Layer(w, 6, 8, mask_source="quantized", order="mask_then_quant")


# ----------------------------------------------------------- mask statistics

def test_mask_flips_matches_numpy_and_invariants():
    """Flip count between consecutive masks ("Dynamic Mask Recomputation":
    how many positions change): numpy's != count; 0 for equal masks; every
    position for complementary masks."""
    w0 = wl.master_weights(32, 128, seed=1)
    w1 = w0 + 0.01 * wl.master_weights(32, 128, seed=2)  # a small update moves some positions
    m0 = oracle.nm_mask(w0, 6, 8)
    m1 = oracle.nm_mask(w1, 6, 8)
    f = oracle.mask_flips(m0, m1)
    assert f == int((m0 != m1).sum()) and 0 < f < m0.size
    assert f % 2 == 0  # exactly n per group: every drop is matched by an entry
    assert oracle.mask_flips(m0, m0) == 0
    assert oracle.mask_flips(m0, 1 - m0) == m0.size


def test_near_zero_matches_numpy_and_gaussian_closed_form():
    """Near-zero mass ("Polarization analysis": |W|/gamma below 0.5) as a
    count: numpy float32 division; for W ~ N(0, s) the fraction tends to
    2 Phi(0.5 sqrt(2/pi)) - 1 = 0.3101 (gamma -> s sqrt(2/pi)); every weight
    counts when gamma == 0."""
    w = wl.master_weights(2048, 2048, seed=7)
    g = oracle.gamma(w)
    c = oracle.near_zero(w, g)
    assert c == int((np.abs(w) / np.float32(g) < np.float32(0.5)).sum())
    frac = c / w.size
    expect = math.erf(0.5 * math.sqrt(2 / math.pi) / math.sqrt(2))
    assert abs(frac - expect) < 1.5e-3, (frac, expect)
    assert oracle.near_zero(np.zeros((4, 16), np.float32), 0.0) == 64
    # exactly 0.5 gamma is not below 0.5; the next float down is
    w2 = np.array([[0.5, np.nextafter(np.float32(0.5), np.float32(0)), 1.0, 0.25] * 4], dtype=np.float32)
    assert oracle.near_zero(w2, 1.0) == 8


def test_block_threshold_brute_force_and_hand_row():
    """Per-block threshold ("Magnitude stratification": the (N+1)-th largest
    |W| of each block): the golden 1x8 row at 6:8 drops 0.05 and 0.0, so
    t = 0.05; brute force by sorting on tie-heavy groups; 0 when n == m;
    never above a kept magnitude."""
    row = np.array([[0.9, -0.1, 0.5, -0.7, 0.05, 0.3, -0.2, 0.0] + [0.0] * 8], dtype=np.float32)
    mask = oracle.nm_mask(row, 6, 8)
    assert oracle.block_threshold(row, mask, 8)[0, 0] == np.float32(0.05)
    rng = np.random.default_rng(5)
    for n, m in [(6, 8), (2, 4), (5, 8), (1, 4), (3, 8)]:
        w = (rng.integers(-3, 4, size=(16, 64)) * 0.25).astype(np.float32)
        mask = oracle.nm_mask(w, n, m)
        t = oracle.block_threshold(w, mask, m)
        a = np.abs(w).reshape(16, 64 // m, m)
        expect = -np.sort(-a, axis=-1)[..., n]
        np.testing.assert_array_equal(t, expect)
        kept_min = np.where(mask.reshape(a.shape) == 1, a, np.inf).min(axis=-1)
        assert (t <= kept_min).all()
    w = wl.master_weights(8, 32, seed=3)
    assert not oracle.block_threshold(w, oracle.nm_mask(w, 8, 8), 8).any()


# ------------------------------------------------------------ activation quant

def test_act_quant_invariants_and_zero_row():
    """Per-token absmax ("Activation Quantization: Per-Token Absmax"): every
    nonzero row reaches |q| = 127 exactly at its absmax, zero rows give q = 0
    and d = 0, and |q| never exceeds 127."""
    x = wl.activations(33, 256, seed=1, outlier_frac=0.01)
    x[5] = 0
    x[6] = 0x8000  # all -0.0
    q, d = oracle.quantize_act(x)
    xf = wl.bf16_bits_to_f32(x)
    for t in range(33):
        if np.abs(xf[t]).max() == 0:
            assert not q[t].any() and d[t] == 0
        else:
            assert np.abs(q[t]).max() == 127
            assert d[t] == np.float32(np.abs(xf[t]).max()) / np.float32(127)
    assert np.abs(q.astype(np.int32)).max() <= 127


def test_act_quant_matches_numpy_float32():
    """Special case reducing to library routines: numpy float32 arithmetic of
    x * fl(127 / a) with rint (half-even)."""
    x = wl.activations(50, 320, seed=2)
    xf = wl.bf16_bits_to_f32(x)
    a = np.abs(xf).max(axis=1)
    r = (np.float32(127) / a).astype(np.float32)
    ref = np.clip(np.rint(xf * r[:, None]), -128, 127).astype(np.int8)
    q, d = oracle.quantize_act(x)
    np.testing.assert_array_equal(q, ref)
    np.testing.assert_array_equal(d, (a / np.float32(127)).astype(np.float32))


def test_act_quant_tiny_by_hand():
    # x = [2, -1, 0.5, 0] -> a = 2, r = 63.5; q = [127, -63.5 -> -64 (half-even), 31.75 -> 32, 0]
    x = wl.f32_to_bf16_bits(np.array([[2.0, -1.0, 0.5, 0.0]], dtype=np.float32))
    q, d = oracle.quantize_act(x)
    np.testing.assert_array_equal(q.ravel(), [127, -64, 32, 0])
    assert d[0] == np.float32(2.0) / np.float32(127.0)


# ---------------------------------------------------------------------- forward

def test_gemm_acc_matches_numpy_int64():
    w = wl.master_weights(96, 256, seed=6)
    layer = oracle.Layer(w, 6, 8)
    q, d = oracle.quantize_act(wl.activations(40, 256, seed=6))
    acc = oracle.gemm_acc(q, layer.weff)
    np.testing.assert_array_equal(acc, q.astype(np.int64) @ layer.weff.astype(np.int64).T)


def test_gemm_acc_brute_force_tiny():
    q = np.array([[1, -2, 3, 127]], dtype=np.int8)
    weff = np.array([[1, 0, -1, 1], [-1, -1, -1, -1]], dtype=np.int8)
    np.testing.assert_array_equal(oracle.gemm_acc(q, weff), [[1 - 3 + 127, -(1 - 2 + 3 + 127)]])


def test_output_matches_fp64_definition():
    """y = s * (W_eff x~) with s = gamma * max|x| / 127 ("The Full
    Sparse-BitLinear Layer", forward step 5) within 1e-6 normwise of an fp64
    numpy evaluation, and the bf16 output equals torch's CPU RNE rounding."""
    w = wl.master_weights(128, 256, seed=0)
    x = wl.activations(64, 256, seed=0, outlier_frac=0.01)
    layer = oracle.Layer(w, 6, 8)
    q, d, acc, y, yb = layer.forward(x)
    ref = (q.astype(np.float64) * d.astype(np.float64)[:, None]) @ \
          (float(layer.gamma) * layer.weff.astype(np.float64)).T
    assert np.abs(y - ref).max() / np.abs(ref).max() < 1e-6
    tb = torch.from_numpy(y).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(yb, tb)


# --------------------------------------------------------------------- backward

def _setup_bwd(n, m, t=24, o=40, k=64, seed=8):
    w = wl.master_weights(o, k, seed=seed)
    x = wl.activations(t, k, seed=seed)
    dy = wl.output_grad(t, o, seed=seed)
    layer = oracle.Layer(w, n, m)
    q, d = oracle.quantize_act(x)
    return w, layer, q, d, dy


def test_backward_matches_numpy_fp64():
    """Dual STE ("dL/dW ~= dL/dW_eff"): dX = gamma dY W_eff, dW = dY^T X~."""
    w, layer, q, d, dy = _setup_bwd(6, 8)
    dx, dw = oracle.backward(dy, layer.weff, layer.gamma, q, d)
    dyf = wl.bf16_bits_to_f32(dy).astype(np.float64)
    np.testing.assert_allclose(dx, float(layer.gamma) * dyf @ layer.weff.astype(np.float64), rtol=1e-12, atol=1e-12)
    xt = q.astype(np.float64) * d.astype(np.float64)[:, None]
    np.testing.assert_allclose(dw, dyf.T @ xt, rtol=1e-12, atol=1e-12)


def test_dual_ste_dw_independent_of_mask_and_dense_at_masked_positions():
    """Dual STE passes the gradient through the mask as identity: dW is the
    same for every n:m and is nonzero at masked positions too."""
    dws = []
    for n, m in [(8, 8), (6, 8), (2, 4), (3, 8)]:
        w, layer, q, d, dy = _setup_bwd(n, m)
        _, dw = oracle.backward(dy, layer.weff, layer.gamma, q, d, want_dx=False)
        dws.append(dw)
        masked = layer.mask == 0
        if masked.any():
            assert (np.abs(dw[masked]) > 0).mean() > 0.99
    for dw in dws[1:]:
        np.testing.assert_array_equal(dw, dws[0])


def test_dx_at_n_equal_m_is_dense_bitlinear():
    """At n = m the layer is dense BitLinear, so dX uses W_q itself."""
    w, layer, q, d, dy = _setup_bwd(8, 8)
    dx, _ = oracle.backward(dy, layer.wq, layer.gamma, q, d, want_dw=False)
    dx2, _ = oracle.backward(dy, layer.weff, layer.gamma, q, d, want_dw=False)
    np.testing.assert_array_equal(dx, dx2)


def test_sampled_variants_agree_with_full():
    w, layer, q, d, dy = _setup_bwd(6, 8, t=16, o=24, k=32)
    dx, dw = oracle.backward(dy, layer.weff, layer.gamma, q, d)
    acc = oracle.gemm_acc(q, layer.weff)
    rng = np.random.default_rng(0)
    it, io, ik = rng.integers(0, 16, 50), rng.integers(0, 24, 50), rng.integers(0, 32, 50)
    np.testing.assert_array_equal(oracle.acc_samples(q, layer.weff, it, io), acc[it, io])
    np.testing.assert_array_equal(oracle.dx_samples(dy, layer.weff, layer.gamma, it, ik), dx[it, ik])
    np.testing.assert_array_equal(oracle.dw_samples(dy, q, d, io, ik), dw[io, ik])


# -------------------------------------------------------- planted-mistake check

def test_pins_catch_planted_mistakes():
    """A plausible slip in the oracle's arithmetic (here re-implemented in
    numpy with a dropped term / wrong tie rule / wrong rounding) fails the
    same pins, which shows the pins have teeth."""
    # wrong tie rule (higher index wins) fails the all-equal case
    keys = np.zeros(8, dtype=np.float32)
    wrong = np.zeros(8, dtype=np.uint8)
    wrong[np.argsort(-keys, kind="stable")[::-1][:6]] = 1
    assert not np.array_equal(wrong, oracle.nm_mask(keys.reshape(1, 8), 6, 8).ravel())
    # round-half-away instead of half-even fails the 0.5 tie
    assert np.float32(np.floor(0.5 + 0.5)) != oracle.ternarize(np.array([0.5], dtype=np.float32), 1.0)[0]
    # sequential instead of pairwise summation fails the order pin
    a = 2.0 ** -53
    seq = 0.0
    for v in [1.0, a, a, a]:
        seq += v
    assert seq != oracle.abs_sum(np.array([1.0, a, a, a], dtype=np.float32))
