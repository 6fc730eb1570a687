"""The packing kernel's threshold forms equal the divisions they replace.

Ternarisation ("Step 2: Rescale and RoundClip", Sparse-BitNet summary
section 3.4) sets W_q != 0 exactly when clamp(rint(fl32(|w| / gamma))) is 1,
and the near-zero count (the "Polarization analysis" of the same summary)
counts fl32(|w| / gamma) < 0.5.  The kernel computes neither division:
it compares |w| with a bound derived once from gamma,

  ternary:   T = the first fp32 strictly above gamma * (0.5 + 2^-25)
  near-zero: B = the first fp32 at or above gamma * (0.5 - 2^-26)

(both products exact in fp64).  These CPU tests restate the two bounds and
check them against the correctly rounded fp32 division (numpy, IEEE
round-to-nearest-even) on the floats around each bound and on random
weights, for scales across the fp32 exponent range.
"""
import numpy as np

F32 = np.float32
INF = F32(np.inf)


def round_up_to_f32(t: float) -> np.float32:
    """The smallest fp32 >= t (t a double)."""
    f = F32(t)
    if float(f) < t:
        f = np.nextafter(f, INF)
    return f


def ternary_threshold(gamma: np.float32) -> np.float32:
    if not gamma > 0:
        return INF
    t = float(gamma) * (0.5 + 2.0 ** -25)
    f = round_up_to_f32(t)
    if float(f) == t:
        f = np.nextafter(f, INF)
    return f


def near_zero_bound(gamma: np.float32) -> np.float32:
    if not gamma > 0:
        return INF
    return round_up_to_f32(float(gamma) * (0.5 - 2.0 ** -26))


def candidates(bound: np.float32, rng, n_random=200):
    """The floats within 4 ulps of the bound, and random ones nearby."""
    c = [bound]
    lo = hi = bound
    for _ in range(4):
        lo, hi = np.nextafter(lo, F32(0)), np.nextafter(hi, INF)
        c += [lo, hi]
    c += list((bound * rng.uniform(0.25, 4.0, n_random)).astype(F32))
    return np.array([v for v in c if np.isfinite(v)], dtype=F32)


def gammas(rng):
    exps = np.arange(-100, 100, 7)
    g = (rng.uniform(1.0, 2.0, exps.size) * 2.0 ** exps).astype(F32)
    return list(g) + [F32(1.0), F32(0.75), F32(0.02), np.nextafter(F32(1.0), F32(2))]


def test_ternary_threshold_equals_the_rounded_division():
    rng = np.random.default_rng(1)
    with np.errstate(over="ignore"):
        for g in gammas(rng):
            thr = ternary_threshold(g)
            x = candidates(thr, rng)
            q = np.clip(np.rint(x / g), 0, 1)              # fl32 division, half-even rounding
            np.testing.assert_array_equal(q == 1, x >= thr, err_msg=f"gamma={g!r}")


def test_near_zero_bound_equals_the_rounded_division():
    rng = np.random.default_rng(2)
    with np.errstate(over="ignore"):
        for g in gammas(rng):
            b = near_zero_bound(g)
            x = candidates(b, rng)
            np.testing.assert_array_equal((x / g) < F32(0.5), x < b, err_msg=f"gamma={g!r}")


def test_boundary_cases_by_hand():
    """gamma = 1: exactly 0.5 rounds to 0 and is not near zero; the float
    just above 0.5 ternarises to 1; the float just below 0.5 is near zero."""
    g = F32(1.0)
    half = F32(0.5)
    up, down = np.nextafter(half, INF), np.nextafter(half, F32(0))
    assert ternary_threshold(g) == up
    assert near_zero_bound(g) == half
    assert np.rint(half / g) == 0 and np.rint(up / g) == 1
    assert not (half / g) < half and (down / g) < half
    assert ternary_threshold(F32(0.0)) == INF and near_zero_bound(F32(0.0)) == INF
