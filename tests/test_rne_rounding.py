"""CPU restatement of the quantisers' rounding: fl32(v + 1.5 * 2^23) in
round-to-nearest-even fp32 leaves rint(v) (half to even) in the low byte of
its bits, for every product the quantiser forms (|v| <= 127 (1 + 2^-24)),
ties included; checked against numpy's rint on every fp32 near each integer
and half-integer of [-128, 128] and on random values, and the packing order
(byte i = code i) against the oracle's activation quantiser."""
import numpy as np

import oracle
from sparsity_sbl_quantize_b200 import workloads as wl

MAGIC = np.float32(12582912.0)


def rne_byte(v):
    s = (np.asarray(v, dtype=np.float32) + MAGIC).astype(np.float32)
    return (s.view(np.uint32) & 0xFF).astype(np.uint8).view(np.int8)


def test_low_byte_is_round_half_even():
    vals = []
    for k in np.arange(-256, 257) / 2.0:  # integers and half-integers
        f = np.float32(k)
        for step in range(-6, 7):
            x = f
            for _ in range(abs(step)):
                x = np.nextafter(x, np.float32(np.inf if step > 0 else -np.inf), dtype=np.float32)
            vals.append(x)
    vals = np.array(vals, dtype=np.float32)
    vals = vals[np.abs(vals) <= np.float32(127.0) * np.float32(1 + 2.0 ** -23)]
    rng = np.random.default_rng(0)
    vals = np.concatenate([vals, rng.uniform(-127.0, 127.0, 100000).astype(np.float32)])
    np.testing.assert_array_equal(rne_byte(vals), np.rint(vals).astype(np.int8))


def test_packed_codes_match_the_oracle_quantiser():
    x = wl.activations(7, 256, seed=3, outlier_frac=0.05)
    q_ref, d_ref = oracle.quantize_act(x)
    xf = wl.bf16_bits_to_f32(x)
    amax = np.abs(xf).max(axis=1)
    r = np.float32(127.0) / amax.astype(np.float32)
    q = rne_byte((xf * r[:, None]).astype(np.float32))
    np.testing.assert_array_equal(q, q_ref)
