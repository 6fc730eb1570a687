"""CPU restatement of the dW operand's power-of-two prescale (the backward's
grad_absmax_kernel and transpose_to_f16_kernel<0>), checked against what it
must achieve and against the oracle's exact Dual-STE dW.

The kernel picks s from the fp32 bits of M = max |fl32(dY d_t)|:
s = clamp(141 - e, -126, 126) with e the biased exponent (at least 1), so that
M 2^s lies in [2^14, 2^15); the operand is fp16(fl32(dY d_t) 2^s) and the GEMM
result is multiplied by 2^-s.  Restated here in numpy (float32 products, the
IEEE fp16 conversion, an fp64 stand-in for the tensor core's fp32
accumulation), it must keep dW within the 1e-3 float tolerance for gradients of
any magnitude -- which the unscaled fp16 operand does not.
"""
import numpy as np
import pytest

import oracle
from sparsity_sbl_quantize_b200 import workloads as wl


def prescale_exponent(m_bits: int) -> int:
    if m_bits == 0:
        return 0
    e = (m_bits >> 23) & 0xFF
    s = 141 - max(e, 1)
    return min(126, max(-126, s))


def test_exponent_puts_max_in_top_binades():
    rng = np.random.default_rng(0)
    # every binade of normal fp32 values, several mantissas each
    for e in range(1, 255):
        for mant in (0, 1, 0x400000, 0x7FFFFF, int(rng.integers(0, 1 << 23))):
            bits = (e << 23) | mant
            m = float(np.array([bits], dtype=np.uint32).view(np.float32)[0])
            s = prescale_exponent(bits)
            scaled = m * 2.0 ** s
            if -126 < 141 - e < 126:
                assert 2.0 ** 14 <= scaled < 2.0 ** 15, (e, mant, s)
            # never above fp16's range, even after rounding to fp16
            assert np.float16(scaled) < np.inf
            assert scaled < 2.0 ** 15
    # subnormal fp32 maxima and zero
    assert prescale_exponent(1) == 126 and prescale_exponent(0x7FFFFF) == 126
    assert prescale_exponent(0) == 0


def dw_fp16_model(dy_bits, q, d, prescale: bool):
    """dW as the GPU forms it: fp16 operands, products accumulated (in fp64
    here: the tensor core's fp32 accumulation adds far less error than the
    fp16 operand rounding), then times 2^-s."""
    dy = (dy_bits.astype(np.uint32) << 16).view(np.float32)
    prod = (dy * d[:, None].astype(np.float32)).astype(np.float32)  # fl32(dY d_t)
    s = 0
    if prescale:
        m = np.abs(prod).max()
        s = prescale_exponent(int(np.array([m], dtype=np.float32).view(np.uint32)[0]))
        prod = (prod * np.float32(2.0 ** s)).astype(np.float32)  # exact
    a = prod.astype(np.float16).astype(np.float64)
    return (a.T @ q.astype(np.float64)) * 2.0 ** -s


def scaled_bits(bits, k):
    v = ((bits.astype(np.uint32) << 16).view(np.float32) * np.float32(2.0 ** k)).astype(np.float32)
    b = v.view(np.uint32)
    assert not (b & 0xFFFF).any()
    return (b >> 16).astype(np.uint16)


@pytest.mark.parametrize("dy_exp", [-30, -20, -10, 0, 6])
def test_prescaled_fp16_operand_meets_tolerance(dy_exp):
    T, O, K = 96, 48, 64
    x = wl.activations(T, K, seed=21)
    dy = scaled_bits(wl.output_grad(T, O, seed=21), dy_exp)
    q, d = oracle.quantize_act(x)
    weff = np.zeros((O, K), dtype=np.int8)
    _, dw_ref = oracle.backward(dy, weff, np.float32(1.0), q, d, want_dx=False)
    den = np.abs(dw_ref).max()
    err = np.abs(dw_fp16_model(dy, q, d, True) - dw_ref).max() / den
    assert err <= 1e-3, err
    if dy_exp <= -20:
        # without the prescale the small products flush to zero in fp16
        err0 = np.abs(dw_fp16_model(dy, q, d, False) - dw_ref).max() / den
        assert err0 > 1e-2, err0
