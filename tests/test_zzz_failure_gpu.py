"""Failure detection on the GPU without a fault: the bounded wait every
kernel uses gives up on an mbarrier that nothing arrives at, records its bit
in the device error word, and the context stays usable (a forward run right
after it still equals the oracle).  Takes the wait limit, about 1 s.
Collected after the other GPU files."""
import numpy as np
import pytest
import torch

import oracle
from sparsity_sbl_quantize_b200 import workloads as wl

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():  # the gpu marker deselects these on CPU hosts
    pytest.skip("needs a CUDA device", allow_module_level=True)

from gpu_case import GpuLayer, bits_of, forward, quantize_act, sbl_mod  # noqa: E402


def test_expired_wait_is_reported_and_the_context_survives():
    sbl = sbl_mod()
    assert sbl.sbl_device_error(clear=True) == 0
    sbl.sbl_selftest_wait_expiry()
    code = sbl.sbl_device_error(clear=True)  # synchronises
    assert code == sbl.SBL_DEVICE_ERROR_SELFTEST
    assert sbl.sbl_device_error() == 0
    w = wl.master_weights(128, 256, seed=4)
    x = wl.activations(64, 256, seed=4)
    layer = GpuLayer(w, 6, 8, sbl.SBL_FMT_I8)
    q, d = quantize_act(x)
    yb, acc = forward(layer, q, d, sbl.SBL_FMT_I8)
    _, _, accr, _, ybr = oracle.Layer(w, 6, 8).forward(x)
    np.testing.assert_array_equal(acc.cpu().numpy(), accr)
    np.testing.assert_array_equal(bits_of(yb), ybr)
    assert sbl.sbl_device_error() == 0
