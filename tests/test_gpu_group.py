"""GPU parity of the grouped int8 forward (sbl_forward_group): several layers
on the same activations in one launch give, bit for bit, the outputs of one
SBL_FMT_I8 sbl_forward per layer (which the parity tests pin to the oracle),
and the oracle's directly on a small case -- for one to four layers, widths
that are not multiples of the 256-column tile, token counts on and off the
CTA-pair path, bf16 and fp32 outputs."""
import numpy as np
import pytest
import torch

import oracle
from sparsity_sbl_quantize_b200 import workloads as wl

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():  # the gpu marker deselects these on CPU hosts
    pytest.skip("needs a CUDA device", allow_module_level=True)

from gpu_case import GpuLayer, bits_of, quantize_act, sbl_mod  # noqa: E402


def packed_layer(O, K, n, m, seed):
    w = wl.master_weights(O, K, seed=seed)
    return GpuLayer(w, n, m, sbl_mod().SBL_FMT_I8), oracle.Layer(w, n, m)


@pytest.mark.parametrize("T,K,outs,fp32", [
    (4096, 896, (4864, 4864), False),        # the MLP's gate and up
    (8192, 1536, (1536, 256, 256), False),   # q, k, v of a 1.5B decoder layer
    (300, 512, (272, 1040, 48, 784), False), # ragged widths and tokens, four groups
    (100, 256, (512, 128), True),            # one CTA-row of tokens (no pairs), fp32
    (1, 64, (16,), False),                   # a single layer, a single token
    (64, 256, (8192, 8192, 8192, 4864), False),  # 256-wide tiles on single CTAs (T <= 128)
    (1000, 256, (4864, 4880, 48), True),     # CTA pairs with a partial last pair of row tiles, fp32
])
def test_group_equals_one_launch_per_layer(T, K, outs, fp32):
    sbl = sbl_mod()
    layers = [packed_layer(O, K, 6, 8, seed=O + 7 * i)[0] for i, O in enumerate(outs)]
    x = wl.activations(T, K, seed=T + K)
    q, d = quantize_act(x)
    dt = torch.float32 if fp32 else torch.bfloat16
    ys = [torch.full((T, O), 7, dtype=dt, device="cuda") for O in outs]
    refs = [torch.empty((T, O), dtype=dt, device="cuda") for O in outs]
    for L, r in zip(layers, refs):
        sbl.sbl_forward(L.desc, q, d, T, L.packed, sbl.SBL_FMT_I8, r, y_is_fp32=fp32)
    sbl.sbl_forward_group([L.desc for L in layers], q, d, T, [L.packed for L in layers], ys, y_is_fp32=fp32)
    torch.cuda.synchronize()
    assert sbl.sbl_device_error() == 0
    for y, r in zip(ys, refs):
        view = torch.int32 if fp32 else torch.int16
        assert torch.equal(y.view(view), r.view(view))


def test_group_matches_the_oracle():
    sbl = sbl_mod()
    T, K, outs = 200, 320, (160, 96)
    pairs = [packed_layer(O, K, 2, 4, seed=31 + O) for O in outs]
    x = wl.activations(T, K, seed=5)
    q, d = quantize_act(x)
    ys = [torch.empty((T, O), dtype=torch.bfloat16, device="cuda") for O in outs]
    sbl.sbl_forward_group([L.desc for L, _ in pairs], q, d, T, [L.packed for L, _ in pairs], ys)
    torch.cuda.synchronize()
    for y, (_, ref) in zip(ys, pairs):
        _, _, _, _, yb = ref.forward(x)
        np.testing.assert_array_equal(bits_of(y), yb)
