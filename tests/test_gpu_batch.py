"""GPU parity of the batched (persistent, streaming) decode forward,
sbl_forward_batch, against the oracle: every output bit-exact.

Independent layers of mixed shapes (both item sizes: 32-row items for
K <= 7168, 16-row items above; ragged last row blocks; fp32 outputs), and
chains in which each layer quantises the previous layer's bf16 output in the
kernel, checked against the oracle run layer by layer (its activation
quantisation of that bf16 output, GEMM and dequantisation).
"""
import numpy as np
import pytest
import torch

import oracle
from sparsity_sbl_quantize_b200 import workloads as wl

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():  # the gpu marker deselects these on CPU hosts
    pytest.skip("needs a CUDA device", allow_module_level=True)

from gpu_case import GpuLayer, bf16_dev, bits_of, quantize_act, sbl_mod  # noqa: E402


def packed_layer(O, K, n, m, seed):
    w = wl.master_weights(O, K, seed=seed)
    return GpuLayer(w, n, m, 1), oracle.Layer(w, n, m)


def oracle_forward_bits(ref, x_bits):
    _, _, _, y, yb = ref.forward(x_bits)
    return y, yb


@pytest.mark.parametrize("T", [1, 3, 8, 9, 16])
def test_batch_independent_layers_bit_exact(T):
    sbl = sbl_mod()
    shapes = [(2560, 6912, 2, 4), (6912, 2560, 2, 4), (48, 320, 6, 8), (64, 8960, 2, 4), (96, 64, 1, 4),
              (272, 1536, 7, 8)]
    entries, keep = [], []
    for i, (O, K, n, m) in enumerate(shapes):
        layer, ref = packed_layer(O, K, n, m, seed=100 + i)
        x = wl.activations(T, K, seed=200 + i)
        q, d = quantize_act(x)
        fp32 = i == 2
        y = torch.empty((T, O), dtype=torch.float32 if fp32 else torch.bfloat16, device="cuda")
        entries.append(sbl.batch_layer(layer.desc, layer.packed, y, q, d, y_is_fp32=fp32))
        keep.append((layer, ref, x, q, d, y, fp32))
    arr = sbl.batch_array(entries)
    ws = sbl.alloc_workspace(sbl.sbl_forward_batch_workspace_bytes(arr, len(entries), T))
    sbl.sbl_forward_batch(arr, len(entries), T, ws)
    torch.cuda.synchronize()
    assert sbl.sbl_device_error() == 0
    for layer, ref, x, q, d, y, fp32 in keep:
        yr, ybr = oracle_forward_bits(ref, x)
        if fp32:
            np.testing.assert_array_equal(y.cpu().numpy().view(np.uint32), yr.view(np.uint32))
        else:
            np.testing.assert_array_equal(bits_of(y), ybr)


@pytest.mark.parametrize("T", [1, 4, 16])
def test_batch_chain_matches_oracle_layer_by_layer(T):
    """A chain of six layers (256 -> 512 -> 256 -> ... and a 7168-wide step):
    each layer after the first reads the previous bf16 output, quantises it
    per token inside the kernel and stores the quantised input and scales."""
    sbl = sbl_mod()
    dims = [256, 512, 256, 7168, 320, 512, 256]
    x0 = wl.activations(T, dims[0], seed=7, outlier_frac=0.01)
    q0, d0 = quantize_act(x0)
    entries, keep = [], []
    for i in range(len(dims) - 1):
        K, O = dims[i], dims[i + 1]
        layer, ref = packed_layer(O, K, 2 if i % 2 else 6, 4 if i % 2 else 8, seed=300 + i)
        y = torch.empty((T, O), dtype=torch.bfloat16, device="cuda")
        if i == 0:
            e = sbl.batch_layer(layer.desc, layer.packed, y, q0, d0)
            xq_out = d_out = None
        else:
            xq_out = torch.full((T, K), 99, dtype=torch.int8, device="cuda")
            d_out = torch.full((max(T, 4),), -1.0, dtype=torch.float32, device="cuda")
            e = sbl.batch_layer(layer.desc, layer.packed, y, chained=True, xq_out=xq_out, d_out=d_out)
        entries.append(e)
        keep.append((ref, y, xq_out, d_out, layer))  # the layer's buffers must outlive the call
    arr = sbl.batch_array(entries)
    nws = sbl.sbl_forward_batch_workspace_bytes(arr, len(entries), T)
    assert nws >= 128 * len(entries)
    ws = sbl.alloc_workspace(nws)
    for rep in range(2):  # a second call on the same workspace starts from zero again
        sbl.sbl_forward_batch(arr, len(entries), T, ws)
        torch.cuda.synchronize()
        assert sbl.sbl_device_error() == 0
        x_bits = x0
        for i, (ref, y, xq_out, d_out, _) in enumerate(keep):
            qr, dr, accr, yr, ybr = ref.forward(x_bits)
            if xq_out is not None:
                np.testing.assert_array_equal(xq_out.cpu().numpy(), qr)
                np.testing.assert_array_equal(d_out.cpu().numpy()[:T], dr)
            np.testing.assert_array_equal(bits_of(y), ybr, err_msg=f"layer {i}")
            x_bits = ybr  # the next layer's input, as the oracle runs it


def test_batch_chain_then_independent_layer():
    """A chained pair followed by an independent layer with its own input."""
    sbl = sbl_mod()
    T = 2
    a, ra = packed_layer(512, 256, 6, 8, seed=1)
    b, rb = packed_layer(256, 512, 6, 8, seed=2)
    c, rc = packed_layer(128, 640, 2, 4, seed=3)
    xa, xc = wl.activations(T, 256, seed=4), wl.activations(T, 640, seed=5)
    qa, da = quantize_act(xa)
    qc, dc = quantize_act(xc)
    ya = torch.empty((T, 512), dtype=torch.bfloat16, device="cuda")
    yb = torch.empty((T, 256), dtype=torch.bfloat16, device="cuda")
    yc = torch.empty((T, 128), dtype=torch.bfloat16, device="cuda")
    arr = sbl.batch_array([sbl.batch_layer(a.desc, a.packed, ya, qa, da),
                           sbl.batch_layer(b.desc, b.packed, yb, chained=True),
                           sbl.batch_layer(c.desc, c.packed, yc, qc, dc)])
    ws = sbl.alloc_workspace(sbl.sbl_forward_batch_workspace_bytes(arr, 3, T))
    sbl.sbl_forward_batch(arr, 3, T, ws)
    torch.cuda.synchronize()
    _, yab = oracle_forward_bits(ra, xa)
    np.testing.assert_array_equal(bits_of(ya), yab)
    np.testing.assert_array_equal(bits_of(yb), oracle_forward_bits(rb, yab)[1])
    np.testing.assert_array_equal(bits_of(yc), oracle_forward_bits(rc, xc)[1])


def test_batch_full_decode_workload_equals_single_launches():
    """The BitNet-2B decode shapes at T = 1, 4, 16 with several weight copies in
    one batch: identical to one sbl_forward (PK2) launch per layer, which the
    parity tests pin to the oracle."""
    sbl = sbl_mod()
    wk = wl.WORKLOADS["bitnet2b_decode"]
    n, m = wk.patterns[0]
    layers = [packed_layer(lin.d_out, lin.d_in, n, m, seed=wk.seed + li)[0] for li, lin in enumerate(wk.linears)]
    for T in wk.tokens:
        entries, outs = [], []
        for rep in range(3):
            for li, lin in enumerate(wk.linears):
                x = wl.activations(T, lin.d_in, seed=wk.seed + 10 * rep + li)
                q, d = quantize_act(x)
                y = torch.empty((T, lin.d_out), dtype=torch.bfloat16, device="cuda")
                y1 = torch.empty_like(y)
                sbl.sbl_forward(layers[li].desc, q, d, T, layers[li].packed, sbl.SBL_FMT_PK2, y1)
                entries.append(sbl.batch_layer(layers[li].desc, layers[li].packed, y, q, d))
                outs.append((y, y1, q, d))
        arr = sbl.batch_array(entries)
        ws = sbl.alloc_workspace(sbl.sbl_forward_batch_workspace_bytes(arr, len(entries), T))
        sbl.sbl_forward_batch(arr, len(entries), T, ws)
        torch.cuda.synchronize()
        for y, y1, _, _ in outs:
            assert torch.equal(y.view(torch.int16), y1.view(torch.int16))
    assert sbl.sbl_device_error() == 0
