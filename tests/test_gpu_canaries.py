"""Guard bands around every output and workspace: each buffer a call writes
sits inside a larger allocation whose 4 KiB before and after hold a fixed
byte; after the call on ragged shapes (partial tiles, K tails, odd token
counts) the bands must be untouched.  This stands in for a memory checker,
which is not available where the GPU tests run."""
import numpy as np
import pytest
import torch

import oracle
from sparsity_sbl_quantize_b200 import workloads as wl

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():  # the gpu marker deselects these on CPU hosts
    pytest.skip("needs a CUDA device", allow_module_level=True)

from gpu_case import bf16_dev, sbl_mod  # noqa: E402

GUARD = 4096
CANARY = 0xA5


class Guarded:
    """Buffers carved out of guard-banded allocations."""

    def __init__(self):
        self.blocks = []

    def take(self, shape, dtype):
        nbytes = int(np.prod(shape)) * torch.empty((), dtype=dtype).element_size()
        nbytes = max(nbytes, 16)
        raw = torch.full((GUARD + nbytes + GUARD,), CANARY, dtype=torch.uint8, device="cuda")
        self.blocks.append((raw, nbytes))
        inner = raw[GUARD:GUARD + nbytes]
        n = int(np.prod(shape))
        return inner.view(dtype)[:n].view(*shape) if n else inner.view(dtype)[:0]

    def check(self):
        torch.cuda.synchronize()
        for raw, nbytes in self.blocks:
            assert bool((raw[:GUARD] == CANARY).all()), "write before the buffer"
            assert bool((raw[GUARD + nbytes:] == CANARY).all()), "write after the buffer"


def _packed(sbl, g, d, formats):
    O, K = d.out_features, d.in_features
    p = sbl.Packed(gamma=g.take((4,), torch.float32))
    rb = lambda f, b=sbl.SBL_BUF_MAIN: sbl.sbl_packed_row_bytes(d, f, b)  # noqa: E731
    if formats & sbl.SBL_FMT_PK2:
        p.pk2 = g.take((O, rb(sbl.SBL_FMT_PK2)), torch.uint8)
    if formats & sbl.SBL_FMT_NM:
        p.nm_values = g.take((O, rb(sbl.SBL_FMT_NM)), torch.uint8)
        p.nm_bitmap = g.take((O, rb(sbl.SBL_FMT_NM, sbl.SBL_BUF_NM_BITMAP)), torch.uint8)
    if formats & sbl.SBL_FMT_I8:
        p.i8 = g.take((O, K), torch.int8)
    if formats & sbl.SBL_FMT_BF16T:
        p.bf16t = g.take((K, O), torch.bfloat16)
    if formats & sbl.SBL_FMT_SP24:
        p.sp24_values = g.take((O, rb(sbl.SBL_FMT_SP24)), torch.int8)
        p.sp24_meta = g.take((O, rb(sbl.SBL_FMT_SP24, sbl.SBL_BUF_SP24_META)), torch.uint8)
    if formats & sbl.SBL_FMT_T24:
        p.t24_lo = g.take((O, rb(sbl.SBL_FMT_T24)), torch.uint8)
        p.t24_hi = g.take((O, rb(sbl.SBL_FMT_T24, sbl.SBL_BUF_T24_HI)), torch.uint8)
    return p


# shapes the parity tests run with every format named here: partial tiles in
# O, T and K (528 x 1040 x 300), and the decode's many-chunk rows (11008)
@pytest.mark.parametrize("O,K,T,n,m", [(528, 1040, 300, 6, 8), (528, 1040, 300, 2, 4), (48, 11008, 7, 2, 4),
                                       (64, 2048, 12, 2, 8)])
def test_guard_bands_pack_act_forward_backward(O, K, T, n, m):
    sbl = sbl_mod()
    g = Guarded()
    d = sbl.desc(O, K, n, m)
    fm = sbl.SBL_FMT_PK2 | sbl.SBL_FMT_NM | sbl.SBL_FMT_I8 | sbl.SBL_FMT_BF16T
    if n <= 2:
        fm |= sbl.SBL_FMT_SP24 | sbl.SBL_FMT_T24
    w = torch.from_numpy(wl.master_weights(O, K, seed=O + K)).cuda()
    p = _packed(sbl, g, d, fm)
    ws = g.take((sbl.sbl_workspace_bytes(d, 0, sbl.SBL_OP_QUANTIZE_MASK_PACK),), torch.uint8)
    sbl.sbl_quantize_mask_pack(d, w, fm, p, ws)
    # the packing writes its buffers exactly as the oracle packs them
    ref = oracle.Layer(wl.master_weights(O, K, seed=O + K), n, m)
    np.testing.assert_array_equal(p.i8.cpu().numpy(), ref.weff)

    x = wl.activations(T, K, seed=T)
    xd = bf16_dev(x)
    q, dv = g.take((T, K), torch.int8), g.take((T,), torch.float32)
    sbl.sbl_quantize_act(xd, T, K, q, dv)
    q2, d2 = g.take((T, K), torch.int8), g.take((T,), torch.float32)
    sbl.sbl_quantize_act_rmsnorm(xd, T, K, None, 1e-5, q2, d2)

    fmts = [sbl.SBL_FMT_I8] + ([sbl.SBL_FMT_SP24] if n <= 2 else [])
    if T <= 16 and K % 64 == 0:
        fmts += [sbl.SBL_FMT_PK2] + ([sbl.SBL_FMT_T24] if n <= 2 else [])
    for fmt in fmts:
        yb = g.take((T, O), torch.bfloat16)
        yf = g.take((T, O), torch.float32)
        acc = g.take((T, O), torch.int32)
        sbl.sbl_forward(d, q, dv, T, p, fmt, yb, False, acc)
        sbl.sbl_forward(d, q, dv, T, p, fmt, yf, True, None)
        res = bf16_dev(wl.activations(T, O, seed=1))
        ye = g.take((T, O), torch.bfloat16)
        sbl.sbl_forward_ex(d, q, dv, T, p, fmt, ye, relu2=True, residual=res)
        ql, dl, yl = g.take((T, K), torch.int8), g.take((T,), torch.float32), g.take((T, O), torch.bfloat16)
        sbl.sbl_linear_forward(d, xd, T, p, fmt, ql, dl, yl)

    dy = bf16_dev(wl.output_grad(T, O, seed=T))
    bws = g.take((sbl.sbl_workspace_bytes(d, T, sbl.SBL_OP_BACKWARD),), torch.uint8)
    dx = g.take((T, K), torch.float32)
    dw = g.take((O, K), torch.float32)
    sbl.sbl_backward_dual_ste(d, dy, q, dv, T, p, dx, True, dw, bws)
    dxb = g.take((T, K), torch.bfloat16)
    sbl.sbl_backward_dual_ste(d, dy, q, dv, T, p, dxb, False, None, bws)
    g.check()
    assert sbl.sbl_device_error(clear=True) == 0


def test_guard_bands_fused_decode_one_token():
    """The fused decode (one launch, CTA 0 also stores Xq and d) at T = 1."""
    sbl = sbl_mod()
    g = Guarded()
    O, K, T = 96, 2560, 1
    d = sbl.desc(O, K, 2, 4)
    p = _packed(sbl, g, d, sbl.SBL_FMT_PK2)
    ws = g.take((sbl.sbl_workspace_bytes(d, 0, sbl.SBL_OP_QUANTIZE_MASK_PACK),), torch.uint8)
    sbl.sbl_quantize_mask_pack(d, torch.from_numpy(wl.master_weights(O, K, seed=3)).cuda(), sbl.SBL_FMT_PK2, p, ws)
    xd = bf16_dev(wl.activations(T, K, seed=4))
    q, dv, y = g.take((T, K), torch.int8), g.take((T,), torch.float32), g.take((T, O), torch.bfloat16)
    sbl.sbl_linear_forward(d, xd, T, p, sbl.SBL_FMT_PK2, q, dv, y)
    g.check()
    qr, dr = oracle.quantize_act(wl.activations(T, K, seed=4))
    np.testing.assert_array_equal(q.cpu().numpy(), qr)
    np.testing.assert_array_equal(dv.cpu().numpy(), dr)
