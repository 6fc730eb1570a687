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


def test_guard_bands_batched_decode_and_sharding():
    """The batched decode (independent layers with ragged row blocks and a
    chain storing its quantised inputs) and the sharded weight side write
    only their buffers, workspaces included."""
    sbl = sbl_mod()
    g = Guarded()
    T = 3
    shapes = [(48, 320), (80, 8960), (272, 1536)]  # items of 4, 1 and 2 tiles, partial last items
    entries, keep = [], []
    for i, (O, K) in enumerate(shapes):
        d = sbl.desc(O, K, 2, 4)
        p = _packed(sbl, g, d, sbl.SBL_FMT_PK2)
        ws = g.take((sbl.sbl_workspace_bytes(d, 0, sbl.SBL_OP_QUANTIZE_MASK_PACK),), torch.uint8)
        sbl.sbl_quantize_mask_pack(d, torch.from_numpy(wl.master_weights(O, K, seed=i)).cuda(), sbl.SBL_FMT_PK2, p, ws)
        q, dv = g.take((T, K), torch.int8), g.take((T,), torch.float32)
        sbl.sbl_quantize_act(bf16_dev(wl.activations(T, K, seed=i)), T, K, q, dv)
        y = g.take((T, O), torch.bfloat16)
        entries.append(sbl.batch_layer(d, p, y, q, dv))
        keep.append((p, q, dv, y))
    # a chained pair 320 -> 64 -> 128 after them (its first layer shares the
    # first input above)
    d1 = sbl.desc(64, 320, 6, 8)
    p1 = _packed(sbl, g, d1, sbl.SBL_FMT_PK2)
    d2 = sbl.desc(128, 64, 6, 8)
    p2 = _packed(sbl, g, d2, sbl.SBL_FMT_PK2)
    for i, (d, p) in enumerate(((d1, p1), (d2, p2))):
        ws = g.take((sbl.sbl_workspace_bytes(d, 0, sbl.SBL_OP_QUANTIZE_MASK_PACK),), torch.uint8)
        w = torch.from_numpy(wl.master_weights(d.out_features, d.in_features, seed=10 + i)).cuda()
        sbl.sbl_quantize_mask_pack(d, w, sbl.SBL_FMT_PK2, p, ws)
    q1, d1v = keep[0][1], keep[0][2]
    y1, y2 = g.take((T, 64), torch.bfloat16), g.take((T, 128), torch.bfloat16)
    xo, do = g.take((T, 64), torch.int8), g.take((T,), torch.float32)
    entries.append(sbl.batch_layer(d1, p1, y1, q1, d1v))
    entries.append(sbl.batch_layer(d2, p2, y2, chained=True, xq_out=xo, d_out=do))
    arr = sbl.batch_array(entries)
    bws = g.take((sbl.sbl_forward_batch_workspace_bytes(arr, len(entries), T),), torch.uint8)
    sbl.sbl_forward_batch(arr, len(entries), T, bws)

    # sharded weight side: two shards of a 1104 x 2048 layer
    O, K = 1104, 2048
    w = torch.from_numpy(wl.master_weights(O, K, seed=5)).cuda()
    from sparsity_sbl_quantize_b200 import sharding
    parts = []
    for first, rows in sharding.column_shards(O, K, 2):
        ds = sbl.desc(rows, K, 6, 8)
        ws = g.take((sbl.sbl_workspace_bytes(ds, 0, sbl.SBL_OP_QUANTIZE_MASK_PACK),), torch.uint8)
        nodes = g.take((sbl.sbl_gamma_node_count(ds),), torch.float64)
        sbl.sbl_gamma_partials(ds, w[first:first + rows].contiguous(), first, nodes, ws)
        parts.append((ds, first, rows, nodes))
    allnodes = torch.cat([n for *_, n in parts])
    for ds, first, rows, _ in parts:
        p = _packed(sbl, g, ds, sbl.SBL_FMT_I8 | sbl.SBL_FMT_PK2)
        sbl.sbl_gamma_combine(allnodes, allnodes.numel(), O * K, p.gamma)
        sbl.sbl_quantize_mask_pack_shard(ds, w[first:first + rows].contiguous(), sbl.SBL_FMT_I8 | sbl.SBL_FMT_PK2, p)
    g.check()
    assert sbl.sbl_device_error(clear=True) == 0


@pytest.mark.parametrize("T,outs", [(300, (528, 48, 784)), (100, (528, 48, 784)),
                                    (1000, (4864, 4880, 48))])  # 128-wide tiles; 256-wide on CTA pairs
def test_guard_bands_grouped_forward(T, outs):
    """The grouped int8 forward writes only each layer's output: ragged
    widths and a partial last token tile, bf16 and fp32."""
    sbl = sbl_mod()
    g = Guarded()
    K = 1040
    descs, packs = [], []
    for i, O in enumerate(outs):
        d = sbl.desc(O, K, 6, 8)
        p = _packed(sbl, g, d, sbl.SBL_FMT_I8)
        ws = g.take((sbl.sbl_workspace_bytes(d, 0, sbl.SBL_OP_QUANTIZE_MASK_PACK),), torch.uint8)
        sbl.sbl_quantize_mask_pack(d, torch.from_numpy(wl.master_weights(O, K, seed=20 + i)).cuda(),
                                   sbl.SBL_FMT_I8, p, ws)
        descs.append(d)
        packs.append(p)
    q, dv = g.take((T, K), torch.int8), g.take((T,), torch.float32)
    sbl.sbl_quantize_act(bf16_dev(wl.activations(T, K, seed=3)), T, K, q, dv)
    for fp32 in (False, True):
        ys = [g.take((T, O), torch.float32 if fp32 else torch.bfloat16) for O in outs]
        sbl.sbl_forward_group(descs, q, dv, T, packs, ys, y_is_fp32=fp32)
    g.check()
    assert sbl.sbl_device_error(clear=True) == 0
