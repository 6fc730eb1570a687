"""GPU parity: the CUDA path through the C ABI against the CPU oracle.

Integer stages (gamma, W_eff in every packed format, q, d, int32 accumulators)
and the forward outputs must match bit for bit; the backward's fp32 results
must be within 1e-3 normwise (max |gpu - ref| / max |ref|), the float
tolerance the benchmark spec states.  Small cases compare every element and span
several tiles with ragged tails; the full workload sizes compare all integer
stages in full and the GEMM outputs at seeded sample coordinates.
"""
import numpy as np
import pytest
import torch

import oracle
from sparsity_sbl_quantize_b200 import workloads as wl

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():  # the gpu marker deselects these on CPU hosts
    pytest.skip("needs a CUDA device", allow_module_level=True)

from gpu_case import (ALL_FORMATS, GpuLayer, bf16_bits_to_f64, bf16_dev, bf16_ulp, bits_of,  # noqa: E402
                      elementwise_rel, f32_to_bf16_bits, forward, normwise, quantize_act, sbl_mod, to_dev)

FWD_TOL = 1e-3  # only used where bit-exactness is not expected (backward)


SP24 = 16
T24 = 32


def check_pack(w, n, m, formats=ALL_FORMATS):
    if n <= 2 and formats == ALL_FORMATS:
        formats |= SP24 | T24  # the 2:4 formats exist for 2:4-compatible masks
    layer = GpuLayer(w, n, m, formats)
    got = layer.host()
    ref = oracle.Layer(w, n, m)
    assert got["gamma"] == ref.gamma, (got["gamma"], ref.gamma)
    if "i8" in got:
        np.testing.assert_array_equal(got["i8"], ref.weff)
    if "pk2" in got:
        np.testing.assert_array_equal(got["pk2"], oracle.pack_pk2(ref.weff))
    if "nm_values" in got:
        vals, bm = oracle.pack_nm(ref.weff, ref.mask, n, m)
        np.testing.assert_array_equal(got["nm_bitmap"], bm)
        np.testing.assert_array_equal(got["nm_values"], vals)
    if "bf16t" in got:
        expect = np.where(ref.weff.T > 0, 0x3F80, np.where(ref.weff.T < 0, 0xBF80, 0)).astype(np.uint16)
        np.testing.assert_array_equal(got["bf16t"], expect)
    if "sp24_values" in got:
        vals, meta = oracle.pack_sp24(ref.weff, ref.mask)
        np.testing.assert_array_equal(got["sp24_values"], vals)
        np.testing.assert_array_equal(got["sp24_meta"], meta)
    if "t24_lo" in got:
        lo, hi = oracle.pack_t24(ref.weff)
        np.testing.assert_array_equal(got["t24_lo"], lo)
        np.testing.assert_array_equal(got["t24_hi"], hi)
    return layer, ref


# ------------------------------------------------------------------- packing

@pytest.mark.parametrize("O,K,n,m", [(128, 256, 6, 8), (48, 80, 6, 8), (64, 96, 2, 4), (32, 64, 1, 4),
                                     (16, 16, 3, 4), (96, 160, 7, 8), (64, 128, 8, 8), (32, 64, 4, 4),
                                     (80, 208, 3, 8), (528, 1040, 5, 8)])
def test_pack_bit_exact(O, K, n, m):
    check_pack(wl.master_weights(O, K, seed=O + K + n), n, m)


def test_pack_gamma_multi_block_tree():
    """> 16384 weights: several first-level partials plus the last-block tree,
    with a count that is not a power of two."""
    check_pack(wl.master_weights(1008, 1040, seed=21), 6, 8)


def test_pack_gamma_summation_order():
    """An input on which the order of the fp64 sum decides gamma's fp32
    rounding: |W| sums to 2^30 + 64 (the mean lands on an fp32 midpoint) plus
    8192 x 2^-35 in the second tree node.  Summed pairwise (as the R1 tree
    does) the tiny values survive and gamma rounds up; added one by one to the
    large partial they are lost and the tie rounds to even (down)."""
    w = np.zeros((64, 256), dtype=np.float32)
    w[0, 0], w[0, 1] = 2.0 ** 30, -64.0
    w.reshape(-1)[8192:] = 2.0 ** -35
    w.reshape(-1)[8192::3] *= -1.0
    seq = 0.0
    for v in np.abs(w.astype(np.float64)).reshape(-1):
        seq += v
    gamma_seq = np.float32(seq / w.size)
    ref = oracle.Layer(w, 6, 8)
    assert ref.gamma != gamma_seq  # the input discriminates the two orders
    assert ref.gamma == np.float32((2.0 ** 30 + 64 + 2.0 ** -22) / w.size)
    check_pack(w, 6, 8)


@pytest.mark.parametrize("n,m", [(6, 8), (2, 4), (2, 8), (1, 4), (3, 4), (7, 8), (5, 8), (3, 8), (1, 8), (4, 8)])
def test_pack_ties_zero_and_signed_zero(n, m):
    """Tie-heavy weights (few distinct magnitudes), all-zero and all -0.0 rows:
    the kept set must follow the lower-index rule in every selection path."""
    w = (np.random.default_rng(3).integers(-2, 3, size=(64, 128)) * 0.125).astype(np.float32)
    w[5] = 0.0
    w[6] = -0.0
    w[7, ::2] = -0.0
    check_pack(w, n, m)


def test_pack_all_zero_matrix_gamma_zero():
    layer, ref = check_pack(np.zeros((32, 64), dtype=np.float32), 6, 8)
    assert ref.gamma == 0.0 and not layer.host()["i8"].any()


def test_pack_rounding_boundaries():
    """Weights at and next to the 0.5 * gamma rounding boundary (gamma = 1
    exactly for these rows) hit the threshold test on both sides."""
    base = np.array([0.5, -0.5, 1.5, -1.5, 2.5, -2.5] + [0.75] * 8 + [0.5, 0.5], dtype=np.float32)
    up = np.nextafter(np.float32(0.5), np.float32(1))
    dn = np.nextafter(np.float32(0.5), np.float32(0))
    w = np.tile(base, (16, 4)).reshape(16, 64)
    w[1, 0], w[2, 0], w[3, 0], w[4, 0] = up, -up, dn, -dn
    check_pack(w, 8, 8)


# -------------------------------------------------------- re-mask statistics

def bitmap_of(mask):
    """Oracle mask (one byte per position) -> keep bitmap rows (bit k%8 of
    byte k/8, rows padded to 16 bytes)."""
    o, k = mask.shape
    rb = oracle.nm_bitmap_row_bytes(k)
    out = np.zeros((o, rb), dtype=np.uint8)
    out[:, : k // 8] = np.packbits(mask.astype(np.uint8).reshape(o, k // 8, 8)[..., ::-1], axis=-1)[..., 0]
    return out


@pytest.mark.parametrize("O,K,n,m", [(128, 256, 6, 8), (48, 80, 2, 4), (96, 160, 7, 8), (64, 128, 8, 8),
                                     (528, 1040, 5, 8), (32, 64, 1, 4), (1008, 1040, 2, 8)])
def test_pack_stats_bit_exact(O, K, n, m):
    """Keep bitmap, flip count against the mask of slightly perturbed
    weights, near-zero count and per-group thresholds: exactly the oracle's,
    with and without the SP24 instantiation."""
    sbl = sbl_mod()
    w_prev = wl.master_weights(O, K, seed=O + K)
    w = w_prev + np.float32(0.003) * wl.master_weights(O, K, seed=O + K + 1)
    ref_prev = oracle.Layer(w_prev, n, m)
    ref = oracle.Layer(w, n, m)
    dsc = sbl.desc(O, K, n, m)
    rb = sbl.keep_bitmap_bytes(dsc)
    prev = to_dev(bitmap_of(ref_prev.mask))
    fmts = sbl.SBL_FMT_I8 | (sbl.SBL_FMT_SP24 if n <= 2 else 0)
    for formats in (fmts, 0):
        p = sbl.alloc_packed(dsc, formats)
        ws = sbl.alloc_workspace(sbl.sbl_workspace_bytes(dsc, 0, sbl.SBL_OP_QUANTIZE_MASK_PACK))
        keep = torch.full((O, rb), 0xAB, dtype=torch.uint8, device="cuda")
        flips = torch.full((1,), -1, dtype=torch.int64, device="cuda")
        nz = torch.full((1,), -1, dtype=torch.int64, device="cuda")
        thr = torch.empty((O, K // m), dtype=torch.float32, device="cuda")
        sbl.sbl_quantize_mask_pack_stats(dsc, to_dev(w), formats, p, ws, prev_keep=prev, keep=keep, flips=flips,
                                         near_zero=nz, block_threshold=thr)
        np.testing.assert_array_equal(keep.cpu().numpy(), bitmap_of(ref.mask))
        assert int(flips.item()) == oracle.mask_flips(ref_prev.mask, ref.mask)
        assert int(nz.item()) == oracle.near_zero(w, ref.gamma)
        np.testing.assert_array_equal(thr.cpu().numpy().view(np.uint32),
                                      oracle.block_threshold(w, ref.mask, m).view(np.uint32))
        if formats & sbl.SBL_FMT_I8:
            np.testing.assert_array_equal(p.i8.cpu().numpy(), ref.weff)
        assert float(p.gamma[0].item()) == ref.gamma


def test_pack_stats_near_zero_boundary_and_zero_gamma():
    """Weights at and next to 0.5 gamma (gamma = 1 exactly): exactly 0.5 is
    not near zero, the float below is; an all-zero matrix counts every
    weight."""
    sbl = sbl_mod()
    base = np.array([0.5, -0.5, 1.5, -1.5, 2.5, -2.5] + [0.75] * 8 + [0.5, 0.5], dtype=np.float32)
    dn = np.nextafter(np.float32(0.5), np.float32(0))
    w = np.tile(base, (16, 4)).reshape(16, 64)
    w[1, 0], w[2, 0] = dn, -dn
    for mat in (w, np.zeros((16, 64), dtype=np.float32)):
        ref = oracle.Layer(mat, 6, 8)
        dsc = sbl.desc(16, 64, 6, 8)
        p = sbl.alloc_packed(dsc, sbl.SBL_FMT_I8)
        ws = sbl.alloc_workspace(sbl.sbl_workspace_bytes(dsc, 0, sbl.SBL_OP_QUANTIZE_MASK_PACK))
        nz = torch.zeros((1,), dtype=torch.int64, device="cuda")
        sbl.sbl_quantize_mask_pack_stats(dsc, to_dev(mat), sbl.SBL_FMT_I8, p, ws, near_zero=nz)
        assert int(nz.item()) == oracle.near_zero(mat, ref.gamma)


# -------------------------------------------------------------- activations

@pytest.mark.parametrize("T,K", [(64, 256), (300, 1040), (1, 16), (7, 8960), (33, 11008), (5, 32768)])
def test_act_quant_bit_exact(T, K):
    x = wl.activations(T, K, seed=T + K, outlier_frac=0.01)
    x[0] = 0  # an all-zero token
    q, d = quantize_act(x)
    qr, dr = oracle.quantize_act(x)
    np.testing.assert_array_equal(q.cpu().numpy(), qr)
    np.testing.assert_array_equal(d.cpu().numpy()[:T], dr)


def _gains(K, seed):
    rng = np.random.default_rng(seed)
    return wl.f32_to_bf16_bits(rng.normal(1.0, 0.25, size=K).astype(np.float32))


def rmsnorm_quantize_act(x_bits, g_bits, eps):
    sbl = sbl_mod()
    t, k = x_bits.shape
    q = torch.empty((t, k), dtype=torch.int8, device="cuda")
    d = torch.empty((max(t, 1),), dtype=torch.float32, device="cuda")
    g = None if g_bits is None else bf16_dev(g_bits)
    sbl.sbl_quantize_act_rmsnorm(bf16_dev(x_bits), t, k, g, eps, q, d)
    return q, d


# every thread-row width (32 .. 1024 threads), 1 .. 8 chunks per thread, ragged
# K within a slot, multi-row CTAs with an inactive tail row
@pytest.mark.parametrize("T,K", [(64, 256), (300, 1040), (1, 16), (7, 8960), (33, 11008), (5, 32768),
                                 (3, 65536), (9, 40960), (130, 2048), (5, 4112)])
@pytest.mark.parametrize("gains", [False, True])
def test_rmsnorm_act_quant_bit_exact(T, K, gains):
    x = wl.activations(T, K, seed=3 * T + K, outlier_frac=0.01)
    x[0] = 0  # an all-zero token: S = 0, r = 1/sqrt(eps), q = 0, d = 0
    if T > 2:
        x[2] = wl.f32_to_bf16_bits(wl.bf16_bits_to_f32(x[2]) * np.float32(1e-30))  # tiny magnitudes
    g = _gains(K, K) if gains else None
    for eps in (1e-5, 1e-6):
        q, d = rmsnorm_quantize_act(x, g, eps)
        qr, dr = oracle.rmsnorm_quantize_act(x, g, eps)
        np.testing.assert_array_equal(q.cpu().numpy(), qr)
        np.testing.assert_array_equal(d.cpu().numpy()[:T], dr)


def test_rmsnorm_act_quant_eps_zero_nonzero_rows():
    x = wl.activations(40, 896, seed=11)
    q, d = rmsnorm_quantize_act(x, None, 0.0)
    qr, dr = oracle.rmsnorm_quantize_act(x, None, 0.0)
    np.testing.assert_array_equal(q.cpu().numpy(), qr)
    np.testing.assert_array_equal(d.cpu().numpy()[:40], dr)


# ------------------------------------------------------------------- forward

def run_forward_full_check(O, K, T, n, m, seed, fmt_name="I8", outliers=0.0):
    sbl = sbl_mod()
    w = wl.master_weights(O, K, seed=seed)
    x = wl.activations(T, K, seed=seed, outlier_frac=outliers)
    layer = GpuLayer(w, n, m, 1 | 4)
    ref = oracle.Layer(w, n, m)
    q, d = quantize_act(x)
    qr, dr, accr, yr, ybr = ref.forward(x)
    np.testing.assert_array_equal(q.cpu().numpy(), qr)
    fmt = {"I8": sbl.SBL_FMT_I8, "PK2": sbl.SBL_FMT_PK2, "SP24": sbl.SBL_FMT_SP24, "T24": sbl.SBL_FMT_T24}[fmt_name]
    if fmt_name in ("SP24", "T24"):
        layer = GpuLayer(w, n, m, fmt)
    yb, acc = forward(layer, q, d, fmt)
    np.testing.assert_array_equal(acc.cpu().numpy(), accr)
    np.testing.assert_array_equal(bits_of(yb), ybr)
    yf, _ = forward(layer, q, d, fmt, fp32=True, want_acc=False)
    np.testing.assert_array_equal(yf.cpu().numpy(), yr)


@pytest.mark.parametrize("O,K,T,n,m", [
    (128, 256, 64, 6, 8),     # the single-layer workload shape
    (528, 1040, 300, 6, 8),   # 3 x 3 tiles, ragged M, N and K
    (256, 128, 128, 2, 4),    # exactly one tile
    (16, 16, 1, 1, 4),        # minimum sizes
    (784, 384, 257, 7, 8),
    (512, 640, 1000, 2, 8),
])
def test_forward_gemm_bit_exact(O, K, T, n, m):
    run_forward_full_check(O, K, T, n, m, seed=O + T)


def test_forward_single_layer_workload_outliers():
    wk = wl.WORKLOADS["single_256x128"]
    lin = wk.linears[0]
    n, m = wk.patterns[0]
    run_forward_full_check(lin.d_out, lin.d_in, wk.tokens[0], n, m, seed=wk.seed, outliers=wk.outlier_frac)


@pytest.mark.parametrize("O,K,T", [(256, 256, 1), (384, 640, 4), (528, 1088, 16), (6912, 2560, 16),
                                   (2560, 6912, 1), (2560, 6912, 9), (16, 64, 3),
                                   (48, 11008, 7),    # 43 K chunks: eight per warp
                                   (32, 16448, 16),   # two rounds of chunks, 64-weight last chunk
                                   (16, 192, 8),      # one partial chunk
                                   (48, 2560, 12)])   # a CTA of two 16-row groups, one past O
def test_forward_decode_pk2_bit_exact(O, K, T):
    run_forward_full_check(O, K, T, 2, 4, seed=O + K + T, fmt_name="PK2")


# T24: the decode kernel from the 6-bit group codes (2:4-compatible masks)
@pytest.mark.parametrize("O,K,T,n,m", [(48, 11008, 7, 2, 4), (32, 16448, 16, 2, 4), (16, 192, 8, 2, 4),
                                       (6912, 2560, 1, 2, 4), (2560, 6912, 16, 2, 4), (96, 1024, 3, 1, 4),
                                       (64, 2048, 12, 2, 8), (32, 512, 1, 1, 8)])
def test_forward_decode_t24_bit_exact(O, K, T, n, m):
    run_forward_full_check(O, K, T, n, m, seed=O + K + T + n, fmt_name="T24")


def test_forward_t24_epilogue_and_packed_planes():
    """Squared ReLU and the residual on the T24 decode; the planes the pack
    wrote next to SP24 equal the oracle's."""
    sbl = sbl_mod()
    O, K, T = 64, 2560, 5
    w = wl.master_weights(O, K, seed=9)
    x = wl.activations(T, K, seed=9)
    layer, ref = check_pack(w, 2, 4)
    _, _, _, yr, _ = ref.forward(x)
    res_bits = wl.activations(T, O, seed=10)
    _, outb = oracle.epilogue(yr, relu2=True, residual_bf16_bits=res_bits)
    q, d = quantize_act(x)
    y = torch.empty((T, O), dtype=torch.bfloat16, device="cuda")
    sbl.sbl_forward_ex(layer.desc, q, d, T, layer.packed, sbl.SBL_FMT_T24, y, relu2=True,
                       residual=bf16_dev(res_bits))
    np.testing.assert_array_equal(bits_of(y), outb)


def test_forward_decode_pk2_six_of_eight():
    run_forward_full_check(896, 4864, 5, 6, 8, seed=11, fmt_name="PK2")


@pytest.mark.parametrize("O,K,T,n,m", [
    (128, 256, 128, 2, 4),    # exactly one tile and one k-block
    (528, 1040, 300, 2, 4),   # ragged O, T, and K (16 past the last 256 block)
    (384, 1536, 520, 2, 8),   # 2:8 run on the 2:4 hardware path
    (16, 16, 5, 1, 4),        # minimum sizes
    (256, 896, 257, 1, 8),    # half k-block tail (896 = 3.5 x 256)
    (4864, 896, 64, 2, 4),    # the MLP gate/up shape, short T
])
def test_forward_sp24_bit_exact(O, K, T, n, m):
    run_forward_full_check(O, K, T, n, m, seed=O + K + T, fmt_name="SP24")


@pytest.mark.parametrize("O,K,T", [(896, 4864, 4096),    # MLP down projection (128-token pair tiles)
                                   (4864, 896, 4096),    # MLP gate/up (224-token pair tiles)
                                   (2048, 1024, 4000),   # 224-token tiles with a ragged last tile
                                   # the 1.5B decoder linears on which the format rule picks the
                                   # sparse kernel at T = 8192 (down, gate/up, q/o)
                                   (1536, 8960, 8192), (8960, 1536, 8192), (1536, 1536, 8192)])
def test_forward_sp24_matches_dense_path_full_size(O, K, T):
    """The sparse and dense tensor-core paths compute the same integers: at
    full workload sizes their accumulators and outputs agree bit for bit, and
    sampled accumulators match the oracle."""
    sbl = sbl_mod()
    w = wl.master_weights(O, K, seed=2)
    x = wl.activations(T, K, seed=2)
    layer = GpuLayer(w, 2, 4, sbl.SBL_FMT_I8 | sbl.SBL_FMT_SP24)
    q, d = quantize_act(x)
    yd, accd = forward(layer, q, d, sbl.SBL_FMT_I8)
    ys, accs = forward(layer, q, d, sbl.SBL_FMT_SP24)
    assert torch.equal(accd, accs)
    np.testing.assert_array_equal(bits_of(yd), bits_of(ys))
    ref = oracle.Layer(w, 2, 4)
    qr, _ = oracle.quantize_act(x)
    rng = np.random.default_rng(7)
    it, io = rng.integers(0, T, 1024), rng.integers(0, O, 1024)
    it[:2], io[:2] = [T - 1, 0], [O - 1, O - 1]
    np.testing.assert_array_equal(accs.cpu().numpy()[it, io], oracle.acc_samples(qr, ref.weff, it, io))


@pytest.mark.parametrize("fmt_name,O,K,T,n,m", [("I8", 528, 1040, 300, 6, 8), ("I8", 256, 128, 64, 2, 4),
                                                ("SP24", 528, 1040, 300, 2, 4), ("SP24", 4864, 896, 96, 2, 4),
                                                ("PK2", 384, 640, 9, 2, 4), ("PK2", 2560, 6912, 1, 2, 4)])
@pytest.mark.parametrize("relu2,residual", [(True, False), (False, True), (True, True)])
@pytest.mark.parametrize("fp32", [False, True])
def test_forward_epilogue_bit_exact(fmt_name, O, K, T, n, m, relu2, residual, fp32):
    """Squared ReLU and the residual add fused into every forward kernel:
    bit for bit the oracle's dequantisation followed by its epilogue."""
    sbl = sbl_mod()
    w = wl.master_weights(O, K, seed=O + T)
    x = wl.activations(T, K, seed=O + T)
    fmt = {"I8": sbl.SBL_FMT_I8, "PK2": sbl.SBL_FMT_PK2, "SP24": sbl.SBL_FMT_SP24}[fmt_name]
    layer = GpuLayer(w, n, m, fmt)
    ref = oracle.Layer(w, n, m)
    q, d = quantize_act(x)
    qr, dr, accr, yr, _ = ref.forward(x)
    res_bits = (wl.activations(T, O, seed=O + T + 1)) if residual else None
    out, outb = oracle.epilogue(yr, relu2=relu2, residual_bf16_bits=res_bits)
    y = torch.empty((T, O), dtype=torch.float32 if fp32 else torch.bfloat16, device="cuda")
    acc = torch.empty((T, O), dtype=torch.int32, device="cuda")
    sbl.sbl_forward_ex(layer.desc, q, d, T, layer.packed, fmt, y, relu2=relu2,
                       residual=bf16_dev(res_bits) if residual else None, acc_out=acc)
    np.testing.assert_array_equal(acc.cpu().numpy(), accr)
    if fp32:
        np.testing.assert_array_equal(y.cpu().numpy().view(np.uint32), out.view(np.uint32))
    else:
        np.testing.assert_array_equal(bits_of(y), outb)


# sbl_linear_forward: Q_a(X) then the forward, one fused launch for the PK2
# decode (T K <= 4096), else the activation and forward kernels
@pytest.mark.parametrize("fmt_name,O,K,T,n,m", [
    ("PK2", 6912, 2560, 1, 2, 4),    # fused, one token
    ("PK2", 96, 4096, 1, 2, 4),      # fused at the size limit, 2 chunks per warp
    ("PK2", 48, 1024, 4, 2, 4),      # fused at the limit, tokens spread over threads
    ("PK2", 32, 256, 16, 2, 4),      # fused, two n8 token blocks
    ("PK2", 16, 192, 8, 6, 8),       # fused, K not a multiple of 256
    ("PK2", 2560, 6912, 1, 2, 4),    # past the limit: two launches
    ("PK2", 64, 2560, 4, 2, 4),      # past the limit: two launches
    ("PK2", 48, 11008, 7, 2, 4),     # too large to fuse: two launches
    ("PK2", 32, 16448, 16, 2, 4),    # too large to fuse: two launches
    ("I8", 528, 1040, 300, 6, 8),    # GEMM path
    ("SP24", 528, 1040, 300, 2, 4),  # sparse GEMM path
])
def test_linear_forward_bit_exact(fmt_name, O, K, T, n, m):
    sbl = sbl_mod()
    w = wl.master_weights(O, K, seed=O + K)
    x = wl.activations(T, K, seed=O + T, outlier_frac=0.01)
    x[0] = 0  # a zero token: q = 0, d = 0, y = 0
    fmt = {"I8": sbl.SBL_FMT_I8, "PK2": sbl.SBL_FMT_PK2, "SP24": sbl.SBL_FMT_SP24}[fmt_name]
    layer = GpuLayer(w, n, m, fmt)
    ref = oracle.Layer(w, n, m)
    qr, dr, _, yr, ybr = ref.forward(x)
    xd = bf16_dev(x)
    q = torch.full((T, K), 99, dtype=torch.int8, device="cuda")
    d = torch.full((T,), -1.0, dtype=torch.float32, device="cuda")
    for fp32 in (False, True):
        y = torch.empty((T, O), dtype=torch.float32 if fp32 else torch.bfloat16, device="cuda")
        sbl.sbl_linear_forward(layer.desc, xd, T, layer.packed, fmt, q, d, y)
        np.testing.assert_array_equal(q.cpu().numpy(), qr)
        np.testing.assert_array_equal(d.cpu().numpy(), dr)
        if fp32:
            np.testing.assert_array_equal(y.cpu().numpy().view(np.uint32), yr.view(np.uint32))
        else:
            np.testing.assert_array_equal(bits_of(y), ybr)
    assert sbl.sbl_device_error(clear=True) == 0


@pytest.mark.parametrize("O,K,T", [(96, 768, 5), (2560, 6912, 16)])  # fused; two launches
def test_linear_forward_fused_decode_epilogue(O, K, T):
    """The fused decode with Squared ReLU and the residual: the oracle's
    quantiser, dequantisation and epilogue, bit for bit."""
    sbl = sbl_mod()
    w = wl.master_weights(O, K, seed=K)
    x = wl.activations(T, K, seed=T)
    layer = GpuLayer(w, 2, 4, sbl.SBL_FMT_PK2)
    ref = oracle.Layer(w, 2, 4)
    _, _, _, yr, _ = ref.forward(x)
    res_bits = wl.activations(T, O, seed=T + 1)
    _, outb = oracle.epilogue(yr, relu2=True, residual_bf16_bits=res_bits)
    q = torch.empty((T, K), dtype=torch.int8, device="cuda")
    d = torch.empty((T,), dtype=torch.float32, device="cuda")
    y = torch.empty((T, O), dtype=torch.bfloat16, device="cuda")
    sbl.sbl_linear_forward(layer.desc, bf16_dev(x), T, layer.packed, sbl.SBL_FMT_PK2, q, d, y, relu2=True,
                           residual=bf16_dev(res_bits))
    np.testing.assert_array_equal(bits_of(y), outb)


def test_forward_zero_tokens_is_noop():
    sbl = sbl_mod()
    layer = GpuLayer(wl.master_weights(32, 64, seed=1), 6, 8, 4)
    q = torch.empty((0, 64), dtype=torch.int8, device="cuda")
    d = torch.empty((1,), dtype=torch.float32, device="cuda")
    y = torch.empty((1, 32), dtype=torch.bfloat16, device="cuda")
    sbl.sbl_forward(layer.desc, q, d, 0, layer.packed, sbl.SBL_FMT_I8, y)


def sampled_forward_check(O, K, T, n, m, seed, n_samples=2048):
    """Full-size launch: integer stages in full, accumulators and outputs at
    seeded sample coordinates through the oracle's sampled routine."""
    w = wl.master_weights(O, K, seed=seed)
    x = wl.activations(T, K, seed=seed)
    layer = GpuLayer(w, n, m, 4)
    ref = oracle.Layer(w, n, m)
    got = layer.host()
    assert got["gamma"] == ref.gamma
    np.testing.assert_array_equal(got["i8"], ref.weff)
    q, d = quantize_act(x)
    qr, dr = oracle.quantize_act(x)
    np.testing.assert_array_equal(q.cpu().numpy(), qr)
    np.testing.assert_array_equal(d.cpu().numpy(), dr)
    yb, acc = forward(layer, q, d, layer.sbl.SBL_FMT_I8)
    rng = np.random.default_rng(seed)
    it, io = rng.integers(0, T, n_samples), rng.integers(0, O, n_samples)
    it[:4], io[:4] = [0, T - 1, 0, T - 1], [0, 0, O - 1, O - 1]  # corners
    acc_s = oracle.acc_samples(qr, ref.weff, it, io)
    acc_g = acc.cpu().numpy()
    np.testing.assert_array_equal(acc_g[it, io], acc_s)
    _, yb_s = oracle.dequant(acc_s.astype(np.int32).reshape(-1, 1), ref.gamma, dr[it])
    np.testing.assert_array_equal(bits_of(yb)[it, io], yb_s.ravel())


@pytest.mark.parametrize("name", ["qwen05b_mlp", "qwen15b_decoder", "qwen3b_train"])
def test_forward_full_workload_sizes_sampled(name):
    wk = wl.WORKLOADS[name]
    for li, lin in enumerate(wk.linears):
        n, m = wk.patterns[li % len(wk.patterns)]
        sampled_forward_check(lin.d_out, lin.d_in, wk.tokens[0], n, m, seed=wk.seed + li)


def test_forward_sweep_patterns_full_width():
    wk = wl.WORKLOADS["qwen15b_decoder"]
    lin = wk.linears[4]  # gate 1536 -> 8960
    for n, m in wk.patterns:
        sampled_forward_check(lin.d_out, lin.d_in, 1024, n, m, seed=n * 8 + m, n_samples=512)


def test_decode_workload_all_token_counts():
    wk = wl.WORKLOADS["bitnet2b_decode"]
    for lin in wk.linears:
        for T in wk.tokens:
            run_forward_full_check(lin.d_out, lin.d_in, T, 2, 4, seed=wk.seed + T, fmt_name="PK2")


# ------------------------------------------------------------------ backward

def scaled_bf16(bits: np.ndarray, exps: np.ndarray) -> np.ndarray:
    """bf16 bit patterns with row i multiplied by 2^exps[i] (exact: the values stay
    inside bf16's normal range)."""
    v = bf16_bits_to_f64(bits) * np.ldexp(1.0, np.asarray(exps, dtype=np.int64))[:, None]
    return f32_to_bf16_bits(v.astype(np.float32))


def backward_inputs(O, K, T, seed, dy_exp=0, d_spread=0):
    """Seeded W, X, dY; dY scaled by 2^dy_exp; with d_spread = s the token rows
    of X are scaled by 2^e, e cycling over -s/2 .. s/2, so the token scales d_t
    span 2^s."""
    w = wl.master_weights(O, K, seed=seed)
    x = wl.activations(T, K, seed=seed)
    dy = wl.output_grad(T, O, seed=seed)
    if d_spread:
        x = scaled_bf16(x, np.arange(T) % (d_spread + 1) - d_spread // 2)
    if dy_exp:
        dy = scaled_bf16(dy, np.full(T, dy_exp))
    return w, x, dy


def run_backward(O, K, T, n, m, seed, dx_fp32=True, dy_exp=0, d_spread=0):
    sbl = sbl_mod()
    w, x, dy = backward_inputs(O, K, T, seed, dy_exp, d_spread)
    layer = GpuLayer(w, n, m, 4 | 8)
    ref = oracle.Layer(w, n, m)
    q, d = quantize_act(x)
    dx = torch.empty((T, K), dtype=torch.float32 if dx_fp32 else torch.bfloat16, device="cuda")
    dw = torch.empty((O, K), dtype=torch.float32, device="cuda")
    ws = sbl.alloc_workspace(sbl.sbl_workspace_bytes(layer.desc, T, sbl.SBL_OP_BACKWARD))
    sbl.sbl_backward_dual_ste(layer.desc, bf16_dev(dy), q, d, T, layer.packed, dx, dx_fp32, dw, ws)
    torch.cuda.synchronize()
    return layer, ref, x, dy, dx, dw


def float_report(gpu, ref):
    return f"normwise {normwise(gpu, ref):.3g}, elementwise {elementwise_rel(gpu, ref):.3g} (|ref| >= 1e-2 max)"


@pytest.mark.parametrize("O,K,T,n,m", [(128, 256, 64, 6, 8), (528, 1040, 300, 6, 8), (256, 192, 70, 2, 4),
                                       (64, 64, 1, 8, 8)])
def test_backward_dual_ste_small(O, K, T, n, m):
    layer, ref, x, dy, dx, dw = run_backward(O, K, T, n, m, seed=O + K)
    qr, dr = oracle.quantize_act(x)
    dxr, dwr = oracle.backward(dy, ref.weff, ref.gamma, qr, dr)
    dxg, dwg = dx.cpu().numpy(), dw.cpu().numpy()
    assert normwise(dxg, dxr) <= FWD_TOL, float_report(dxg, dxr)
    assert normwise(dwg, dwr) <= FWD_TOL, float_report(dwg, dwr)
    # Dual STE: the gradient reaches masked weights too
    masked = ref.mask == 0
    if masked.any():
        assert (np.abs(dwg[masked]) > 0).mean() > 0.99


@pytest.mark.parametrize("dy_exp,d_spread", [(-30, 0), (-20, 0), (-10, 0), (6, 0), (0, 20), (-20, 20)])
def test_backward_dw_gradient_scales(dy_exp, d_spread):
    """dW at gradient magnitudes from 2^-30 to 2^6 of N(0, 1), and with token
    scales d_t spread over 2^20: products dY d_t of 1e-11 .. 1e+1, most of
    which an unscaled fp16 operand would flush to zero or lose to subnormals.
    The per-call power-of-two prescale keeps dW within the float tolerance."""
    O, K, T = 256, 320, 200
    layer, ref, x, dy, dx, dw = run_backward(O, K, T, 6, 8, seed=11, dy_exp=dy_exp, d_spread=d_spread)
    qr, dr = oracle.quantize_act(x)
    if d_spread:
        assert dr.max() / dr[dr > 0].min() >= 2.0 ** (d_spread - 1)
    dxr, dwr = oracle.backward(dy, ref.weff, ref.gamma, qr, dr)
    assert np.abs(dwr).max() > 0
    dwg, dxg = dw.cpu().numpy(), dx.cpu().numpy()
    assert normwise(dwg, dwr) <= FWD_TOL, float_report(dwg, dwr)
    assert normwise(dxg, dxr) <= FWD_TOL, float_report(dxg, dxr)


def test_backward_dw_zero_gradient():
    """dY == 0: the prescale is 2^0 and dW is exactly zero."""
    sbl = sbl_mod()
    O, K, T = 64, 128, 96
    w, x, _ = backward_inputs(O, K, T, seed=3)
    layer = GpuLayer(w, 6, 8, 4 | 8)
    q, d = quantize_act(x)
    dy = torch.zeros((T, O), dtype=torch.bfloat16, device="cuda")
    dw = torch.full((O, K), 7.0, dtype=torch.float32, device="cuda")
    ws = sbl.alloc_workspace(sbl.sbl_workspace_bytes(layer.desc, T, sbl.SBL_OP_BACKWARD))
    sbl.sbl_backward_dual_ste(layer.desc, dy, q, d, T, layer.packed, None, False, dw, ws)
    torch.cuda.synchronize()
    assert not dw.cpu().numpy().any()


def check_bf16_dx(dx_bits, ref, ref_abs):
    """bf16 dX against the exact (fp64) dX: every element within one bf16 ulp of
    the exact value, plus 2^-20 of sum_o |gamma dY W_eff| for the fp32
    accumulation order (it matters only where the sum cancels: for a typical
    element that allowance is about 2^-14 of its value, against the ulp's
    2^-8); and the normwise error within bf16's rounding (2^-9) plus the float
    tolerance."""
    g = bf16_bits_to_f64(dx_bits)
    err = np.abs(g - ref)
    tol = bf16_ulp(ref) + 2.0 ** -20 * ref_abs
    bad = err > tol
    assert not bad.any(), (f"{int(bad.sum())} of {bad.size} bf16 dX entries off by more than one ulp; worst "
                           f"{float((err / tol).max()):.3g} x the bound; {float_report(g, ref)}")
    assert normwise(g, ref) <= 2.0 ** -9 + FWD_TOL, float_report(g, ref)


def test_backward_bf16_dx():
    layer, ref, x, dy, dx, dw = run_backward(256, 256, 128, 6, 8, seed=5, dx_fp32=False)
    qr, dr = oracle.quantize_act(x)
    dxr, _ = oracle.backward(dy, ref.weff, ref.gamma, qr, dr, want_dw=False)
    dxa, _ = oracle.backward(dy & 0x7FFF, np.abs(ref.weff), ref.gamma, qr, dr, want_dw=False)
    check_bf16_dx(bits_of(dx), dxr, dxa)


def test_backward_training_workload_sampled():
    """The 3B training linears at full size (T = 16384, the bench's step): fp32
    dX and dW at seeded samples within the float tolerance, and the bf16 dX the
    training step writes within one bf16 ulp at 4096 samples."""
    wk = wl.WORKLOADS["qwen3b_train"]
    T = wk.tokens[0]
    for li, lin in enumerate(wk.linears):
        layer, ref, x, dy, dx, dw = run_backward(lin.d_out, lin.d_in, T, 6, 8, seed=wk.seed + li)
        qr, dr = oracle.quantize_act(x)
        rng = np.random.default_rng(li)
        it, ik, io = rng.integers(0, T, 256), rng.integers(0, lin.d_in, 256), rng.integers(0, lin.d_out, 256)
        dx_s = oracle.dx_samples(dy, ref.weff, ref.gamma, it, ik)
        dw_s = oracle.dw_samples(dy, qr, dr, io, ik)
        dxg, dwg = dx.cpu().numpy()[it, ik], dw.cpu().numpy()[io, ik]
        assert normwise(dxg, dx_s) <= FWD_TOL, float_report(dxg, dx_s)
        assert normwise(dwg, dw_s) <= FWD_TOL, float_report(dwg, dw_s)
        del dx, dw
        # the bf16 dX of the benchmarked step, same inputs
        sbl = layer.sbl
        q, d = quantize_act(x)
        dxb = torch.empty((T, lin.d_in), dtype=torch.bfloat16, device="cuda")
        ws = sbl.alloc_workspace(sbl.sbl_workspace_bytes(layer.desc, T, sbl.SBL_OP_BACKWARD))
        sbl.sbl_backward_dual_ste(layer.desc, bf16_dev(dy), q, d, T, layer.packed, dxb, False, None, ws)
        torch.cuda.synchronize()
        it, ik = rng.integers(0, T, 4096), rng.integers(0, lin.d_in, 4096)
        ref_s = oracle.dx_samples(dy, ref.weff, ref.gamma, it, ik)
        abs_s = oracle.dx_samples(dy & 0x7FFF, np.abs(ref.weff), ref.gamma, it, ik)
        check_bf16_dx(bits_of(dxb)[it, ik], ref_s, abs_s)


# -------------------------------------------------- ablation variants (f3)

VARIANTS = [("bf16", "master", "quant_then_mask"), ("fp32", "quantized", "quant_then_mask"),
            ("fp32", "master", "mask_then_quant"), ("bf16", "master", "mask_then_quant"),
            ("bf16", "quantized", "quant_then_mask")]


@pytest.mark.parametrize("dtype,mask_source,order", VARIANTS)
@pytest.mark.parametrize("O,K,n,m", [(128, 256, 6, 8), (48, 80, 2, 4), (528, 1040, 3, 8), (64, 128, 1, 8),
                                     (1008, 1040, 2, 4)])
def test_pack_variants_bit_exact(dtype, mask_source, order, O, K, n, m):
    """The weight-side ablation arms (bf16 master weights, mask from |W_q|,
    gamma over the survivors): gamma and every packed format bit for bit
    against the oracle run with the same variant, plus the statistics."""
    sbl = sbl_mod()
    w = wl.master_weights(O, K, seed=O + K + n)
    if dtype == "bf16":
        wbits = (w.view(np.uint32) >> 16).astype(np.uint16)  # truncated to bf16 (any bf16 value will do)
        w_dev = torch.from_numpy(wbits.view(np.int16)).view(torch.bfloat16).to("cuda")
        ref = oracle.Layer(wbits, n, m, mask_source=mask_source, order=order)
    else:
        w_dev = to_dev(w)
        ref = oracle.Layer(w, n, m, mask_source=mask_source, order=order)
    dsc = sbl.desc(O, K, n, m)
    fmts = sbl.SBL_FMT_I8 | sbl.SBL_FMT_PK2 | sbl.SBL_FMT_NM | (sbl.SBL_FMT_SP24 if n <= 2 else 0)
    p = sbl.alloc_packed(dsc, fmts)
    ws = sbl.alloc_workspace(sbl.sbl_workspace_bytes(dsc, 0, sbl.SBL_OP_QUANTIZE_MASK_PACK))
    keep = torch.empty((O, sbl.keep_bitmap_bytes(dsc)), dtype=torch.uint8, device="cuda")
    nz = torch.zeros((1,), dtype=torch.int64, device="cuda")
    thr = torch.empty((O, K // m), dtype=torch.float32, device="cuda")
    src = {"master": sbl.SBL_MASK_FROM_MASTER, "quantized": sbl.SBL_MASK_FROM_QUANTIZED}[mask_source]
    odr = {"quant_then_mask": sbl.SBL_QUANT_THEN_MASK, "mask_then_quant": sbl.SBL_MASK_THEN_QUANT}[order]
    sbl.sbl_quantize_mask_pack_ex(dsc, w_dev, fmts, p, ws, mask_source=src, order=odr, keep=keep, near_zero=nz,
                                  block_threshold=thr)
    torch.cuda.synchronize()
    assert float(p.gamma[0].item()) == ref.gamma
    np.testing.assert_array_equal(p.i8.cpu().numpy(), ref.weff)
    np.testing.assert_array_equal(p.pk2.cpu().numpy(), oracle.pack_pk2(ref.weff))
    vals, bm = oracle.pack_nm(ref.weff, ref.mask, n, m)
    np.testing.assert_array_equal(p.nm_bitmap.cpu().numpy(), bm)
    np.testing.assert_array_equal(p.nm_values.cpu().numpy(), vals)
    np.testing.assert_array_equal(keep.cpu().numpy(), bitmap_of(ref.mask))
    if n <= 2:
        sv, sm = oracle.pack_sp24(ref.weff, ref.mask)
        np.testing.assert_array_equal(p.sp24_values.cpu().numpy(), sv)
        np.testing.assert_array_equal(p.sp24_meta.cpu().numpy(), sm)
    assert int(nz.item()) == oracle.near_zero(ref.w, ref.gamma)
    np.testing.assert_array_equal(thr.cpu().numpy().view(np.uint32),
                                  oracle.block_threshold(ref.w, ref.mask, m).view(np.uint32))


def test_pack_variant_circular_combination_is_unsupported():
    sbl = sbl_mod()
    dsc = sbl.desc(32, 64, 6, 8)
    p = sbl.alloc_packed(dsc, sbl.SBL_FMT_I8)
    ws = sbl.alloc_workspace(sbl.sbl_workspace_bytes(dsc, 0, sbl.SBL_OP_QUANTIZE_MASK_PACK))
    with pytest.raises(sbl.SblError):
        sbl.sbl_quantize_mask_pack_ex(dsc, to_dev(wl.master_weights(32, 64, seed=1)), sbl.SBL_FMT_I8, p, ws,
                                      mask_source=sbl.SBL_MASK_FROM_QUANTIZED, order=sbl.SBL_MASK_THEN_QUANT)


@pytest.mark.parametrize("O,K,T,n,m", [(128, 256, 64, 6, 8), (528, 1040, 300, 2, 4), (96, 80, 33, 5, 8)])
def test_backward_mask_gated_dw(O, K, T, n, m):
    """The mask-gated dW ablation: dW = (dY^T Xtilde) * M, exactly zero at
    the pruned positions and within the float tolerance elsewhere; dX as
    ungated."""
    sbl = sbl_mod()
    w = wl.master_weights(O, K, seed=O + T)
    x = wl.activations(T, K, seed=O + T)
    dy = wl.output_grad(T, O, seed=O + T)
    layer = GpuLayer(w, n, m, 4 | 8)
    ref = oracle.Layer(w, n, m)
    q, d = quantize_act(x)
    keep = to_dev(bitmap_of(ref.mask))
    dx = torch.empty((T, K), dtype=torch.float32, device="cuda")
    dw = torch.empty((O, K), dtype=torch.float32, device="cuda")
    ws = sbl.alloc_workspace(sbl.sbl_workspace_bytes(layer.desc, T, sbl.SBL_OP_BACKWARD))
    sbl.sbl_backward_dual_ste_ex(layer.desc, bf16_dev(dy), q, d, T, layer.packed, dx, True, dw, keep, ws)
    torch.cuda.synchronize()
    qr, dr = oracle.quantize_act(x)
    dxr, dwr = oracle.backward(dy, ref.weff, ref.gamma, qr, dr)
    dwg = dw.cpu().numpy()
    assert not dwg[ref.mask == 0].any()
    assert normwise(dwg, dwr * ref.mask) <= FWD_TOL
    assert normwise(dx.cpu().numpy(), dxr) <= FWD_TOL


def test_device_error_word_clear():
    sbl = sbl_mod()
    assert sbl.sbl_device_error(clear=True) == 0
