"""Host-side checks of the C ABI that need no GPU: the library loads, exports
every function include/sbl.h declares, sizes its buffers like the oracle's
formats, and rejects invalid arguments before touching a device."""
import ctypes
import os
import re

import pytest

from conftest import ROOT

HEADER = os.path.join(ROOT, "include", "sbl.h")


@pytest.fixture(scope="module")
def sbl():
    from sparsity_sbl_quantize_b200 import build
    build.build()
    from sparsity_sbl_quantize_b200 import sbl as mod
    return mod


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(sbl_[a-z0-9_]+)\s*\(", text)))


def test_library_exports_every_declared_symbol(sbl):
    decl = declared_functions()
    assert "sbl_forward" in decl and "sbl_quantize_mask_pack" in decl
    lib = ctypes.CDLL(sbl.LIB_PATH)
    for name in decl:
        assert hasattr(lib, name), f"{name} declared in sbl.h but not exported"
    assert sorted(sbl.EXPORTED) == decl


def test_status_strings_and_version(sbl):
    for code in range(8):
        assert sbl.sbl_status_string(code)
    assert sbl.sbl_version() >= 100


@pytest.mark.parametrize("O,K,n,m", [(128, 256, 6, 8), (4864, 896, 2, 4), (2560, 6912, 2, 4),
                                     (16, 16, 1, 4), (48, 80, 3, 8)])
def test_row_bytes_match_oracle_formats(sbl, O, K, n, m):
    import oracle
    d = sbl.desc(O, K, n, m)
    assert sbl.sbl_packed_row_bytes(d, sbl.SBL_FMT_PK2) == oracle.pk2_row_bytes(K)
    assert sbl.sbl_packed_row_bytes(d, sbl.SBL_FMT_NM) == oracle.nm_value_row_bytes(K, n, m)
    assert sbl.sbl_packed_row_bytes(d, sbl.SBL_FMT_NM, sbl.SBL_BUF_NM_BITMAP) == oracle.nm_bitmap_row_bytes(K)
    assert sbl.sbl_packed_row_bytes(d, sbl.SBL_FMT_I8) == K
    assert sbl.sbl_packed_row_bytes(d, sbl.SBL_FMT_BF16T) == 2 * O
    assert sbl.sbl_packed_row_bytes(d, sbl.SBL_FMT_SP24) == oracle.sp24_value_row_bytes(K)
    assert sbl.sbl_packed_row_bytes(d, sbl.SBL_FMT_SP24, sbl.SBL_BUF_SP24_META) == oracle.sp24_meta_row_bytes(K)
    assert sbl.sbl_packed_row_bytes(d, sbl.SBL_FMT_T24) == oracle.t24_lo_row_bytes(K)
    assert sbl.sbl_packed_row_bytes(d, sbl.SBL_FMT_T24, sbl.SBL_BUF_T24_HI) == oracle.t24_hi_row_bytes(K)


@pytest.mark.parametrize("O,K,n,m", [(0, 256, 6, 8), (128, 250, 6, 8), (128, 256, 9, 8),
                                     (128, 256, 0, 8), (128, 256, 3, 6), (20, 256, 2, 4),
                                     (128, 8, 2, 4), (128, 131072, 2, 4)])
def test_invalid_descriptors_are_rejected(sbl, O, K, n, m):
    d = sbl.desc(O, K, n, m)
    assert sbl.sbl_packed_row_bytes(d, sbl.SBL_FMT_PK2) == 0
    assert sbl.sbl_workspace_bytes(d, 16, sbl.SBL_OP_BACKWARD) == 0


def test_workspace_sizes(sbl):
    d = sbl.desc(11008, 2048, 6, 8)
    ws = sbl.sbl_workspace_bytes(d, 16384, sbl.SBL_OP_BACKWARD)
    assert ws >= (11008 + 2048) * 16384 * 2
    assert sbl.sbl_workspace_bytes(d, 0, sbl.SBL_OP_QUANTIZE_MASK_PACK) >= 16384 * 8


class _FakePtr:
    """Stands in for a device tensor: only data_ptr() is read by the binding."""

    def __init__(self, addr, nbytes=1 << 20):
        self.addr, self.nbytes = addr, nbytes

    def data_ptr(self):
        return self.addr

    def numel(self):
        return self.nbytes

    def element_size(self):
        return 1


def _raw(sbl, fn, *args):
    return getattr(sbl._lib, fn)(*args)


def test_validation_happens_before_any_device_access(sbl):
    """Bad shapes, null pointers and misalignment return their status codes;
    the device is only looked up after the arguments pass, so on a host
    without a GPU a valid call reports SBL_ERR_DEVICE and launches nothing."""
    good = 0x10000
    P = ctypes.c_void_p
    # act quant: shape, null, alignment, then device
    assert _raw(sbl, "sbl_quantize_act", P(good), 4, 250, P(good), P(good), None) == 2
    assert _raw(sbl, "sbl_quantize_act", None, 4, 256, P(good), P(good), None) == 1
    assert _raw(sbl, "sbl_quantize_act", P(good + 4), 4, 256, P(good), P(good), None) == 3
    assert _raw(sbl, "sbl_quantize_act", P(good), 0, 256, P(good), P(good), None) == 0  # T == 0: no-op
    # linear forward: descriptor, null, alignment, then device
    lf = "sbl_linear_forward"
    dd = sbl.desc(128, 256, 6, 8)
    pw = sbl.sbl_packed(None, None, None, good, good, good)
    assert _raw(sbl, lf, ctypes.byref(dd), P(good), -1, ctypes.byref(pw), sbl.SBL_FMT_PK2, P(good), P(good),
                P(good), 0, None, None) == 2
    assert _raw(sbl, lf, ctypes.byref(dd), P(good), 0, ctypes.byref(pw), sbl.SBL_FMT_PK2, P(good), P(good),
                P(good), 0, None, None) == 0
    assert _raw(sbl, lf, ctypes.byref(dd), None, 4, ctypes.byref(pw), sbl.SBL_FMT_PK2, P(good), P(good),
                P(good), 0, None, None) == 1
    assert _raw(sbl, lf, ctypes.byref(dd), P(good), 4, ctypes.byref(pw), sbl.SBL_FMT_PK2, None, P(good),
                P(good), 0, None, None) == 1
    assert _raw(sbl, lf, ctypes.byref(dd), P(good + 8), 4, ctypes.byref(pw), sbl.SBL_FMT_PK2, P(good),
                P(good), P(good), 0, None, None) == 3
    assert _raw(sbl, lf, ctypes.byref(dd), P(good), 4, ctypes.byref(pw), sbl.SBL_FMT_PK2, P(good), P(good),
                P(good), 0, None, None) == 1  # no PK2 buffer: invalid before the device lookup
    pk = sbl.sbl_packed(good, None, None, None, None, good)
    assert _raw(sbl, lf, ctypes.byref(dd), P(good), 4, ctypes.byref(pk), sbl.SBL_FMT_PK2, P(good), P(good),
                P(good), 0, None, None) == 7  # valid: no sm_100 device here
    F = ctypes.c_float
    rms = "sbl_quantize_act_rmsnorm"
    assert _raw(sbl, rms, P(good), 4, 250, None, F(1e-5), P(good), P(good), None) == 2
    assert _raw(sbl, rms, P(good), 4, 2 * 65536, None, F(1e-5), P(good), P(good), None) == 2
    assert _raw(sbl, rms, None, 4, 256, None, F(1e-5), P(good), P(good), None) == 1
    assert _raw(sbl, rms, P(good), 4, 256, None, F(-1.0), P(good), P(good), None) == 1
    assert _raw(sbl, rms, P(good), 4, 256, None, F(float("nan")), P(good), P(good), None) == 1
    assert _raw(sbl, rms, P(good), 4, 256, None, F(float("inf")), P(good), P(good), None) == 1
    assert _raw(sbl, rms, P(good), 4, 256, P(good + 2), F(1e-5), P(good), P(good), None) == 3
    assert _raw(sbl, rms, P(good), 0, 256, None, F(1e-5), P(good), P(good), None) == 0
    assert _raw(sbl, rms, P(good), 4, 256, None, F(1e-5), P(good), P(good), None) == 7  # no sm_100 device here
    assert _raw(sbl, rms, P(good), 4, 256, P(good), F(0.0), P(good), P(good), None) == 7
    d = sbl.desc(128, 256, 6, 8)
    w = sbl.sbl_packed(None, None, None, good, good, good)
    st = _raw(sbl, "sbl_forward", ctypes.byref(d), P(good), P(good), 64, ctypes.byref(w),
              sbl.SBL_FMT_I8, P(good), 0, None, None)
    try:
        import torch
        has_gpu = torch.cuda.is_available()
    except Exception:
        has_gpu = False
    if not has_gpu:
        assert st == 7  # SBL_ERR_DEVICE: no launch was attempted
    # unsupported forward format, bad n:m, missing workspace
    assert _raw(sbl, "sbl_forward", ctypes.byref(d), P(good), P(good), 64, ctypes.byref(w),
                sbl.SBL_FMT_NM, P(good), 0, None, None) in (4, 7)
    bad = sbl.desc(128, 256, 3, 6)
    assert _raw(sbl, "sbl_forward", ctypes.byref(bad), P(good), P(good), 64, ctypes.byref(w),
                sbl.SBL_FMT_I8, P(good), 0, None, None) == 4
    assert _raw(sbl, "sbl_quantize_mask_pack", ctypes.byref(d), P(good), sbl.SBL_FMT_I8,
                ctypes.byref(w), None, 0, None) == 5
    assert _raw(sbl, "sbl_quantize_mask_pack", ctypes.byref(d), P(good), 1 << 7,
                ctypes.byref(w), P(good), 1 << 20, None) == 1
    # BF16T needs the int8 copy in the same call
    assert _raw(sbl, "sbl_quantize_mask_pack", ctypes.byref(d), P(good), sbl.SBL_FMT_BF16T,
                ctypes.byref(w), P(good), 1 << 20, None) == 4
    # decode path: more than 16 tokens is unsupported
    wp = sbl.sbl_packed(good, None, None, None, None, good)
    assert _raw(sbl, "sbl_forward", ctypes.byref(d), P(good), P(good), 17, ctypes.byref(wp),
                sbl.SBL_FMT_PK2, P(good), 0, None, None) in (4, 7)


def test_sp24_validation(sbl):
    """The sparse MMA operand exists only for masks with at most two kept
    weights per group of four (n <= 2): other n:m are unsupported in both the
    pack and the forward; missing or misaligned buffers are rejected first."""
    good = 0x10000
    P = ctypes.c_void_p
    ws = P(good)
    d68 = sbl.desc(128, 256, 6, 8)
    d24 = sbl.desc(128, 256, 2, 4)
    w = sbl.sbl_packed(None, None, None, None, None, good, good, good)
    assert _raw(sbl, "sbl_quantize_mask_pack", ctypes.byref(d68), P(good), sbl.SBL_FMT_SP24,
                ctypes.byref(w), ws, 1 << 20, None) == 4
    assert _raw(sbl, "sbl_forward", ctypes.byref(d68), P(good), P(good), 64, ctypes.byref(w),
                sbl.SBL_FMT_SP24, P(good), 0, None, None) in (4, 7)
    nometa = sbl.sbl_packed(None, None, None, None, None, good, good, None)
    assert _raw(sbl, "sbl_quantize_mask_pack", ctypes.byref(d24), P(good), sbl.SBL_FMT_SP24,
                ctypes.byref(nometa), ws, 1 << 20, None) == 1
    skew = sbl.sbl_packed(None, None, None, None, None, good, good + 8, good)
    assert _raw(sbl, "sbl_quantize_mask_pack", ctypes.byref(d24), P(good), sbl.SBL_FMT_SP24,
                ctypes.byref(skew), ws, 1 << 20, None) == 3


def test_t24_validation(sbl):
    """The 6-bit group code exists for the same masks as SP24 (n <= 2): other
    n:m are unsupported in the pack; missing or misaligned planes are
    rejected first; the decode takes at most 16 tokens."""
    good = 0x10000
    P = ctypes.c_void_p
    ws = P(good)
    d68 = sbl.desc(128, 256, 6, 8)
    d24 = sbl.desc(128, 256, 2, 4)
    w = sbl.sbl_packed(None, None, None, None, None, good, None, None, good, good)
    assert _raw(sbl, "sbl_quantize_mask_pack", ctypes.byref(d68), P(good), sbl.SBL_FMT_T24,
                ctypes.byref(w), ws, 1 << 20, None) == 4
    nohi = sbl.sbl_packed(None, None, None, None, None, good, None, None, good, None)
    assert _raw(sbl, "sbl_quantize_mask_pack", ctypes.byref(d24), P(good), sbl.SBL_FMT_T24,
                ctypes.byref(nohi), ws, 1 << 20, None) == 1
    skew = sbl.sbl_packed(None, None, None, None, None, good, None, None, good + 8, good)
    assert _raw(sbl, "sbl_quantize_mask_pack", ctypes.byref(d24), P(good), sbl.SBL_FMT_T24,
                ctypes.byref(skew), ws, 1 << 20, None) == 3
    assert _raw(sbl, "sbl_forward", ctypes.byref(d24), P(good), P(good), 17, ctypes.byref(w),
                sbl.SBL_FMT_T24, P(good), 0, None, None) in (4, 7)


def test_forward_format_recommendation(sbl):
    """The recommended forward operand: the dense int8 MMA unless the mask
    is 2:4-compatible (n <= 2) and the GEMM is long in K and large in T x O."""
    F = sbl.sbl_forward_format
    assert F(sbl.desc(4864, 896, 2, 4), 4096) == sbl.SBL_FMT_I8      # short K
    assert F(sbl.desc(896, 4864, 2, 4), 4096) == sbl.SBL_FMT_I8      # few output tiles
    assert F(sbl.desc(8960, 1536, 2, 4), 8192) == sbl.SBL_FMT_SP24
    assert F(sbl.desc(1536, 8960, 2, 8), 8192) == sbl.SBL_FMT_SP24   # 2:8 runs as 2:4
    assert F(sbl.desc(2048, 11008, 6, 8), 16384) == sbl.SBL_FMT_I8   # 6:8 is not 2:4
    assert F(sbl.desc(2048, 11008, 3, 4), 16384) == sbl.SBL_FMT_I8
    assert F(sbl.desc(20, 256, 2, 4), 64) == 0                       # invalid descriptor
    assert F(sbl.desc(128, 256, 2, 4), -1) == 0


def test_mask_stats_validation(sbl):
    """Statistics arguments are checked before any device access: a flip
    count needs the previous bitmap; counters must be 8-byte and arrays
    16-byte aligned."""
    good = 0x10000
    P = ctypes.c_void_p
    d = sbl.desc(128, 256, 6, 8)
    w = sbl.sbl_packed(None, None, None, good, None, good)
    no_prev = sbl.sbl_mask_stats(None, good, good, None, None)
    assert _raw(sbl, "sbl_quantize_mask_pack_stats", ctypes.byref(d), P(good), sbl.SBL_FMT_I8, ctypes.byref(w),
                ctypes.byref(no_prev), P(good), 1 << 20, None) == 1
    odd_counter = sbl.sbl_mask_stats(good, None, good + 4, None, None)
    assert _raw(sbl, "sbl_quantize_mask_pack_stats", ctypes.byref(d), P(good), sbl.SBL_FMT_I8, ctypes.byref(w),
                ctypes.byref(odd_counter), P(good), 1 << 20, None) == 3
    odd_thr = sbl.sbl_mask_stats(None, None, None, None, good + 4)
    assert _raw(sbl, "sbl_quantize_mask_pack_stats", ctypes.byref(d), P(good), sbl.SBL_FMT_I8, ctypes.byref(w),
                ctypes.byref(odd_thr), P(good), 1 << 20, None) == 3


def test_forward_epilogue_validation(sbl):
    good = 0x10000
    P = ctypes.c_void_p
    d = sbl.desc(128, 256, 6, 8)
    w = sbl.sbl_packed(None, None, None, good, None, good)
    epi = sbl.sbl_epilogue(1, good + 2)  # misaligned residual
    assert _raw(sbl, "sbl_forward_ex", ctypes.byref(d), P(good), P(good), 64, ctypes.byref(w), sbl.SBL_FMT_I8,
                P(good), 0, None, ctypes.byref(epi), None) == 3


def test_binding_refuses_to_load_without_the_library(tmp_path):
    """No CPU fallback: the binding, placed where no libsbl.so sits, raises on
    import instead of offering any other implementation."""
    import importlib.util
    src = os.path.join(ROOT, "sparsity_sbl_quantize_b200", "sbl.py")
    dst = tmp_path / "sbl.py"
    dst.write_text(open(src).read())
    spec = importlib.util.spec_from_file_location("sbl_without_library", dst)
    mod = importlib.util.module_from_spec(spec)
    with pytest.raises(ImportError, match="libsbl.so is missing"):
        spec.loader.exec_module(mod)


def test_compute_calls_fail_loudly_without_a_device(sbl):
    """On a host without a CUDA device the compute entry points raise (the
    binding's stream lookup, or the library's device check); nothing runs
    elsewhere and the outputs stay untouched."""
    import torch
    if torch.cuda.is_available():
        pytest.skip("a CUDA device is present")
    d = sbl.desc(32, 64, 6, 8)
    x = torch.zeros((4, 64), dtype=torch.bfloat16)
    q = torch.zeros((4, 64), dtype=torch.int8)
    dv = torch.zeros((4,), dtype=torch.float32)
    with pytest.raises((sbl.SblError, RuntimeError)):
        sbl.sbl_quantize_act(x, 4, 64, q, dv)
    p = sbl.Packed(gamma=torch.zeros(4, dtype=torch.float32), i8=torch.zeros((32, 64), dtype=torch.int8))
    y = torch.zeros((4, 32), dtype=torch.bfloat16)
    with pytest.raises((sbl.SblError, RuntimeError)):
        sbl.sbl_forward(d, q, dv, 4, p, sbl.SBL_FMT_I8, y)
    assert torch.count_nonzero(y) == 0 and torch.count_nonzero(q) == 0


def test_c99_program_against_the_library(sbl, tmp_path):
    """The header compiles as strict C99 (no CUDA header, no C++), every
    declared function links against libsbl.so, and a plain C program sees
    the documented sizes, format rule and argument checks."""
    import subprocess
    import torch
    lib_dir = os.path.dirname(sbl.LIB_PATH)
    exe = tmp_path / "abi_host_check"
    subprocess.run(["gcc", "-std=c99", "-pedantic", "-Wall", "-Wextra", "-Werror",
                    "-I", os.path.join(ROOT, "include"), os.path.join(ROOT, "tests", "abi_host_check.c"),
                    "-L", lib_dir, "-lsbl", f"-Wl,-rpath,{lib_dir}", "-o", str(exe)], check=True)
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stderr
    if not torch.cuda.is_available():
        assert "(no device)" in r.stdout


def test_argument_fuzzing_without_a_device(sbl):
    """Random descriptors, token counts, format bits and pointers (null,
    misaligned, plausible) through every entry point: each call returns a
    documented status and none crashes.  Runs only when the library reports
    that no device is present, so no pointer here can reach a kernel."""
    import random
    code = ctypes.c_uint32(0)
    if _raw(sbl, "sbl_device_error", ctypes.byref(code), 0) != 7:
        pytest.skip("a device is present: fake pointers must not reach kernels")
    rnd = random.Random(3)
    P = ctypes.c_void_p
    ints = [-(1 << 31), -1, 0, 1, 2, 3, 4, 6, 7, 8, 9, 15, 16, 17, 64, 80, 256, 1040, 65536, 65552, 1 << 20,
            (1 << 31) - 1]

    def ptr():
        return rnd.choice([None, P(0x10000), P(0x10008), P(0x20000), P(0x30001)])

    def desc():
        return sbl.desc(rnd.choice(ints), rnd.choice(ints), rnd.choice(ints), rnd.choice(ints))

    def packed():
        return sbl.sbl_packed(*[rnd.choice([None, 0x40000, 0x40004]) for _ in range(10)])

    statuses = set()
    for _ in range(4000):
        d, w, T, f = desc(), packed(), rnd.choice(ints), rnd.choice([0, 1, 2, 4, 8, 16, 32, 63, 64, 1 << 31])
        which = rnd.randrange(9)
        if which == 0:
            st = _raw(sbl, "sbl_forward", ctypes.byref(d), ptr(), ptr(), T, ctypes.byref(w), f, ptr(),
                      rnd.randint(0, 1), ptr(), None)
        elif which == 1:
            st = _raw(sbl, "sbl_quantize_act", ptr(), T, rnd.choice(ints), ptr(), ptr(), None)
        elif which == 2:
            st = _raw(sbl, "sbl_quantize_act_rmsnorm", ptr(), T, rnd.choice(ints), ptr(),
                      ctypes.c_float(rnd.choice([0.0, 1e-5, -1.0, float("nan")])), ptr(), ptr(), None)
        elif which == 3:
            st = _raw(sbl, "sbl_linear_forward", ctypes.byref(d), ptr(), T, ctypes.byref(w), f, ptr(), ptr(),
                      ptr(), 0, None, None)
        elif which == 4:
            st = _raw(sbl, "sbl_backward_dual_ste", ctypes.byref(d), ptr(), ptr(), ptr(), T, ctypes.byref(w),
                      ptr(), 1, ptr(), ptr(), rnd.choice([0, 256, 1 << 30]), None)
        elif which == 5:
            st = _raw(sbl, "sbl_quantize_mask_pack", ctypes.byref(d), ptr(), f, ctypes.byref(w), ptr(),
                      rnd.choice([0, 256, 1 << 20]), None)
        elif which == 6:
            st = _raw(sbl, "sbl_quantize_mask_pack_noalloc", ctypes.byref(d), ptr(), f, ctypes.byref(w), None)
        elif which == 7:
            n = _raw(sbl, "sbl_packed_row_bytes", ctypes.byref(d), f, rnd.randrange(5))
            n2 = _raw(sbl, "sbl_workspace_bytes", ctypes.byref(d), T, rnd.randrange(3))
            st = 0 if n >= 0 and n2 >= 0 else -1
        else:
            fmt = _raw(sbl, "sbl_forward_format", ctypes.byref(d), T)
            st = 0 if fmt in (0, 4, 16) else -1
        statuses.add(st)
    assert statuses <= set(range(8))
    assert {1, 2, 7} <= statuses  # invalid arguments, bad sizes, and calls that reached the device check


def test_batch_forward_validation_before_device(sbl):
    """sbl_forward_batch: count, T, descriptors, K limits, null pointers, chain
    rules, alignment and the workspace are checked before the device lookup;
    a valid call on a host without a GPU reports SBL_ERR_DEVICE."""
    good = 0x10000

    def layer(O=128, K=256, chained=False, y_fp32=0, xq=good, pk2=good):
        return sbl.sbl_batch_layer(sbl.desc(O, K, 2, 4), pk2, good, xq, good, good, y_fp32, 1 if chained else 0,
                                   None, None)

    def call(layers, T=4, ws=None, ws_bytes=0, count=None):
        arr = sbl.batch_array(layers)
        return _raw(sbl, "sbl_forward_batch", arr, len(layers) if count is None else count, T,
                    ctypes.c_void_p(ws) if ws else None, ws_bytes, None)

    assert _raw(sbl, "sbl_forward_batch", None, 1, 4, None, 0, None) == 1
    assert call([layer()], T=0) == 2 and call([layer()], T=17) == 2
    assert call([layer()], count=0) == 2 and call([layer()], count=257) == 2
    assert call([layer(K=250)]) == 2                       # invalid descriptor
    assert call([layer(K=272)]) == 4                       # K not a multiple of 64
    assert call([layer(K=13888)]) == 4                     # K above the stage limit (13824)
    assert call([layer(pk2=None)]) == 1 and call([layer(xq=None)]) == 1
    assert call([layer(pk2=good + 8)]) == 3
    assert call([layer(chained=True)]) == 1                # a chain needs a previous layer
    assert call([layer(O=256), layer(O=128, K=512, chained=True)]) == 1   # shapes do not chain
    assert call([layer(O=512, y_fp32=1), layer(K=512, chained=True)]) == 1  # fp32 output cannot chain
    chain = [layer(O=512), layer(K=512, chained=True, xq=None)]
    nws = sbl.sbl_forward_batch_workspace_bytes(sbl.batch_array(chain), 2, 4)
    # completion words of two layers (256) + the first layer's prepared input (4 x 256 + 256)
    assert nws == 256 + 1024 + 256
    one = sbl.sbl_forward_batch_workspace_bytes(sbl.batch_array([layer()]), 1, 4)
    assert one == 1024 + 256
    # two layers on one input share its prepared copy; a second input gets its own
    assert sbl.sbl_forward_batch_workspace_bytes(sbl.batch_array([layer(), layer()]), 2, 4) == one
    assert sbl.sbl_forward_batch_workspace_bytes(sbl.batch_array([layer(), layer(xq=good + 4096)]), 2, 4) == 2 * one
    assert sbl.sbl_forward_batch_workspace_bytes(sbl.batch_array([layer()]), 1, 0) == 0
    assert call(chain) == 5 and call(chain, ws=good, ws_bytes=nws - 1) == 5
    assert call(chain, ws=good + 16, ws_bytes=nws) == 3
    assert call(chain, ws=good, ws_bytes=nws) == 7         # valid: no sm_100 device here
    big = [layer(), layer(O=64, K=13824)]
    assert call(big, T=16) == 5
    nb = sbl.sbl_forward_batch_workspace_bytes(sbl.batch_array(big), 2, 16)
    assert call(big, T=16, ws=good, ws_bytes=nb) == 7


def test_sharding_calls_validate_before_device(sbl):
    good = 0x10000
    P = ctypes.c_void_p
    d = sbl.desc(64, 1040, 6, 8)
    assert sbl.sbl_gamma_node_count(d) == (64 * 1040 + 8191) // 8192
    assert sbl.sbl_gamma_node_count(sbl.desc(64, 250, 6, 8)) == 0
    nb = sbl.sbl_workspace_bytes(d, 0, sbl.SBL_OP_QUANTIZE_MASK_PACK)
    part = "sbl_gamma_partials"
    assert _raw(sbl, part, ctypes.byref(d), None, 0, P(good), P(good), nb, None) == 1
    assert _raw(sbl, part, ctypes.byref(d), P(good), 16, P(good), P(good), nb, None) == 2   # misaligned shard
    assert _raw(sbl, part, ctypes.byref(d), P(good), -8, P(good), P(good), nb, None) == 2
    assert _raw(sbl, part, ctypes.byref(d), P(good + 4), 0, P(good), P(good), nb, None) == 3
    assert _raw(sbl, part, ctypes.byref(d), P(good), 0, P(good), P(good), nb - 1, None) == 5
    assert _raw(sbl, part, ctypes.byref(d), P(good), 0, P(good), P(good), nb, None) == 7  # no device here
    comb = "sbl_gamma_combine"
    assert _raw(sbl, comb, None, 4, 4 * 8192, P(good), None) == 1
    assert _raw(sbl, comb, P(good), 3, 4 * 8192, P(good), None) == 2
    assert _raw(sbl, comb, P(good), 1, 0, P(good), None) == 2
    assert _raw(sbl, comb, P(good), 5, 4 * 8192 + 1, P(good), None) == 7
    w = sbl.sbl_packed(None, None, None, good, None, good)
    assert _raw(sbl, "sbl_quantize_mask_pack_shard", ctypes.byref(d), P(good), sbl.SBL_FMT_I8, ctypes.byref(w),
                None) == 7
    assert _raw(sbl, "sbl_quantize_mask_pack_shard", ctypes.byref(d), None, sbl.SBL_FMT_I8, ctypes.byref(w),
                None) == 1


def test_group_forward_validation_before_device(sbl):
    """sbl_forward_group: count, descriptors, shared in_features, null and
    misaligned pointers are checked before the device lookup; a valid call on
    a host without a GPU reports SBL_ERR_DEVICE."""
    good = 0x10000
    P = ctypes.c_void_p

    def call(descs, ws, ys, T=64, xq=good, d=good, count=None):
        n = len(descs)
        darr = (ctypes.POINTER(sbl.sbl_layer_desc) * max(n, 1))(*[ctypes.pointer(x) for x in descs])
        warr = (ctypes.POINTER(sbl.sbl_packed) * max(n, 1))(*[ctypes.pointer(w) for w in ws])
        yarr = (P * max(n, 1))(*[P(y) if y else None for y in ys])
        return _raw(sbl, "sbl_forward_group", darr, n if count is None else count, P(xq) if xq else None,
                    P(d) if d else None, T, warr, yarr, 0, None)

    w = sbl.sbl_packed(None, None, None, good, None, good)
    d1, d2 = sbl.desc(4864, 896, 6, 8), sbl.desc(4864, 896, 6, 8)
    assert _raw(sbl, "sbl_forward_group", None, 1, P(good), P(good), 64, None, None, 0, None) == 1
    assert call([d1, d2], [w, w], [good, good], count=0) == 1
    assert call([d1, d2], [w, w], [good, good], count=5) == 1
    assert call([d1, sbl.desc(4864, 250, 6, 8)], [w, w], [good, good]) == 2      # invalid descriptor
    assert call([d1, sbl.desc(4864, 1024, 6, 8)], [w, w], [good, good]) == 2     # in_features differ
    assert call([d1, d2], [w, w], [good, good], T=-1) == 2
    assert call([d1, d2], [w, w], [good, good], T=0) == 0                        # nothing to do
    assert call([d1, d2], [w, w], [good, good], xq=None) == 1
    assert call([d1, d2], [w, w], [good, None]) == 1
    assert call([d1, d2], [w, sbl.sbl_packed(None, None, None, None, None, good)], [good, good]) == 1  # no I8
    assert call([d1, d2], [w, w], [good, good + 8]) == 3
    assert call([d1, d2], [w, sbl.sbl_packed(None, None, None, good + 4, None, good)], [good, good]) == 3
    assert call([d1, d2], [w, w], [good, good], d=good + 4) == 3
    assert call([d1, d2, d1, d2], [w] * 4, [good] * 4) == 7                      # valid: no sm_100 device here
