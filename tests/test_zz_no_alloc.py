"""The no-allocation packing entry point against the regular one.

sbl_quantize_mask_pack_noalloc serves callers that cannot obtain device
memory where they call the layer (a plugin whose host framework owns every
allocation, a runtime with a budget fixed up front, a path that must not risk
cudaMalloc's implicit synchronisation).  It must give exactly what
sbl_quantize_mask_pack gives with a caller workspace -- packing is integer
work, so the comparison is bit for bit -- on consecutive calls that reuse
its static scratch.  This file is collected last on purpose.
"""
import numpy as np
import pytest
import torch

from sparsity_sbl_quantize_b200 import workloads as wl

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)


def _sbl():
    from sparsity_sbl_quantize_b200 import build
    build.build()
    from sparsity_sbl_quantize_b200 import sbl
    return sbl


FORMATS = 1 | 2 | 4 | 8  # PK2 | NM | I8 | BF16T


def _both(sbl, w, n, m):
    o, k = w.shape
    dsc = sbl.desc(o, k, n, m)
    wd = torch.from_numpy(w).cuda()
    ref = sbl.alloc_packed(dsc, FORMATS)
    ws = sbl.alloc_workspace(sbl.sbl_workspace_bytes(dsc, 0, sbl.SBL_OP_QUANTIZE_MASK_PACK))
    sbl.sbl_quantize_mask_pack(dsc, wd, FORMATS, ref, ws)
    got = sbl.alloc_packed(dsc, FORMATS)
    sbl.sbl_quantize_mask_pack_noalloc(dsc, wd, FORMATS, got)
    torch.cuda.synchronize()
    return ref, got


def _equal(a, b):
    for name in ("gamma", "pk2", "nm_values", "nm_bitmap", "i8", "bf16t"):
        ta, tb = getattr(a, name), getattr(b, name)
        if name == "gamma":
            ta, tb = ta[:1], tb[:1]
        assert torch.equal(ta.view(torch.uint8), tb.view(torch.uint8)), name


def test_noalloc_matches_workspace_entry_point_on_consecutive_calls():
    sbl = _sbl()
    cases = [((528, 1040), 6, 8, 1), ((1008, 1040), 2, 4, 2), ((128, 256), 6, 8, 3)]
    for (o, k), n, m, seed in cases:  # several calls in a row share the static scratch
        w = wl.master_weights(o, k, seed=seed)
        ref, got = _both(sbl, w, n, m)
        _equal(ref, got)
    # the same layer twice more: the scratch's left-over contents must not leak in
    w = wl.master_weights(1008, 1040, seed=7)
    for _ in range(2):
        ref, got = _both(sbl, w, 5, 8)
        _equal(ref, got)
    assert sbl.sbl_device_error() == 0


def test_noalloc_matches_the_oracle():
    """gamma and W_eff from the no-allocation call against the oracle
    directly (besides the regular entry point), twice in a row."""
    import oracle
    sbl = _sbl()
    w = wl.master_weights(528, 1040, seed=11)
    ref = oracle.Layer(w, 6, 8)
    for _ in range(2):
        _, got = _both(sbl, w, 6, 8)
        assert np.float32(got.gamma[0].item()) == ref.gamma
        np.testing.assert_array_equal(got.i8.cpu().numpy(), ref.weff)
        np.testing.assert_array_equal(got.pk2.cpu().numpy(), oracle.pack_pk2(ref.weff))


def test_noalloc_rejects_layers_beyond_its_scratch():
    sbl = _sbl()
    # 2^28 weights is the limit; 16384 x 16400 is over it -> SBL_ERR_SHAPE
    dsc = sbl.desc(16384, 16400, 2, 4)
    tiny = torch.empty(16, dtype=torch.float32, device="cuda")
    p = sbl.Packed(gamma=torch.empty(4, dtype=torch.float32, device="cuda"), i8=tiny)
    with pytest.raises(sbl.SblError) as e:
        sbl.sbl_quantize_mask_pack_noalloc(dsc, tiny, 4, p)
    assert e.value.status == 2
