"""A packed layer stored with save_packed and read back with load_packed
drives the forward exactly as the freshly packed one does (the container
itself is host code, tested in test_container.py; this checks the device
copies around it).  Collected after the other GPU files."""
import pytest
import torch

from sparsity_sbl_quantize_b200 import workloads as wl

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():  # the gpu marker deselects these on CPU hosts
    pytest.skip("needs a CUDA device", allow_module_level=True)

from gpu_case import bf16_dev, sbl_mod  # noqa: E402

BUFFERS = ["pk2", "nm_values", "nm_bitmap", "i8", "bf16t", "sp24_values", "sp24_meta", "t24_lo", "t24_hi"]


def test_saved_and_loaded_layer_gives_the_same_forward(tmp_path):
    sbl = sbl_mod()
    O, K, T = 96, 2560, 4
    d = sbl.desc(O, K, 2, 4)
    fm = sbl.SBL_FMT_PK2 | sbl.SBL_FMT_I8 | sbl.SBL_FMT_SP24 | sbl.SBL_FMT_T24
    p = sbl.alloc_packed(d, fm)
    ws = sbl.alloc_workspace(sbl.sbl_workspace_bytes(d, 0, sbl.SBL_OP_QUANTIZE_MASK_PACK))
    sbl.sbl_quantize_mask_pack(d, torch.from_numpy(wl.master_weights(O, K, seed=9)).cuda(), fm, p, ws)
    path = str(tmp_path / "layer.sblp")
    sbl.save_packed(path, d, fm, p)
    d2, f2, p2 = sbl.load_packed(path)
    assert (d2.out_features, d2.in_features, d2.n, d2.m, f2) == (O, K, 2, 4, fm)
    assert torch.equal(p.gamma[:1], p2.gamma[:1])
    for name in BUFFERS:
        a, b = getattr(p, name), getattr(p2, name)
        assert (a is None) == (b is None), name
        if a is not None:
            assert b.is_cuda and torch.equal(a, b), name
    x = bf16_dev(wl.activations(T, K, seed=9))
    q = torch.empty((T, K), dtype=torch.int8, device="cuda")
    dv = torch.empty((T,), dtype=torch.float32, device="cuda")
    sbl.sbl_quantize_act(x, T, K, q, dv)
    for fmt in (sbl.SBL_FMT_PK2, sbl.SBL_FMT_T24, sbl.SBL_FMT_I8, sbl.SBL_FMT_SP24):
        y1 = torch.empty((T, O), dtype=torch.bfloat16, device="cuda")
        y2 = torch.empty((T, O), dtype=torch.bfloat16, device="cuda")
        sbl.sbl_forward(d, q, dv, T, p, fmt, y1)
        sbl.sbl_forward(d2, q, dv, T, p2, fmt, y2)
        torch.cuda.synchronize()
        assert torch.equal(y1, y2), fmt
    assert sbl.sbl_device_error(clear=True) == 0
