"""GPU parity of the column-parallel weight side, the ranks emulated one after
another on one device (no rank waits on another): each shard's first-level
sums (sbl_gamma_partials), concatenated in row order and finished by
sbl_gamma_combine, give the oracle's gamma bit for bit, and packing each shard
with it (sbl_quantize_mask_pack_shard) gives the oracle's rows of W_eff and
PK2.  Misaligned shards and a wrong node count are refused."""
import numpy as np
import pytest
import torch

import oracle
from sparsity_sbl_quantize_b200 import sharding
from sparsity_sbl_quantize_b200 import workloads as wl

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():  # the gpu marker deselects these on CPU hosts
    pytest.skip("needs a CUDA device", allow_module_level=True)

from gpu_case import sbl_mod, to_dev  # noqa: E402


@pytest.mark.parametrize("O,K,n,m,world", [(1104, 2048, 6, 8, 2), (896, 1536, 2, 4, 3), (4864, 896, 6, 8, 2),
                                           (2048, 11008, 6, 8, 2), (11008, 2048, 6, 8, 4)])
def test_sharded_gamma_and_packing_equal_unsharded(O, K, n, m, world):
    sbl = sbl_mod()
    w = wl.master_weights(O, K, seed=O + K)
    ref = oracle.Layer(w, n, m)
    shards = sharding.column_shards(O, K, world)
    counts = sharding.node_counts(shards, K)
    fmts = sbl.SBL_FMT_I8 | sbl.SBL_FMT_PK2
    pieces = []
    nodes = []
    for first, rows in shards:
        dsc = sbl.desc(rows, K, n, m)
        ws_ = sbl.alloc_workspace(sbl.sbl_workspace_bytes(dsc, 0, sbl.SBL_OP_QUANTIZE_MASK_PACK))
        wd = to_dev(w[first:first + rows])
        part = torch.empty(sbl.sbl_gamma_node_count(dsc), dtype=torch.float64, device="cuda")
        sbl.sbl_gamma_partials(dsc, wd, first, part, ws_)
        nodes.append(part)
        pieces.append((dsc, wd, first, rows))
    assert [p.numel() for p in nodes] == counts
    allnodes = torch.cat(nodes)
    for dsc, wd, first, rows in pieces:
        out = sbl.alloc_packed(dsc, fmts)
        sbl.sbl_gamma_combine(allnodes, allnodes.numel(), O * K, out.gamma)
        sbl.sbl_quantize_mask_pack_shard(dsc, wd, fmts, out)
        torch.cuda.synchronize()
        assert np.float32(out.gamma[0].item()) == ref.gamma
        np.testing.assert_array_equal(out.i8.cpu().numpy(), ref.weff[first:first + rows])
        np.testing.assert_array_equal(out.pk2.cpu().numpy(), oracle.pack_pk2(ref.weff)[first:first + rows])
    assert sbl.sbl_device_error() == 0


def test_sharding_refuses_misaligned_shards_and_node_counts():
    sbl = sbl_mod()
    K = 1040
    dsc = sbl.desc(64, K, 6, 8)
    wd = torch.zeros((64, K), dtype=torch.float32, device="cuda")
    ws_ = sbl.alloc_workspace(sbl.sbl_workspace_bytes(dsc, 0, sbl.SBL_OP_QUANTIZE_MASK_PACK))
    part = torch.empty(16, dtype=torch.float64, device="cuda")
    with pytest.raises(sbl.SblError) as e:
        sbl.sbl_gamma_partials(dsc, wd, 16, part, ws_)  # 16 x 1040 weights: not on a first-level boundary
    assert e.value.status == 2
    g = torch.empty(4, dtype=torch.float32, device="cuda")
    with pytest.raises(sbl.SblError) as e:
        sbl.sbl_gamma_combine(part, 3, 8192 * 4, g)  # four nodes expected
    assert e.value.status == 2
