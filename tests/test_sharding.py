"""Column-parallel sharding on the CPU: the shard plan, and two and three gloo
ranks exchanging gamma's first-level block sums.

Each rank takes its block sums from the oracle (its R1 tree over each 8192-
weight block of its own rows, exactly what sbl_gamma_partials computes on a
GPU), the ranks gather them with the same helper the GPU path uses, and the
rest of the tree is finished in rank order.  The result must be the oracle's
sum over the whole matrix bit for bit, and gamma the oracle's gamma; packing a
shard's rows with it must give the unsharded layer's rows.
"""
import json
import os
import socket
import subprocess
import sys

import numpy as np
import pytest

from conftest import ROOT
from sparsity_sbl_quantize_b200 import sharding


def tree(parts):
    """The pairwise tree of gamma's definition over a list of node sums:
    split at the largest power of two below n (zero padding adds exact 0)."""
    n = len(parts)
    if n == 1:
        return parts[0]
    h = 1
    while h * 2 < n:
        h *= 2
    return tree(parts[:h]) + tree(parts[h:])


@pytest.mark.parametrize("O,K,world", [(11008, 2048, 2), (2048, 11008, 2), (4864, 896, 2), (896, 4864, 3),
                                       (6912, 2560, 4), (256, 1536, 2), (8960, 1536, 8)])
def test_shard_plan_covers_rows_on_tree_boundaries(O, K, world):
    shards = sharding.column_shards(O, K, world)
    assert len(shards) == world and shards[0][0] == 0
    assert sum(r for _, r in shards) == O
    for (a, ra), (b, _) in zip(shards, shards[1:]):
        assert a + ra == b
    for first, rows in shards:
        assert rows % 16 == 0 and rows > 0
        sharding.check_shard(first, K)
    sizes = [r for _, r in shards[:-1]]
    assert max(sizes) - min(sizes) <= sharding.row_unit(K) if sizes else True


def test_misaligned_boundary_and_too_many_ranks_are_refused():
    with pytest.raises(ValueError):
        sharding.check_shard(16, 1040)      # 16 x 1040 is not a multiple of 8192
    sharding.check_shard(64, 128)           # 8192 exactly
    with pytest.raises(ValueError):
        sharding.column_shards(64, 256, 4)  # units of 32 rows: only two


def test_tree_over_block_sums_equals_the_whole_tree():
    """Single process: block sums of any aligned split, finished by the tree,
    equal the oracle's sum over the whole matrix (bit for bit)."""
    import oracle
    from sparsity_sbl_quantize_b200 import workloads as wl
    for O, K in ((528, 1040), (96, 2560), (80, 208)):
        w = wl.master_weights(O, K, seed=O)
        flat = w.reshape(-1)
        blocks = [oracle.abs_sum(flat[i:i + 8192]) for i in range(0, flat.size, 8192)]
        assert tree(blocks) == oracle.abs_sum(w)


RANK_SCRIPT = r"""
import json, sys
sys.path.insert(0, {root!r}); sys.path.insert(0, {tests!r})
import numpy as np, torch, torch.distributed as dist
import oracle
from sparsity_sbl_quantize_b200 import sharding, workloads as wl
from test_sharding import tree
dist.init_process_group("gloo")
rank, world = dist.get_rank(), dist.get_world_size()
O, K, n, m = {O}, {K}, 6, 8
w = wl.master_weights(O, K, seed=13)
shards = sharding.column_shards(O, K, world)
first, rows = shards[rank]
mine = w[first:first + rows].reshape(-1)
local = torch.tensor([oracle.abs_sum(mine[i:i + 8192]) for i in range(0, mine.size, 8192)], dtype=torch.float64)
nodes = sharding.gather_node_sums(dist, local, sharding.node_counts(shards, K))
s = tree([float(v) for v in nodes])
g = np.float32(s / (O * K))
weff = oracle.apply_mask(oracle.ternarize(w[first:first + rows], g), oracle.nm_mask(w[first:first + rows], n, m))
ref = oracle.Layer(w, n, m)
print(json.dumps({{"rank": rank, "sum_equal": s == oracle.abs_sum(w), "gamma_equal": bool(g == ref.gamma),
                   "rows_equal": bool(np.array_equal(weff, ref.weff[first:first + rows]))}}))
dist.destroy_process_group()
"""


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


@pytest.mark.parametrize("O,K,world", [(1104, 2048, 2), (896, 1536, 3)])
def test_gloo_ranks_gather_block_sums_to_the_unsharded_gamma(O, K, world):
    port = _free_port()
    script = RANK_SCRIPT.format(root=ROOT, tests=os.path.join(ROOT, "tests"), O=O, K=K)
    procs = []
    for rank in range(world):
        env = dict(os.environ, RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank),
                   MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
        procs.append(subprocess.Popen([sys.executable, "-c", script], env=env, stdout=subprocess.PIPE,
                                      stderr=subprocess.PIPE, text=True))
    for p in procs:
        out, err = p.communicate(timeout=180)
        assert p.returncode == 0, err[-2000:]
        r = json.loads(out.strip().splitlines()[-1])
        assert r["sum_equal"] and r["gamma_equal"] and r["rows_equal"], r
