"""Column-parallel sharding of one Sparse-BitLinear layer over ranks (one
process per GPU, torch.distributed for the exchange).

Rank r holds rows [first_row, first_row + rows) of the fp32 master weights.
The N:M groups run along in_features, so masking, ternarisation and packing
are row-local; the only whole-matrix quantity is gamma = mean |W|, whose fp64
pairwise tree has as its first level the sums of consecutive 8192-weight
blocks.  With every shard boundary on a multiple of 8192 weights each rank's
block sums are blocks of the whole matrix: the ranks exchange those (a few KB)
and finish the same tree, so every rank packs its rows with exactly the gamma
of the unsharded layer.  The forward of a column shard needs no exchange (the
activations are replicated; each rank produces its own output columns).

The arithmetic runs in libsbl.so (sbl_gamma_partials, sbl_gamma_combine,
sbl_quantize_mask_pack_shard); this module only plans the shards and moves the
block sums between ranks.
"""
from __future__ import annotations

import math
from typing import List, Sequence, Tuple

GAMMA_BLOCK = 8192  # weights per first-level node of gamma's tree


def row_unit(in_features: int) -> int:
    """Smallest row count that keeps a shard boundary on the tree's first
    level (rows * K % 8192 == 0) and on the library's 16-row granularity."""
    need = GAMMA_BLOCK // math.gcd(in_features, GAMMA_BLOCK)
    return need * 16 // math.gcd(need, 16)


def check_shard(first_row: int, in_features: int) -> None:
    if (first_row * in_features) % GAMMA_BLOCK:
        raise ValueError(f"shard boundary at row {first_row} (x {in_features} weights) is not on a multiple of "
                         f"{GAMMA_BLOCK} weights: gamma's tree would not split there")


def column_shards(out_features: int, in_features: int, world: int) -> List[Tuple[int, int]]:
    """(first_row, rows) of every rank: near-equal shares of whole row units,
    boundaries aligned for gamma's tree; the last rank takes any remainder
    that is not a whole unit (it ends the matrix, so its last block may be
    partial)."""
    unit = row_unit(in_features)
    units, rest = divmod(out_features, unit)
    if units < world:
        raise ValueError(f"{out_features} rows in units of {unit} do not give {world} ranks a share each")
    out, first = [], 0
    for r in range(world):
        share = (units // world + (1 if r < units % world else 0)) * unit
        if r == world - 1:
            share += rest
        out.append((first, share))
        first += share
    return out


def node_counts(shards: Sequence[Tuple[int, int]], in_features: int) -> List[int]:
    return [-(-rows * in_features // GAMMA_BLOCK) for _, rows in shards]


def gather_node_sums(dist, local, counts: Sequence[int], group=None):
    """Every rank's first-level sums, concatenated in rank order (the order of
    the rows).  Ranks pad to the largest count so one all-gather serves."""
    import torch
    width = max(counts)
    buf = torch.zeros(width, dtype=local.dtype, device=local.device)
    buf[: local.numel()] = local
    parts = [torch.empty_like(buf) for _ in counts]
    dist.all_gather(parts, buf, group=group)
    return torch.cat([p[:c] for p, c in zip(parts, counts)])


def quantize_mask_pack_column_parallel(dist, shard_desc, W_shard, first_row: int, out_features: int,
                                       formats: int, out, workspace, counts: Sequence[int], group=None):
    """This rank's part of the sharded weight side: its block sums, the
    exchange, gamma from all of them (into out.gamma), then its rows packed.
    Every rank takes the same collective step."""
    import torch

    from . import sbl
    K = shard_desc.in_features
    check_shard(first_row, K)
    local = torch.empty(sbl.sbl_gamma_node_count(shard_desc), dtype=torch.float64, device=W_shard.device)
    sbl.sbl_gamma_partials(shard_desc, W_shard, first_row, local, workspace)
    nodes = gather_node_sums(dist, local, counts, group)
    sbl.sbl_gamma_combine(nodes, nodes.numel(), out_features * K, out.gamma)
    sbl.sbl_quantize_mask_pack_shard(shard_desc, W_shard, formats, out)
