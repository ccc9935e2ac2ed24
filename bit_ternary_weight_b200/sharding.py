"""Column-parallel (N-split) decode across the GPUs of one node.

A ternary weight [N, K] is split by output rows: rank r owns rows
[r * R, min(N, (r + 1) * R)) with R a whole number of 8-row groups, the same
for every rank but the last.  In the packed layout TL the bytes of one 8-row
group (all of K) are one contiguous slab of 2 K bytes, so a rank's share of
the packed weight is one contiguous byte range: a view, no repacking.  The
weight scale gamma is per tensor and the activation scale per token, so every
rank uses the whole tensor's gamma (computed once, over all rows, by the
packer) and quantises the whole token itself; the rank's outputs are then
exactly the rows the unsplit product would give.  One all-gather of the bf16
(or fp32) outputs, 2 R bytes per rank and token, rebuilds y on every rank.

This is the split the decode GEMV allows without changing any integer result:
no partial sums cross GPUs, so parity with the single-GPU product is exact.
Prefill needs no exchange at all (tokens split across ranks, weights
replicated).  Pages: "How to Run BitNet Inference on GPU Using CUDA Kernels:
A Complete Guide", section "Understanding the Two-Phase Architecture" (the
decode phase is the memory-bound INT8 x INT2 linear); the pages themselves run
on one device, so the partition is this library's.

The all-gather goes through ``torch.distributed`` (NCCL between GPUs, gloo on
the host for tests).  No TMA multicast and no library kernel ever reads a
peer's memory here: each rank's kernels read only its own shard.
"""
from __future__ import annotations

from dataclasses import dataclass

import torch

GROUP_ROWS = 8  # rows of one packed row group


@dataclass(frozen=True)
class RowShard:
    rank: int
    world: int
    row0: int        # first output row of this rank
    row1: int        # one past the last (row1 - row0 may be 0 for a tail rank)
    rows_per_rank: int  # R: rows every rank's slot in the gather buffer holds

    @property
    def rows(self) -> int:
        return self.row1 - self.row0


def row_partition(N: int, world: int) -> list[RowShard]:
    """Rows of an N-row weight for each of `world` ranks, in whole 8-row groups:
    every rank owns R = ceil(ceil(N / 8) / world) * 8 rows, the last ones fewer
    (possibly none).  The shards tile [0, N) in rank order."""
    if N < 1 or world < 1:
        raise ValueError("N and world must be positive")
    groups = (N + GROUP_ROWS - 1) // GROUP_ROWS
    gpr = (groups + world - 1) // world
    R = gpr * GROUP_ROWS
    out = []
    for r in range(world):
        row0 = min(N, r * R)
        row1 = min(N, (r + 1) * R)
        out.append(RowShard(r, world, row0, row1, R))
    return out


def packed_byte_range(K: int, shard: RowShard) -> tuple[int, int]:
    """Byte range [b0, b1) of the TL packed array holding the shard's rows:
    its row groups' slabs, 2 K bytes each (K / 4 bytes per row, 8 rows)."""
    slab = 2 * K
    g0 = shard.row0 // GROUP_ROWS
    g1 = (shard.row1 + GROUP_ROWS - 1) // GROUP_ROWS
    return g0 * slab, g1 * slab


def shard_weight(w, shard: RowShard):
    """The rank's part of a packed weight as a TernaryWeight view (shared
    packed storage and the whole tensor's gamma), or None for an empty shard."""
    from . import TernaryWeight
    if shard.rows == 0:
        return None
    b0, b1 = packed_byte_range(w.K, shard)
    return TernaryWeight(w.packed[b0:b1], w.w_scale, shard.rows, w.K)


class ColumnParallelDecode:
    """Decode BitLinears split by output rows over the ranks of a process group.

    ``products``: TernaryWeights sharing K (for instance q, k and v).  Each call
    runs this rank's shards in one fused launch (quantise, product, rescale),
    writing straight into the rank's slot of one gather buffer per product,
    then all-gathers every product's outputs; ``outputs()`` returns the full
    [M, N] views.  Ranks with an empty shard still take part in the gather.
    """

    def __init__(self, products, group=None, M: int = 1, out_dtype=torch.bfloat16,
                 device=None):
        import torch.distributed as dist
        self.group = group
        self.world = dist.get_world_size(group) if dist.is_initialized() else 1
        self.rank = dist.get_rank(group) if dist.is_initialized() else 0
        self.M = M
        self.K = products[0].K
        if any(p.K != self.K for p in products):
            raise ValueError("products must share K")
        device = device or products[0].packed.device
        self.full = []     # per product: flat gather buffer, world slots of M * R
        self.local = []    # per product: this rank's slot, viewed [M, R]
        self.shards = []
        for p in products:
            sh = row_partition(p.N, self.world)[self.rank]
            slot = M * sh.rows_per_rank
            buf = torch.zeros(self.world * slot, dtype=out_dtype, device=device)
            self.full.append(buf)
            self.local.append(buf[self.rank * slot:(self.rank + 1) * slot].view(M, sh.rows_per_rank))
            self.shards.append((p, sh, shard_weight(p, sh)))

    def outputs(self):
        """Full outputs [M, N] per product (valid after __call__ and the gather).
        The gather buffer is rank-major, so for M = 1 the N valid rows are its
        first N elements (a view); for M > 1 the tokens' rows are reassembled
        into a new tensor."""
        outs = []
        for (p, sh, _), buf in zip(self.shards, self.full):
            R = sh.rows_per_rank
            if self.M == 1:
                outs.append(buf.view(1, self.world * R)[:, :p.N])
            else:
                outs.append(buf.view(self.world, self.M, R).permute(1, 0, 2)
                            .reshape(self.M, self.world * R)[:, :p.N])
        return outs

    def __call__(self, x: torch.Tensor, pdl: bool = False):
        from . import gemv_fused_multi
        live = [(w, loc[:, :sh.rows]) for (p, sh, w), loc in zip(self.shards, self.local)
                if w is not None]
        if live:
            gemv_fused_multi([w for w, _ in live], x, outs=[o for _, o in live], pdl=pdl)
        self.gather()
        return self.outputs()

    def gather(self):
        if self.world == 1:
            return
        import torch.distributed as dist
        # in place: each rank's input is its own slot of the output buffer
        for buf, loc in zip(self.full, self.local):
            dist.all_gather_into_tensor(buf, loc.view(-1), group=self.group)
