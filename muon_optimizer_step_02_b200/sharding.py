"""Host-side logic for running the batched Muon step on several GPUs.

Every matrix of a Muon step is an independent unit of work, so a model's
matrices can be split across ranks: each rank steps the matrices it owns and
the updated weights are then shared.  This module holds the parts of that
which need no GPU: the assignment of matrices to ranks (longest-processing-
time first on the step's FLOP count) and two exchange patterns, written
against torch.distributed so that they run on NCCL (GPUs) and on gloo (CPU
tests) alike: per-matrix reduce and broadcast (`sharded_step`), and flat
owner-ordered buffers with one reduce-scatter of the gradients, momentum kept
only by the owner, and one all-gather of the weights (`ShardLayout`,
`sharded_step_flat`).

Context: PR #1893 "Record: L_ParallelResiduals_UNetSkips_DepthRecur_Muon_
1.0901", table "Architecture and training stack", row "Train context"
(8-way distributed); PR #1396 section "Reproduction" (torchrun
--nproc_per_node=8).
"""

from __future__ import annotations

import heapq
from typing import Callable, List, Sequence, Tuple


def matrix_cost(rows: int, cols: int, ns_steps: int) -> float:
    """Relative cost of one matrix: Newton-Schulz FLOPs plus the elementwise
    passes (weighted by a nominal FLOP:byte balance of the GPU)."""
    m, n = min(rows, cols), max(rows, cols)
    flops = ns_steps * (4.0 * m * m * n + 2.0 * m * m * m)
    elementwise_bytes = 20.0 * rows * cols
    return flops + 200.0 * elementwise_bytes


def partition_matrices(shapes: Sequence[Tuple[int, int]], world: int,
                       ns_steps: int = 5) -> List[int]:
    """Owner rank of every matrix.  Longest-processing-time first: matrices
    in decreasing cost, each to the currently least-loaded rank (ties to the
    lowest rank, equal costs in list order), so every rank computes the same
    answer without communicating."""
    if world < 1:
        raise ValueError("world must be >= 1")
    order = sorted(range(len(shapes)),
                   key=lambda i: (-matrix_cost(*shapes[i], ns_steps), i))
    heap = [(0.0, r) for r in range(world)]
    owner = [0] * len(shapes)
    for i in order:
        load, r = heapq.heappop(heap)
        owner[i] = r
        heapq.heappush(heap, (load + matrix_cost(*shapes[i], ns_steps), r))
    return owner


def rank_loads(shapes, owner, world, ns_steps=5) -> List[float]:
    loads = [0.0] * world
    for (r, c), o in zip(shapes, owner):
        loads[o] += matrix_cost(r, c, ns_steps)
    return loads


def sharded_step(W, M, G_local, owner, rank, step_fn: Callable, group=None):
    """One data-parallel Muon step with matrix ownership.

    W, M, G_local: per-matrix tensors on this rank (W replicated, M only
    meaningful on the owner, G_local this rank's gradient contribution).
      1. every gradient is summed onto its owner (reduce to owner);
      2. each rank steps the matrices it owns: step_fn(indices) updates
         W[i] and M[i] in place for i in indices;
      3. the owner broadcasts each updated weight to every rank.
    Every rank issues the same collectives in the same order."""
    import torch.distributed as dist
    for i, o in enumerate(owner):
        dist.reduce(G_local[i], dst=o, op=dist.ReduceOp.SUM, group=group)
    mine = [i for i, o in enumerate(owner) if o == rank]
    if mine:
        step_fn(mine)
    for i, o in enumerate(owner):
        dist.broadcast(W[i], src=o, group=group)
    return mine


class ShardLayout:
    """Flat, owner-ordered buffers for a sharded step with one reduce-scatter
    and one all-gather.

    The matrices are laid out rank by rank (rank 0's matrices, then rank
    1's, ...), each rank's segment padded to the longest segment (`seg`
    elements), so that

      * the gradients (a flat buffer of world * seg elements on every rank,
        each rank's own contribution) reduce-scatter into the owner's segment
        in one collective: every rank receives exactly the summed gradients of
        the matrices it owns;
      * the momentum lives only on the owner (seg elements per rank);
      * the updated weights (a flat buffer of world * seg elements) are
        all-gathered from the owners' segments in one collective.

    `offset[i]` is matrix i's first element in the flat buffers;
    `local_offset[i]` its first element inside its owner's segment."""

    def __init__(self, shapes: Sequence[Tuple[int, int]], world: int, ns_steps: int = 5,
                 align: int = 8):
        self.shapes = [(int(r), int(c)) for r, c in shapes]
        self.world = world
        self.owner = partition_matrices(self.shapes, world, ns_steps)
        self.mine = [[i for i, o in enumerate(self.owner) if o == r] for r in range(world)]
        # every matrix starts `align` elements into a segment: 8 elements keep
        # 16-byte alignment for both the bf16 gradients and the fp32 states
        self.local_offset = [0] * len(self.shapes)
        seg_len = [0] * world
        for r in range(world):
            off = 0
            for i in self.mine[r]:
                self.local_offset[i] = off
                n = self.shapes[i][0] * self.shapes[i][1]
                off += (n + align - 1) // align * align
            seg_len[r] = off
        self.seg = max(max(seg_len), align)
        self.offset = [self.owner[i] * self.seg + self.local_offset[i]
                       for i in range(len(self.shapes))]

    def numel(self) -> int:
        return self.world * self.seg

    def views(self, flat, idx=None):
        """Views of the listed matrices (all by default) in a flat buffer of
        world * seg elements."""
        idx = range(len(self.shapes)) if idx is None else idx
        return [flat[self.offset[i]:self.offset[i] + self.shapes[i][0] * self.shapes[i][1]]
                .view(self.shapes[i]) for i in idx]

    def local_views(self, seg_buf, rank):
        """Views of rank's matrices in a segment buffer of seg elements."""
        return [seg_buf[self.local_offset[i]:self.local_offset[i] +
                        self.shapes[i][0] * self.shapes[i][1]].view(self.shapes[i])
                for i in self.mine[rank]]


def sharded_step_flat(layout: ShardLayout, W_flat, M_seg, G_flat, G_seg, rank,
                      step_fn: Callable, group=None):
    """One data-parallel Muon step on the flat layout:
      1. reduce-scatter the gradients: G_seg (seg elements) <- the sum over
         ranks of their G_flat segment for this rank;
      2. step this rank's matrices: step_fn(W_views, M_views, G_views) on
         views of its segment of W_flat, of M_seg and of G_seg;
      3. all-gather the updated segments of W_flat to every rank.
    Every rank issues the same two collectives."""
    import torch.distributed as dist
    dist.reduce_scatter_tensor(G_seg, G_flat, op=dist.ReduceOp.SUM, group=group)
    own = W_flat[rank * layout.seg:(rank + 1) * layout.seg]
    if layout.mine[rank]:
        step_fn(layout.local_views(own, rank), layout.local_views(M_seg, rank),
                layout.local_views(G_seg, rank))
    dist.all_gather_into_tensor(W_flat, own.clone(), group=group)


def max_over_ranks(value: float, device=None, group=None) -> float:
    """The slowest rank's time (the timing rule of the benchmark)."""
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX, group=group)
    return float(t.item())
