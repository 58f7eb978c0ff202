"""Host-side logic for running the batched Muon step on several GPUs.

Every matrix of a Muon step is an independent unit of work, so a model's
matrices can be split across ranks: each rank steps the matrices it owns and
the updated weights are then shared.  This module holds the parts of that
which need no GPU: the assignment of matrices to ranks (longest-processing-
time first on the step's FLOP count) and the exchange pattern, written
against torch.distributed so that it runs on NCCL (GPUs) and on gloo (CPU
tests) alike.

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


def max_over_ranks(value: float, device=None, group=None) -> float:
    """The slowest rank's time (the timing rule of the benchmark)."""
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX, group=group)
    return float(t.item())
