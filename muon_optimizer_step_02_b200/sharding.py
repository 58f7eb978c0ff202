"""Host-side logic for running the batched Muon step on several GPUs.

Every matrix of a Muon step is an independent unit of work, so a model's
matrices can be split across ranks: each rank steps the matrices it owns and
the updated weights are then shared.  This module holds the parts of that
which need no GPU, written against torch.distributed so that they run on
NCCL (GPUs) and on gloo (CPU tests) alike:

* the assignment of matrices to ranks (longest-processing-time first on the
  step's cost);
* `ShardLayout` / `sharded_step_flat`: flat owner-ordered buffers, one
  reduce-scatter of the gradients into each owner's segment, the owners'
  steps (momentum kept by the owner only), one all-gather of the weights;
* `BucketedLayout` / `sharded_step_bucketed`: the same over buckets of
  consecutive matrices, with the reduce-scatter of later buckets overlapping
  the step of earlier ones and each bucket's all-gather overlapping the
  steps after it (a communication stream beside the compute stream), and an
  option to reduce the gradients in fp32;
* in both, an optional EMA of the weights each rank owns, updated by the
  owner right after its step (the average shards like the momentum, with no
  exchange of its own).

Context: PR #1893 "Record: L_ParallelResiduals_UNetSkips_DepthRecur_Muon_
1.0901", table "Architecture and training stack", row "Train context"
(8-way distributed) and row "EMA" (EMA_DECAY=0.9965); PR #1396 section
"Reproduction" (torchrun --nproc_per_node=8).
"""

from __future__ import annotations

import heapq
from contextlib import nullcontext
from typing import Callable, List, Optional, Sequence, Tuple


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
                      step_fn: Callable, group=None, E_seg=None,
                      ema_fn: Optional[Callable] = None):
    """One data-parallel Muon step on the flat layout:
      1. reduce-scatter the gradients: G_seg (seg elements) <- the sum over
         ranks of their G_flat segment for this rank;
      2. step this rank's matrices: step_fn(W_views, M_views, G_views) on
         views of its segment of W_flat, of M_seg and of G_seg;
         with `ema_fn`, then ema_fn(E_views, W_views): the average of the
         weights this rank owns, in E_seg (seg elements), from the updated
         weights -- the EMA shards like the momentum, with no exchange;
      3. all-gather the updated segments of W_flat to every rank.
    Every rank issues the same two collectives."""
    import torch.distributed as dist
    dist.reduce_scatter_tensor(G_seg, G_flat, op=dist.ReduceOp.SUM, group=group)
    own = W_flat[rank * layout.seg:(rank + 1) * layout.seg]
    if layout.mine[rank]:
        w_views = layout.local_views(own, rank)
        step_fn(w_views, layout.local_views(M_seg, rank), layout.local_views(G_seg, rank))
        if ema_fn is not None:
            ema_fn(layout.local_views(E_seg, rank), w_views)
    dist.all_gather_into_tensor(W_flat, own.clone(), group=group)


class BucketedLayout:
    """The matrices split into `n_buckets` buckets of consecutive plan entries
    of about equal cost (so that each bucket's step takes about as long), each
    bucket laid out by its own `ShardLayout` (ownership balanced inside the
    bucket).  `buckets[b]` lists bucket b's matrices (global indices);
    `layouts[b]` indexes them 0 .. len(buckets[b]) - 1."""

    def __init__(self, shapes: Sequence[Tuple[int, int]], world: int, n_buckets: int,
                 ns_steps: int = 5, align: int = 8):
        self.shapes = [(int(r), int(c)) for r, c in shapes]
        self.world = world
        n = len(self.shapes)
        if not 1 <= n_buckets <= max(n, 1):
            raise ValueError("need 1 <= n_buckets <= number of matrices")
        cost = [matrix_cost(r, c, ns_steps) for r, c in self.shapes]
        total = sum(cost)
        self.buckets: List[List[int]] = []
        cur, acc = [], 0.0
        for i in range(n):
            cur.append(i)
            acc += cost[i]
            left_mats = n - i - 1
            left_buckets = n_buckets - len(self.buckets) - 1
            # close the bucket at its share of the cost, keeping at least one
            # matrix for every bucket still to come
            if left_buckets > 0 and (acc >= total * (len(self.buckets) + 1) / n_buckets
                                     or left_mats == left_buckets):
                self.buckets.append(cur)
                cur = []
        self.buckets.append(cur)
        self.layouts = [ShardLayout([self.shapes[i] for i in bk], world, ns_steps, align)
                        for bk in self.buckets]


class BucketBuffers:
    """One bucket's buffers on one rank (all flat, 1-D):
      W_flat  world * seg  weights (replicated after the all-gather);
      M_seg   seg          momentum of the matrices this rank owns;
      G_flat  world * seg  this rank's gradient contribution (bf16, or fp32 to
                           reduce in fp32);
      G_seg   seg          the summed gradients of this rank's matrices, in
                           G_flat's dtype;
      G_step  seg          the gradients the step reads: G_seg itself when the
                           reduction is in the step's dtype, else a bf16 buffer
                           that `to_step_dtype` fills from G_seg;
      E_seg   seg or None  the average (EMA) of the weights this rank owns."""

    def __init__(self, W_flat, M_seg, G_flat, G_seg, G_step=None, E_seg=None):
        self.W_flat, self.M_seg, self.G_flat, self.G_seg = W_flat, M_seg, G_flat, G_seg
        self.G_step = G_seg if G_step is None else G_step
        self.E_seg = E_seg

    @classmethod
    def allocate(cls, layout: ShardLayout, weight_dtype, grad_dtype, step_grad_dtype,
                 device=None, with_ema=False):
        import torch
        W = torch.zeros(layout.numel(), dtype=weight_dtype, device=device)
        M = torch.zeros(layout.seg, dtype=weight_dtype, device=device)
        Gf = torch.zeros(layout.numel(), dtype=grad_dtype, device=device)
        Gs = torch.zeros(layout.seg, dtype=grad_dtype, device=device)
        Gt = None if step_grad_dtype == grad_dtype else \
            torch.zeros(layout.seg, dtype=step_grad_dtype, device=device)
        E = torch.zeros(layout.seg, dtype=weight_dtype, device=device) if with_ema else None
        return cls(W, M, Gf, Gs, Gt, E)


def sharded_step_bucketed(layout: BucketedLayout, bufs: Sequence[BucketBuffers], rank: int,
                          step_fns: Sequence[Callable], group=None, comm_stream=None,
                          to_step_dtype: Optional[Callable] = None,
                          ema_fns: Optional[Sequence[Callable]] = None):
    """One data-parallel Muon step over the buckets of `layout`.

      1. the reduce-scatters of every bucket's gradients are issued at once, in
         bucket order, on `comm_stream` (after the gradients on the current
         stream are ready);
      2. for each bucket in order, the current stream waits for that bucket's
         reduce-scatter only, rounds the summed gradients to the step's dtype
         with `to_step_dtype(G_step, G_seg)` if the reduction ran in another
         dtype, and runs `step_fns[b](W_views, M_views, G_views)` on views of
         this rank's segment, then, with `ema_fns`, ema_fns[b](E_views,
         W_views) on its E_seg (the average of the weights it owns, no
         exchange); so bucket b's step overlaps the reduce-scatters of the
         buckets after it;
      3. the all-gathers of the updated weights are issued on `comm_stream` in
         bucket order, each waiting for its own bucket's step only, so that
         bucket b's all-gather overlaps the steps of the buckets after it;
         the current stream finally waits for all of them.

    Every rank issues the same collectives in the same order (all
    reduce-scatters, then all all-gathers).  On CPU tensors (gloo) the waits
    are host waits and `comm_stream` must be None."""
    import torch
    import torch.distributed as dist
    cuda = bufs[0].W_flat.is_cuda
    if comm_stream is not None and not cuda:
        raise ValueError("comm_stream needs CUDA buffers")
    compute = torch.cuda.current_stream() if cuda else None
    side = torch.cuda.stream(comm_stream) if comm_stream is not None else nullcontext()
    if comm_stream is not None:
        comm_stream.wait_stream(compute)
    with side:
        rs = [dist.reduce_scatter_tensor(bf.G_seg, bf.G_flat, op=dist.ReduceOp.SUM,
                                         group=group, async_op=True) for bf in bufs]
    done = []
    for b, (L, bf) in enumerate(zip(layout.layouts, bufs)):
        rs[b].wait()
        if bf.G_step is not bf.G_seg:
            if to_step_dtype is None:
                raise ValueError("a reduction dtype other than the step's needs "
                                 "to_step_dtype")
            to_step_dtype(bf.G_step, bf.G_seg)
        own = bf.W_flat[rank * L.seg:(rank + 1) * L.seg]
        if L.mine[rank]:
            w_views = L.local_views(own, rank)
            step_fns[b](w_views, L.local_views(bf.M_seg, rank),
                        L.local_views(bf.G_step, rank))
            if ema_fns is not None:
                ema_fns[b](L.local_views(bf.E_seg, rank), w_views)
        if comm_stream is not None:
            ev = torch.cuda.Event()
            ev.record(compute)
            done.append(ev)
    ag = []
    with side:
        for b, (L, bf) in enumerate(zip(layout.layouts, bufs)):
            if comm_stream is not None:
                comm_stream.wait_event(done[b])
            own = bf.W_flat[rank * L.seg:(rank + 1) * L.seg]
            ag.append(dist.all_gather_into_tensor(bf.W_flat, own.clone(), group=group,
                                                  async_op=True))
    for w in ag:
        w.wait()


def max_over_ranks(value: float, device=None, group=None) -> float:
    """The slowest rank's time (the timing rule of the benchmark)."""
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX, group=group)
    return float(t.item())
