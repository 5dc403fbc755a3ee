"""Data-parallel Lloyd over several processes, one GPU each, in two splits.

Point blocks (lloyd_data_parallel): the points of every batch split into
contiguous blocks, one per rank.

The pages' large-N path splits the N points into contiguous block
partitions, one per GPU; each GPU runs its own assign and partial update over
its block, the partial centroid sums and counts are reduced over the GPUs,
and the new centroids are the same everywhere ("flash-kmeans and the return
of exact K-Means on the GPU", section "Multi-GPU scaling without a NCCL
dependency").  Here every rank is one process driving one GPU; the exchange
is one all-reduce of the sums (B*K*d fp32) and one of the counts (B*K int32)
per iteration through torch.distributed (NCCL over NVLink / NVSwitch), and
every rank then runs the same finalize, so the centroids stay identical
without a broadcast.  Each per-rank step is one call into libfk
(fk_lloyd_step_partial, fk_update_finalize); a rank's block may sit in device
memory or in pinned host memory (then it is streamed in chunks).

    n0, n1 = block_of(N, rank, world)
    iters = lloyd_data_parallel(x[:, n0:n1], init, max_iter, tol, ids, centers)

Batch shares (lloyd_batch_split): the B batches of a problem are independent
K-Means problems, so each rank takes a contiguous share of them and runs the
whole Lloyd loop on its share with no exchange of data at all; the only
collective in the loop is a max of one float per iteration when tol > 0 (the
stop rule is one global max-shift test over every batch), and the results
are gathered once at the end (gather_batches).

    b0, b1 = block_of(B, rank, world)
    iters = lloyd_batch_split(x[b0:b1], init[b0:b1], max_iter, tol, ids_share, centers_share)
    ids_all = gather_batches(ids_share, B)
"""
from __future__ import annotations

import torch
import torch.distributed as dist


def block_of(N: int, rank: int, world: int) -> tuple[int, int]:
    """[n0, n1): the contiguous block of rank `rank`; the first N % world ranks
    hold one point more than the others."""
    base, extra = divmod(N, world)
    n0 = rank * base + min(rank, extra)
    return n0, n0 + base + (1 if rank < extra else 0)


def initial_centers_over_blocks(x: torch.Tensor, K: int, seed: int = 0, group=None) -> torch.Tensor:
    """The initial centroids of a problem split into contiguous blocks, on every rank.

    x is this rank's block (B, n, d); the blocks in rank order make up the whole
    problem of N = (sum of n) points per batch.  Returns (B, K, d) in x's dtype on
    x's device: the points at init_indices(B, N, K, seed) of the whole problem,
    the centroids a single process with all the points would start from.  Every
    rank takes the same collective steps: one all-gather of the block sizes, one
    all-reduce that assembles the rows, each owned by exactly one rank (summed
    as integer bits with zeros, so every value arrives exactly).
    """
    from .kmeans import init_indices
    B, n, d = x.shape
    group_rank = dist.get_rank(group)
    world = dist.get_world_size(group)
    on_gpu = dist.get_backend(group) == "nccl"
    cdev = torch.device("cuda", torch.cuda.current_device()) if on_gpu else torch.device("cpu")
    size = torch.tensor([n], dtype=torch.int64, device=cdev)
    sizes = [torch.empty_like(size) for _ in range(world)]
    dist.all_gather(sizes, size, group=group)
    sizes = [int(t.item()) for t in sizes]
    N, n0 = sum(sizes), sum(sizes[:group_rank])
    if K > N:  # every rank knows N now, so every rank raises
        raise ValueError(f"K = {K} clusters but only {N} points over the ranks")
    idx = init_indices(B, N, K, seed)
    rows = torch.zeros((B, K, d), dtype=x.dtype)
    for b in range(B):
        mine = ((idx[b] >= n0) & (idx[b] < n0 + n)).nonzero().flatten()
        if mine.numel():
            rows[b, mine] = x[b].index_select(0, (idx[b, mine] - n0).to(x.device)).cpu()
    words = rows.view(torch.int32) if x.element_size() == 4 or d % 2 == 0 else rows.to(torch.float32)
    words = words.to(cdev)
    dist.all_reduce(words, op=dist.ReduceOp.SUM, group=group)
    out = words.view(x.dtype) if words.dtype == torch.int32 else words.to(x.dtype)
    return out.to(x.device).contiguous()


class CudaSteps:
    """The per-rank steps of lloyd_data_parallel and lloyd_batch_split, each one call into libfk."""

    def __init__(self, stream=None, chunk_points: int = 0):
        from . import fk_init_centers, fk_lloyd_step_partial, fk_point_norms, fk_update_finalize
        self._init, self._partial = fk_init_centers, fk_lloyd_step_partial
        self._norms, self._final = fk_point_norms, fk_update_finalize
        self.stream, self.chunk_points = stream, chunk_points

    def point_norms(self, x):
        # fp16 / bf16 points resident on the device: ||x||^2 once per run
        if x.dtype == torch.float32 or not x.is_cuda or x.shape[1] == 0:
            return None
        xn = torch.empty(x.shape[:2], dtype=torch.float32, device=x.device)
        return self._norms(x, xn, stream=self.stream)

    def init_centers(self, init, centers):
        self._init(init, centers, stream=self.stream)

    def partial(self, x, xn, centers_dt, ids, sums, counts):
        self._partial(x, xn, centers_dt, ids, sums, counts, stream=self.stream,
                      chunk_points=self.chunk_points)

    def finalize(self, sums, counts, centers, centers_dt, shift, dtype):
        self._final(sums, counts, centers, centers_dt, shift, dtype=dtype, stream=self.stream)


def lloyd_data_parallel(x: torch.Tensor, init_centers: torch.Tensor, max_iter: int, tol: float,
                        ids: torch.Tensor, centers: torch.Tensor, group=None, steps=None) -> int:
    """Lloyd's iterations over this rank's block of points.

    x             (B, n, d): this rank's block (device or pinned host memory).
    init_centers  (B, K, d) in x's dtype on this rank's device, identical on every rank.
    ids           (B, n) int32 out (device): the block's assignment of the last iteration.
    centers       (B, K, d) out (device): the centroids of the last update, identical on
                  every rank.
    group         torch.distributed group of the ranks (default: the world, when a
                  process group is initialised; otherwise this process alone).
    Stops after max_iter iterations or when the max centroid shift is below tol (strict);
    every rank sees the same shift, so every rank stops after the same iteration and takes
    the same collective steps.  Returns the number of iterations run.
    """
    steps = steps or CudaSteps()
    B, _, d = x.shape
    K = init_centers.shape[1]
    dev = centers.device
    reduce = dist.is_available() and dist.is_initialized()
    sums = torch.empty((B, K, d), dtype=centers.dtype, device=dev)
    counts = torch.empty((B, K), dtype=torch.int32, device=dev)
    shift = torch.zeros((1,), dtype=centers.dtype, device=dev)
    steps.init_centers(init_centers, centers)
    low = x.dtype in (torch.float16, torch.bfloat16)
    # the assign takes centroids in x's dtype: the initial ones first, then the
    # rounded copy every finalize writes (fp32 points: the fp32 centroids)
    centers_dt = torch.empty_like(init_centers) if low else None
    cur = init_centers if low else centers
    xn = steps.point_norms(x)
    it = 0
    while it < max_iter:
        steps.partial(x, xn, cur, ids, sums, counts)
        if reduce:
            dist.all_reduce(sums, op=dist.ReduceOp.SUM, group=group)
            dist.all_reduce(counts, op=dist.ReduceOp.SUM, group=group)
        steps.finalize(sums, counts, centers, centers_dt, shift, x.dtype)
        it += 1
        if low:
            cur = centers_dt
        if tol > 0 and float(shift.item()) < tol:
            break
    return it


def lloyd_batch_split(x: torch.Tensor, init_centers: torch.Tensor, max_iter: int, tol: float,
                      ids: torch.Tensor, centers: torch.Tensor, group=None, steps=None) -> int:
    """Lloyd's iterations over this rank's share of the batches.

    x             (b, N, d): this rank's contiguous share of the batches (b may be 0).
    init_centers  (b, K, d) in x's dtype: their initial centroids.
    ids, centers  (b, N) int32 and (b, K, d) out.
    The batches never exchange data.  With tol > 0 the ranks agree on the stop:
    after every iteration one all-reduce takes the max of the ranks' max shifts,
    so every rank stops after the iteration a single process over all the
    batches would stop after.  With tol <= 0 the loop takes no collective step.
    Returns the number of iterations run.
    """
    steps = steps or CudaSteps()
    b, _, d = x.shape
    K = init_centers.shape[1]
    dev = centers.device
    agree = tol > 0 and dist.is_available() and dist.is_initialized()
    shift = torch.zeros((1,), dtype=centers.dtype, device=dev)
    if b > 0:
        sums = torch.empty((b, K, d), dtype=centers.dtype, device=dev)
        counts = torch.empty((b, K), dtype=torch.int32, device=dev)
        steps.init_centers(init_centers, centers)
    low = x.dtype in (torch.float16, torch.bfloat16)
    centers_dt = torch.empty_like(init_centers) if low else None
    cur = init_centers if low else centers
    xn = steps.point_norms(x) if b > 0 else None
    it = 0
    while it < max_iter:
        if b > 0:
            steps.partial(x, xn, cur, ids, sums, counts)
            steps.finalize(sums, counts, centers, centers_dt, shift, x.dtype)
        it += 1
        if low:
            cur = centers_dt
        if tol > 0:
            if agree:
                dist.all_reduce(shift, op=dist.ReduceOp.MAX, group=group)
            if float(shift.item()) < tol:
                break
    return it


def gather_batches(share: torch.Tensor, B: int, group=None) -> torch.Tensor:
    """The (B, ...) tensor whose batches [b0, b1) are each rank's `share`
    (block_of(B, rank, world)), on every rank: one all-gather of the shares
    padded to the largest one."""
    world = dist.get_world_size(group)
    per = -(-B // world)
    pad = torch.zeros((per,) + tuple(share.shape[1:]), dtype=share.dtype, device=share.device)
    pad[: share.shape[0]] = share
    parts = [torch.empty_like(pad) for _ in range(world)]
    dist.all_gather(parts, pad, group=group)
    out = [parts[r][: block_of(B, r, world)[1] - block_of(B, r, world)[0]] for r in range(world)]
    return torch.cat(out, dim=0)
